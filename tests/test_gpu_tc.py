"""Parity of the tensor-core path (tcgen05 kind::i8, or kind::f16 on the
codes widened to fp16, T >= 16, Q8_0 weights) with the CPU oracle, through
the C ABI."""
import numpy as np
import pytest
import torch

from quantized_latent_moe_b200 import synth
from helpers import gpu_layer, oracle_layer, oracle_forward, max_abs_rel

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def E():
    from quantized_latent_moe_b200 import build, elq
    build.build()
    elq.lib()
    return elq


@pytest.mark.parametrize("N,K,T", [(128, 128, 64), (256, 512, 100), (1792, 4096, 128), (4096, 1792, 300),
                                   (384, 1280, 77)])
def test_tc_latent_proj_exact(E, orc, N, K, T):
    W = synth.normal(21, N + K, (N, K), 0.02)
    X = synth.normal(22, T, (T, K))
    m = E.QMatrix.from_f32(W.cuda(), 8)
    xq = E.quantize_q8_1(X.cuda())
    y = E.latent_proj(m, xq, T).cpu().numpy()
    ref = orc.qmatmul(8, orc.quantize(8, W.numpy()), N, K, orc.quantize(orc.Q8_1, X.numpy()), T)
    assert np.array_equal(y, ref)


def test_f16_codes_layout(E):
    """elq_pack_f16 against the layout the header states, built here from the
    quantised weights' codes: per (tile, block) [code/16][row/8][(code%16)/8]
    [row%8][8 fp16], the value of row r's code c of the block."""
    n_rows, k = 256, 128
    W = synth.normal(23, 7, (n_rows, k), 0.02)
    m = E.QMatrix.from_f32(W.cuda(), 8).pack_f16()
    # the codes by row, independent of the int8 arena: the Q8_0 quantiser's blocks
    import oracle
    oracle.lib()
    codes = np.frombuffer(oracle.quantize(8, W.numpy()).tobytes(), np.uint8).reshape(n_rows, k // 32, 34)[:, :, 2:]
    codes = codes.view(np.int8)
    got = m.q16.cpu().numpy().view(np.float16).reshape(n_rows // 128, k // 32, 4096)
    exp = np.zeros_like(got)
    for r in range(128):
        for c in range(32):
            dst = ((c // 16) * 4096 + (r // 8) * 256 + ((c % 16) // 8) * 128 + (r % 8) * 16 + (c % 8) * 2) // 2
            exp[:, :, dst] = codes[r::128, :, c].astype(np.float16).reshape(n_rows // 128, k // 32)
    assert np.array_equal(got, exp)


@pytest.mark.parametrize("f16", [False, True], ids=["i8", "f16"])
@pytest.mark.parametrize("T", [64, 100, 257])
def test_tc_layer_tiny_exact(E, orc, T, f16):
    wl = synth.WORKLOADS["tiny"]
    ly = gpu_layer(wl)
    if f16:
        ly.enable_f16()
    assert ly.kernel_count(T) == 10
    x = synth.make_x(wl, T=T)
    y = E.moe_layer(ly, x.cuda()).cpu().numpy()
    assert E.workspace_status(ly.workspace(T)) == 0
    ol = oracle_layer(orc, wl)
    tr = ol.forward(x.numpy(), trace=True)
    v = lambda n: E.workspace_view(ly, T, n).cpu().numpy()
    assert np.array_equal(v("z").reshape(T, -1), tr["z"])
    assert np.array_equal(v("zq").reshape(T, -1), tr["zq"])
    assert np.array_equal(v("idx").reshape(T, -1), tr["idx"])
    assert np.array_equal(v("perm"), tr["perm"])
    assert np.array_equal(v("y_lat").reshape(T, -1), tr["y_lat"])
    assert np.array_equal(v("ylq").reshape(T, -1), tr["ylq"])
    assert max_abs_rel(y, tr["y"]) <= 1e-3
    assert np.array_equal(y, tr["y"])


@pytest.mark.parametrize("f16", [False, True], ids=["i8", "f16"])
def test_tc_experts_grouped_exact(E, orc, f16):
    wl = synth.WORKLOADS["tiny"]
    T = 96
    ly = gpu_layer(wl)
    if f16:
        ly.enable_f16()
    ol = oracle_layer(orc, wl)
    tr = ol.forward(synth.make_x(wl, T=T).numpy(), trace=True)
    y_lat = E.moe_experts_grouped(ly, torch.from_numpy(tr["zq"]).cuda(), torch.from_numpy(tr["idx"]).cuda(),
                                  torch.from_numpy(tr["w"]).cuda()).cpu().numpy()
    assert np.array_equal(y_lat, tr["y_lat"])


def _threads(fn, parts):
    from concurrent.futures import ThreadPoolExecutor
    import os
    with ThreadPoolExecutor(max_workers=min(16, os.cpu_count() or 1)) as ex:
        return list(ex.map(fn, parts))


@pytest.mark.parametrize("f16", [False, True], ids=["i8", "f16"])
def test_tc_prefill_full_size(E, orc, f16):
    """The prefill workload at full size (T=2048, 128 experts, Zipf-skewed
    router), through the layer call:
     - z and its Q8_1 rows for all 2048 tokens against the oracle's quantised
       matmul (the oracle quantises x and D itself);
     - the routing of all 2048 tokens (logits, idx, weights) against the
       oracle's router on the oracle's z, and the bucket arrays against the
       oracle's bucketing of those ids;
     - y for sampled tokens, the oracle computing them alone (the layer is
       token-wise independent): the last pair of every expert group (each lands
       in that expert's last, usually partial, 64-token tile), every token of
       the smallest group, the first and last tokens of the largest, tokens 0
       and 2047."""
    wl = synth.WORKLOADS["prefill"]
    ly = gpu_layer(wl)
    if f16:
        ly.enable_f16()
    x = synth.make_x(wl)
    y = E.moe_layer(ly, x.cuda()).cpu().numpy()
    assert E.workspace_status(ly.workspace(wl.T)) == 0
    v = lambda n: E.workspace_view(ly, wl.T, n).cpu().numpy()
    T, L, H, k = wl.T, wl.L, wl.H, wl.k
    # z for every token (rows of tokens split over host threads)
    dw = synth.dense_weights(wl, 0)
    Dq = orc.quantize(8, dw["D"].numpy())
    xq = orc.quantize(orc.Q8_1, x.float().numpy())
    assert np.array_equal(v("xq").reshape(T, -1), xq)
    rows = [(t0, min(T, t0 + 128)) for t0 in range(0, T, 128)]
    zs = _threads(lambda r: orc.qmatmul(8, Dq, L, H, xq[r[0]:r[1]], r[1] - r[0]), rows)
    z_ref = np.concatenate(zs)
    assert np.array_equal(v("z").reshape(T, L), z_ref)
    assert np.array_equal(v("zq").reshape(T, -1), orc.quantize(orc.Q8_1, z_ref))
    # routing of every token
    ridx, rw, rlg = orc.router_topk(z_ref, dw["router_w"].numpy(), dw["router_bias"].numpy(), k)
    assert np.array_equal(v("logits").reshape(T, -1), rlg)
    idx = v("idx").reshape(T, k)
    assert np.array_equal(idx, ridx)
    assert np.array_equal(v("weights").reshape(T, k), rw)
    counts, offsets, perm, pos = orc.bucket(ridx, wl.E)
    assert np.array_equal(v("counts"), counts) and np.array_equal(v("offsets"), offsets)
    assert np.array_equal(v("perm"), perm) and np.array_equal(v("pos"), pos)
    # sampled outputs
    sample = {0, T - 1}
    for e in range(wl.E):
        if counts[e]:
            sample.add(int(perm[offsets[e + 1] - 1]) // k)
    e_min = int(np.argmin(np.where(counts > 0, counts, 1 << 30)))
    e_max = int(np.argmax(counts))
    sample |= {int(p) // k for p in perm[offsets[e_min]:offsets[e_min + 1]]}
    sample |= {int(perm[offsets[e_max]]) // k, int(perm[offsets[e_max + 1] - 1]) // k}
    sample = sorted(sample)
    ol = oracle_layer(orc, wl, experts=sorted(set(ridx[sample].reshape(-1).tolist())))
    xs = x.float().numpy()
    parts = [sample[i:i + 8] for i in range(0, len(sample), 8)]
    ref = np.concatenate(_threads(lambda ts: ol.forward(xs[ts]), parts))
    assert max_abs_rel(y[sample], ref) <= 1e-3
    assert np.array_equal(y[sample], ref)


def test_int8_rate_kernel_runs(E):
    """The measurement kernel behind the int8 peak: no wait runs out, and every
    CTA's accumulator word is the same nonzero value (same operands)."""
    sink, err = E.test_mma_i8_rate(64)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    s = sink.cpu()
    assert (s == s[0]).all() and int(s[0]) != 0


def test_f32x2_rate_kernel_runs(E):
    """The measurement kernel behind the epilogue bound runs and leaves
    finite values."""
    sink = E.test_f32x2_rate(16)
    torch.cuda.synchronize()
    assert torch.isfinite(sink).all()
