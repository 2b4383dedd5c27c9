"""Parity of the NVFP4 expert paths (through the C ABI) with the CPU oracle.

Cluster GEMV (T <= 8): the quantiser's bytes, the packed arena and every
intermediate of a layer with NVFP4 experts (z's and h's NVFP4 blocks, the
expert outputs o, the combine) must be bit-exact; the layer output too, since
both sides take the same micro-block order and the same scale products.

Block-scaled tensor cores (more tokens): z, its NVFP4 rows and the routing are
bit-exact (the int8 tensor-core D projection and the same quantiser); the
expert sums are the tensor core's fp32 accumulation, whose order is not the
oracle's chain.  Every micro-block term (a small integer times two E4M3
scales) is exact in fp32, so the sums agree whenever no partial sum rounds --
which holds on every workload below: the outputs are asserted bit-exact, and
within the layer tolerance (max-abs-rel 1e-3) on activations spread over a
wide range.
"""
import numpy as np
import pytest
import torch

from quantized_latent_moe_b200 import synth
from helpers import add_experts, gpu_layer, max_abs_rel, nvfp4_globals, oracle_forward, oracle_layer

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def E():
    from quantized_latent_moe_b200 import build, elq
    build.build()
    elq.lib()
    assert torch.cuda.is_available()
    return elq


def _special_rows():
    """Blocks that reach the rounding rules' edges: every E2M1 midpoint and its
    neighbours under an exact scale of 1 (amax 6), values that round to a
    signed zero, zero blocks, and micro-blocks whose scale saturates."""
    rows = []
    grid = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0], np.float32)
    mids = (grid[:-1] + grid[1:]) / 2
    vals = []
    for m in mids:
        vals += [m, np.nextafter(m, np.float32(0)), np.nextafter(m, np.float32(9))]
    vals = np.array(vals, np.float32)
    for sign in (1.0, -1.0):
        v = np.resize(vals, 15) * sign
        rows.append(np.concatenate([[6.0], v, [-6.0], -v]).astype(np.float32))
    rows.append(np.array([6.0] + [-0.1, -0.2, -0.24, 0.1, -0.0, 0.0] * 2 + [-0.25, 0.25, 0.26]
                         + [1e-3] * 16, np.float32))
    rows.append(np.zeros(32, np.float32))
    rows.append(np.array([3e4] * 8 + [-2e4] * 8 + [1.0] * 16, np.float32))   # amax / 6 > 448: saturated scale
    return np.stack(rows)


@pytest.mark.parametrize("g", [1.0, 2.0 ** -6, 0.37, "amax"])
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_quantize_nvfp4_bytes(E, orc, g, dtype):
    x = synth.normal(21, 3, (37, 256), 1.0)
    x[5] *= 1e-3
    x[7] *= 300.0
    sp = torch.from_numpy(_special_rows())
    x[10:10 + sp.shape[0], :32] = sp
    x = x.to(dtype)
    xf = x.float().numpy()
    if g == "amax":
        g = float(nvfp4_globals(x.float()[None])[0])
    got = E.quantize_nvfp4(x.cuda(), g).cpu().numpy()
    ref = orc.quantize_nvfp4(xf, g)
    assert np.array_equal(got, ref)


def test_quantize_nvfp4_ragged_and_empty(E, orc):
    for rows, cols in ((1, 32), (3, 96), (129, 64)):
        x = synth.normal(22, rows, (rows, cols), 2.0)
        assert np.array_equal(E.quantize_nvfp4(x.cuda(), 0.5).cpu().numpy(), orc.quantize_nvfp4(x.numpy(), 0.5))
    assert E.quantize_nvfp4(torch.empty(0, 64, device="cuda"), 1.0).numel() == 0


def test_arena_pack_nvfp4(E, orc):
    """NVFP4 blocks pack in the Q4_0 byte geometry (the oracle's Q4_0 packing
    of the same bytes), each tile's scales followed by the same bytes as the
    tensor cores' scale atoms (built here from the header's statement)."""
    n_rows, k = 256, 512
    nb, tiles = k // 32, n_rows // 128
    w = synth.normal(23, 1, (n_rows, k), 0.02)
    g = float(nvfp4_globals(w[None])[0])
    aos = orc.quantize_nvfp4(w.numpy(), g)
    m = E.QMatrix.from_aos(torch.from_numpy(aos).cuda(), E.NVFP4, n_rows, k)
    q, d = orc.arena_pack(orc.Q4_0, aos, n_rows, k)
    assert np.array_equal(m.q.cpu().numpy(), q)
    md = m.d.cpu().numpy().reshape(tiles, 2, nb * 256)
    assert np.array_equal(md[:, 0], d.reshape(tiles, nb * 256))
    sc = aos.reshape(tiles, 128, nb, 18)[..., :2]            # [tile][row m][block][byte]
    atoms = np.zeros((tiles, nb // 2, 512), np.uint8)
    for m_ in range(128):
        for kb in range(nb):
            o = (m_ % 32) * 16 + (m_ // 32) * 4 + (kb % 2) * 2
            atoms[:, kb // 2, o:o + 2] = sc[:, m_, kb]
    assert np.array_equal(md[:, 1], atoms.reshape(tiles, nb * 256))


NV_TINY = synth.Workload("nv_tiny", 9, 3, 512, 256, 8, 2, 256, synth.Q8_0, synth.F32, "normal",
                         ex_fmt=synth.NVFP4)
NV_TINY4 = synth.Workload("nv_tiny4", 10, 8, 512, 512, 16, 8, 256, synth.Q4_0, synth.BF16, "none",
                          ex_fmt=synth.NVFP4)


def _check(E, ly, T, tr):
    v = lambda n: E.workspace_view(ly, T, n).cpu().numpy()
    assert np.array_equal(v("z").reshape(T, -1), tr["z"])
    assert np.array_equal(v("zq").reshape(T, -1), tr["zq"])
    assert np.array_equal(v("idx").reshape(T, -1), tr["idx"])
    assert np.array_equal(v("weights").reshape(T, -1), tr["w"])
    pos = tr["pos"]
    assert np.array_equal(v("hq").reshape(T * ly.k, -1)[pos], tr["hq"])
    assert np.array_equal(v("o").reshape(T * ly.k, -1)[pos], tr["o"])
    assert np.array_equal(v("y_lat").reshape(T, -1), tr["y_lat"])
    assert np.array_equal(v("ylq").reshape(T, -1), tr["ylq"])


@pytest.mark.parametrize("wl", [NV_TINY, NV_TINY4], ids=["q8du", "q4du_bf16"])
def test_nvfp4_layer_exact(E, orc, wl):
    ly = gpu_layer(wl)
    assert ly.kernel_count(wl.T) == 5
    ol = oracle_layer(orc, wl)
    # both sides take the same global scales from the same fp32 weights
    assert np.array_equal(ly.gate_up.gs.cpu().numpy(), ol.gate_g)
    assert np.array_equal(ly.down.gs.cpu().numpy(), ol.down_g)
    for T in sorted({1, 2, wl.T}):
        x = synth.make_x(wl, T=T)
        y = E.moe_layer(ly, x.cuda()).cpu().numpy()
        assert E.workspace_status(ly.workspace(T)) == 0
        tr = ol.forward(x.float().numpy(), trace=True)
        _check(E, ly, T, tr)
        assert np.array_equal(y, tr["y"]), T


def test_nvfp4_layer_refuses_q4_du_above_8_tokens(E):
    """Beyond the cluster GEMV's sizes the NVFP4 experts run on the tensor
    cores, whose D and U projections are Q8_0 only."""
    ly = gpu_layer(NV_TINY4)
    x = synth.make_x(NV_TINY4, T=9).cuda()
    assert ly.kernel_count(9) == 0
    with pytest.raises(E.ElqError) as ei:
        E.moe_layer(ly, x, ws=torch.zeros(1 << 20, dtype=torch.uint8, device="cuda"))
    assert ei.value.status == -2


def _check_tc(E, ly, T, tr):
    v = lambda n: E.workspace_view(ly, T, n).cpu().numpy()
    assert np.array_equal(v("z").reshape(T, -1), tr["z"])
    assert np.array_equal(v("zq").reshape(T, -1), tr["zq"])
    assert np.array_equal(v("idx").reshape(T, -1), tr["idx"])
    assert np.array_equal(v("weights").reshape(T, -1), tr["w"])
    assert np.array_equal(v("offsets"), tr["offsets"])
    return v("y_lat").reshape(T, -1)


@pytest.mark.parametrize("T,f16", [(9, False), (16, False), (64, False), (127, False), (128, False),
                                   (129, False), (300, False), (16, True), (129, True)])
def test_nvfp4_tc_layer(E, orc, T, f16):
    """The block-scaled tensor-core experts (eleven kernels), from just above
    the GEMV's sizes through several 128-slot tiles per expert and ragged last
    tiles; D and U on int8 or fp16-widened codes."""
    wl = NV_TINY
    ly = gpu_layer(wl)
    if f16:
        ly.enable_f16()
    assert ly.kernel_count(T) == 11
    ol = oracle_layer(orc, wl)
    x = synth.make_x(wl, T=T)
    y = E.moe_layer(ly, x.cuda()).cpu().numpy()
    assert E.workspace_status(ly.workspace(T)) == 0
    tr = ol.forward(x.float().numpy(), trace=True)
    y_lat = _check_tc(E, ly, T, tr)
    assert max_abs_rel(y, tr["y"]) <= 1e-3
    assert np.array_equal(y_lat, tr["y_lat"])
    assert np.array_equal(y, tr["y"])
    # the same bits again (the combine counters reset themselves)
    assert np.array_equal(E.moe_layer(ly, x.cuda()).cpu().numpy(), y)


@pytest.mark.parametrize("spread", [4.0, 8.0])
def test_nvfp4_tc_wide_range_activations(E, orc, spread):
    """D's rows scaled by 2^u, u uniform in [-spread, spread]: z's micro-block
    scales cover many binades (some saturate, some flush), so the expert sums
    are no longer small: the layer stays within the tolerance of the oracle."""
    wl = NV_TINY
    T = 200
    ly = gpu_layer(wl)
    dw = synth.dense_weights(wl, 0)
    f = (2.0 ** (synth.normal(31, 1, wl.L).numpy().clip(-1.7, 1.7) / 1.7 * spread)).astype(np.float32)
    D = (dw["D"].numpy() * f[:, None]).astype(np.float32)
    ly.set_dense(torch.from_numpy(D).cuda(), dw["U"].cuda())
    torch.cuda.synchronize()
    w = {k: (None if v is None else v.numpy()) for k, v in dw.items()}
    w.update(D=D, gate=None, act_gz=synth.NVFP4_ACT_GSCALE, act_gh=synth.NVFP4_ACT_GSCALE)
    ol = orc.Layer(wl.H, wl.L, wl.E, wl.k, wl.I, orc.Q8_0, orc.NVFP4, w)
    add_experts(ol, wl, range(wl.E))
    x = synth.make_x(wl, T=T)
    y = E.moe_layer(ly, x.cuda()).cpu().numpy()
    tr = ol.forward(x.float().numpy(), trace=True)
    _check_tc(E, ly, T, tr)
    assert max_abs_rel(y, tr["y"]) <= 1e-3


def test_nvfp4_tc_prefill_full_size(E, orc):
    """The prefill shapes with NVFP4 experts (T = 2048, 128 experts, top-8,
    Zipf-skewed router): z's NVFP4 rows and the routing for every token, y for
    sampled tokens (the last pair of every expert group, every token of the
    smallest group, tokens 0 and 2047), the oracle computing them alone."""
    wl = synth.WORKLOADS["prefill_nvfp4"]
    ly = gpu_layer(wl)
    assert ly.kernel_count(wl.T) == 11
    x = synth.make_x(wl)
    y = E.moe_layer(ly, x.cuda()).cpu().numpy()
    assert E.workspace_status(ly.workspace(wl.T)) == 0
    v = lambda n: E.workspace_view(ly, wl.T, n).cpu().numpy()
    T, k = wl.T, wl.k
    idx = v("idx").reshape(T, k)
    perm = v("perm")
    offsets = v("offsets")
    sample = {0, T - 1}
    sizes = np.diff(offsets)
    for e in range(wl.E):
        if sizes[e]:
            sample.add(int(perm[offsets[e + 1] - 1]) // k)
    small = int(np.argmin(np.where(sizes > 0, sizes, 1 << 30)))
    sample |= {int(p) // k for p in perm[offsets[small]:offsets[small + 1]]}
    sample = sorted(sample)
    ol = oracle_layer(orc, wl, experts=[])
    xs = x.float().numpy()[sample]
    tr = oracle_forward(orc, ol, wl, xs, trace=True)
    zq = v("zq").reshape(T, -1)[sample]
    assert np.array_equal(v("z").reshape(T, -1)[sample], tr["z"])
    assert np.array_equal(zq, tr["zq"])
    assert np.array_equal(idx[sample], tr["idx"])
    assert max_abs_rel(y[sample], tr["y"]) <= 1e-3
    assert np.array_equal(y[sample], tr["y"])


def test_nvfp4_experts_grouped_exact(E, orc):
    wl = NV_TINY4
    ly = gpu_layer(wl)
    ol = oracle_layer(orc, wl)
    tr = ol.forward(synth.make_x(wl).float().numpy(), trace=True)
    zq = torch.from_numpy(tr["zq"]).cuda()
    idx = torch.from_numpy(tr["idx"]).cuda()
    w = torch.from_numpy(tr["w"]).cuda()
    y_lat = E.moe_experts_grouped(ly, zq, idx, w).cpu().numpy()
    assert np.array_equal(y_lat, tr["y_lat"])


@pytest.mark.parametrize("T", [1, 8])
def test_nvfp4_decode_full_size(E, orc, T):
    """The decode shapes with NVFP4 experts (128 experts, top-8, L = 1792,
    I = 1024): the whole output equals the oracle's (the oracle supplied with
    the routed experts only)."""
    wl = synth.WORKLOADS["decode_nvfp4"]
    ly = gpu_layer(wl)
    x = synth.make_x(wl, T=T)
    y = E.moe_layer(ly, x.cuda()).cpu().numpy()
    assert E.workspace_status(ly.workspace(T)) == 0
    ol = oracle_layer(orc, wl, experts=[])
    tr = oracle_forward(orc, ol, wl, x.float().numpy(), trace=True)
    routed = sorted(set(tr["idx"].reshape(-1).tolist()))
    assert np.array_equal(ly.gate_up.gs.cpu().numpy()[routed], ol.gate_g[routed])
    _check(E, ly, T, tr)
    assert np.array_equal(y, tr["y"])
    # repeated calls give the same bits (the combine counters reset themselves)
    assert np.array_equal(E.moe_layer(ly, x.cuda()).cpu().numpy(), y)


def test_fp4_rate_kernel_runs(E):
    """The measurement kernel behind the fp4 peak: no wait runs out, and every
    CTA's accumulator is n_mma x 64 (all values and scales 1.0, K = 64), which
    also pins the block-scaled MMA's operand and scale-factor plumbing."""
    n = 37
    sink, err = E.test_mma_nvf4_rate(n)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    s = sink.cpu().numpy().view(np.float32)
    assert (s == np.float32(64.0 * n)).all(), s[:4]
