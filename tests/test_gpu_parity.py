"""Parity of the CUDA path (through the C ABI) with the CPU oracle.

Integer and byte results (quantised blocks, block isums, router indices,
bucket arrays) must be bit-exact.  The floating-point results follow the same
accumulation order and the same exp on both sides, so they are compared for
exact equality as well; the layer outputs are additionally held to the
required max-abs-rel <= 1e-3.
"""
import numpy as np
import pytest
import torch

from quantized_latent_moe_b200 import synth
from helpers import gpu_layer, oracle_layer, oracle_forward, max_abs_rel, add_experts

pytestmark = pytest.mark.gpu
TOL = 1e-3


@pytest.fixture(scope="module")
def E():
    from quantized_latent_moe_b200 import build, elq
    build.build()
    elq.lib()
    assert torch.cuda.is_available()
    return elq


def _gen(seed, tid, shape, sigma=1.0):
    return synth.normal(seed, tid, shape, sigma)


def test_synth_gpu_equals_cpu(E):
    a = synth.normal(9, 3, (3, 1000), 0.02)
    b = synth.normal(9, 3, (3, 1000), 0.02, device="cuda").cpu()
    assert torch.equal(a, b)
    x = synth.make_x(synth.WORKLOADS["decode"], device="cuda").cpu()
    assert torch.equal(x, synth.make_x(synth.WORKLOADS["decode"]))


def test_expf_bitwise(E, orc):
    xs = np.concatenate([np.linspace(-110, 95, 20001), np.random.default_rng(0).uniform(-30, 30, 5000)])
    xs = xs.astype(np.float32)
    g = E.test_expf(torch.from_numpy(xs).cuda()).cpu().numpy()
    ref = np.array([orc.expf(float(v)) for v in xs], np.float32)
    assert np.array_equal(g.view(np.uint32), ref.view(np.uint32))


@pytest.mark.parametrize("wfmt", [8, 2])
def test_block_isums_exact(E, orc, wfmt):
    n = 4096
    w = _gen(1, 1, (n, 32), 0.02).numpy()
    a = _gen(1, 2, (n, 32)).numpy()
    wb = orc.quantize(wfmt, w)
    ab = orc.quantize(orc.Q8_1, a)
    isum, term = E.test_block_isums(wfmt, torch.from_numpy(wb).cuda(), torch.from_numpy(ab).cuda(), n)
    isum, term = isum.cpu().numpy(), term.cpu().numpy()
    ref_i = np.array([orc.block_isum(wfmt, wb[i], ab[i]) for i in range(n)])
    ref_t = np.array([orc.block_term(wfmt, wb[i], ab[i]) for i in range(n)], np.float32)
    assert np.array_equal(isum, ref_i)
    assert np.array_equal(term, ref_t)                    # within 1e-7: here identical
    assert np.abs(term - ref_t).max() <= 1e-7


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("rows,cols", [(1, 32), (3, 4096), (37, 1792), (64, 96)])
def test_quantize_q8_1_bytes(E, orc, dtype, rows, cols):
    x = _gen(2, rows * 7 + cols, (rows, cols))
    x[0, :32] = torch.tensor([127.0, 2.5, -2.5, 0.5, -0.5, 1.5, -1.5] + [0.0] * 25)
    if rows > 1:
        x[1, :32] = 0.0
        x[1, 40 % cols] = -3.0
    x = x.to(dtype)
    g = E.quantize_q8_1(x.cuda()).cpu().numpy()
    ref = orc.quantize(orc.Q8_1, x.float().numpy())
    assert np.array_equal(g, ref)


@pytest.mark.parametrize("fmt", [8, 2])
def test_quantize_weights_and_pack(E, orc, fmt):
    rows, k = 384, 288
    w = _gen(3, fmt, (rows, k), 0.02)
    w[5, :32] = 0.0
    m = E.QMatrix.from_f32(w.cuda(), fmt)
    aos = orc.quantize(fmt, w.numpy())
    q_ref, d_ref = orc.arena_pack(fmt, aos, rows, k)
    assert np.array_equal(m.q.cpu().numpy(), q_ref)
    assert np.array_equal(m.d.cpu().numpy(), d_ref)
    m2 = E.QMatrix.from_aos(torch.from_numpy(aos).cuda(), fmt, rows, k)
    assert np.array_equal(m2.q.cpu().numpy(), q_ref)
    assert np.array_equal(m2.d.cpu().numpy(), d_ref)


def test_gate_up_interleave(E, orc):
    Ex, I, L = 2, 128, 64
    g = _gen(4, 1, (Ex, I, L), 0.02)
    u = _gen(4, 2, (Ex, I, L), 0.02)
    ly = E.QMatrix(8, Ex * 2 * I, L)
    from quantized_latent_moe_b200.elq import _lib, _ptr, _stream
    assert _lib().elq_quantize_gate_up(8, _ptr(g.cuda()), _ptr(u.cuda()), Ex, I, L, _ptr(ly.q), _ptr(ly.d),
                                       _stream()) == 0
    rows = []
    for e in range(Ex):
        for j in range(I // 64):
            rows.append(g[e, 64 * j:64 * j + 64])
            rows.append(u[e, 64 * j:64 * j + 64])
    ref_rows = torch.cat(rows).numpy()
    q_ref, d_ref = orc.arena_pack(8, orc.quantize(8, ref_rows), Ex * 2 * I, L)
    assert np.array_equal(ly.q.cpu().numpy(), q_ref)
    assert np.array_equal(ly.d.cpu().numpy(), d_ref)


@pytest.mark.parametrize("fmt", [8, 2])
@pytest.mark.parametrize("N,K,T", [(128, 128, 1), (256, 384, 3), (1792, 4096, 1), (384, 1280, 6),
                                   (512, 512, 33), (128, 2048, 32), (4096, 1792, 2), (256, 640, 70)])
def test_latent_proj_exact(E, orc, fmt, N, K, T):
    W = _gen(5, N + K, (N, K), 0.02)
    X = _gen(6, T, (T, K))
    m = E.QMatrix.from_f32(W.cuda(), fmt)
    xq = E.quantize_q8_1(X.cuda())
    y = E.latent_proj(m, xq, T).cpu().numpy()
    ref = orc.qmatmul(fmt, orc.quantize(fmt, W.numpy()), N, K, orc.quantize(orc.Q8_1, X.numpy()), T)
    assert np.array_equal(y, ref)


@pytest.mark.parametrize("T,L,E_,k,bias", [(1, 1792, 128, 8, True), (6, 1280, 128, 8, False),
                                            (37, 256, 8, 2, False), (5, 64, 33, 32, True),
                                            (300, 256, 128, 8, True), (2000, 64, 33, 32, True),
                                            (2048, 1792, 128, 8, True)])
def test_router_exact(E, orc, T, L, E_, k, bias):
    z = _gen(7, T, (T, L), 1.3)
    W = _gen(7, 100 + L, (E_, L), 0.02)
    b = _gen(7, 200, (E_,)) if bias else None
    idx, w, lg = E.router_topk(z.cuda(), W.cuda(), None if b is None else b.cuda(), k)
    ridx, rw, rlg = orc.router_topk(z.numpy(), W.numpy(), None if b is None else b.numpy(), k)
    assert np.array_equal(lg.cpu().numpy(), rlg)
    assert np.array_equal(idx.cpu().numpy(), ridx)
    assert np.array_equal(w.cpu().numpy(), rw)


def test_router_ties(E, orc):
    z = torch.ones(2, 64)
    W = torch.zeros(16, 64)
    W[[3, 7, 9, 12]] = 0.25
    idx, w, _ = E.router_topk(z.cuda(), W.cuda(), None, 6)
    ridx, rw, _ = orc.router_topk(z.numpy(), W.numpy(), None, 6)
    assert np.array_equal(idx.cpu().numpy(), ridx)
    assert list(ridx[0][:4]) == [3, 7, 9, 12] and list(ridx[0][4:]) == [0, 1]
    assert np.array_equal(w.cpu().numpy(), rw)


@pytest.mark.parametrize("T,k,E_", [(1, 8, 128), (6, 8, 128), (2048, 8, 128), (37, 2, 5), (1, 1, 1)])
def test_bucket_exact(E, orc, T, k, E_):
    r = np.random.default_rng(T + E_)
    if E_ >= 64:   # skewed, as the routed workloads are
        p = np.exp(-np.arange(E_) / 20.0)
        p /= p.sum()
        idx = np.stack([r.choice(E_, k, replace=False, p=p) for _ in range(T)]).astype(np.int32)
    else:
        idx = np.stack([r.choice(E_, k, replace=False) for _ in range(T)]).astype(np.int32)
    out = E.route_bucket(torch.from_numpy(idx).cuda(), E_)
    ref = orc.bucket(idx, E_)
    for a, b in zip(out, ref):
        assert np.array_equal(a.cpu().numpy(), b)


def _check_intermediates(E, ly, T, tr):
    """Every intermediate of the last layer call against the oracle's trace."""
    v = lambda n: E.workspace_view(ly, T, n).cpu().numpy()
    assert np.array_equal(v("z").reshape(T, -1), tr["z"])
    assert np.array_equal(v("zq").reshape(T, -1), tr["zq"])
    assert np.array_equal(v("logits").reshape(T, -1), tr["logits"])
    assert np.array_equal(v("idx").reshape(T, -1), tr["idx"])
    assert np.array_equal(v("weights").reshape(T, -1), tr["w"])
    assert np.array_equal(v("counts"), tr["counts"])
    assert np.array_equal(v("offsets"), tr["offsets"])
    assert np.array_equal(v("perm"), tr["perm"])
    assert np.array_equal(v("pos"), tr["pos"])
    # hq and o are stored by pair position on the GPU, by pair id in the trace
    # (the tensor-core path keeps them in padded per-expert slots instead)
    if ly.kernel_count(T) != 10:
        pos = tr["pos"]
        assert np.array_equal(v("hq").reshape(T * ly.k, -1)[pos], tr["hq"])
        assert np.array_equal(v("o").reshape(T * ly.k, -1)[pos], tr["o"])
    assert np.array_equal(v("y_lat").reshape(T, -1), tr["y_lat"])
    assert np.array_equal(v("ylq").reshape(T, -1), tr["ylq"])


@pytest.mark.parametrize("fused", [True, False])
@pytest.mark.parametrize("name", ["tiny", "decode", "verify"])
def test_layer_exact(E, orc, name, fused):
    """Every intermediate and the output, on the fused single-kernel path and
    on the separate-kernel sequence."""
    wl = synth.WORKLOADS[name]
    ly = gpu_layer(wl)
    if fused:
        ly.flags = E.LAYER_FUSED
    assert ly.kernel_count(wl.T) == (1 if fused else 5)
    x = synth.make_x(wl)
    y = E.moe_layer(ly, x.cuda()).cpu().numpy()
    assert E.workspace_status(ly.workspace(wl.T)) == 0
    ol = oracle_layer(orc, wl, experts=[])
    tr = oracle_forward(orc, ol, wl, x.float().numpy(), trace=True)
    ref = tr["y"]
    assert max_abs_rel(y, ref) <= TOL
    _check_intermediates(E, ly, wl.T, tr)
    assert np.array_equal(y, ref)


@pytest.mark.parametrize("name,T", [("tiny", 9), ("tiny", 15), ("tiny", 16), ("tiny", 33), ("verify", 12),
                                    ("verify", 24)])
def test_layer_exact_larger_T(E, orc, name, T):
    """Above 8 tokens the activation quantiser runs as its own kernel; from 16
    tokens Q8_0 layers take the tensor-core path (ten kernels), Q4_0 layers
    stay on the GEMV path."""
    wl = synth.WORKLOADS[name]
    ly = gpu_layer(wl)
    x = synth.make_x(wl, T=T)
    y = E.moe_layer(ly, x.cuda()).cpu().numpy()
    assert ly.kernel_count(T) == (10 if (wl.fmt == "q8_0" and T >= 16) else 6)
    ol = oracle_layer(orc, wl, experts=[])
    tr = oracle_forward(orc, ol, wl, x.float().numpy(), trace=True)
    _check_intermediates(E, ly, T, tr)
    xq = E.workspace_view(ly, T, "xq").cpu().numpy().reshape(T, -1)
    assert np.array_equal(xq, tr["xq"])
    assert np.array_equal(y, tr["y"])


STREAMED = [synth.Workload("wide", 11, 200, 512, 256, 128, 8, 128, synth.Q8_0, synth.F32, "zipf"),
            synth.Workload("wide4", 12, 160, 512, 256, 128, 8, 128, synth.Q4_0, synth.F32, "normal"),
            synth.Workload("tiny1500", 0, 1500, 512, 256, 8, 2, 256, synth.Q8_0, synth.F32, "none")]


@pytest.mark.parametrize("wl", STREAMED, ids=[w.name for w in STREAMED])
def test_layer_streamed_router(E, orc, wl):
    """Token counts at which the router runs 16 experts per CTA and a CTA
    streams several 8-token blocks through its two-stage ring (top-k by the
    last CTA to finish each block, bucketing by the last block): every routing
    output, every intermediate and y equal the oracle's."""
    ly = gpu_layer(wl)
    x = synth.make_x(wl)
    y = E.moe_layer(ly, x.cuda()).cpu().numpy()
    assert E.workspace_status(ly.workspace(wl.T)) == 0
    ol = oracle_layer(orc, wl)
    tr = ol.forward(x.float().numpy(), trace=True)
    _check_intermediates(E, ly, wl.T, tr)
    assert np.array_equal(y, tr["y"])
    y2 = E.moe_layer(ly, x.cuda()).cpu().numpy()        # the counters reset themselves
    assert np.array_equal(y2, y)


def test_layer_repeat_and_ragged_T(E, orc):
    """Same bits on repeated calls (counters self-reset) and for ragged T."""
    wl = synth.WORKLOADS["tiny"]
    ly = gpu_layer(wl)
    ol = oracle_layer(orc, wl)
    for T in (1, 3, 8, 9, 33, 4, 4, 40):
        x = synth.normal(wl.seed, 77 + T, (T, wl.H))
        y = E.moe_layer(ly, x.cuda()).cpu().numpy()
        ref = ol.forward(x.numpy())
        assert np.array_equal(y, ref), T


def test_experts_grouped_exact(E, orc):
    wl = synth.WORKLOADS["verify"]
    ly = gpu_layer(wl)
    ol = oracle_layer(orc, wl, experts=[])
    x = synth.make_x(wl).float().numpy()
    tr = oracle_forward(orc, ol, wl, x, trace=True)
    zq = torch.from_numpy(tr["zq"]).cuda()
    idx = torch.from_numpy(tr["idx"]).cuda()
    w = torch.from_numpy(tr["w"]).cuda()
    y_lat = E.moe_experts_grouped(ly, zq, idx, w).cpu().numpy()
    assert np.array_equal(y_lat, tr["y_lat"])


def test_router_nan_inputs_give_valid_ids(E, orc):
    """R18 on the GPU: NaN latent rows and a NaN bias route exactly as the
    oracle's (NaN ranks as -inf), so no invalid expert id reaches the
    bucketing or the expert kernels."""
    T, L, E_, k = 5, 1792, 128, 8
    z = _gen(9, 600, (T, L))
    z[1, 100] = float("nan")
    w = _gen(9, 601, (E_, L), 0.02)
    b = _gen(9, 602, E_)
    ref_idx0, _, _ = orc.router_topk(z[:1].numpy(), w.numpy(), b.numpy(), k)
    b[int(ref_idx0[0, 0])] = float("nan")
    idx, wts, lg = E.router_topk(z.cuda(), w.cuda(), b.cuda(), k)
    ridx, rw, rlg = orc.router_topk(z.numpy(), w.numpy(), b.numpy(), k)
    assert np.array_equal(idx.cpu().numpy(), ridx)
    assert np.array_equal(wts.cpu().numpy(), rw, equal_nan=True)
    assert np.array_equal(lg.cpu().numpy(), rlg, equal_nan=True)
    assert ridx[1].tolist() == list(range(k)) and int(ref_idx0[0, 0]) not in ridx[0].tolist()


def test_layer_with_a_nan_token(E, orc):
    """A NaN token does not fault the layer; the other tokens' outputs are
    exactly the oracle's."""
    wl = synth.WORKLOADS["tiny"]
    ly = gpu_layer(wl)
    ol = oracle_layer(orc, wl)
    for T in (3, 12):
        x = synth.normal(wl.seed, 610 + T, (T, wl.H))
        x[1, 3] = float("nan")
        y = E.moe_layer(ly, x.cuda()).cpu().numpy()
        assert E.workspace_status(ly.workspace(T)) == 0
        ref = ol.forward(x.numpy())
        keep = [t for t in range(T) if t != 1]
        assert np.array_equal(y[keep], ref[keep])
