"""Pins of the oracle's NVFP4 expert format (readings R19-R21).

The element conversions are checked against torch's float8_e4m3fn type and
against brute-force nearest search on the E2M1 grid; the block layout against
a hand-derived worked block under tests/golden/; the quantiser against the
format's error bound; the dot and the layer against fp64 arithmetic on the
dequantised operands.
"""
import json
import os

import numpy as np
import pytest
import torch

from quantized_latent_moe_b200 import synth

GOLD = os.path.join(os.path.dirname(__file__), "golden")
EPS32 = 2.0 ** -24
GRID = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])


def _torch_e4m3(v):
    return int(torch.tensor([v], dtype=torch.float32).to(torch.float8_e4m3fn).view(torch.uint8)[0])


def _e4m3_values():
    b = torch.arange(0, 127, dtype=torch.uint8)
    return b.view(torch.float8_e4m3fn).float().numpy().astype(np.float64)


def _parse(blocks, nblk):
    """Independent parse: (scale bytes [nblk,2], signed E2M1 values [nblk,32])."""
    raw = np.asarray(blocks, np.uint8).reshape(nblk, 18)
    codes = np.empty((nblk, 32), np.int64)
    codes[:, 0::2] = raw[:, 2:] & 15
    codes[:, 1::2] = raw[:, 2:] >> 4
    val = GRID[codes & 7] * np.where(codes & 8, -1.0, 1.0)
    return raw[:, :2], val


def _dec_scales(sbytes):
    t = torch.from_numpy(np.ascontiguousarray(sbytes, np.uint8).reshape(-1))
    return t.view(torch.float8_e4m3fn).float().numpy().astype(np.float64).reshape(sbytes.shape)


# --------------------------------------------------------------------------
# element formats

def test_e4m3_decode_matches_torch(orc):
    for b in range(256):
        ref = float(torch.tensor([b], dtype=torch.uint8).view(torch.float8_e4m3fn).float()[0])
        got = orc.e4m3_to_f32(b & 0x7F)        # the oracle's scales carry no sign
        ref = abs(ref)
        assert (np.isnan(got) and np.isnan(ref)) or got == ref, b


def test_e4m3_encode_matches_torch_round_to_nearest_even(orc):
    vals = _e4m3_values()                      # 0 .. 448, increasing
    xs = set()
    for a, b in zip(vals[:-1], vals[1:]):
        m = np.float32((a + b) / 2)            # exact midpoint (representable)
        for v in (np.float32(a), np.float32(b), m, np.nextafter(m, np.float32(0)),
                  np.nextafter(m, np.float32(1e9))):
            xs.add(float(v))
    r = np.random.default_rng(0)
    xs.update(float(v) for v in np.exp(r.uniform(np.log(1e-4), np.log(448), 3000)).astype(np.float32))
    for v in sorted(xs):
        if v <= 0.0 or v > 448.0:
            continue
        assert orc.f32_to_e4m3(v) == _torch_e4m3(v), v


def test_e4m3_encode_saturates_and_zeroes(orc):
    for v in (448.0, 449.0, 463.99, 464.0, 500.0, 1e30, float("inf")):
        assert orc.f32_to_e4m3(v) == 0x7E
    for v in (0.0, -0.0, -1.0, float("nan"), 2.0 ** -11, 1e-30):
        assert orc.f32_to_e4m3(v) == 0
    assert orc.f32_to_e4m3(2.0 ** -10 * 1.0001) == 1     # above half the smallest subnormal
    assert orc.f32_to_e4m3(2.0 ** -9) == 1
    assert orc.f32_to_e4m3(2.0 ** -6) == 0x08             # smallest normal


def test_e2m1_brute_force_nearest_even(orc):
    xs = [0.0]
    for a, b in zip(GRID[:-1], GRID[1:]):
        m = (a + b) / 2
        xs += [a, b, m, float(np.nextafter(np.float32(m), np.float32(0))),
               float(np.nextafter(np.float32(m), np.float32(9)))]
    xs += list(np.linspace(0, 9, 901)) + [6.0001, 7.0, 100.0, 1e30]
    for v in xs:
        for s in (1.0, -1.0):
            x = np.float32(s * v)
            d = np.abs(GRID - abs(float(x)))
            best = np.flatnonzero(d == d.min())
            code = int(best[0]) if len(best) == 1 else int([c for c in best if c % 2 == 0][0])
            if abs(float(x)) > 6.0:
                code = 7                                   # saturation
            want = code | (8 if x < 0 else 0)
            assert orc.f32_to_e2m1(float(x)) == want, (float(x), orc.f32_to_e2m1(float(x)), want)
            assert abs(orc.e2m1_to_f32(want)) == GRID[code]


# --------------------------------------------------------------------------
# blocks

def test_nvfp4_worked_block(orc):
    with open(os.path.join(GOLD, "nvfp4_block.json")) as f:
        gold = json.load(f)
    x = np.array(gold["x"], np.float32)
    assert list(orc.quantize_nvfp4(x, 1.0)) == gold["g1_bytes"]
    assert list(orc.quantize_nvfp4(x, 2.0)) == gold["g2_bytes"]
    assert list(orc.quantize_nvfp4(np.zeros(32, np.float32), 1.0)) == [0] * 18


@pytest.mark.parametrize("sigma,gmode", [(1.0, "one"), (0.02, "global"), (1e-3, "one"),
                                         (1e-3, "pow2"), (40.0, "global"), (40.0, "one")])
def test_nvfp4_roundtrip_bound_and_scale(orc, sigma, gmode):
    r = np.random.default_rng(int(sigma * 1000) + len(gmode))
    x = (r.standard_normal(32 * 400) * sigma).astype(np.float32)
    x[r.integers(0, x.size, 40)] = 0.0
    weights = gmode == "global"
    g = {"one": 1.0, "pow2": 2.0 ** -6, "global": orc.nvfp4_global(x) if weights else 0}[gmode]
    if weights:
        assert g == np.float32(np.float32(np.abs(x).max()) / np.float32(2688.0))
    q = orc.quantize_nvfp4(x, g)
    sb, val = _parse(q, 400)
    ds = _dec_scales(sb)
    amax = np.abs(x.astype(np.float64)).reshape(-1, 16).max(axis=1).reshape(400, 2)
    target = amax / 6.0 / g
    normal = target >= 2.0 ** -6
    # the scale is E4M3 of amax / 6 / g: relative error at most 2^-4 in the normal range,
    # half the smallest subnormal step below it, 448 at the top
    top = np.minimum(target, 448.0)
    assert np.all(np.abs(ds - top)[normal] <= 2.0 ** -4 * top[normal] * (1 + 1e-6))
    assert np.all(np.abs(ds - target)[~normal] <= 2.0 ** -10 * (1 + 1e-6))
    # a value inside the grid's range (6 steps) is within one step of its
    # input (E2M1's widest half-gap is 1); one beyond it (the scale rounded
    # down, or saturated) gives 6 steps of its sign; a zero scale zeroes its
    # micro-block
    deq = orc.dequantize_nvfp4(q, x.size, g).reshape(400, 32)
    step = np.repeat(ds, 16, axis=1) * g
    xr = x.reshape(400, 32).astype(np.float64)
    inside = np.abs(xr) <= 6 * step * (1 + 1e-6)
    ok_in = np.abs(deq - xr) <= step * (1 + 1e-6) + 1e-30
    ok_out = deq == np.sign(xr) * 6 * step
    assert np.all(np.where(inside, ok_in, ok_out))
    assert np.all(deq[np.repeat(ds == 0, 16, axis=1)] == 0)
    # in the normal range nothing lies beyond the grid but by the scale's rounding
    assert np.all((inside | ~np.repeat(normal & (target <= 448.0), 16, axis=1))
                  | (np.abs(xr) <= 6 * step * (1 + 2.0 ** -4) * (1 + 1e-6)))
    # dequantize agrees with the independent parse
    assert np.array_equal(deq, val * np.repeat(ds, 16, axis=1) * np.float64(np.float32(g)))
    # the global scale uses the top of the E4M3 range without overflowing it
    if weights:
        assert sb.max() <= 0x7E and sb.max() >= 0x7C


# --------------------------------------------------------------------------
# dot

@pytest.mark.parametrize("N,K,T", [(3, 32, 1), (5, 256, 2), (4, 512, 3), (7, 1792, 1)])
def test_qmatmul_nvfp4_vs_fp64(orc, N, K, T):
    r = np.random.default_rng(N * K + T)
    W = (r.standard_normal((N, K)) * 0.02).astype(np.float32)
    X = r.standard_normal((T, K)).astype(np.float32)
    g = orc.nvfp4_global(W)
    Wq = orc.quantize_nvfp4(W, g)
    ga = 2.0 ** -5 if K % 64 else 0.75
    Xq = orc.quantize_nvfp4(X, ga)
    Y = orc.qmatmul_nvfp4(Wq, g, N, K, Xq, T, ga)
    Wd = orc.dequantize_nvfp4(Wq, N * K, g).reshape(N, K)
    Xd = orc.dequantize_nvfp4(Xq, T * K, ga).reshape(T, K)
    ref = Xd @ Wd.T
    gamma = (2 * (K // 16) + 10) * EPS32
    assert np.all(np.abs(Y - ref) <= gamma * (np.abs(Xd) @ np.abs(Wd).T) + 1e-30)
    # one micro-block with integer values is exact
    if K == 32:
        # every micro-block holds a 6: both scales are exactly 1
        w = np.array([1, -2, 3, 0.5, 6, 4, -1.5, 0] * 4, np.float32)
        a = np.array([2, 1, -1, 4, -6, 0.5, 1, 3] * 4, np.float32)
        Y1 = orc.qmatmul_nvfp4(orc.quantize_nvfp4(w, 1.0), 1.0, 1, 32, orc.quantize_nvfp4(a, 1.0), 1)
        assert Y1[0, 0] == float((w * a).sum())


# --------------------------------------------------------------------------
# layer with NVFP4 experts

def _nv_layer(orc, T=3):
    wl = synth.Workload("nv_tiny", 9, T, 512, 256, 8, 2, 256, synth.Q8_0, synth.F32, "normal",
                        ex_fmt=synth.NVFP4)
    w = synth.layer_weights(wl)
    wn = {k: (v.numpy() if isinstance(v, torch.Tensor) else v) for k, v in w.items()}
    for key in ("gate", "up", "down"):
        wn[key] = [a.numpy() for a in w[key]]
    ly = orc.Layer(wl.H, wl.L, wl.E, wl.k, wl.I, orc.Q8_0, orc.NVFP4, wn)
    return wl, ly, wn, synth.make_x(wl).float().numpy()


def test_nvfp4_layer_stages_vs_fp64(orc):
    wl, ly, wn, x = _nv_layer(orc)
    T, L, k, I = wl.T, wl.L, wl.k, wl.I
    tr = ly.forward(x, trace=True)

    def check(got, A, B):
        ref = A @ B.T
        bound = (2 * (B.shape[1] // 16) + 10) * EPS32 * (np.abs(A) @ np.abs(B).T) + 1e-30
        assert np.all(np.abs(got - ref) <= bound)

    # gate and up of an expert share one global scale, from both matrices
    for e in range(wl.E):
        gu = np.concatenate([wn["gate"][e].ravel(), wn["up"][e].ravel()])
        assert ly.gate_g[e] == np.float32(np.float32(np.abs(gu).max()) / np.float32(2688.0))
        assert ly.down_g[e] == np.float32(np.float32(np.abs(wn["down"][e]).max()) / np.float32(2688.0))
    gz, gh = synth.NVFP4_ACT_GSCALE, synth.NVFP4_ACT_GSCALE
    assert ly.act_gz == gz and ly.act_gh == gh
    assert np.array_equal(tr["zq"], orc.quantize_nvfp4(tr["z"], gz))
    zd = orc.dequantize_nvfp4(tr["zq"], T * L, gz).reshape(T, L)
    for p in range(T * k):
        t, e = p // k, int(tr["idx"].reshape(-1)[p])
        gd = orc.dequantize_nvfp4(ly.gate[e], I * L, ly.gate_g[e]).reshape(I, L)
        ud = orc.dequantize_nvfp4(ly.up[e], I * L, ly.gate_g[e]).reshape(I, L)
        check(tr["g"][p:p + 1], zd[t:t + 1], gd)
        check(tr["u"][p:p + 1], zd[t:t + 1], ud)
        g = tr["g"][p].astype(np.float64)
        h = g / (1.0 + np.exp(-g)) * tr["u"][p]
        hd = orc.dequantize_nvfp4(tr["hq"][p], I, gh)
        sb, _ = _parse(tr["hq"][p], I // 32)
        step = np.repeat(_dec_scales(sb), 16, axis=1).reshape(-1) * gh
        assert np.all(sb > 0x08)                  # normal-range scales: nothing flushed
        assert np.all(np.abs(hd - h) <= step * (1 + 1e-5) + 1e-4 * np.abs(h) + 1e-30)
        dd = orc.dequantize_nvfp4(ly.down[e], L * I, ly.down_g[e]).reshape(L, I)
        check(tr["o"][p:p + 1], hd[None, :], dd)
    # the rest of the layer (combine, U) is the Q8 path's, pinned elsewhere;
    # here: the output is close to the unquantised experts' output
    assert np.all(np.isfinite(tr["y"]))


def test_nvfp4_layer_close_to_q8_layer(orc):
    """NVFP4 experts move the layer output by far less than its own size."""
    wl, ly, wn, x = _nv_layer(orc)
    y_nv = ly.forward(x)
    ly8 = orc.Layer(wl.H, wl.L, wl.E, wl.k, wl.I, orc.Q8_0, orc.Q8_0, wn)
    y8 = ly8.forward(x)
    rel = np.linalg.norm(y_nv - y8) / np.linalg.norm(y8)
    assert 1e-4 < rel < 0.35, rel
