"""Stage-by-stage pins of the oracle's layer on the tiny workload.

Each stage is recomputed in fp64 from the oracle's own quantised inputs to that
stage (numpy dequantisation and matmul, an independent library path); the
oracle's fp32 result must sit within the rounding bound of that fp64 value.
A dropped term, a wrong sign, a swapped gate/up, a transposed matrix or a wrong
token/expert index moves a stage far outside its bound.
"""
import math

import numpy as np
import pytest
import torch

from quantized_latent_moe_b200 import synth

EPS32 = 2.0 ** -24


def _deq(orc, fmt, raw, rows, cols):
    return orc.dequantize(fmt, raw, rows * cols).reshape(rows, cols)


def _oracle_layer(orc, wl, T=None):
    fmt = {"q8_0": orc.Q8_0, "q4_0": orc.Q4_0}[wl.fmt]
    w = synth.layer_weights(wl)
    wn = {k: (v.numpy() if isinstance(v, torch.Tensor) else v) for k, v in w.items()}
    wn["gate"] = [g.numpy() for g in w["gate"]]
    wn["up"] = [g.numpy() for g in w["up"]]
    wn["down"] = [g.numpy() for g in w["down"]]
    ly = orc.Layer(wl.H, wl.L, wl.E, wl.k, wl.I, fmt, fmt, wn)
    x = synth.make_x(wl, T=T).float().numpy()
    return ly, wn, x, fmt


@pytest.mark.parametrize("name", ["tiny"])
def test_layer_stages_vs_fp64(orc, name):
    wl = synth.WORKLOADS[name]
    ly, wn, x, fmt = _oracle_layer(orc, wl)
    T, H, L, E, k, I = wl.T, wl.H, wl.L, wl.E, wl.k, wl.I
    tr = ly.forward(x, trace=True)

    def check(got, A, B):       # got ~ A @ B.T in fp64, bound by |A| @ |B|.T
        ref = A @ B.T
        bound = (2 * (B.shape[1] // 32) + 8) * EPS32 * (np.abs(A) @ np.abs(B).T) + 1e-30
        assert np.all(np.abs(got - ref) <= bound)

    # a1/a2: xq is Q8_1 of x; z = D . xq
    xq = tr["xq"]
    assert np.array_equal(xq, orc.quantize(orc.Q8_1, x))
    check(tr["z"], _deq(orc, orc.Q8_1, xq, T, H), _deq(orc, fmt, ly.D, L, H))
    # a3: router on fp32 z
    lg = tr["z"].astype(np.float64) @ wn["router_w"].astype(np.float64).T
    assert np.all(np.abs(tr["logits"] - lg) <= 16 * EPS32 * (np.abs(tr["z"]) @ np.abs(wn["router_w"]).T))
    for t in range(T):
        assert list(tr["idx"][t]) == list(np.argsort(-lg[t], kind="stable")[:k])
    # a4, a5
    assert np.array_equal(tr["zq"], orc.quantize(orc.Q8_1, tr["z"]))
    zd = _deq(orc, orc.Q8_1, tr["zq"], T, L)
    # a6: gate / up per pair from the matching expert's own matrices
    for p in range(T * k):
        t, e = divmod(p, k)[0], tr["idx"].reshape(-1)[p]
        check(tr["g"][p:p + 1], zd[t:t + 1], _deq(orc, fmt, ly.gate[e], I, L))
        check(tr["u"][p:p + 1], zd[t:t + 1], _deq(orc, fmt, ly.up[e], I, L))
        # a7: h = silu(g) * u, then Q8_1
        g = tr["g"][p].astype(np.float64)
        h = g / (1.0 + np.exp(-g)) * tr["u"][p]
        hq = tr["hq"][p]
        hd = _deq(orc, orc.Q8_1, hq, 1, I)[0]
        d = orc.dequantize(orc.Q8_1, hq, I).reshape(-1, 32)
        scale = np.abs(h.reshape(-1, 32)).max(axis=1) / 127.0
        assert np.all(np.abs(hd - h).reshape(-1, 32) <= scale[:, None] * 0.5 * (1 + 1e-3) + 127 * scale[:, None] * 2.0 ** -11 + 1e-30)
        # a8: down
        check(tr["o"][p:p + 1], hd[None, :], _deq(orc, fmt, ly.down[e], L, I))
    # a9: weighted combine in rank order
    o = tr["o"].reshape(T, k, L).astype(np.float64)
    ref = (tr["w"][:, :, None] * o).sum(axis=1)
    assert np.all(np.abs(tr["y_lat"] - ref) <= 2 * k * EPS32 * (np.abs(tr["w"][:, :, None] * o)).sum(axis=1) + 1e-30)
    assert np.array_equal(tr["ylq"], orc.quantize(orc.Q8_1, tr["y_lat"]))
    # a10
    check(tr["y"], _deq(orc, orc.Q8_1, tr["ylq"], T, L), _deq(orc, fmt, ly.U, H, L))


def test_layer_close_to_unquantised_fp64(orc):
    """The quantised layer approximates the same layer in fp64 without any
    quantisation (quantisation noise only, a few percent)."""
    wl = synth.WORKLOADS["tiny"]
    ly, wn, x, fmt = _oracle_layer(orc, wl)
    y = ly.forward(x)
    X = x.astype(np.float64)
    z = X @ wn["D"].T
    lg = z @ wn["router_w"].T
    yl = np.zeros((wl.T, wl.L))
    for t in range(wl.T):
        sel = np.argsort(-lg[t], kind="stable")[:wl.k]
        e = np.exp(lg[t, sel] - lg[t, sel[0]])
        w = e / e.sum()
        for j, ex in enumerate(sel):
            g = wn["gate"][ex] @ z[t]
            u = wn["up"][ex] @ z[t]
            yl[t] += w[j] * (wn["down"][ex] @ (g / (1 + np.exp(-g)) * u))
    ref = yl @ wn["U"].T
    rel = np.abs(y - ref).max() / np.abs(ref).max()
    assert rel < 0.05, rel


def test_sampled_tokens_equal_full_batch(orc):
    """The layer is token-wise independent: a token computed alone gives the
    same bits as in the batch (the basis of sampled checks at full size)."""
    wl = synth.WORKLOADS["tiny"]
    ly, wn, x, fmt = _oracle_layer(orc, wl)
    y = ly.forward(x)
    for t in (0, 3):
        assert np.array_equal(ly.forward(x[t:t + 1])[0], y[t])


def test_missing_expert_is_refused(orc):
    wl = synth.WORKLOADS["tiny"]
    ly, wn, x, fmt = _oracle_layer(orc, wl)
    idx, _ = ly.route(x)
    e = int(idx[0, 0])
    ly.gate[e] = None
    with pytest.raises(ValueError):
        ly.forward(x)
