"""Pins of the oracle's Q5_1 / Q4_K / Q5_K expert formats (readings R22-R24).

The decoding is checked against hand-derived worked blocks (the 6-bit scale
packing included, tests/golden/kquant_blocks.json); the block dot against
brute-force integer sums of the decoded codes and the quantised activation
sum; the row dot against fp64 arithmetic on the dequantised operands; a layer
with these experts stage by stage.
"""
import json
import os
import struct

import numpy as np
import pytest

from quantized_latent_moe_b200 import synth

GOLD = os.path.join(os.path.dirname(__file__), "golden")
EPS32 = 2.0 ** -24
FMTS = {"q5_1": 7, "q3_k": 11, "q4_k": 12, "q5_k": 13}


def _fixture():
    with open(os.path.join(GOLD, "kquant_blocks.json")) as f:
        return json.load(f)


def _kq_block(fx, q5):
    b = bytearray(struct.pack("<HH", fx["kq_d_bits"], fx["kq_dmin_bits"]))
    b += bytes(fx["kq_scales_bytes"])
    if q5:
        b += bytes(range(32))                          # qh byte l = l
    for p in range(4):
        for l in range(32):
            b.append((l & 15) | ((15 - (l & 15)) << 4))
    return np.frombuffer(bytes(b), np.uint8)


def _kq_expected(fx, q5):
    vals = []
    for j in range(8):
        for l in range(32):
            q = (l & 15) if j % 2 == 0 else 15 - (l & 15)
            if q5:
                q += 16 * ((l >> j) & 1)
            vals.append(fx["kq_d"] * fx["kq_scale"][j] * q - fx["kq_dmin"] * fx["kq_min"][j])
    return np.array(vals)


def _q51_block(fx):
    b = struct.pack("<HHI", fx["q51_d_bits"], fx["q51_m_bits"], fx["q51_qh"])
    b += bytes(j | ((15 - j) << 4) for j in range(16))
    return np.frombuffer(b, np.uint8)


def _q51_expected(fx):
    qh = fx["q51_qh"]
    out = []
    for i in range(32):
        lo = i if i < 16 else 15 - (i - 16)
        out.append(fx["q51_d"] * (lo + 16 * ((qh >> i) & 1)) + fx["q51_m"])
    return np.array(out)


def _q3k_block(fx):
    b = bytearray(range(32))                                       # hmask[l] = l
    b += bytes(((3 * l + n) & 255) for n in range(2) for l in range(32))
    b += bytes(fx["q3k_scales_bytes"])
    b += struct.pack("<H", fx["q3k_d_bits"])
    return np.frombuffer(bytes(b), np.uint8)


def test_q3_k_worked_block(orc):
    fx = _fixture()
    blk = _q3k_block(fx)
    assert blk.size == 110
    vals = orc.dequantize_ext(orc.Q3_K, blk, 1, 256)[0]
    for i, v in fx["q3k_spot"].items():
        assert vals[int(i)] == v, i
    # every value is 0.5 * scale(i / 16) * q with q in -4 .. 3 (the scale table by hand)
    sc = np.repeat(np.array(fx["q3k_scale"], np.float64), 16)
    q = vals / (0.5 * sc)
    assert np.all(q == np.rint(q)) and q.min() >= -4 and q.max() <= 3


def test_row_bytes_are_gguf_sizes(orc):
    assert orc.row_bytes(orc.Q5_1, 32) == 24
    assert orc.row_bytes(orc.Q4_K, 256) == 144
    assert orc.row_bytes(orc.Q5_K, 256) == 176
    assert orc.row_bytes(orc.Q4_K, 1792) == 7 * 144
    assert orc.row_bytes(orc.Q3_K, 256) == 110


def test_worked_blocks_decode(orc):
    fx = _fixture()
    assert np.array_equal(orc.dequantize_ext(orc.Q4_K, _kq_block(fx, False), 1, 256)[0], _kq_expected(fx, False))
    assert np.array_equal(orc.dequantize_ext(orc.Q5_K, _kq_block(fx, True), 1, 256)[0], _kq_expected(fx, True))
    assert np.array_equal(orc.dequantize_ext(orc.Q5_1, _q51_block(fx), 1, 32)[0], _q51_expected(fx))


def _q81(orc, r, n):
    return orc.quantize(orc.Q8_1, (r.standard_normal(n) * 0.7 + 0.3).astype(np.float32))


def _codes(name, row, K):
    """Independent parse of a row's codes (numpy, from the GGUF layouts)."""
    row = np.asarray(row, np.uint8)
    if name == "q5_1":
        b = row.reshape(K // 32, 24)
        qh = b[:, 4:8].copy().view(np.uint32).reshape(-1).astype(np.int64)
        lo = np.concatenate([b[:, 8:] & 15, b[:, 8:] >> 4], axis=1).astype(np.int64)
        bits = (qh[:, None] >> np.arange(32)[None, :]) & 1
        return (lo + 16 * bits).reshape(-1)
    if name == "q3_k":
        b = row.reshape(K // 256, 110).astype(np.int64)
        i = np.arange(256)
        n, j, l = i // 128, (i % 128) // 32, i % 32
        low = (b[:, 32 + 32 * n + l] >> (2 * j)) & 3
        high = (b[:, l] >> (4 * n + j)) & 1
        return (low - 4 * (1 - high)).reshape(-1)
    bb = 176 if name == "q5_k" else 144
    b = row.reshape(K // 256, bb)
    qs = b[:, bb - 128:].reshape(-1, 4, 32).astype(np.int64)
    q = np.stack([qs & 15, qs >> 4], axis=2).reshape(-1, 8, 32)           # [super][sub-block j][l]
    if name == "q5_k":
        qh = b[:, 16:48].astype(np.int64)                                   # [super][l]
        q = q + 16 * ((qh[:, None, :] >> np.arange(8)[None, :, None]) & 1)
    return q.reshape(-1)


@pytest.mark.parametrize("name", ["q5_1", "q3_k", "q4_k", "q5_k"])
def test_block_sums_brute_force(orc, name):
    """isum and sumq are the exact integer sums of the codes with the
    activation codes (the min term's sum is the quantised one, not s / d)."""
    fmt = FMTS[name]
    fx = _fixture()
    r = np.random.default_rng(fmt)
    K = 256
    rows = synth.ext_blocks(name, 3, fmt, 4, K).numpy()
    for n in range(4):
        qw_all = _codes(name, rows[n], K)
        lo, hi = {"q3_k": (-4, 3), "q4_k": (0, 15)}.get(name, (0, 31))
        assert qw_all.min() >= lo and qw_all.max() <= hi
        a = _q81(orc, r, K)
        for kb in range(K // 32):
            isum, sumq, sd, sm = orc.block_ext(fmt, rows[n], kb, a[kb * 36:(kb + 1) * 36])
            qa = a[kb * 36 + 4:(kb + 1) * 36].view(np.int8).astype(np.int64)
            qw = qw_all[kb * 32:(kb + 1) * 32]
            if name == "q3_k":
                # the two 16-value halves' sums (no min term)
                assert isum == int((qw[:16] * qa[:16]).sum())
                assert sumq == int((qw[16:] * qa[16:]).sum())
                continue
            assert sumq == int(qa.sum())
            assert isum == int((qw * qa).sum())
    # the worked K block against an activation block of ones: sums per sub-block by hand
    a = orc.quantize(orc.Q8_1, np.full(256, 1.0, np.float32))       # every code 127
    kq = _kq_block(fx, False)
    for j in range(8):
        isum, sumq, _, _ = orc.block_ext(orc.Q4_K, kq, j, a[j * 36:(j + 1) * 36])
        assert sumq == 32 * 127
        assert isum == 127 * (sum(range(16)) * 2)          # q = l & 15 or 15 - (l & 15), 32 values


@pytest.mark.parametrize("name,N,K,T", [("q5_1", 3, 64, 1), ("q5_1", 5, 512, 2), ("q4_k", 4, 256, 1),
                                        ("q4_k", 3, 1792, 2), ("q5_k", 4, 512, 3), ("q3_k", 4, 256, 1),
                                        ("q3_k", 3, 1792, 2)])
def test_qmatmul_ext_vs_fp64(orc, name, N, K, T):
    fmt = FMTS[name]
    r = np.random.default_rng(N * K + T)
    W = synth.ext_blocks(name, 5, fmt, N, K).numpy()
    X = r.standard_normal((T, K)).astype(np.float32)
    Xq = orc.quantize(orc.Q8_1, X)
    Y = orc.qmatmul_ext(fmt, W, N, K, Xq, T)
    Wd = orc.dequantize_ext(fmt, W, N, K)
    Xd = orc.dequantize(orc.Q8_1, Xq, T * K).reshape(T, K)
    ref = Xd @ Wd.T
    gamma = (4 * (K // 32) + 8) * EPS32
    assert np.all(np.abs(Y - ref) <= gamma * (np.abs(Xd) @ np.abs(Wd).T) + 1e-30)


@pytest.mark.parametrize("name", ["q5_1", "q3_k", "q4_k", "q5_k"])
def test_ext_layer_stages_vs_fp64(orc, name):
    wl = synth.Workload("ext_tiny", 12, 3, 512, 256, 8, 2, 256, synth.Q8_0, synth.F32, "normal", ex_fmt=name)
    fmt = FMTS[name]
    dw = synth.dense_weights(wl)
    w = {k: (None if v is None else v.numpy()) for k, v in dw.items()}
    blocks = [synth.expert_blocks(wl, e) for e in range(wl.E)]
    w.update(gate=[b[0].numpy() for b in blocks], up=[b[1].numpy() for b in blocks],
             down=[b[2].numpy() for b in blocks])
    ly = orc.Layer(wl.H, wl.L, wl.E, wl.k, wl.I, orc.Q8_0, fmt, w)
    x = synth.make_x(wl).numpy()
    tr = ly.forward(x, trace=True)
    T, L, k, I = wl.T, wl.L, wl.k, wl.I
    zd = orc.dequantize(orc.Q8_1, tr["zq"], T * L).reshape(T, L)

    def check(got, A, B):
        ref = A @ B.T
        bound = (4 * (B.shape[1] // 32) + 8) * EPS32 * (np.abs(A) @ np.abs(B).T) + 1e-30
        assert np.all(np.abs(got - ref) <= bound)

    for p in range(T * k):
        t, e = p // k, int(tr["idx"].reshape(-1)[p])
        check(tr["g"][p:p + 1], zd[t:t + 1], orc.dequantize_ext(fmt, w["gate"][e], I, L))
        check(tr["u"][p:p + 1], zd[t:t + 1], orc.dequantize_ext(fmt, w["up"][e], I, L))
        hd = orc.dequantize(orc.Q8_1, tr["hq"][p], I)[None, :]
        check(tr["o"][p:p + 1], hd, orc.dequantize_ext(fmt, w["down"][e], L, I))
    assert np.all(np.isfinite(tr["y"]))
