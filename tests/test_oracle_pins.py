"""Pins of the CPU oracle against what the formats and the mathematics fix.

None of these re-types the oracle's own formula as the only check: each
compares with an independent library routine (numpy's fp16 conversion and
fp64 arithmetic), a closed-form bound or invariant, a hand-derived worked
example under tests/golden/, or brute force on tiny inputs.
"""
import json
import math
import os

import numpy as np
import pytest

GOLD = os.path.join(os.path.dirname(__file__), "golden")
EPS32 = 2.0 ** -24          # unit roundoff of fp32


def _rng(seed):
    return np.random.default_rng(seed)


def _f16(bits):
    return np.array(bits, np.uint16).view(np.float16).astype(np.float64)


def parse_blocks(fmt, raw, nblk):
    """Independent parse of AoS blocks -> (d fp64 [nblk], q int [nblk,32])."""
    raw = np.asarray(raw, np.uint8).reshape(nblk, -1)
    d = raw[:, 0:2].copy().view(np.uint16).reshape(-1)
    if fmt == 8:
        q = raw[:, 2:34].view(np.int8).astype(np.int64)
        return _f16(d), q, None
    if fmt == 9:
        s = raw[:, 2:4].copy().view(np.uint16).reshape(-1)
        q = raw[:, 4:36].view(np.int8).astype(np.int64)
        return _f16(d), q, _f16(s)
    nib = raw[:, 2:18].astype(np.int64)
    q = np.concatenate([nib & 15, nib >> 4], axis=1)   # element j, j+16
    return _f16(d), q, None


# --------------------------------------------------------------------------
# number formats

def test_fp16_rne_matches_numpy(orc):
    r = _rng(0)
    vals = np.concatenate([
        r.standard_normal(4000).astype(np.float32),
        (r.standard_normal(2000) * 1e-5).astype(np.float32),   # fp16 subnormal range
        (r.standard_normal(2000) * 3e4).astype(np.float32),    # near overflow
        np.array([0.0, -0.0, 65504.0, 65519.99, 65520.0, 1e6, -1e6, 2.0 ** -24,
                  2.0 ** -25, 2.0 ** -25 * 1.0001, 3 * 2.0 ** -26, 2.0 ** -14,
                  2.0 ** -14 * (1 - 2 ** -12), 1e-30, np.inf, -np.inf], np.float32),
    ])
    # exact ties between adjacent fp16 values
    base = np.array([1.0, 1.0009765625, 2.0, 1000.0, 2.0 ** -20], np.float64)
    ulp = np.array([2 ** -10, 2 ** -10, 2 ** -9, 0.5, 2 ** -24])
    vals = np.concatenate([vals, (base + ulp / 2).astype(np.float32)])
    for v in vals:
        mine = orc.f32_to_f16_bits(float(v))
        with np.errstate(over="ignore"):
            ref = int(np.float32(v).astype(np.float16).view(np.uint16))
        assert mine == ref, (v, hex(mine), hex(ref))


def test_fp16_to_f32_matches_numpy(orc):
    for h in list(range(0, 0x7C01, 7)) + [0x0001, 0x03FF, 0x0400, 0x7BFF, 0x7C00, 0xFC00, 0x8001]:
        mine = orc.f16_bits_to_f32(h)
        ref = float(np.array(h, np.uint16).view(np.float16))
        assert mine == ref, hex(h)


def _ulp32(x):
    x = abs(x)
    if x < 2.0 ** -126:
        return 2.0 ** -149
    return 2.0 ** (math.floor(math.log2(x)) - 23)


def test_bf16_to_f32_matches_torch(orc):
    """Every bf16 bit pattern widens to the fp32 torch's bfloat16 conversion
    gives (NaNs: a NaN), plus values fixed by the format: 0x3F80 = 1.0,
    0xC000 = -2.0, 0x7F80 = +inf, 0x0001 = 2^-133 (the smallest subnormal)."""
    import torch
    bits = np.arange(65536, dtype=np.uint16)
    ref = torch.from_numpy(bits.astype(np.int16)).view(torch.bfloat16).float().numpy()
    got = np.array([orc.lib().orc_bf16_to_f32(int(b)) for b in bits], np.float32)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan].view(np.uint32), ref[~nan].view(np.uint32))
    f = orc.lib().orc_bf16_to_f32
    assert f(0x3F80) == 1.0 and f(0xC000) == -2.0 and f(0x7F80) == math.inf
    assert f(0x0001) == 2.0 ** -133


def test_expf_within_two_ulp_of_fp64(orc):
    r = _rng(1)
    xs = np.concatenate([np.linspace(-20, 20, 4001), r.uniform(-87, 88, 3000),
                         r.uniform(-103.9, -87.4, 500), [0.0, 1e-8, -1e-8, 0.5, -0.5]])
    for x in xs.astype(np.float32):
        got = orc.expf(float(x))
        ref = math.exp(float(x))
        assert abs(got - ref) <= 2 * _ulp32(ref), (x, got, ref)


def test_expf_special_values(orc):
    assert orc.expf(0.0) == 1.0
    assert orc.expf(100.0) == math.inf
    assert orc.expf(-200.0) == 0.0
    assert orc.expf(89.0) == math.inf
    assert 0.0 < orc.expf(-100.0) < 2.0 ** -126      # subnormal result
    assert orc.expf(float(np.float32(88.72))) < 3.5e38


def test_silu_matches_fp64(orc):
    for g in np.linspace(-30, 30, 1201).astype(np.float32):
        ref = float(g) / (1.0 + math.exp(-float(g)))
        got = orc.silu(float(g))
        assert abs(got - ref) <= 4 * _ulp32(ref) + 1e-45, (g, got, ref)


# --------------------------------------------------------------------------
# quantisers

def test_q8_1_worked_example(orc):
    ex = json.load(open(os.path.join(GOLD, "q8_1_ties.json")))
    out = orc.quantize(orc.Q8_1, np.array(ex["x"], np.float32))
    assert out.size == 36
    assert int(out[0]) | (int(out[1]) << 8) == ex["d_bits"]
    assert int(out[2]) | (int(out[3]) << 8) == ex["s_bits"]
    assert list(out[4:36].view(np.int8)) == ex["q"]


@pytest.mark.parametrize("fmt", [8, 9])
def test_q8_invariants(orc, fmt):
    r = _rng(2)
    nblk = 3000
    x = r.standard_normal((nblk, 32)).astype(np.float32) * r.uniform(1e-3, 1e3, (nblk, 1)).astype(np.float32)
    raw = orc.quantize(fmt, x.reshape(-1))
    d16, q, s16 = parse_blocks(fmt, raw, nblk)
    assert np.abs(q).max() <= 127
    amax = np.abs(x).max(axis=1)
    d32 = (amax / np.float32(127)).astype(np.float64)       # numpy fp32 divide, IEEE RN
    # the element of largest magnitude maps to +-127
    arg = np.abs(x).argmax(axis=1)
    assert np.all(np.abs(q[np.arange(nblk), arg]) == 127)
    # stored d is the fp16 rounding of amax/127
    assert np.all(d16 == np.float32(d32).astype(np.float16).astype(np.float64))
    # round trip against the fp16 scale: |x - d16 q| <= d/2 + 127 |d - d16| (+ rounding slack)
    err = np.abs(x.astype(np.float64) - d16[:, None] * q)
    bound = d32[:, None] * (0.5 + 4 * EPS32) + 127 * np.abs(d32 - d16)[:, None]
    assert np.all(err <= bound)
    # q is the nearest integer to x/d (fp32 quotient), halves away from zero
    quot = (x / np.float32(d32)[:, None].astype(np.float32)).astype(np.float64)
    nearest = np.sign(quot) * np.floor(np.abs(quot) + 0.5)
    assert np.array_equal(q, nearest.astype(np.int64))
    if fmt == 9:
        sq = q.sum(axis=1)
        # s = fp16(d * sum q): within one fp16 rounding (+ one fp32 rounding) of d*sum(q)
        exact = d32 * sq
        assert np.all(np.abs(s16 - exact) <= np.abs(exact) * (2.0 ** -11 + 2 * EPS32) + 2.0 ** -24)


def test_q8_special_blocks(orc):
    z = np.zeros(32, np.float32)
    for fmt in (8, 9):
        raw = orc.quantize(fmt, z)
        assert not raw.any()
        one = z.copy()
        one[5] = -3.0
        d, q, s = parse_blocks(fmt, orc.quantize(fmt, one), 1)
        assert q[0, 5] == -127 and np.count_nonzero(q) == 1
        assert d[0] == float(np.float16(np.float32(3.0) / np.float32(127)))
        if fmt == 9:
            assert s[0] == float(np.float16(np.float32(np.float32(3.0) / np.float32(127)) * np.float32(-127)))


def test_q4_0_invariants_and_nibble_order(orc):
    r = _rng(3)
    nblk = 3000
    x = r.standard_normal((nblk, 32)).astype(np.float32) * r.uniform(1e-3, 1e3, (nblk, 1)).astype(np.float32)
    raw = orc.quantize(orc.Q4_0, x.reshape(-1))
    assert raw.size == nblk * 18
    d16, q, _ = parse_blocks(2, raw, nblk)
    assert q.min() >= 0 and q.max() <= 15
    arg = np.abs(x).argmax(axis=1)
    m = x[np.arange(nblk), arg].astype(np.float64)
    assert np.all(q[np.arange(nblk), arg] == 0)          # the signed max maps to -8
    assert np.all(np.sign(d16) == -np.sign(m))
    assert np.all(d16 == np.float32(m / -8.0).astype(np.float16).astype(np.float64))
    d32 = np.abs(m) / 8.0
    err = np.abs(x.astype(np.float64) - d16[:, None] * (q - 8))
    bound = d32[:, None] * (1.0 + 8 * EPS32) + 16 * np.abs(np.abs(d16) - d32)[:, None]
    assert np.all(err <= bound)                          # the clamp side costs up to one step
    inside = np.abs(x.astype(np.float64) / d32[:, None]) <= 7.0
    assert np.all(err[inside] <= (d32[:, None] * (0.5 + 8 * EPS32) + 16 * np.abs(np.abs(d16) - d32)[:, None]).repeat(32, 1)[inside])
    # nibble order: element j -> low nibble of byte j, element j+16 -> high nibble
    for j in (0, 7, 15):
        e = np.zeros(32, np.float32)
        e[j] = 8.0
        e[j + 16] = -8.0      # q = 16 -> clamped to 15
        b = orc.quantize(orc.Q4_0, e)
        assert b[2 + j] == (0 | (15 << 4)) or b[2 + j] == (0 | (15 << 4))
        assert all(b[2 + i] == 0x88 for i in range(16) if i != j)
    # all zeros: m = +0, d = 0 / -8 = -0 (IEEE), every nibble 8
    assert list(orc.quantize(orc.Q4_0, np.zeros(32, np.float32))) == [0, 0x80] + [0x88] * 16


def test_dequantize_matches_parse(orc):
    r = _rng(4)
    x = r.standard_normal(32 * 50).astype(np.float32)
    for fmt in (2, 8, 9):
        raw = orc.quantize(fmt, x)
        d, q, _ = parse_blocks(fmt, raw, 50)
        ref = (d[:, None] * ((q - 8) if fmt == 2 else q)).reshape(-1)
        assert np.array_equal(orc.dequantize(fmt, raw, x.size), ref)


# --------------------------------------------------------------------------
# block dots

@pytest.mark.parametrize("wfmt", [8, 2])
def test_block_isum_brute_force_and_term(orc, wfmt):
    r = _rng(5)
    for _ in range(500):
        w = r.standard_normal(32).astype(np.float32) * 0.02
        a = r.standard_normal(32).astype(np.float32)
        wb = orc.quantize(wfmt, w)
        ab = orc.quantize(orc.Q8_1, a)
        dw, qw, _ = parse_blocks(wfmt, wb, 1)
        da, qa, _ = parse_blocks(9, ab, 1)
        qw = qw - 8 if wfmt == 2 else qw
        isum = int((qw[0] * qa[0]).sum())
        assert orc.block_isum(wfmt, wb, ab) == isum
        assert abs(isum) <= (32 * 127 * 127 if wfmt == 8 else 32 * 8 * 127)
        term = orc.block_term(wfmt, wb, ab)
        exact = float(dw[0] * da[0] * isum)          # fp64 dequantised dot, exact here
        assert abs(term - exact) <= 2 * EPS32 * abs(exact) + 1e-45


def test_q4_isum_uses_quantised_sum_not_s(orc):
    """R7: the offset term is -8 * sum(q8) of the quantised activations."""
    r = _rng(6)
    for _ in range(200):
        wb = orc.quantize(orc.Q4_0, r.standard_normal(32).astype(np.float32))
        ab = orc.quantize(orc.Q8_1, r.standard_normal(32).astype(np.float32) + 0.7)
        _, qw, _ = parse_blocks(2, wb, 1)
        _, qa, _ = parse_blocks(9, ab, 1)
        assert orc.block_isum(2, wb, ab) == int((qw[0] * qa[0]).sum() - 8 * qa[0].sum())


# --------------------------------------------------------------------------
# matmul, router, bucketing

@pytest.mark.parametrize("wfmt,N,K,T", [(8, 5, 32, 1), (8, 7, 96, 3), (8, 3, 512, 2),
                                        (2, 4, 288, 2), (2, 9, 256, 1)])
def test_qmatmul_vs_fp64_dequantised(orc, wfmt, N, K, T):
    r = _rng(7 + N + K)
    W = r.standard_normal((N, K)).astype(np.float32) * 0.02
    X = r.standard_normal((T, K)).astype(np.float32)
    Wq = orc.quantize(wfmt, W)
    Xq = orc.quantize(orc.Q8_1, X)
    Y = orc.qmatmul(wfmt, Wq, N, K, Xq, T)
    Wd = orc.dequantize(wfmt, Wq, N * K).reshape(N, K)
    Xd = orc.dequantize(orc.Q8_1, Xq, T * K).reshape(T, K)
    ref = Xd @ Wd.T
    absterm = np.abs(Xd) @ np.abs(Wd).T
    nb = K // 32
    gamma = (2 * nb + 8) * EPS32
    assert np.all(np.abs(Y - ref) <= gamma * absterm + 1e-30)
    # a transposed or mis-indexed operand is far outside this bound
    assert Y.shape == (T, N)


def test_router_invariants(orc):
    r = _rng(8)
    T, L, E, k = 5, 64, 16, 4
    z = r.standard_normal((T, L)).astype(np.float32)
    Wr = (r.standard_normal((E, L)) * 0.1).astype(np.float32)
    b = r.standard_normal(E).astype(np.float32)
    idx, w, lg = orc.router_topk(z, Wr, b, k)
    ref = z.astype(np.float64) @ Wr.astype(np.float64).T + b
    absd = np.abs(z.astype(np.float64)) @ np.abs(Wr.astype(np.float64)).T + np.abs(b)
    assert np.all(np.abs(lg - ref) <= (L // 32 + 7) * EPS32 * absd)
    for t in range(T):
        assert len(set(idx[t])) == k
        sel = lg[t, idx[t]]
        rest = np.delete(lg[t], idx[t])
        assert sel.min() >= rest.max()
        assert np.all(np.diff(sel) <= 0)
        assert list(idx[t]) == list(np.argsort(-ref[t], kind="stable")[:k])
        assert np.all(np.diff(w[t]) <= 0)
        assert abs(w[t].sum() - 1.0) <= 4 * k * EPS32
        e = np.exp(sel.astype(np.float64) - sel[0])
        assert np.allclose(w[t], e / e.sum(), rtol=8 * EPS32 * k, atol=0)


def test_router_ties_prefer_lower_id(orc):
    L, E, k = 32, 8, 3
    z = np.ones((1, L), np.float32)
    Wr = np.zeros((E, L), np.float32)
    Wr[[1, 4, 6]] = 0.5
    idx, w, _ = orc.router_topk(z, Wr, None, k)
    assert list(idx[0]) == [1, 4, 6]
    assert np.all(w[0] == np.float32(1.0 / 3.0))
    idx, _, _ = orc.router_topk(z, np.zeros((E, L), np.float32), None, 4)
    assert list(idx[0]) == [0, 1, 2, 3]


def test_bucket_brute_force(orc):
    r = _rng(9)
    for T, k, E in [(1, 8, 128), (6, 8, 128), (37, 2, 5), (4, 2, 8)]:
        idx = np.stack([r.choice(E, k, replace=False) for _ in range(T)]).astype(np.int32)
        counts, offsets, perm, pos = orc.bucket(idx, E)
        flat = idx.reshape(-1)
        assert np.array_equal(counts, np.bincount(flat, minlength=E))
        assert offsets[0] == 0 and np.array_equal(np.diff(offsets), counts)
        assert sorted(perm) == list(range(T * k))
        assert np.all(np.diff(flat[perm]) >= 0)
        for e in range(E):
            seg = perm[offsets[e]:offsets[e + 1]]
            assert np.all(flat[seg] == e) and np.all(np.diff(seg) > 0)
        assert np.array_equal(perm[pos], np.arange(T * k))


# --------------------------------------------------------------------------
# byte sizes printed on the pages, and the arena layout

def test_byte_sizes_from_pages(orc):
    g = json.load(open(os.path.join(GOLD, "byte_sizes.json")))
    lib = orc.lib()
    assert lib.orc_block_bytes(8) * (160 // 32) == g["row_160_q8_0_bytes"]
    assert lib.orc_block_bytes(2) * (160 // 32) == g["row_160_18byte_block_bytes"]
    blob = 3 * orc.quantize(8, np.zeros((2560, 640), np.float32)).size
    assert blob == g["expert_2560x640_q8_0_bytes"]
    assert (384 * blob) // (1 << 20) == g["ring_384_q8_0_mib_floor"]


def test_arena_pack_spot_positions(orc):
    r = _rng(10)
    n, K = 256, 96
    nb = K // 32
    aos = r.integers(0, 256, n * nb * 34).astype(np.uint8)
    q, d = orc.arena_pack(8, aos, n, K)
    blk = aos.reshape(n, nb, 34)
    # row 9 (tile 0, slice 0, r 9), block 2, code 17:
    #   0 + 0 + 2*1024 + (9//8)*256 + (17//16)*128 + (9%8)*16 + 1
    assert q[2 * 1024 + 256 + 128 + 16 + 1] == blk[9, 2, 2 + 17]
    # row 130 (tile 1, slice 0, r 2), block 0, code 0
    assert q[1 * nb * 4096 + 0 + 0 + 2 * 16] == blk[130, 0, 2]
    # row 200 (tile 1, slice 2, r 8), block 1, code 31
    assert q[1 * nb * 4096 + 2 * nb * 1024 + 1 * 1024 + 1 * 256 + 128 + 0 + 15] == blk[200, 1, 2 + 31]
    # scale of row 130, block 1
    sel = 1 * nb * 128 + 0 + 1 * 32 + 2
    assert bytes(d[2 * sel:2 * sel + 2]) == bytes(blk[130, 1, 0:2])
    assert np.array_equal(np.sort(q), np.sort(blk[:, :, 2:].reshape(-1)))
    aos4 = r.integers(0, 256, n * nb * 18).astype(np.uint8)
    q4, d4 = orc.arena_pack(2, aos4, n, K)
    b4 = aos4.reshape(n, nb, 18)
    # row 133 (tile 1, slice 0, r 5), block 2, nibble byte 7
    assert q4[1 * nb * 2048 + 0 + 2 * 512 + 5 * 16 + 7] == b4[133, 2, 2 + 7]
    # row 255 (tile 1, slice 3, r 31), block 0, byte 0
    assert q4[1 * nb * 2048 + 3 * nb * 512 + 0 + 31 * 16] == b4[255, 0, 2]


# ---- R18: NaN router logits rank as -infinity --------------------------------

def test_router_nan_logits_rank_last(orc):
    rng = np.random.default_rng(11)
    L, E, k = 64, 8, 3
    Wr = rng.normal(size=(E, L)).astype(np.float32)
    z = rng.normal(size=(2, L)).astype(np.float32)
    z[1, 7] = np.nan                                   # token 1: every logit NaN
    idx, w, logits = orc.router_topk(z, Wr, None, k)
    assert np.isnan(logits[1]).all()
    assert idx[1].tolist() == [0, 1, 2]                # all tie at -inf: lower ids first
    # a NaN bias removes that expert from the choice of a finite token
    ref_idx, _, _ = orc.router_topk(z[:1], Wr, None, k)
    bias = np.zeros(E, np.float32)
    bias[ref_idx[0, 0]] = np.nan
    idx2, w2, _ = orc.router_topk(z[:1], Wr, bias, k)
    assert ref_idx[0, 0] not in idx2[0].tolist()
    assert np.isfinite(w2).all() and abs(float(w2.sum()) - 1.0) < 1e-6
    assert idx2[0, :k - 1].tolist() == ref_idx[0, 1:].tolist()


# ---- the stack's RMS normalisation -------------------------------------------

def test_rmsnorm_constant_row_closed_form(orc):
    for c, H in ((3.0, 64), (0.5, 4096), (-2.0, 1792)):
        h = np.full((1, H), c, np.float32)
        ms = np.float32(c * c)                         # the sum of H equal squares is exact here
        r = np.sqrt(ms + np.float32(1e-6), dtype=np.float32)
        assert np.array_equal(orc.rmsnorm(h), np.full((1, H), np.float32(c) / r, np.float32))


def test_rmsnorm_single_spike(orc):
    H = 256
    h = np.zeros((1, H), np.float32)
    h[0, 77] = 16.0
    out = orc.rmsnorm(h)
    r = np.sqrt(np.float32(256.0 / H) + np.float32(1e-6), dtype=np.float32)
    assert out[0, 77] == np.float32(16.0) / r and np.count_nonzero(out) == 1


def test_rmsnorm_against_fp64(orc):
    rng = np.random.default_rng(5)
    h = (rng.normal(size=(6, 4096)) * np.array([[1e-3], [1.0], [7.0], [100.0], [0.3], [42.0]])).astype(np.float32)
    out = orc.rmsnorm(h).astype(np.float64)
    hd = h.astype(np.float64)
    ref = hd / np.sqrt((hd * hd).mean(axis=1, keepdims=True) + 1e-6)
    assert np.abs(out - ref).max() <= 4e-6 * np.abs(ref).max()
    # unit RMS afterwards where eps is negligible; 1/sqrt(2) where mean(h^2) == eps
    rms = np.sqrt((out * out).mean(axis=1))
    assert np.allclose(rms[1:], 1.0, rtol=1e-5)
    ms0 = (hd[0] * hd[0]).mean()
    assert abs(rms[0] - np.sqrt(ms0 / (ms0 + 1e-6))) < 1e-6
