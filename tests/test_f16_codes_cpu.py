"""The arithmetic the fp16-operand tensor-core GEMMs rely on, checked on the
CPU: int8 codes are exact in fp16, and a 32-code block's sum of products,
accumulated in fp32 in any order and any grouping, is the exact integer sum
(every partial sum is an integer below 2^24), so the fp32 accumulator equals
the int32 one the int8 GEMMs convert."""
import numpy as np


def test_int8_codes_exact_in_fp16():
    q = np.arange(-128, 128, dtype=np.int64)
    assert np.array_equal(q.astype(np.float16).astype(np.int64), q)


def _fp32_sum(vals, order, group):
    """Sum in fp32: products added in `order`, first within groups of `group`
    (as a K = 16 instruction might), then the group sums."""
    acc = np.float32(0.0)
    v = vals[order].astype(np.float32)
    for g0 in range(0, len(v), group):
        part = np.float32(0.0)
        for x in v[g0:g0 + group]:
            part = np.float32(part + x)
        acc = np.float32(acc + part)
    return acc


def test_block_sums_exact_in_fp32_any_order():
    rng = np.random.default_rng(5)
    cases = [rng.integers(-127, 128, (2, 32)) for _ in range(200)]
    cases += [np.full((2, 32), 127), np.stack([np.full(32, 127), np.full(32, -127)]),
              np.stack([np.r_[127, np.ones(31, int)], np.r_[127, -np.ones(31, int)]])]
    for a, b in cases:
        prods = (a.astype(np.int64) * b.astype(np.int64))
        exact = int(prods.sum())
        assert abs(exact) < 2 ** 24
        for group in (1, 4, 8, 16, 32):
            for _ in range(3):
                order = rng.permutation(32)
                assert int(_fp32_sum(prods, order, group)) == exact
    # the bound itself: the largest magnitude a block can reach
    assert 32 * 127 * 127 < 2 ** 24
