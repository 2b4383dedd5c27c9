"""The allocation-free projection entry point, elq_latent_proj_noalloc.

It serves callers that cannot allocate device memory (an engine plugin given
only input and output pointers, an engine that reserves all of HBM for its
resident weights up front): its scratch is a static device array of the
library.  This file runs last so that a failure here leaves every other test
already run; it also passes on its own in a fresh process.
"""
import numpy as np
import pytest
import torch

from quantized_latent_moe_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def E():
    from quantized_latent_moe_b200 import build, elq
    build.build()
    elq.lib()
    assert torch.cuda.is_available()
    return elq


@pytest.mark.parametrize("fmt,N,K,T", [(8, 1792, 4096, 1), (8, 4096, 1792, 3), (2, 1280, 3072, 6),
                                       (8, 256, 512, 64)])
def test_noalloc_matches_workspace_entry(E, fmt, N, K, T):
    W = synth.normal(11, N + K, (N, K), 0.02).cuda()
    X = synth.normal(12, T, (T, K)).cuda()
    m = E.QMatrix.from_f32(W, fmt)
    xq = E.quantize_q8_1(X)
    ref = E.latent_proj(m, xq, T)
    # two calls in a row share (and leave behind) the same static scratch
    for _ in range(2):
        y = E.latent_proj_noalloc(m, xq, T)
        torch.cuda.synchronize()
        assert torch.equal(y, ref)      # the projection tests' tolerance: bit-identical
        assert E.latent_proj_noalloc_status() == 0


@pytest.mark.parametrize("fmt,N,K,T", [(8, 1792, 4096, 36), (2, 384, 1280, 5)])
def test_noalloc_matches_oracle(E, orc, fmt, N, K, T):
    """Against the CPU oracle's quantised matmul (the oracle quantises the
    weights and activations itself); T = 36 is the largest token count whose
    scratch fits the 4 MiB array for a 1792 x 4096 Q8_0 matrix."""
    W = synth.normal(13, N + K, (N, K), 0.02)
    X = synth.normal(14, T, (T, K))
    m = E.QMatrix.from_f32(W.cuda(), fmt)
    xq = E.quantize_q8_1(X.cuda())
    y = E.latent_proj_noalloc(m, xq, T).cpu().numpy()
    assert E.latent_proj_noalloc_status() == 0
    ref = orc.qmatmul(fmt, orc.quantize(fmt, W.numpy()), N, K, orc.quantize(orc.Q8_1, X.numpy()), T)
    assert np.array_equal(y, ref)


def test_noalloc_rejects_oversize(E):
    # 1792 x 4096 Q8_0: 16 chunks x T tokens x 1792 rows x 4 B of partial sums;
    # T = 36 fits the 4 MiB array (above), T = 37 does not
    N, K = 1792, 4096
    m = E.QMatrix(8, N, K)
    for T in (37, 64):
        xq = torch.zeros(T, K // 32 * 36, dtype=torch.uint8, device="cuda")
        with pytest.raises(E.ElqError) as ex:
            E.latent_proj_noalloc(m, xq, T)
        assert ex.value.status == -4
