"""Parity of the tensor-core path (tcgen05 kind::i8, T >= 16, Q8_0 weights)
with the CPU oracle, through the C ABI."""
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


@pytest.mark.parametrize("T", [64, 100, 257])
def test_tc_layer_tiny_exact(E, orc, T):
    wl = synth.WORKLOADS["tiny"]
    ly = gpu_layer(wl)
    assert ly.kernel_count(T) == 9
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


def test_tc_experts_grouped_exact(E, orc):
    wl = synth.WORKLOADS["tiny"]
    T = 96
    ly = gpu_layer(wl)
    ol = oracle_layer(orc, wl)
    tr = ol.forward(synth.make_x(wl, T=T).numpy(), trace=True)
    y_lat = E.moe_experts_grouped(ly, torch.from_numpy(tr["zq"]).cuda(), torch.from_numpy(tr["idx"]).cuda(),
                                  torch.from_numpy(tr["w"]).cuda()).cpu().numpy()
    assert np.array_equal(y_lat, tr["y_lat"])


def test_tc_prefill_full_size_sampled(E, orc):
    """The prefill workload at full size (T=2048, 128 experts, Zipf-skewed
    router): all routing decisions and sampled tokens' outputs against the
    oracle computing those tokens alone (the layer is token-wise independent)."""
    wl = synth.WORKLOADS["prefill"]
    ly = gpu_layer(wl)
    x = synth.make_x(wl)
    y = E.moe_layer(ly, x.cuda()).cpu().numpy()
    assert E.workspace_status(ly.workspace(wl.T)) == 0
    counts = E.workspace_view(ly, wl.T, "counts").cpu().numpy()
    assert counts.sum() == wl.T * wl.k and counts.max() <= wl.T
    ol = oracle_layer(orc, wl, experts=[])
    sample = [0, 1, 511, 1024, 2047]
    xs = x.float().numpy()[sample]
    ref = oracle_forward(orc, ol, wl, xs, trace=True)
    idx = E.workspace_view(ly, wl.T, "idx").cpu().numpy().reshape(wl.T, -1)
    assert np.array_equal(idx[sample], ref["idx"])
    assert np.array_equal(y[sample], ref["y"])


def test_int8_rate_kernel_runs(E):
    """The measurement kernel behind the int8 peak: no wait runs out, and every
    CTA's accumulator word is the same nonzero value (same operands)."""
    sink, err = E.test_mma_i8_rate(64)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    s = sink.cpu()
    assert (s == s[0]).all() and int(s[0]) != 0
