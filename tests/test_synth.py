"""The seeded input recipe: determinism, range addressing, moments."""
import numpy as np
import torch

from quantized_latent_moe_b200 import synth


def test_deterministic_and_range_addressable():
    a = synth.normal(5, 7, 10000, 0.02)
    b = synth.normal(5, 7, 10000, 0.02)
    assert torch.equal(a, b)
    c = synth.normal(5, 7, 3000, 0.02, start=4000)
    assert torch.equal(a[4000:7000], c)
    assert not torch.equal(a, synth.normal(5, 8, 10000, 0.02))
    assert not torch.equal(a, synth.normal(6, 7, 10000, 0.02))


def test_chunking_does_not_change_values():
    a = synth.normal(1, 2, 5000, 1.0)
    b = synth.normal(1, 2, 5000, 1.0, chunk=777)
    assert torch.equal(a, b)


def test_moments_and_support():
    x = synth.normal(3, 1, 1 << 20, 0.02).double()
    assert abs(x.mean().item()) < 1e-4
    assert abs(x.std().item() / 0.02 - 1) < 5e-3
    assert x.abs().max().item() <= 0.02 * 3.4642
    k = ((x / x.std()) ** 4).mean().item()
    assert 2.68 < k < 2.72         # Irwin-Hall(4): kurtosis 3 - 6/(5*4) = 2.7


def test_permutation_and_zipf_bias():
    p = synth.permutation(3, 8, 128)
    assert sorted(p.tolist()) == list(range(128))
    wl = synth.WORKLOADS["prefill"]
    b = synth.router_bias(wl)
    assert b.shape == (128,)
    assert b.max().item() == 0.0
    assert np.isclose(b.min().item(), -0.3 * 1.1 * np.log(128), rtol=1e-6)


def test_bf16_input_is_rne_of_fp32_draw():
    wl = synth.WORKLOADS["decode"]
    x = synth.make_x(wl)
    assert x.dtype == torch.bfloat16 and x.shape == (1, 4096)
    f = synth.normal(wl.seed, synth.x_tid(0), (1, 4096))
    assert torch.equal(x, f.to(torch.bfloat16))
