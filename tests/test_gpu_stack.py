"""A stack of layers on one fp32 residual stream (elq_moe_stack: h = x, then
h = h + layer_l(h) for each layer) against the oracle layer by layer.

Every token's path through a layer is independent of the other tokens (the
grouping of pairs by expert changes the order of work, not a value), so at
the full stack shape the oracle follows sampled tokens alone.
"""
import numpy as np
import pytest
import torch

from quantized_latent_moe_b200 import synth
from helpers import add_experts, gpu_layer, oracle_layer

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def E():
    from quantized_latent_moe_b200 import build, elq
    build.build()
    elq.lib()
    assert torch.cuda.is_available()
    return elq


def _oracle_stack(orc, wl, n_layers, x, all_experts=True):
    """h = x, then h = h + layer_l(rms(h)) in fp32; with all_experts False
    each layer gets only the experts its tokens route to (of that layer)."""
    h = x.astype(np.float32)
    for l in range(n_layers):
        ol = oracle_layer(orc, wl, layer=l, experts=None if all_experts else [])
        xn = orc.rmsnorm(h)
        if not all_experts:
            idx, _ = ol.route(xn)
            add_experts(ol, wl, sorted(set(idx.reshape(-1).tolist())), layer=l)
        h = (h + ol.forward(xn)).astype(np.float32)
    return h


@pytest.mark.parametrize("T", [3, 9, 33])
def test_small_stack_exact(E, orc, T):
    """Four distinct tiny layers; T = 3 takes the raw-x D path, 9 and 33 the
    quantiser kernel; fp32 and bf16 first inputs."""
    wl = synth.WORKLOADS["tiny"]
    layers = [gpu_layer(wl, layer=l) for l in range(4)]
    for dt in (torch.float32, torch.bfloat16):
        x = synth.normal(wl.seed, 4000 + T, (T, wl.H)).to(dt)
        h = E.moe_stack(layers, x.cuda()).cpu().numpy()
        assert E.workspace_status(layers[0].stack_workspace(T)) == 0
        ref = _oracle_stack(orc, wl, 4, x.float().numpy())
        assert np.array_equal(h, ref), dt


def test_stack_shape_sampled_tokens(E, orc):
    """The stack workload's layer shape (H=4096, L=1792, 128 experts top-8,
    I=1024, Q8_0, bf16 tokens, router bias N(0,1)) at T = 32, three layers;
    the oracle follows tokens 0, 17 and 31."""
    wl = synth.WORKLOADS["stack"]
    n = 3
    layers = [gpu_layer(wl, layer=l) for l in range(n)]
    x = synth.make_x(wl, step=0)
    h = E.moe_stack(layers, x.cuda()).cpu().numpy()
    assert E.workspace_status(layers[0].stack_workspace(wl.T)) == 0
    rows = [0, 17, 31]
    ref = _oracle_stack(orc, wl, n, x.float().numpy()[rows], all_experts=False)
    assert np.array_equal(h[rows], ref)


def test_stack_matches_layer_calls(E, orc):
    """The stack equals single layer calls fed the oracle's normalised rows,
    with the fp32 residual add done by torch between them (the same IEEE
    adds)."""
    wl = synth.WORKLOADS["tiny"]
    layers = [gpu_layer(wl, layer=l) for l in range(3)]
    x = synth.normal(wl.seed, 4100, (9, wl.H)).cuda()
    h = E.moe_stack(layers, x)
    r = x.clone()
    for ly in layers:
        xn = torch.from_numpy(orc.rmsnorm(r.cpu().numpy())).cuda()
        r = r + E.moe_layer(ly, xn)
    assert torch.equal(h, r)


def _oracle_layer_on_demand(orc, wl, layer):
    """Oracle layer whose experts are drawn when a routing needs them (drawn
    by the input recipe on the GPU and copied over: the same bits as on the
    host; the oracle quantises them itself)."""
    from helpers import ORC_FMT
    dw = synth.dense_weights(wl, layer)
    w = {kk: (None if v is None else v.numpy()) for kk, v in dw.items()}
    w["gate"] = None
    return orc.Layer(wl.H, wl.L, wl.E, wl.k, wl.I, ORC_FMT[wl.fmt], ORC_FMT[wl.fmt], w)


def _add_experts_drawn_on_gpu(ol, wl, experts, layer):
    g, u, d = [None] * wl.E, [None] * wl.E, [None] * wl.E
    for e in experts:
        if ol.gate[e] is None:
            a, b, c = synth.expert_weights(wl, int(e), layer, device="cuda")
            g[e], u[e], d[e] = a.cpu().numpy(), b.cpu().numpy(), c.cpu().numpy()
    ol.set_experts({"gate": g, "up": u, "down": d}, [e for e in experts if g[e] is not None])


def test_stack_48_layers_steps_0_and_63(E, orc):
    """The stack workload at full depth: 48 distinct layers (each with its own
    128 experts, about 36 GB of arena), the step-0 and step-63 token batches
    of 32 tokens each; the oracle follows two tokens of each step through all
    48 layers (rms-normalised input, fp32 residual), drawing each layer's
    experts as its routing needs them.  Exact, and finite everywhere."""
    wl = synth.WORKLOADS["stack"]
    layers = [gpu_layer(wl, layer=l) for l in range(wl.layers)]
    ols = [_oracle_layer_on_demand(orc, wl, l) for l in range(wl.layers)]
    for step, rows in ((0, [0, 31]), (wl.steps - 1, [5, 17])):
        x = synth.make_x(wl, step=step)
        h = E.moe_stack(layers, x.cuda()).cpu().numpy()
        assert E.workspace_status(layers[0].stack_workspace(wl.T)) == 0
        assert np.isfinite(h).all()
        r = x.float().numpy()[rows]
        for l in range(wl.layers):
            ol = ols[l]
            xn = orc.rmsnorm(r)
            idx, _ = ol.route(xn)
            _add_experts_drawn_on_gpu(ol, wl, sorted(set(idx.reshape(-1).tolist())), l)
            r = (r + ol.forward(xn)).astype(np.float32)
        assert np.array_equal(h[rows], r), step
