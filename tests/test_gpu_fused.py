"""The fused small-T layer kernel (the whole layer as one cooperative
persistent launch, T <= 8 and T * k <= 64, selected by the layer flag
LAYER_FUSED) against the CPU oracle, element by element, and against the
separate-kernel sequence.

The arithmetic of every step is the one the separate kernels use (same
accumulation order, same exp, same quantiser), so every output and every
intermediate is compared for exact equality.
"""
import numpy as np
import pytest
import torch

from quantized_latent_moe_b200 import synth
from helpers import add_experts, gpu_layer, oracle_forward, oracle_layer

pytestmark = pytest.mark.gpu

ELQ_ERR_TIMEOUT = -6
VIEWS = ["z", "zq", "logits", "idx", "weights", "counts", "offsets", "perm", "pos", "hq", "o", "y_lat",
         "ylq", "n_act"]


@pytest.fixture(scope="module")
def E():
    from quantized_latent_moe_b200 import build, elq
    build.build()
    elq.lib()
    assert torch.cuda.is_available()
    return elq


@pytest.fixture(scope="module")
def tiny(E, orc):
    wl = synth.WORKLOADS["tiny"]
    ly = gpu_layer(wl)
    ly.flags = E.LAYER_FUSED
    return wl, ly, oracle_layer(orc, wl)


def _views(E, ly, T):
    return {n: E.workspace_view(ly, T, n).cpu().numpy().copy() for n in VIEWS}


def test_kernel_counts(E, tiny):
    wl, ly, _ = tiny
    for T in range(1, 9):
        assert ly.kernel_count(T) == 1, T
    assert ly.kernel_count(9) == 6
    ly.flags = 0
    try:
        assert ly.kernel_count(4) == 5
    finally:
        ly.flags = E.LAYER_FUSED


def test_every_T_both_input_types(E, tiny):
    """T = 1 .. 8, fp32 and bf16 input: identical to the oracle."""
    wl, ly, ol = tiny
    for T in range(1, 9):
        for dt in (torch.float32, torch.bfloat16):
            x = synth.normal(wl.seed, 500 + T, (T, wl.H)).to(dt)
            y = E.moe_layer(ly, x.cuda()).cpu().numpy()
            ref = ol.forward(x.float().numpy())
            assert np.array_equal(y, ref), (T, dt)
        assert E.workspace_status(ly.workspace(T)) == 0


def test_repeated_calls_reset_their_flags(E, orc):
    """Consecutive decode steps on one workspace: the phase flags and tile
    counters return to zero at the end of each call."""
    wl = synth.WORKLOADS["decode"]
    ly = gpu_layer(wl)
    ly.flags = E.LAYER_FUSED
    assert ly.kernel_count(1) == 1
    ol = oracle_layer(orc, wl, experts=[])
    xs = [synth.make_x(wl, step=s) for s in range(5)]
    ys = [E.moe_layer(ly, x.cuda()).cpu().numpy() for x in xs]
    assert E.workspace_status(ly.workspace(1)) == 0
    for x, y in zip(xs, ys):
        ref = oracle_forward(orc, ol, wl, x.float().numpy())
        assert np.array_equal(y, ref)


def test_fused_equals_separate_kernels(E, orc):
    """The verify window (T = 6, Q4_0): every intermediate of the fused call
    equals that of the separate-kernel sequence, and y equals the oracle's."""
    wl = synth.WORKLOADS["verify"]
    ly = gpu_layer(wl)
    x = synth.make_x(wl).cuda()
    ly.flags = E.LAYER_FUSED
    assert ly.kernel_count(wl.T) == 1
    y_f = E.moe_layer(ly, x).cpu().numpy()
    v_f = _views(E, ly, wl.T)
    ly.flags = 0
    assert ly.kernel_count(wl.T) == 5
    y_s = E.moe_layer(ly, x).cpu().numpy()
    v_s = _views(E, ly, wl.T)
    assert np.array_equal(y_f, y_s)
    n = int(v_f["n_act"][0])
    for name in VIEWS:
        a, b = v_f[name], v_s[name]
        assert np.array_equal(a, b), name
    ol = oracle_layer(orc, wl, experts=[])
    tr = oracle_forward(orc, ol, wl, x.float().cpu().numpy(), trace=True)
    assert np.array_equal(y_f, tr["y"])
    assert n == len(set(tr["idx"].reshape(-1).tolist()))


@pytest.mark.parametrize("du,ex", [(8, 2), (2, 8)])
def test_mixed_formats(E, orc, du, ex):
    """D/U and the experts in different formats (the kernel's other template
    instances), T = 1 and 5."""
    from quantized_latent_moe_b200 import elq
    wl = synth.Workload("mixed", 7, 1, 1024, 512, 16, 4, 256, synth.Q8_0, synth.F32, "normal")
    dw = synth.dense_weights(wl)
    ly = elq.Layer.allocate(wl.H, wl.L, wl.E, wl.k, wl.I, du, ex, dw["router_w"].cuda(),
                            dw["router_bias"].cuda())
    ly.set_dense(dw["D"].cuda(), dw["U"].cuda())
    ws_ = [synth.expert_weights(wl, e, device="cuda") for e in range(wl.E)]
    ly.set_experts(0, torch.stack([w[0] for w in ws_]), torch.stack([w[1] for w in ws_]),
                   torch.stack([w[2] for w in ws_]))
    ly.flags = E.LAYER_FUSED
    w = {k: (None if v is None else v.numpy()) for k, v in dw.items()}
    w["gate"] = None
    ol = orc.Layer(wl.H, wl.L, wl.E, wl.k, wl.I, du, ex, w)
    add_experts(ol, wl, range(wl.E))
    for T in (1, 5):
        assert ly.kernel_count(T) == 1
        x = synth.normal(wl.seed, 900 + T, (T, wl.H))
        y = E.moe_layer(ly, x.cuda()).cpu().numpy()
        assert np.array_equal(y, ol.forward(x.numpy())), T


def test_graph_replay(E, tiny):
    """Fused calls captured in a CUDA graph replay to the oracle's results."""
    wl, ly, ol = tiny
    T = 3
    xs = [synth.normal(wl.seed, 700 + i, (T, wl.H)).cuda() for i in range(3)]
    ys = [torch.empty(T, wl.H, device="cuda") for _ in range(3)]
    ws = ly.workspace(T)
    for x, y in zip(xs, ys):          # eager first: opt-in and first-use set-up outside capture
        E.moe_layer(ly, x, y, ws)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for x, y in zip(xs, ys):
            E.moe_layer(ly, x, y, ws)
    for y in ys:
        y.zero_()
    for _ in range(2):
        g.replay()
    torch.cuda.synchronize()
    assert E.workspace_status(ws) == 0
    for x, y in zip(xs, ys):
        assert np.array_equal(y.cpu().numpy(), ol.forward(x.cpu().numpy()))
    del g


def test_bounded_wait_reports_timeout(E, tiny):
    """Failure detection without a fault: the routing is withheld, the expert
    phases' waits run out after 20 ms, the kernel drains its own copies and
    returns, and the workspace error word says so.  A zero-filled workspace
    then serves a normal call."""
    wl, ly, ol = tiny
    T = 2
    x = synth.normal(wl.seed, 800, (T, wl.H)).cuda()
    ws = torch.zeros(ly.workspace_bytes(T) + 256, dtype=torch.uint8, device="cuda")
    off = (-ws.data_ptr()) % 256
    ws = ws[off:off + ly.workspace_bytes(T)]
    assert E.test_fused_timeout(ly, x, ws, 20_000_000) == 0
    torch.cuda.synchronize()
    assert E.workspace_status(ws) == ELQ_ERR_TIMEOUT
    ws.zero_()
    y = E.moe_layer(ly, x, ws=ws).cpu().numpy()
    assert E.workspace_status(ws) == 0
    assert np.array_equal(y, ol.forward(x.cpu().numpy()))
