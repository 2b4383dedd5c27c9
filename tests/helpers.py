"""Shared helpers of the test-suite: build the same synthetic layer for the
CUDA library (quantised by its own kernels) and for the CPU oracle (quantised
by the oracle)."""
import numpy as np
import torch

from quantized_latent_moe_b200 import synth

ORC_FMT = {"q8_0": 8, "q4_0": 2}


def gpu_layer(wl, layer=0, device="cuda", expert_batch=16):
    from quantized_latent_moe_b200 import elq
    fmt = elq.FMT[wl.fmt]
    dw = synth.dense_weights(wl, layer, device=device)
    rb = dw["router_bias"]
    ly = elq.Layer.allocate(wl.H, wl.L, wl.E, wl.k, wl.I, fmt, fmt, dw["router_w"],
                            None if rb is None else rb.to(device))
    ly.set_dense(dw["D"], dw["U"])
    for e0 in range(0, wl.E, expert_batch):
        es = range(e0, min(wl.E, e0 + expert_batch))
        ws = [synth.expert_weights(wl, e, layer, device=device) for e in es]
        ly.set_experts(e0, torch.stack([w[0] for w in ws]), torch.stack([w[1] for w in ws]),
                       torch.stack([w[2] for w in ws]))
    torch.cuda.synchronize()
    return ly


def oracle_layer(orc, wl, layer=0, experts=None):
    """Oracle layer with only ``experts`` supplied (None = all)."""
    fmt = ORC_FMT[wl.fmt]
    dw = synth.dense_weights(wl, layer)
    w = {k: (None if v is None else v.numpy()) for k, v in dw.items()}
    w["gate"] = None
    ly = orc.Layer(wl.H, wl.L, wl.E, wl.k, wl.I, fmt, fmt, w)
    if experts is None:
        experts = range(wl.E)
    add_experts(ly, wl, experts, layer)
    return ly


def add_experts(ly, wl, experts, layer=0):
    g = [None] * wl.E
    u = [None] * wl.E
    d = [None] * wl.E
    for e in experts:
        if ly.gate[e] is None:
            a, b, c = synth.expert_weights(wl, int(e), layer)
            g[e], u[e], d[e] = a.numpy(), b.numpy(), c.numpy()
    ly.set_experts({"gate": g, "up": u, "down": d}, [e for e in experts if g[e] is not None])


def oracle_forward(orc, ly, wl, x, trace=False):
    """Route first to learn the needed experts, supply them, then run."""
    idx, _ = ly.route(x)
    add_experts(ly, wl, sorted(set(idx.reshape(-1).tolist())))
    return ly.forward(x, trace=trace)


def max_abs_rel(a, b):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    return float(np.abs(a - b).max() / max(np.abs(b).max(), 1e-30))
