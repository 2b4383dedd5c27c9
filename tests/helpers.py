"""Shared helpers of the test-suite: build the same synthetic layer for the
CUDA library (quantised by its own kernels) and for the CPU oracle (quantised
by the oracle)."""
import numpy as np
import torch

from quantized_latent_moe_b200 import synth

ORC_FMT = {"q8_0": 8, "q4_0": 2, "nvfp4": 100, "q5_1": 7, "q3_k": 11, "q4_k": 12, "q5_k": 13}
EXT = ("q5_1", "q3_k", "q4_k", "q5_k")


def nvfp4_globals(w: torch.Tensor) -> torch.Tensor:
    """Per-matrix NVFP4 global scales of w [n, ...]: amax / 2688 (fp32), 1 for
    an all-zero matrix -- computed here, on either side's device, from the
    seeded fp32 weights."""
    amax = w.reshape(w.shape[0], -1).abs().amax(dim=1)
    g = amax / torch.tensor(2688.0, dtype=torch.float32, device=w.device)
    return torch.where(amax > 0, g, torch.ones_like(g))


def gpu_layer(wl, layer=0, device="cuda", expert_batch=16):
    from quantized_latent_moe_b200 import elq
    fmt = elq.FMT[wl.fmt]
    efmt = elq.FMT[wl.expert_fmt]
    dw = synth.dense_weights(wl, layer, device=device)
    rb = dw["router_bias"]
    ly = elq.Layer.allocate(wl.H, wl.L, wl.E, wl.k, wl.I, fmt, efmt, dw["router_w"],
                            None if rb is None else rb.to(device))
    ly.set_dense(dw["D"], dw["U"])
    if efmt == elq.NVFP4:
        ly.act_gz = ly.act_gh = synth.NVFP4_ACT_GSCALE
    for e0 in range(0, wl.E, expert_batch):
        es = range(e0, min(wl.E, e0 + expert_batch))
        if wl.expert_fmt in EXT:
            bs = [synth.expert_blocks(wl, e, layer) for e in es]
            ly.set_expert_blocks(e0, *(torch.stack([b[i] for b in bs]).to(device) for i in range(3)))
            continue
        ws = [synth.expert_weights(wl, e, layer, device=device) for e in es]
        g, u, d = (torch.stack([w[i] for w in ws]) for i in range(3))
        if efmt == elq.NVFP4:
            ly.set_experts_nvfp4(e0, g, u, d, nvfp4_globals(torch.cat([g, u], dim=1)), nvfp4_globals(d))
        else:
            ly.set_experts(e0, g, u, d)
        del ws, g, u, d
    torch.cuda.synchronize()
    return ly


def oracle_layer(orc, wl, layer=0, experts=None):
    """Oracle layer with only ``experts`` supplied (None = all)."""
    dw = synth.dense_weights(wl, layer)
    w = {k: (None if v is None else v.numpy()) for k, v in dw.items()}
    w["gate"] = None
    if wl.expert_fmt == synth.NVFP4:
        w["act_gz"] = w["act_gh"] = synth.NVFP4_ACT_GSCALE
    ly = orc.Layer(wl.H, wl.L, wl.E, wl.k, wl.I, ORC_FMT[wl.fmt], ORC_FMT[wl.expert_fmt], w)
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
            if wl.expert_fmt in EXT:
                a, b, c = synth.expert_blocks(wl, int(e), layer)
            else:
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
