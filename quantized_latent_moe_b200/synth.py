"""Seeded synthetic inputs, identical on CPU and on the GPU.

This module holds the input recipe and nothing of the layer's arithmetic: no
quantiser, no dot product, no routing.  Both the CUDA path (through the
benchmark and the tests) and the CPU oracle (through the tests) take their
inputs from here.

Generator.  Every tensor is addressed by (seed, tensor id, element index).  An
element's two 32-bit words are a keyed hash of its 41-bit counter
``2 * index + lane``: three rounds of the MurmurHash3 32-bit finaliser
(fmix32), with the key derived from (seed, tensor id) by the same finaliser.
Only integer operations on values below 2^50 are used, so torch gives the same
bits on CPU and CUDA, and any element range can be regenerated on its own.

Normal values.  The four 16-bit halves of the two words are summed
(Irwin-Hall with n = 4, an exact integer), centred, and scaled to the target
standard deviation by one fp64 multiply, then rounded to fp32 (and to bf16
where the workload asks for bf16).  Every step is exact or one IEEE rounding,
so CPU and GPU agree bit for bit.  The distribution is the sum of four
uniforms: mean 0, the requested variance, support +-3.46 sigma.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import torch

M32 = 0xFFFFFFFF


def _mul32(x: torch.Tensor, c: int) -> torch.Tensor:
    """(x * c) mod 2^32 for x holding uint32 values in int64, c < 2^32."""
    lo, hi = c & 0xFFFF, c >> 16
    return (x * lo + (((x * hi) & 0xFFFF) << 16)) & M32


def _fmix32(h: torch.Tensor) -> torch.Tensor:
    h = h ^ (h >> 16)
    h = _mul32(h, 0x85EBCA6B)
    h = h ^ (h >> 13)
    h = _mul32(h, 0xC2B2AE35)
    return h ^ (h >> 16)


def _fmix32_int(h: int) -> int:
    h &= M32
    h ^= h >> 16
    h = (h * 0x85EBCA6B) & M32
    h ^= h >> 13
    h = (h * 0xC2B2AE35) & M32
    return h ^ (h >> 16)


def _keys(seed: int, tid: int):
    k0 = _fmix32_int(seed * 0x9E3779B9 + 0x632BE5AB)
    k1 = _fmix32_int(k0 ^ (tid * 0x85EBCA77 + 0x165667B1))
    k2 = _fmix32_int(k1 + 0x27D4EB2F)
    k3 = _fmix32_int(k2 ^ 0x61C88647)
    return k1, k2, k3


def words(seed: int, tid: int, start: int, n: int, lane: int, device="cpu") -> torch.Tensor:
    """32-bit hash words (int64 tensor) of elements start .. start+n-1."""
    k1, k2, k3 = _keys(seed, tid)
    c = (torch.arange(start, start + n, dtype=torch.int64, device=device) * 2) + lane
    lo = c & M32
    hi = c >> 32
    h = _fmix32(lo ^ k1)
    h = _fmix32(h ^ _mul32(hi ^ k2, 0x9E3779B9))
    h = _fmix32((h + k3) & M32)
    return h


_IH_STD = math.sqrt((65536.0 ** 2 - 1.0) / 3.0)   # std of the sum of four U{0..65535}
_IH_MEAN = 2 * 65535                               # mean of that sum


def normal(seed: int, tid: int, shape, sigma: float = 1.0, device="cpu",
           start: int = 0, chunk: int = 1 << 26) -> torch.Tensor:
    """fp32 tensor of the given shape with the recipe's normal values;
    element i of the flattened tensor is element ``start + i`` of the stream."""
    if isinstance(shape, int):
        shape = (shape,)
    n = 1
    for s in shape:
        n *= s
    out = torch.empty(n, dtype=torch.float32, device=device)
    scale = float(sigma) / _IH_STD
    for s0 in range(0, n, chunk):
        m = min(chunk, n - s0)
        w0 = words(seed, tid, start + s0, m, 0, device)
        w1 = words(seed, tid, start + s0, m, 1, device)
        tot = (w0 & 0xFFFF) + (w0 >> 16) + (w1 & 0xFFFF) + (w1 >> 16) - _IH_MEAN
        out[s0:s0 + m] = (tot.to(torch.float64) * scale).to(torch.float32)
        del w0, w1, tot
    return out.view(*shape)


def permutation(seed: int, tid: int, n: int) -> torch.Tensor:
    """A seeded permutation of 0..n-1 (argsort of hash words, index breaks ties)."""
    w = words(seed, tid, 0, n, 0)
    key = w * n + torch.arange(n, dtype=torch.int64)
    return torch.argsort(key)


# ---------------------------------------------------------------------------
# pre-quantised weights: GGUF blocks drawn directly (random codes, 6-bit
# sub-block scales and mins, fp16 super-block scales in a fixed binade)

Q5_1, Q3_K, Q4_K, Q5_K = "q5_1", "q3_k", "q4_k", "q5_k"
EXT_ROW_BYTES = {Q5_1: (32, 24), Q3_K: (256, 110), Q4_K: (256, 144), Q5_K: (256, 176)}   # values, bytes per block
# fp16 exponent fields of the block scales: (d, m or dmin), so that values
# land within about +-0.1 and Q5_1's m is negative
_EXT_FIELDS = {Q5_1: (4, 8), Q3_K: (5, None), Q4_K: (1, 5), Q5_K: (1, 6)}


def ext_row_bytes(fmt: str, k: int) -> int:
    vals, nb = EXT_ROW_BYTES[fmt]
    return k // vals * nb


def ext_blocks(fmt: str, seed: int, tid: int, rows: int, k: int, row0: int = 0) -> torch.Tensor:
    """uint8 [rows, row bytes] of GGUF blocks of format fmt (q5_1, q3_k, q4_k, q5_k):
    every byte from the counter hash, then each block's fp16 scale fields
    set to a positive fp16 of exponent field f_d (d) and, for the second
    field, f_m (negative for Q5_1's m, positive for the K-quants' dmin), the
    fraction bits from the hash.  Rows row0 .. row0+rows-1 of the stream."""
    vals, bb = EXT_ROW_BYTES[fmt]
    rb = k // vals * bb
    nw = (rb + 3) // 4                    # hash words per row (the last one partly used)
    w = words(seed, tid, row0 * nw, rows * nw, 0)
    by = torch.stack([(w >> (8 * i)) & 0xFF for i in range(4)], dim=1).reshape(rows, nw * 4)[:, :rb]
    by = by.reshape(rows, k // vals, bb).clone()
    fd, fm = _EXT_FIELDS[fmt]
    if fmt == Q3_K:
        # the super-block scale d is the block's last two bytes
        d = (fd << 10) | ((by[:, :, 108] | (by[:, :, 109] << 8)) & 0x3FF)
        by[:, :, 108], by[:, :, 109] = d & 0xFF, d >> 8
        return by.reshape(rows, rb).to(torch.uint8)
    d = (fd << 10) | ((by[:, :, 0] | (by[:, :, 1] << 8)) & 0x3FF)
    m = (fm << 10) | ((by[:, :, 2] | (by[:, :, 3] << 8)) & 0x3FF)
    if fmt == Q5_1:
        m = m | 0x8000
    by[:, :, 0], by[:, :, 1] = d & 0xFF, d >> 8
    by[:, :, 2], by[:, :, 3] = m & 0xFF, m >> 8
    return by.reshape(rows, rb).to(torch.uint8)


def expert_blocks(wl: "Workload", e: int, layer: int = 0):
    """Expert e's gate [I, L], up [I, L] and down [L, I] as GGUF blocks of
    the workload's expert format (uint8 rows)."""
    fmt = wl.expert_fmt
    return (ext_blocks(fmt, wl.seed, tid(layer, TID_GATE), wl.I, wl.L, row0=e * wl.I),
            ext_blocks(fmt, wl.seed, tid(layer, TID_UP), wl.I, wl.L, row0=e * wl.I),
            ext_blocks(fmt, wl.seed, tid(layer, TID_DOWN), wl.L, wl.I, row0=e * wl.L))


# ---------------------------------------------------------------------------
# workloads

F32, BF16 = "f32", "bf16"
Q8_0, Q4_0, NVFP4 = "q8_0", "q4_0", "nvfp4"


@dataclass(frozen=True)
class Workload:
    name: str
    seed: int
    T: int
    H: int
    L: int
    E: int
    k: int
    I: int
    fmt: str                 # weight format of D and U (and of the experts unless ex_fmt)
    x_dtype: str             # activation input dtype
    bias: str                # "none" | "normal" | "zipf"
    layers: int = 1
    steps: int = 1
    zipf_s: float = 1.1
    zipf_c: float = 0.3
    residual: bool = False   # stack: x_{l+1} = x_l + y_l in fp32
    extra: dict = field(default_factory=dict)
    ex_fmt: str = ""         # expert weight format when it differs from fmt

    @property
    def expert_fmt(self) -> str:
        return self.ex_fmt or self.fmt


WORKLOADS = {
    # tiny layer: T=4, H=512, L=256, 8 experts top-2, I=256, Q8_0, fp32 input
    "tiny": Workload("tiny", 0, 4, 512, 256, 8, 2, 256, Q8_0, F32, "none"),
    # decode: one token, 1792-wide latent, 128 experts top-8, Q8_0, bf16 input,
    # router bias N(0, 1) per expert
    "decode": Workload("decode", 1, 1, 4096, 1792, 128, 8, 1024, Q8_0, BF16, "normal"),
    # speculative verify window: six tokens, 1280-wide latent, Q4_0 everywhere,
    # other distributions as the tiny layer (fp32 input, no router bias)
    "verify": Workload("verify", 2, 6, 3072, 1280, 128, 8, 768, Q4_0, F32, "none"),
    # prefill: 2048 tokens, Zipf(1.1)-skewed router over the 128 experts
    "prefill": Workload("prefill", 3, 2048, 4096, 1792, 128, 8, 1024, Q8_0, BF16, "zipf"),
    # decode with NVFP4 latent experts (D/U stay Q8_0): the decode shapes
    "decode_nvfp4": Workload("decode_nvfp4", 5, 1, 4096, 1792, 128, 8, 1024, Q8_0, BF16, "normal",
                             ex_fmt=NVFP4),
    # prefill with NVFP4 latent experts: the prefill shapes and router skew
    "prefill_nvfp4": Workload("prefill_nvfp4", 6, 2048, 4096, 1792, 128, 8, 1024, Q8_0, BF16, "zipf",
                              ex_fmt=NVFP4),
    # decode with Q4_K latent experts (D/U Q8_0): the decode shapes
    "decode_q4_k": Workload("decode_q4_k", 7, 1, 4096, 1792, 128, 8, 1024, Q8_0, BF16, "normal", ex_fmt="q4_k"),
    # decode with Q3_K latent experts (D/U Q8_0): the decode shapes
    "decode_q3_k": Workload("decode_q3_k", 8, 1, 4096, 1792, 128, 8, 1024, Q8_0, BF16, "normal", ex_fmt="q3_k"),
    # resident stack: 48 layers, 32 sequences decoding one token per step
    "stack": Workload("stack", 4, 32, 4096, 1792, 128, 8, 1024, Q8_0, BF16, "normal",
                      layers=48, steps=64, residual=True),
}

WEIGHT_SIGMA = 0.02

# Static fp32 global scales of the NVFP4 experts' inputs (the latent z and the
# SwiGLU output h), as a calibrated checkpoint would carry them: 2^-6 puts
# every micro-block of these workloads' activations in E4M3's normal range and
# leaves room up to |x| = 6 * 448 / 64 = 42.
NVFP4_ACT_GSCALE = 2.0 ** -6

# tensor ids within a layer
TID_X, TID_D, TID_U, TID_RW, TID_RB, TID_GATE, TID_UP, TID_DOWN, TID_ZIPF = range(9)


def tid(layer: int, what: int) -> int:
    return 64 * layer + what


def x_tid(step: int) -> int:
    return (1 << 20) + step


def make_x(wl: Workload, step: int = 0, T: int | None = None, device="cpu",
           token0: int = 0) -> torch.Tensor:
    """Layer input [T, H]: fp32, or bf16 (RNE from the fp32 draw) for bf16 workloads."""
    T = wl.T if T is None else T
    x = normal(wl.seed, x_tid(step), (T, wl.H), 1.0, device, start=token0 * wl.H)
    return x.to(torch.bfloat16) if wl.x_dtype == BF16 else x


def router_bias(wl: Workload, layer: int = 0):
    """Per-expert router bias (fp32 [E]) or None."""
    if wl.bias == "none":
        return None
    if wl.bias == "normal":
        return normal(wl.seed, tid(layer, TID_RB), wl.E, 1.0)
    # Zipf skew: bias_e = -c * s * ln(rank_e), rank a seeded permutation of 1..E
    rank = permutation(wl.seed, tid(layer, TID_ZIPF), wl.E).to(torch.float64) + 1.0
    return (-wl.zipf_c * wl.zipf_s * torch.log(rank)).to(torch.float32)


def dense_weights(wl: Workload, layer: int = 0, device="cpu"):
    """D [L,H], U [H,L], router_w [E,L] (fp32) and router bias."""
    s = WEIGHT_SIGMA
    return dict(
        D=normal(wl.seed, tid(layer, TID_D), (wl.L, wl.H), s, device),
        U=normal(wl.seed, tid(layer, TID_U), (wl.H, wl.L), s, device),
        router_w=normal(wl.seed, tid(layer, TID_RW), (wl.E, wl.L), s, device),
        router_bias=router_bias(wl, layer),
    )


def expert_weights(wl: Workload, e: int, layer: int = 0, device="cpu"):
    """gate [I,L], up [I,L], down [L,I] (fp32) of expert e."""
    s = WEIGHT_SIGMA
    nGU = wl.I * wl.L
    return (normal(wl.seed, tid(layer, TID_GATE), (wl.I, wl.L), s, device, start=e * nGU),
            normal(wl.seed, tid(layer, TID_UP), (wl.I, wl.L), s, device, start=e * nGU),
            normal(wl.seed, tid(layer, TID_DOWN), (wl.L, wl.I), s, device, start=e * nGU))


def layer_weights(wl: Workload, layer: int = 0, experts=None, device="cpu"):
    """All fp32 weights of a layer; ``experts`` limits which experts are drawn
    (others are None)."""
    w = dense_weights(wl, layer, device)
    es = range(wl.E) if experts is None else experts
    gate = [None] * wl.E
    up = [None] * wl.E
    down = [None] * wl.E
    for e in es:
        gate[e], up[e], down[e] = expert_weights(wl, e, layer, device)
    w.update(gate=gate, up=up, down=down)
    if wl.expert_fmt == NVFP4:
        w.update(act_gz=NVFP4_ACT_GSCALE, act_gh=NVFP4_ACT_GSCALE)
    return w
