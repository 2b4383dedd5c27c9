"""Scalar CPU oracle of the quantized latent-MoE layer -- TEST INFRASTRUCTURE.

Only the tests, the package's ``smoke()`` check and the benchmark's CPU
baseline leg may use this package.  The CUDA library never imports, links or
calls it, and it imports nothing from the CUDA library.  What it computes is
stated in ``elq_oracle.h`` (readings R1-R25) and written out in
``elq_oracle.c`` as plain loops; this module only builds the C file with gcc
and marshals numpy arrays into it.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "elq_oracle.c")
HDR = os.path.join(HERE, "elq_oracle.h")
LIB = os.path.join(HERE, "libelq_oracle.so")

Q4_0, Q5_1, Q8_0, Q8_1, Q3_K, Q4_K, Q5_K, NVFP4 = 2, 7, 8, 9, 11, 12, 13, 100
BLOCK_BYTES = {Q4_0: 18, Q8_0: 34, Q8_1: 36, NVFP4: 18, Q5_1: 24}
EXT = (Q5_1, Q3_K, Q4_K, Q5_K)     # expert formats given as GGUF blocks (R22-R25)

CFLAGS = ["-O2", "-ffp-contract=off", "-fno-fast-math", "-std=c11", "-fPIC",
          "-shared", "-Wall", "-Wextra"]


def build(force: bool = False) -> str:
    """Compile elq_oracle.c into libelq_oracle.so (plain gcc, no GPU)."""
    newest = max(os.path.getmtime(SRC), os.path.getmtime(HDR))
    if force or not os.path.exists(LIB) or os.path.getmtime(LIB) < newest:
        tmp = LIB + ".tmp%d" % os.getpid()
        subprocess.run(["gcc", *CFLAGS, "-o", tmp, SRC, "-lm"], check=True)
        os.replace(tmp, LIB)
    return LIB


_lib = None


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build())
        _declare(_lib)
    return _lib


P = ctypes.c_void_p
I32, I64, F32 = ctypes.c_int32, ctypes.c_int64, ctypes.c_float


class OrcLayer(ctypes.Structure):
    _fields_ = [("H", ctypes.c_int), ("L", ctypes.c_int), ("E", ctypes.c_int),
                ("k", ctypes.c_int), ("I", ctypes.c_int),
                ("du_fmt", ctypes.c_int), ("ex_fmt", ctypes.c_int),
                ("D", P), ("U", P), ("router_w", P), ("router_bias", P),
                ("gate", P), ("up", P), ("down", P),
                ("gate_g", P), ("up_g", P), ("down_g", P),
                ("act_gz", F32), ("act_gh", F32)]


class OrcTrace(ctypes.Structure):
    _fields_ = [(n, P) for n in ("xq", "z", "logits", "idx", "w", "zq", "counts",
                                 "offsets", "perm", "pos", "g", "u", "hq", "o",
                                 "y_lat", "ylq")]


def _declare(L):
    sig = {
        "orc_block_bytes": (ctypes.c_int, [ctypes.c_int]),
        "orc_f32_to_f16": (ctypes.c_uint16, [F32]),
        "orc_f16_to_f32": (F32, [ctypes.c_uint16]),
        "orc_bf16_to_f32": (F32, [ctypes.c_uint16]),
        "orc_expf": (F32, [F32]),
        "orc_silu": (F32, [F32]),
        "orc_quantize_q8_1": (None, [P, I64, P]),
        "orc_quantize_q8_0": (None, [P, I64, P]),
        "orc_quantize_q4_0": (None, [P, I64, P]),
        "orc_dequantize": (None, [ctypes.c_int, P, I64, P]),
        "orc_block_isum": (I32, [ctypes.c_int, P, P]),
        "orc_block_term": (F32, [ctypes.c_int, P, P]),
        "orc_qmatmul": (None, [ctypes.c_int, P, ctypes.c_int, ctypes.c_int, P,
                               ctypes.c_int, P]),
        "orc_router_topk": (None, [P, P, P] + [ctypes.c_int] * 4 + [P, P, P]),
        "orc_bucket": (None, [P] + [ctypes.c_int] * 3 + [P, P, P, P]),
        "orc_rmsnorm": (None, [P, ctypes.c_int, ctypes.c_int, P]),
        "orc_moe_layer": (ctypes.c_int, [ctypes.POINTER(OrcLayer), P, ctypes.c_int,
                                         P, ctypes.POINTER(OrcTrace)]),
        "orc_route": (ctypes.c_int, [ctypes.POINTER(OrcLayer), P, ctypes.c_int, P, P]),
        "orc_arena_pack": (None, [ctypes.c_int, P, ctypes.c_int, ctypes.c_int, P, P]),
        "orc_row_bytes": (I64, [ctypes.c_int, I64]),
        "orc_dequantize_ext": (None, [ctypes.c_int, P, ctypes.c_int, ctypes.c_int, P]),
        "orc_block_ext": (None, [ctypes.c_int, P, ctypes.c_int, P, P, P, P, P]),
        "orc_qmatmul_ext": (None, [ctypes.c_int, P, ctypes.c_int, ctypes.c_int, P, ctypes.c_int, P]),
        "orc_f32_to_e2m1": (ctypes.c_uint8, [F32]),
        "orc_e2m1_to_f32": (F32, [ctypes.c_uint8]),
        "orc_f32_to_e4m3": (ctypes.c_uint8, [F32]),
        "orc_e4m3_to_f32": (F32, [ctypes.c_uint8]),
        "orc_nvfp4_global": (F32, [P, I64]),
        "orc_quantize_nvfp4": (None, [P, I64, F32, P]),
        "orc_dequantize_nvfp4": (None, [P, I64, F32, P]),
        "orc_qmatmul_nvfp4": (None, [P, F32, ctypes.c_int, ctypes.c_int, P, F32, ctypes.c_int, P]),
    }
    for name, (res, args) in sig.items():
        f = getattr(L, name)
        f.restype = res
        f.argtypes = args


def _p(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _f32(x):
    return np.ascontiguousarray(x, dtype=np.float32)


# -- thin wrappers ---------------------------------------------------------

def f32_to_f16_bits(x: float) -> int:
    return int(lib().orc_f32_to_f16(float(x)))


def f16_bits_to_f32(h: int) -> float:
    return float(lib().orc_f16_to_f32(int(h)))


def expf(x: float) -> float:
    return float(lib().orc_expf(float(x)))


def silu(x: float) -> float:
    return float(lib().orc_silu(float(x)))


def quantize(fmt: int, x) -> np.ndarray:
    """fp32 array (last dim % 32 == 0) -> uint8 array of AoS blocks, shape
    x.shape[:-1] + (x.shape[-1]//32 * block_bytes,)."""
    x = _f32(x)
    n = x.size
    out = np.empty(x.shape[:-1] + (x.shape[-1] // 32 * BLOCK_BYTES[fmt],), np.uint8)
    fn = {Q8_1: lib().orc_quantize_q8_1, Q8_0: lib().orc_quantize_q8_0,
          Q4_0: lib().orc_quantize_q4_0}[fmt]
    fn(_p(x), n, _p(out))
    return out


def dequantize(fmt: int, blocks: np.ndarray, n: int) -> np.ndarray:
    blocks = np.ascontiguousarray(blocks, dtype=np.uint8)
    out = np.empty(n, np.float64)
    lib().orc_dequantize(fmt, _p(blocks), n, _p(out))
    return out


def block_isum(wfmt: int, wblk: np.ndarray, ablk: np.ndarray) -> int:
    wblk = np.ascontiguousarray(wblk, np.uint8)
    ablk = np.ascontiguousarray(ablk, np.uint8)
    return int(lib().orc_block_isum(wfmt, _p(wblk), _p(ablk)))


def block_term(wfmt: int, wblk: np.ndarray, ablk: np.ndarray) -> float:
    wblk = np.ascontiguousarray(wblk, np.uint8)
    ablk = np.ascontiguousarray(ablk, np.uint8)
    return float(lib().orc_block_term(wfmt, _p(wblk), _p(ablk)))


def qmatmul(wfmt: int, W: np.ndarray, N: int, K: int, Xq: np.ndarray, T: int) -> np.ndarray:
    W = np.ascontiguousarray(W, np.uint8)
    Xq = np.ascontiguousarray(Xq, np.uint8)
    assert W.size == N * (K // 32) * BLOCK_BYTES[wfmt]
    assert Xq.size == T * (K // 32) * 36
    Y = np.empty((T, N), np.float32)
    lib().orc_qmatmul(wfmt, _p(W), N, K, _p(Xq), T, _p(Y))
    return Y


def router_topk(z, Wr, bias, k: int):
    z = _f32(z)
    Wr = _f32(Wr)
    T, L = z.shape
    E = Wr.shape[0]
    b = None if bias is None else _f32(bias)
    idx = np.empty((T, k), np.int32)
    w = np.empty((T, k), np.float32)
    logits = np.empty((T, E), np.float32)
    lib().orc_router_topk(_p(z), _p(Wr), _p(b), T, L, E, k, _p(idx), _p(w), _p(logits))
    return idx, w, logits


def rmsnorm(h):
    """Rows of h divided by sqrt(mean(h^2) + 1e-6) (the stack's layer input)."""
    h = _f32(h)
    T, H = h.shape
    out = np.empty((T, H), np.float32)
    lib().orc_rmsnorm(_p(h), T, H, _p(out))
    return out


def bucket(idx: np.ndarray, E: int):
    idx = np.ascontiguousarray(idx, np.int32)
    T, k = idx.shape
    counts = np.empty(E, np.int32)
    offsets = np.empty(E + 1, np.int32)
    perm = np.empty(T * k, np.int32)
    pos = np.empty(T * k, np.int32)
    lib().orc_bucket(_p(idx), T, k, E, _p(counts), _p(offsets), _p(perm), _p(pos))
    return counts, offsets, perm, pos


def f32_to_e2m1(x: float) -> int:
    return int(lib().orc_f32_to_e2m1(float(x)))


def e2m1_to_f32(c: int) -> float:
    return float(lib().orc_e2m1_to_f32(int(c)))


def f32_to_e4m3(x: float) -> int:
    return int(lib().orc_f32_to_e4m3(float(x)))


def e4m3_to_f32(b: int) -> float:
    return float(lib().orc_e4m3_to_f32(int(b)))


def nvfp4_global(x) -> float:
    """Global scale of a weight matrix: amax / (6 * 448), 1 when all zero (R20)."""
    x = _f32(x)
    return float(lib().orc_nvfp4_global(_p(x), x.size))


def quantize_nvfp4(x, g: float = 1.0) -> np.ndarray:
    """fp32 array (last dim % 32 == 0) -> 18-byte NVFP4 blocks under global scale g."""
    x = _f32(x)
    out = np.empty(x.shape[:-1] + (x.shape[-1] // 32 * 18,), np.uint8)
    lib().orc_quantize_nvfp4(_p(x), x.size, float(g), _p(out))
    return out


def dequantize_nvfp4(blocks: np.ndarray, n: int, g: float) -> np.ndarray:
    blocks = np.ascontiguousarray(blocks, dtype=np.uint8)
    out = np.empty(n, np.float64)
    lib().orc_dequantize_nvfp4(_p(blocks), n, float(g), _p(out))
    return out


def qmatmul_nvfp4(W: np.ndarray, gw: float, N: int, K: int, Xq: np.ndarray, T: int,
                  ga: float = 1.0) -> np.ndarray:
    W = np.ascontiguousarray(W, np.uint8)
    Xq = np.ascontiguousarray(Xq, np.uint8)
    assert W.size == N * (K // 32) * 18 and Xq.size == T * (K // 32) * 18
    Y = np.empty((T, N), np.float32)
    lib().orc_qmatmul_nvfp4(_p(W), float(gw), N, K, _p(Xq), float(ga), T, _p(Y))
    return Y


def row_bytes(fmt: int, k: int) -> int:
    return int(lib().orc_row_bytes(fmt, k))


def dequantize_ext(fmt: int, W: np.ndarray, N: int, K: int) -> np.ndarray:
    """fp64 values of N rows of Q5_1 / Q4_K / Q5_K blocks (R22)."""
    W = np.ascontiguousarray(W, np.uint8)
    assert W.size == N * row_bytes(fmt, K)
    out = np.empty((N, K), np.float64)
    lib().orc_dequantize_ext(fmt, _p(W), N, K, _p(out))
    return out


def block_ext(fmt: int, row: np.ndarray, kb: int, ablk: np.ndarray):
    """(isum, sumq, sd, sm) of 32-value block kb of a row against a Q8_1 block (R23, R24)."""
    row = np.ascontiguousarray(row, np.uint8)
    ablk = np.ascontiguousarray(ablk, np.uint8)
    isum, sumq = ctypes.c_int32(), ctypes.c_int32()
    sd, sm = ctypes.c_float(), ctypes.c_float()
    lib().orc_block_ext(fmt, _p(row), kb, _p(ablk), ctypes.byref(isum), ctypes.byref(sumq), ctypes.byref(sd),
                        ctypes.byref(sm))
    return isum.value, sumq.value, sd.value, sm.value


def qmatmul_ext(fmt: int, W: np.ndarray, N: int, K: int, Xq: np.ndarray, T: int) -> np.ndarray:
    W = np.ascontiguousarray(W, np.uint8)
    Xq = np.ascontiguousarray(Xq, np.uint8)
    assert W.size == N * row_bytes(fmt, K) and Xq.size == T * (K // 32) * 36
    Y = np.empty((T, N), np.float32)
    lib().orc_qmatmul_ext(fmt, _p(W), N, K, _p(Xq), T, _p(Y))
    return Y


def arena_pack(fmt: int, aos: np.ndarray, n_rows: int, k: int):
    aos = np.ascontiguousarray(aos, np.uint8)
    nb = k // 32
    slab = 4096 if fmt == Q8_0 else 2048
    q = np.zeros((n_rows // 128) * nb * slab, np.uint8)
    d = np.zeros((n_rows // 128) * nb * 256, np.uint8)
    lib().orc_arena_pack(fmt, _p(aos), n_rows, k, _p(q), _p(d))
    return q, d


class Layer:
    """Quantised weights of one layer in the oracle's AoS form.

    ``w`` holds fp32 arrays D [L,H], U [H,L], router_w [E,L], router_bias [E]
    or None, gate/up [E][I,L], down [E][L,I]; expert entries may be None
    (not supplied).  Quantisation is the oracle's own."""

    def __init__(self, H, L, E, k, I, du_fmt, ex_fmt, w):
        self.H, self.L, self.E, self.k, self.I = H, L, E, k, I
        self.du_fmt, self.ex_fmt = du_fmt, ex_fmt
        self.D = quantize(du_fmt, w["D"])
        self.U = quantize(du_fmt, w["U"])
        self.router_w = _f32(w["router_w"])
        self.router_bias = None if w.get("router_bias") is None else _f32(w["router_bias"])
        self.gate = [None] * E
        self.up = [None] * E
        self.down = [None] * E
        # NVFP4 experts: one global scale per expert gate/up pair and per down (R20)
        self.gate_g = np.ones(E, np.float32)
        self.down_g = np.ones(E, np.float32)
        # and static global scales of the experts' NVFP4 inputs z and h
        self.act_gz = float(w.get("act_gz", 1.0))
        self.act_gh = float(w.get("act_gh", 1.0))
        self.set_experts(w, range(E))

    def set_experts(self, w, experts):
        for e in experts:
            g = w["gate"][e] if w.get("gate") is not None else None
            if g is None:
                continue
            if self.ex_fmt in EXT:
                # given as GGUF blocks (uint8 rows)
                self.gate[e] = np.ascontiguousarray(g, np.uint8)
                self.up[e] = np.ascontiguousarray(w["up"][e], np.uint8)
                self.down[e] = np.ascontiguousarray(w["down"][e], np.uint8)
                continue
            if self.ex_fmt == NVFP4:
                gu = np.concatenate([_f32(g).ravel(), _f32(w["up"][e]).ravel()])
                self.gate_g[e] = nvfp4_global(gu)
                self.down_g[e] = nvfp4_global(w["down"][e])
                self.gate[e] = quantize_nvfp4(g, self.gate_g[e])
                self.up[e] = quantize_nvfp4(w["up"][e], self.gate_g[e])
                self.down[e] = quantize_nvfp4(w["down"][e], self.down_g[e])
                continue
            self.gate[e] = quantize(self.ex_fmt, g)
            self.up[e] = quantize(self.ex_fmt, w["up"][e])
            self.down[e] = quantize(self.ex_fmt, w["down"][e])

    def _struct(self):
        E = self.E
        arr = ctypes.c_void_p * E
        self._g = arr(*[_p(a) for a in self.gate])
        self._u = arr(*[_p(a) for a in self.up])
        self._d = arr(*[_p(a) for a in self.down])
        return OrcLayer(self.H, self.L, self.E, self.k, self.I, self.du_fmt, self.ex_fmt,
                        _p(self.D), _p(self.U), _p(self.router_w), _p(self.router_bias),
                        ctypes.cast(self._g, P), ctypes.cast(self._u, P),
                        ctypes.cast(self._d, P), _p(self.gate_g), _p(self.gate_g),
                        _p(self.down_g), self.act_gz, self.act_gh)

    def route(self, x):
        x = _f32(x)
        T = x.shape[0]
        idx = np.empty((T, self.k), np.int32)
        w = np.empty((T, self.k), np.float32)
        s = self._struct()
        rc = lib().orc_route(ctypes.byref(s), _p(x), T, _p(idx), _p(w))
        if rc:
            raise ValueError("orc_route failed: %d" % rc)
        return idx, w

    def forward(self, x, trace: bool = False):
        x = _f32(x)
        T = x.shape[0]
        H, L, E, k, I = self.H, self.L, self.E, self.k, self.I
        P_ = T * k
        y = np.empty((T, H), np.float32)
        tr = None
        bufs = {}
        if trace:
            xb = 18 if self.ex_fmt == NVFP4 else 36
            bufs = dict(
                xq=np.empty((T, H // 32 * 36), np.uint8), z=np.empty((T, L), np.float32),
                logits=np.empty((T, E), np.float32), idx=np.empty((T, k), np.int32),
                w=np.empty((T, k), np.float32), zq=np.empty((T, L // 32 * xb), np.uint8),
                counts=np.empty(E, np.int32), offsets=np.empty(E + 1, np.int32),
                perm=np.empty(P_, np.int32), pos=np.empty(P_, np.int32),
                g=np.empty((P_, I), np.float32), u=np.empty((P_, I), np.float32),
                hq=np.empty((P_, I // 32 * xb), np.uint8), o=np.empty((P_, L), np.float32),
                y_lat=np.empty((T, L), np.float32), ylq=np.empty((T, L // 32 * 36), np.uint8))
            tr = OrcTrace(**{n: _p(a) for n, a in bufs.items()})
        s = self._struct()
        rc = lib().orc_moe_layer(ctypes.byref(s), _p(x), T, _p(y),
                                 ctypes.byref(tr) if tr is not None else None)
        if rc:
            raise ValueError("orc_moe_layer failed: %d" % rc)
        if trace:
            bufs["y"] = y
            return bufs
        return y
