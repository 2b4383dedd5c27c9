"""ctypes binding of libelq.so (the C ABI in include/elq.h).

Argument marshalling only: every function here hands torch tensors' device
pointers and the current CUDA stream to one C entry point and raises if it
returns an error status.  All computation runs in the library's CUDA kernels;
there is no fallback of any kind, so a missing or unloadable library raises.
"""
from __future__ import annotations

import ctypes
import os

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libelq.so")

F32, Q4_0, Q5_1, Q8_0, Q8_1, Q3_K, Q4_K, Q5_K, BF16, NVFP4 = 0, 2, 7, 8, 9, 11, 12, 13, 30, 100
LAYER_FUSED = 1            # elq_layer.flags: small T as one persistent kernel
FMT = {"q8_0": Q8_0, "q4_0": Q4_0, "nvfp4": NVFP4, "q5_1": Q5_1, "q3_k": Q3_K, "q4_k": Q4_K, "q5_k": Q5_K}
SLAB = {Q8_0: 4096, Q4_0: 2048, NVFP4: 2048, Q5_1: 2560, Q3_K: 2048, Q4_K: 2048, Q5_K: 2560}   # code bytes per (tile, block)
SCALE_SLAB = {NVFP4: 512, Q5_1: 512, Q3_K: 512, Q4_K: 512, Q5_K: 512}                       # scale bytes per (tile, block)
EXT = (Q5_1, Q3_K, Q4_K, Q5_K)


class ElqError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__("%s: %s (%d)" % (what, _lib().elq_status_string(status).decode(), status))


class QMat(ctypes.Structure):
    _fields_ = [("fmt", ctypes.c_int32), ("n_rows", ctypes.c_int32), ("k", ctypes.c_int32),
                ("gs_rows", ctypes.c_int32), ("q", ctypes.c_void_p), ("d", ctypes.c_void_p),
                ("gs", ctypes.c_void_p), ("q16", ctypes.c_void_p)]


class LayerC(ctypes.Structure):
    _fields_ = [("H", ctypes.c_int32), ("L", ctypes.c_int32), ("E", ctypes.c_int32),
                ("k", ctypes.c_int32), ("I", ctypes.c_int32), ("flags", ctypes.c_int32),
                ("D", QMat), ("U", QMat), ("router_w", ctypes.c_void_p),
                ("router_bias", ctypes.c_void_p), ("gate_up", QMat), ("down", QMat),
                ("act_gz", ctypes.c_float), ("act_gh", ctypes.c_float)]


_L = None
V, I32, I64, SZ = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t

SIGNATURES = {
    "elq_status_string": (ctypes.c_char_p, [I32]),
    "elq_version": (I32, []),
    "elq_arena_bytes": (SZ, [I32, I32, I32, ctypes.POINTER(SZ), ctypes.POINTER(SZ)]),
    "elq_arena_pack": (I32, [I32, V, I32, I32, V, V, V]),
    "elq_f16_bytes": (SZ, [V]),
    "elq_pack_f16": (I32, [V, V, V]),
    "elq_quantize_weights": (I32, [I32, V, I32, I32, V, V, V]),
    "elq_quantize_gate_up": (I32, [I32, V, V, I32, I32, I32, V, V, V]),
    "elq_quantize_q8_1": (I32, [V, I32, I64, I64, V, V]),
    "elq_quantize_nvfp4": (I32, [V, I32, I64, I64, ctypes.c_float, V, V]),
    "elq_router_topk": (I32, [V, V, V, I32, I32, I32, I32, V, V, V, V]),
    "elq_route_bucket": (I32, [V, I32, I32, I32, V, V, V, V, V]),
    "elq_latent_proj_workspace_bytes": (SZ, [ctypes.POINTER(QMat), I32]),
    "elq_latent_proj": (I32, [ctypes.POINTER(QMat), V, I32, V, V, SZ, V]),
    "elq_latent_proj_noalloc": (I32, [ctypes.POINTER(QMat), V, I32, V, V]),
    "elq_latent_proj_noalloc_status": (I32, [V]),
    "elq_moe_experts_grouped": (I32, [ctypes.POINTER(LayerC), V, V, V, I32, V, V, SZ, V]),
    "elq_workspace_bytes": (SZ, [ctypes.POINTER(LayerC), I32]),
    "elq_moe_layer": (I32, [ctypes.POINTER(LayerC), V, I32, I32, V, V, SZ, V]),
    "elq_moe_stack": (I32, [ctypes.POINTER(LayerC), I32, V, I32, I32, V, V, SZ, V]),
    "elq_stack_workspace_bytes": (SZ, [ctypes.POINTER(LayerC), I32]),
    "elq_workspace_status": (I32, [V, V]),
    "elq_layer_kernel_count": (I32, [ctypes.POINTER(LayerC), I32]),
    "elq_workspace_view": (I32, [ctypes.POINTER(LayerC), I32, I32, ctypes.POINTER(SZ), ctypes.POINTER(SZ)]),
    "elq_moe_layer_profiled": (I32, [ctypes.POINTER(LayerC), V, I32, I32, V, V, SZ, V, I32, V]),
    "elq_test_block_isums": (I32, [I32, V, V, I64, V, V, V]),
    "elq_test_expf": (I32, [V, V, I64, V]),
    "elq_test_mma_i8_rate": (I32, [I32, V, V, V]),
    "elq_test_mma_f16_rate": (I32, [I32, V, V, V]),
    "elq_test_mma_nvf4_rate": (I32, [I32, I32, I32, V, V, V]),
    "elq_sm_count": (I32, []),
    "elq_test_f32x2_rate": (I32, [I32, V, V]),
    "elq_test_fused_timeout": (I32, [ctypes.POINTER(LayerC), V, I32, I32, V, V, SZ, ctypes.c_uint64, V]),
}


def _lib() -> ctypes.CDLL:
    global _L
    if _L is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError("libelq.so is not built (%s); run `python -m quantized_latent_moe_b200.build`"
                               % LIB_PATH)
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _L = L
    return _L


lib = _lib


def _ck(status: int, what: str):
    if status != 0:
        raise ElqError(status, what)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _dev_empty(nbytes: int, device, align: int = 256) -> torch.Tensor:
    t = torch.empty(nbytes + align, dtype=torch.uint8, device=device)
    off = (-t.data_ptr()) % align
    return t[off:off + nbytes]


# --------------------------------------------------------------------------
# arena matrices

class QMatrix:
    """One matrix in the device tile-slab arena (codes ``q`` and scales ``d``)."""

    def __init__(self, fmt: int, n_rows: int, k: int, device="cuda", gs_rows: int = 0):
        qb, db = SZ(), SZ()
        if not _lib().elq_arena_bytes(fmt, n_rows, k, ctypes.byref(qb), ctypes.byref(db)):
            raise ElqError(-2, "elq_arena_bytes")
        self.fmt, self.n_rows, self.k = fmt, n_rows, k
        self.q = _dev_empty(qb.value, device)
        self.d = _dev_empty(db.value, device)
        # NVFP4: one fp32 global scale per gs_rows rows (all rows by default)
        self.gs_rows = (gs_rows or n_rows) if fmt == NVFP4 else 0
        self.gs = (torch.ones(n_rows // self.gs_rows, dtype=torch.float32, device=device)
                   if fmt == NVFP4 else None)
        self.q16 = None         # fp16 codes for the fp16-operand tensor-core GEMMs (Q8_0), or None

    @classmethod
    def from_f32(cls, w: torch.Tensor, fmt: int, stream=None) -> "QMatrix":
        w = w.contiguous()
        m = cls(fmt, w.shape[0], w.shape[1], w.device)
        _ck(_lib().elq_quantize_weights(fmt, _ptr(w), m.n_rows, m.k, _ptr(m.q), _ptr(m.d),
                                        _stream(stream)), "elq_quantize_weights")
        return m

    @classmethod
    def from_aos(cls, aos: torch.Tensor, fmt: int, n_rows: int, k: int, stream=None) -> "QMatrix":
        m = cls(fmt, n_rows, k, aos.device)
        _ck(_lib().elq_arena_pack(fmt, _ptr(aos), n_rows, k, _ptr(m.q), _ptr(m.d), _stream(stream)),
            "elq_arena_pack")
        return m

    def struct(self) -> QMat:
        return QMat(self.fmt, self.n_rows, self.k, self.gs_rows, self.q.data_ptr(), self.d.data_ptr(),
                    None if self.gs is None else self.gs.data_ptr(),
                    None if self.q16 is None else self.q16.data_ptr())

    def pack_f16(self, stream=None) -> "QMatrix":
        """Fills ``q16`` with the codes widened to fp16 (elq_pack_f16); Q8_0 only."""
        m = self.struct()
        m.q16 = None
        n = _lib().elq_f16_bytes(ctypes.byref(m))
        if not n:
            raise ElqError(-2, "elq_f16_bytes")
        self.q16 = _dev_empty(n, self.q.device)
        _ck(_lib().elq_pack_f16(ctypes.byref(m), _ptr(self.q16), _stream(stream)), "elq_pack_f16")
        return self

    def drop_f16(self):
        self.q16 = None


class Layer:
    """Device weights of one latent-MoE layer, quantised by the library."""

    def __init__(self, H, L, E, k, I, D: QMatrix, U: QMatrix, router_w, router_bias,
                 gate_up: QMatrix, down: QMatrix):
        self.H, self.L, self.E, self.k, self.I = H, L, E, k, I
        self.D, self.U, self.gate_up, self.down = D, U, gate_up, down
        self.router_w = router_w.contiguous()
        self.router_bias = None if router_bias is None else router_bias.contiguous()
        self.flags = 0          # LAYER_FUSED: small T as one persistent kernel
        # NVFP4 experts: static global scales of their inputs z and h
        self.act_gz, self.act_gh = 1.0, 1.0
        self._ws = {}

    @classmethod
    def allocate(cls, H, L, E, k, I, du_fmt, ex_fmt, router_w, router_bias, device="cuda"):
        return cls(H, L, E, k, I, QMatrix(du_fmt, L, H, device), QMatrix(du_fmt, H, L, device),
                   router_w, router_bias, QMatrix(ex_fmt, E * 2 * I, L, device, gs_rows=2 * I),
                   QMatrix(ex_fmt, E * L, I, device, gs_rows=L))

    def enable_f16(self, stream=None):
        """Builds the fp16 codes of every Q8_0 matrix of the layer, so that calls
        with T >= 16 multiply fp16 operands (same results; twice the codes' bytes
        held in addition)."""
        for m in (self.D, self.U, self.gate_up, self.down):
            if m.fmt == FMT["q8_0"]:
                m.pack_f16(stream)
        self._ws = {}
        return self

    def disable_f16(self):
        for m in (self.D, self.U, self.gate_up, self.down):
            m.drop_f16()
        self._ws = {}
        return self

    def set_dense(self, D: torch.Tensor, U: torch.Tensor, stream=None):
        for m, w in ((self.D, D), (self.U, U)):
            w = w.contiguous()
            _ck(_lib().elq_quantize_weights(m.fmt, _ptr(w), m.n_rows, m.k, _ptr(m.q), _ptr(m.d),
                                            _stream(stream)), "elq_quantize_weights")

    def set_experts(self, e0: int, gate: torch.Tensor, up: torch.Tensor, down: torch.Tensor,
                    stream=None):
        """Quantise experts e0 .. e0+n-1 from fp32 gate/up [n, I, L] and down [n, L, I]."""
        n = gate.shape[0]
        gu, dn = self.gate_up, self.down
        per_q = (2 * self.I // 128) * (self.L // 32) * SLAB[gu.fmt]
        per_d = (2 * self.I // 128) * (self.L // 32) * 256
        gate, up, down = gate.contiguous(), up.contiguous(), down.contiguous()
        _ck(_lib().elq_quantize_gate_up(gu.fmt, _ptr(gate), _ptr(up), n, self.I, self.L,
                                        ctypes.c_void_p(gu.q.data_ptr() + e0 * per_q),
                                        ctypes.c_void_p(gu.d.data_ptr() + e0 * per_d),
                                        _stream(stream)), "elq_quantize_gate_up")
        dq = (self.L // 128) * (self.I // 32) * SLAB[dn.fmt]
        dd = (self.L // 128) * (self.I // 32) * 256
        _ck(_lib().elq_quantize_weights(dn.fmt, _ptr(down.view(n * self.L, self.I)), n * self.L,
                                        self.I, ctypes.c_void_p(dn.q.data_ptr() + e0 * dq),
                                        ctypes.c_void_p(dn.d.data_ptr() + e0 * dd),
                                        _stream(stream)), "elq_quantize_weights")

    def set_experts_nvfp4(self, e0: int, gate: torch.Tensor, up: torch.Tensor, down: torch.Tensor,
                          g_gate_up: torch.Tensor, g_down: torch.Tensor, stream=None):
        """NVFP4 experts e0 .. e0+n-1 from fp32 gate/up [n, I, L] and down [n, L, I]
        under the given per-expert global scales (fp32 [n] each): the library's
        NVFP4 quantiser, then the arena packing (gate and up interleaved by
        64-row halves)."""
        n, I, L = gate.shape
        gu, dn = self.gate_up, self.down
        # interleave: tile j of expert e holds gate rows 64j.. then up rows 64j..
        gi = torch.stack([gate.reshape(n, I // 64, 64, L), up.reshape(n, I // 64, 64, L)], dim=2)
        gi = gi.reshape(n, 2 * I, L).contiguous()
        aos_gu = torch.empty(n, 2 * I, L // 32 * 18, dtype=torch.uint8, device=gate.device)
        aos_dn = torch.empty(n, L, I // 32 * 18, dtype=torch.uint8, device=gate.device)
        for e in range(n):
            _ck(_lib().elq_quantize_nvfp4(_ptr(gi[e]), F32, 2 * I, L, float(g_gate_up[e]), _ptr(aos_gu[e]),
                                          _stream(stream)), "elq_quantize_nvfp4")
            de = down[e].contiguous()
            _ck(_lib().elq_quantize_nvfp4(_ptr(de), F32, L, I, float(g_down[e]), _ptr(aos_dn[e]),
                                          _stream(stream)), "elq_quantize_nvfp4")
        per_q = (2 * I // 128) * (L // 32) * SLAB[NVFP4]
        per_d = (2 * I // 128) * (L // 32) * SCALE_SLAB[NVFP4]   # per-row scales, then the scale atoms
        _ck(_lib().elq_arena_pack(NVFP4, _ptr(aos_gu), n * 2 * I, L,
                                  ctypes.c_void_p(gu.q.data_ptr() + e0 * per_q),
                                  ctypes.c_void_p(gu.d.data_ptr() + e0 * per_d), _stream(stream)),
            "elq_arena_pack")
        dq = (L // 128) * (I // 32) * SLAB[NVFP4]
        dd = (L // 128) * (I // 32) * SCALE_SLAB[NVFP4]
        _ck(_lib().elq_arena_pack(NVFP4, _ptr(aos_dn), n * L, I, ctypes.c_void_p(dn.q.data_ptr() + e0 * dq),
                                  ctypes.c_void_p(dn.d.data_ptr() + e0 * dd), _stream(stream)),
            "elq_arena_pack")
        gu.gs[e0:e0 + n].copy_(g_gate_up)
        dn.gs[e0:e0 + n].copy_(g_down)

    def set_expert_blocks(self, e0: int, gate: torch.Tensor, up: torch.Tensor, down: torch.Tensor, stream=None):
        """Experts e0 .. e0+n-1 from GGUF blocks (uint8 rows) of the layer's
        expert format (Q5_1, Q4_K, Q5_K): gate / up [n, I, row bytes of L],
        down [n, L, row bytes of I], packed into the arena (gate and up
        interleaved by 64-row halves)."""
        n, I = gate.shape[0], self.I
        gu, dn = self.gate_up, self.down
        rb = gate.shape[2]
        gi = torch.stack([gate.reshape(n, I // 64, 64, rb), up.reshape(n, I // 64, 64, rb)], dim=2)
        gi = gi.reshape(n * 2 * I, rb).contiguous()
        per_q = (2 * I // 128) * (self.L // 32) * SLAB[gu.fmt]
        per_d = (2 * I // 128) * (self.L // 32) * SCALE_SLAB[gu.fmt]
        _ck(_lib().elq_arena_pack(gu.fmt, _ptr(gi), n * 2 * I, self.L,
                                  ctypes.c_void_p(gu.q.data_ptr() + e0 * per_q),
                                  ctypes.c_void_p(gu.d.data_ptr() + e0 * per_d), _stream(stream)), "elq_arena_pack")
        dq = (self.L // 128) * (I // 32) * SLAB[dn.fmt]
        dd = (self.L // 128) * (I // 32) * SCALE_SLAB[dn.fmt]
        down = down.reshape(n * self.L, -1).contiguous()
        _ck(_lib().elq_arena_pack(dn.fmt, _ptr(down), n * self.L, I, ctypes.c_void_p(dn.q.data_ptr() + e0 * dq),
                                  ctypes.c_void_p(dn.d.data_ptr() + e0 * dd), _stream(stream)), "elq_arena_pack")

    def struct(self) -> LayerC:
        return LayerC(self.H, self.L, self.E, self.k, self.I, self.flags, self.D.struct(), self.U.struct(),
                      self.router_w.data_ptr(),
                      None if self.router_bias is None else self.router_bias.data_ptr(),
                      self.gate_up.struct(), self.down.struct(), self.act_gz, self.act_gh)

    def kernel_count(self, T: int) -> int:
        s = self.struct()
        return int(_lib().elq_layer_kernel_count(ctypes.byref(s), T))

    def workspace_bytes(self, T: int) -> int:
        s = self.struct()
        return int(_lib().elq_workspace_bytes(ctypes.byref(s), T))

    def workspace(self, T: int) -> torch.Tensor:
        """A zero-filled device workspace for T tokens (cached per T and flags)."""
        key = (T, self.flags)
        ws = self._ws.get(key)
        if ws is None:
            n = self.workspace_bytes(T)
            if n == 0:
                raise ElqError(-1, "elq_workspace_bytes")
            ws = torch.zeros(n + 256, dtype=torch.uint8, device=self.router_w.device)
            off = (-ws.data_ptr()) % 256
            ws = ws[off:off + n]
            self._ws[key] = ws
        return ws

    def stack_workspace(self, T: int) -> torch.Tensor:
        """A zero-filled workspace for elq_moe_stack over layers of this shape."""
        key = ("stack", T)
        ws = self._ws.get(key)
        if ws is None:
            s = self.struct()
            n = int(_lib().elq_stack_workspace_bytes(ctypes.byref(s), T))
            if n == 0:
                raise ElqError(-1, "elq_stack_workspace_bytes")
            ws = torch.zeros(n + 256, dtype=torch.uint8, device=self.router_w.device)
            off = (-ws.data_ptr()) % 256
            ws = ws[off:off + n]
            self._ws[key] = ws
        return ws

    def share_workspace(self, T: int, ws: torch.Tensor):
        """Use `ws` (another layer's workspace of the same shape) for T tokens:
        calls that run one after another on one stream may share it."""
        self._ws[(T, self.flags)] = ws


# --------------------------------------------------------------------------
# hot-path entry points

def quantize_q8_1(x: torch.Tensor, stream=None) -> torch.Tensor:
    x = x.contiguous()
    rows, cols = x.shape
    xt = {torch.float32: F32, torch.bfloat16: BF16}[x.dtype]
    out = torch.empty(rows, cols // 32 * 36, dtype=torch.uint8, device=x.device)
    _ck(_lib().elq_quantize_q8_1(_ptr(x), xt, rows, cols, _ptr(out), _stream(stream)),
        "elq_quantize_q8_1")
    return out


def quantize_nvfp4(x: torch.Tensor, g: float, stream=None) -> torch.Tensor:
    """NVFP4 blocks (18 bytes per 32 values) of x [rows, cols] under global scale g."""
    x = x.contiguous()
    rows, cols = x.shape
    xt = {torch.float32: F32, torch.bfloat16: BF16}[x.dtype]
    out = torch.empty(rows, cols // 32 * 18, dtype=torch.uint8, device=x.device)
    _ck(_lib().elq_quantize_nvfp4(_ptr(x), xt, rows, cols, float(g), _ptr(out), _stream(stream)),
        "elq_quantize_nvfp4")
    return out


def router_topk(z: torch.Tensor, w_router: torch.Tensor, bias, k: int, stream=None):
    T, L = z.shape
    E = w_router.shape[0]
    idx = torch.empty(T, k, dtype=torch.int32, device=z.device)
    w = torch.empty(T, k, dtype=torch.float32, device=z.device)
    logits = torch.empty(T, E, dtype=torch.float32, device=z.device)
    _ck(_lib().elq_router_topk(_ptr(z), _ptr(w_router), _ptr(bias), T, L, E, k, _ptr(idx), _ptr(w),
                               _ptr(logits), _stream(stream)), "elq_router_topk")
    return idx, w, logits


def route_bucket(idx: torch.Tensor, E: int, stream=None):
    T, k = idx.shape
    dev = idx.device
    counts = torch.empty(E, dtype=torch.int32, device=dev)
    offsets = torch.empty(E + 1, dtype=torch.int32, device=dev)
    perm = torch.empty(T * k, dtype=torch.int32, device=dev)
    pos = torch.empty(T * k, dtype=torch.int32, device=dev)
    _ck(_lib().elq_route_bucket(_ptr(idx.contiguous()), T, k, E, _ptr(counts), _ptr(offsets),
                                _ptr(perm), _ptr(pos), _stream(stream)), "elq_route_bucket")
    return counts, offsets, perm, pos


def latent_proj(m: QMatrix, xq: torch.Tensor, T: int, ws=None, stream=None) -> torch.Tensor:
    s = m.struct()
    y = torch.empty(T, m.n_rows, dtype=torch.float32, device=m.q.device)
    if ws is None:
        n = _lib().elq_latent_proj_workspace_bytes(ctypes.byref(s), T)
        ws = torch.zeros(n + 256, dtype=torch.uint8, device=m.q.device)
        off = (-ws.data_ptr()) % 256
        ws = ws[off:off + n]
    _ck(_lib().elq_latent_proj(ctypes.byref(s), _ptr(xq), T, _ptr(y), _ptr(ws), ws.numel(),
                               _stream(stream)), "elq_latent_proj")
    return y


def latent_proj_noalloc(m: QMatrix, xq: torch.Tensor, T: int, y: torch.Tensor | None = None,
                        stream=None) -> torch.Tensor:
    """elq_latent_proj_noalloc: the projection with the library's own static
    scratch instead of a workspace (for callers that cannot allocate).  Calls
    share that scratch, so they must not overlap on the GPU."""
    s = m.struct()
    if y is None:
        y = torch.empty(T, m.n_rows, dtype=torch.float32, device=m.q.device)
    _ck(_lib().elq_latent_proj_noalloc(ctypes.byref(s), _ptr(xq), T, _ptr(y), _stream(stream)),
        "elq_latent_proj_noalloc")
    return y


def latent_proj_noalloc_status(stream=None) -> int:
    """Blocking: the outcome of the last elq_latent_proj_noalloc call on this
    device (0, or the timeout status)."""
    return int(_lib().elq_latent_proj_noalloc_status(_stream(stream)))


def moe_experts_grouped(layer: Layer, zq: torch.Tensor, idx: torch.Tensor, w: torch.Tensor,
                        stream=None) -> torch.Tensor:
    T = idx.shape[0]
    s = layer.struct()
    ws = layer.workspace(T)
    y = torch.empty(T, layer.L, dtype=torch.float32, device=zq.device)
    _ck(_lib().elq_moe_experts_grouped(ctypes.byref(s), _ptr(zq), _ptr(idx.contiguous()),
                                       _ptr(w.contiguous()), T, _ptr(y), _ptr(ws), ws.numel(),
                                       _stream(stream)), "elq_moe_experts_grouped")
    return y


def moe_layer(layer: Layer, x: torch.Tensor, y: torch.Tensor | None = None, ws=None,
              stream=None) -> torch.Tensor:
    x = x.contiguous()
    T = x.shape[0]
    xt = {torch.float32: F32, torch.bfloat16: BF16}[x.dtype]
    if y is None:
        y = torch.empty(T, layer.H, dtype=torch.float32, device=x.device)
    if ws is None:
        ws = layer.workspace(T)
    s = layer.struct()
    _ck(_lib().elq_moe_layer(ctypes.byref(s), _ptr(x), xt, T, _ptr(y), _ptr(ws), ws.numel(),
                             _stream(stream)), "elq_moe_layer")
    return y


def moe_stack(layers, x: torch.Tensor, h: torch.Tensor | None = None, ws=None, stream=None) -> torch.Tensor:
    """h = fp32(x), then h = h + layer(rms(h)) for each layer in turn (one
    residual stream, fp32).  All layers of one shape; one workspace serves them."""
    x = x.contiguous()
    T = x.shape[0]
    xt = {torch.float32: F32, torch.bfloat16: BF16}[x.dtype]
    if h is None:
        h = torch.empty(T, layers[0].H, dtype=torch.float32, device=x.device)
    if ws is None:
        ws = layers[0].stack_workspace(T)
    arr = (LayerC * len(layers))(*[ly.struct() for ly in layers])
    _ck(_lib().elq_moe_stack(arr, len(layers), _ptr(x), xt, T, _ptr(h), _ptr(ws), ws.numel(), _stream(stream)),
        "elq_moe_stack")
    return h


def moe_layer_profiled(layer: Layer, x: torch.Tensor, y: torch.Tensor, events, ws=None,
                       stream=None):
    """elq_moe_layer with a CUDA event recorded before and after each kernel."""
    T = x.shape[0]
    xt = {torch.float32: F32, torch.bfloat16: BF16}[x.dtype]
    if ws is None:
        ws = layer.workspace(T)
    arr = (ctypes.c_void_p * len(events))(*[e.cuda_event for e in events])
    s = layer.struct()
    _ck(_lib().elq_moe_layer_profiled(ctypes.byref(s), _ptr(x), xt, T, _ptr(y), _ptr(ws), ws.numel(),
                                      arr, len(events), _stream(stream)), "elq_moe_layer_profiled")
    return y


VIEWS = {"xq": 0, "z": 1, "zq": 2, "logits": 3, "idx": 4, "weights": 5, "counts": 6, "offsets": 7,
         "perm": 8, "pos": 9, "hq": 10, "o": 11, "y_lat": 12, "ylq": 13, "n_act": 14}
VIEW_DTYPE = {"z": torch.float32, "logits": torch.float32, "weights": torch.float32, "o": torch.float32,
              "y_lat": torch.float32, "idx": torch.int32, "counts": torch.int32, "offsets": torch.int32,
              "perm": torch.int32, "pos": torch.int32, "n_act": torch.int32}


def workspace_view(layer: Layer, T: int, name: str, ws=None) -> torch.Tensor:
    """An intermediate of the last elq_moe_layer call on ``ws`` (a view; read
    it after the stream has reached the end of that call)."""
    if ws is None:
        ws = layer.workspace(T)
    off, n = SZ(), SZ()
    s = layer.struct()
    _ck(_lib().elq_workspace_view(ctypes.byref(s), T, VIEWS[name], ctypes.byref(off), ctypes.byref(n)),
        "elq_workspace_view")
    v = ws[off.value:off.value + n.value]
    dt = VIEW_DTYPE.get(name)
    return v.view(dt) if dt is not None else v


def workspace_status(ws: torch.Tensor, stream=None) -> int:
    return int(_lib().elq_workspace_status(_ptr(ws), _stream(stream)))


def test_block_isums(wfmt: int, w_aos: torch.Tensor, xq: torch.Tensor, n: int, stream=None):
    isum = torch.empty(n, dtype=torch.int32, device=w_aos.device)
    term = torch.empty(n, dtype=torch.float32, device=w_aos.device)
    _ck(_lib().elq_test_block_isums(wfmt, _ptr(w_aos), _ptr(xq), n, _ptr(isum), _ptr(term),
                                    _stream(stream)), "elq_test_block_isums")
    return isum, term


def test_fused_timeout(layer: Layer, x: torch.Tensor, ws: torch.Tensor, budget_ns: int,
                       stream=None) -> int:
    """The fused layer kernel with its routing withheld: returns the call's
    status (the kernel's own outcome is in the workspace error word)."""
    x = x.contiguous()
    T = x.shape[0]
    xt = {torch.float32: F32, torch.bfloat16: BF16}[x.dtype]
    y = torch.empty(T, layer.H, dtype=torch.float32, device=x.device)
    s = layer.struct()
    return int(_lib().elq_test_fused_timeout(ctypes.byref(s), _ptr(x), xt, T, _ptr(y), _ptr(ws), ws.numel(),
                                             budget_ns, _stream(stream)))


def test_mma_i8_rate(n_mma: int, device="cuda", stream=None):
    """Launches the int8 tensor-core rate kernel (elq_test_mma_i8_rate) on the
    current stream; returns (sink, err) device tensors.  The caller times it."""
    n = int(_lib().elq_sm_count())
    sink = torch.zeros(n, dtype=torch.int32, device=device)
    err = torch.zeros(1, dtype=torch.int32, device=device)
    _ck(_lib().elq_test_mma_i8_rate(n_mma, _ptr(sink), _ptr(err), _stream(stream)), "elq_test_mma_i8_rate")
    return sink, err


def test_mma_f16_rate(n_mma: int, device="cuda", stream=None):
    """Launches the fp16 tensor-core rate kernel (elq_test_mma_f16_rate) on the
    current stream; returns (sink, err) device tensors.  The caller times it."""
    n = int(_lib().elq_sm_count())
    sink = torch.zeros(n, dtype=torch.int32, device=device)
    err = torch.zeros(1, dtype=torch.int32, device=device)
    _ck(_lib().elq_test_mma_f16_rate(n_mma, _ptr(sink), _ptr(err), _stream(stream)), "elq_test_mma_f16_rate")
    return sink, err


def test_mma_nvf4_rate(n_mma: int, n_cols: int = 256, cp_each: bool = False, device="cuda", stream=None):
    """Launches the fp4 block-scaled tensor-core rate kernel
    (elq_test_mma_nvf4_rate) on the current stream; returns (sink, err)."""
    n = int(_lib().elq_sm_count())
    sink = torch.zeros(n, dtype=torch.int32, device=device)
    err = torch.zeros(1, dtype=torch.int32, device=device)
    _ck(_lib().elq_test_mma_nvf4_rate(n_mma, n_cols, int(cp_each), _ptr(sink), _ptr(err), _stream(stream)),
        "elq_test_mma_nvf4_rate")
    return sink, err


def test_f32x2_rate(n: int, device="cuda", stream=None) -> torch.Tensor:
    """Launches the packed-fp32 rate kernel (elq_test_f32x2_rate) on the
    current stream; returns its sink.  The caller times it."""
    sink = torch.empty(2 * sm_count() * 1024, dtype=torch.float32, device=device)
    _ck(_lib().elq_test_f32x2_rate(n, _ptr(sink), _stream(stream)), "elq_test_f32x2_rate")
    return sink


def sm_count() -> int:
    return int(_lib().elq_sm_count())


def test_expf(x: torch.Tensor, stream=None) -> torch.Tensor:
    out = torch.empty_like(x)
    _ck(_lib().elq_test_expf(_ptr(x), _ptr(out), x.numel(), _stream(stream)), "elq_test_expf")
    return out
