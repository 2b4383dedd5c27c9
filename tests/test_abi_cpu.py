"""The C-ABI library on a machine without a GPU: it loads, exports every
symbol include/elq.h declares, reports its sizes, and refuses bad arguments on
the host before any launch (every case here fails validation, so nothing is
ever enqueued)."""
import ctypes
import os
import re

import pytest

from quantized_latent_moe_b200 import build, elq

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    build.build()
    return elq.lib()


def declared_functions():
    src = open(os.path.join(ROOT, "include", "elq.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(elq_[a-z0-9_]+)\s*\(", src)))


def test_exports_every_declared_symbol(L):
    names = declared_functions()
    assert len(names) >= 17
    for n in names:
        assert hasattr(L, n), n
    assert set(names) == set(elq.SIGNATURES)


def test_status_strings_and_version(L):
    assert L.elq_version() == 3
    assert L.elq_status_string(0) == b"ok"
    assert L.elq_status_string(-4).startswith(b"workspace")
    assert L.elq_status_string(123) == b"unknown status"


def test_arena_bytes(L):
    q, d = elq.SZ(), elq.SZ()
    # an expert of the pages' synthetic 2560/640 shape: gate+up as 1280 rows? use the D of the decode shape
    assert L.elq_arena_bytes(8, 1792, 4096, ctypes.byref(q), ctypes.byref(d)) == 1792 * 128 * 34
    assert q.value == 1792 * 128 * 32 and d.value == 1792 * 128 * 2
    assert L.elq_arena_bytes(2, 1280, 3072, None, None) == 1280 * 96 * 18
    assert L.elq_arena_bytes(8, 100, 64, None, None) == 0          # rows not a multiple of 128
    assert L.elq_arena_bytes(8, 128, 48, None, None) == 0          # k not a multiple of 32
    assert L.elq_arena_bytes(3, 128, 64, None, None) == 0          # unknown format


def _qm(fmt, rows, k, q=1 << 20, d=2 << 20):
    return elq.QMat(fmt, rows, k, 0, q, d)


def _layer(H=512, L_=256, E=8, k=2, I=256, fmt=8, **over):
    base = 1 << 24
    ly = elq.LayerC(H, L_, E, k, I, 0, _qm(fmt, L_, H, base, base + 4096), _qm(fmt, H, L_, base + 8192, base + 12288),
                    base + 16384, None, _qm(fmt, E * 2 * I, L_, base + 20480, base + 24576),
                    _qm(fmt, E * L_, I, base + 28672, base + 32768))
    for k_, v in over.items():
        setattr(ly, k_, v)
    return ly


def test_layer_validation(L):
    ws_small = ctypes.c_void_p(1 << 26)
    x = ctypes.c_void_p(1 << 27)
    y = ctypes.c_void_p(1 << 28)
    good = _layer()
    assert L.elq_workspace_bytes(ctypes.byref(good), 4) > 0
    # the separate-kernel sequence by default; one fused kernel on request for
    # T <= 8 and T*k <= 64
    assert L.elq_layer_kernel_count(ctypes.byref(good), 4) == 5
    assert L.elq_layer_kernel_count(ctypes.byref(_layer(flags=1)), 4) == 1
    assert L.elq_layer_kernel_count(ctypes.byref(_layer(k=8, flags=1)), 8) == 1  # 64 pairs
    assert L.elq_layer_kernel_count(ctypes.byref(_layer(k=8, flags=1)), 9) == 6  # T > 8
    assert L.elq_layer_kernel_count(ctypes.byref(_layer(E=128, k=16, flags=1)), 8) == 5  # 128 pairs
    assert L.elq_layer_kernel_count(ctypes.byref(good), 9) == 6
    assert L.elq_layer_kernel_count(ctypes.byref(good), 15) == 6
    assert L.elq_layer_kernel_count(ctypes.byref(good), 16) == 10                # tensor cores from 16 tokens
    assert L.elq_layer_kernel_count(ctypes.byref(_layer(fmt=2)), 32) == 6         # Q4_0 stays on the GEMV path
    assert L.elq_layer_kernel_count(None, 4) == 0
    assert L.elq_layer_kernel_count(ctypes.byref(_layer(L_=2176)), 4) == 0      # router rows: L <= 2048
    assert L.elq_layer_kernel_count(ctypes.byref(_layer(L_=2048)), 4) == 5
    # the fused path keeps its phase flags and counters in the workspace
    assert L.elq_workspace_bytes(ctypes.byref(_layer(flags=1)), 4) > L.elq_workspace_bytes(ctypes.byref(good), 4)
    # unknown flag bits are refused
    assert L.elq_layer_kernel_count(ctypes.byref(_layer(flags=2)), 4) == 0
    assert L.elq_moe_layer(ctypes.byref(_layer(flags=6)), x, 0, 4, y, ws_small, 1 << 30, None) == -1
    # workspace too small -> refused before any launch
    assert L.elq_moe_layer(ctypes.byref(good), x, 0, 4, y, ws_small, 16, None) == -4
    assert L.elq_moe_layer(ctypes.byref(good), x, 0, 4, y, None, 1 << 30, None) == -4
    assert L.elq_moe_layer(ctypes.byref(good), None, 0, 4, y, ws_small, 1 << 30, None) == -1
    assert L.elq_moe_layer(ctypes.byref(good), x, 5, 4, y, ws_small, 1 << 30, None) == -2
    assert L.elq_moe_layer(ctypes.byref(good), ctypes.c_void_p((1 << 27) + 2), 0, 4, y, ws_small, 1 << 30, None) == -3
    assert L.elq_moe_layer(ctypes.byref(_layer(k=9)), x, 0, 4, y, ws_small, 1 << 30, None) == -1
    assert L.elq_moe_layer(ctypes.byref(_layer(fmt=9)), x, 0, 4, y, ws_small, 1 << 30, None) == -2
    assert L.elq_moe_layer(ctypes.byref(_layer(I=96)), x, 0, 4, y, ws_small, 1 << 30, None) == -2
    bad = _layer()
    bad.D = _qm(8, 256, 512, (1 << 20) + 16)
    assert L.elq_moe_layer(ctypes.byref(bad), x, 0, 4, y, ws_small, 1 << 30, None) == -3
    bad = _layer()
    bad.U = _qm(8, 512, 128)
    assert L.elq_moe_layer(ctypes.byref(bad), x, 0, 4, y, ws_small, 1 << 30, None) == -1
    bad = _layer()
    bad.router_w = None
    assert L.elq_moe_layer(ctypes.byref(bad), x, 0, 4, y, ws_small, 1 << 30, None) == -1
    assert L.elq_moe_layer(None, x, 0, 4, y, ws_small, 1 << 30, None) == -1
    assert L.elq_moe_layer(ctypes.byref(good), x, 0, -1, y, ws_small, 1 << 30, None) == -1


def _nv_layer(T_ok=True, **over):
    """A layer with NVFP4 experts (Q8_0 D/U): global scales per expert matrix."""
    ly = _layer(L_=256, I=256)
    base = 1 << 25
    ly.gate_up = elq.QMat(elq.NVFP4, 8 * 2 * 256, 256, 2 * 256, base, base + 4096, base + 8192)
    ly.down = elq.QMat(elq.NVFP4, 8 * 256, 256, 256, base + 12288, base + 16384, base + 20480)
    ly.act_gz, ly.act_gh = 2.0 ** -6, 2.0 ** -6
    for k_, v in over.items():
        setattr(ly, k_, v)
    return ly


def test_nvfp4_layer_validation(L):
    x = ctypes.c_void_p(1 << 27)
    y = ctypes.c_void_p(1 << 28)
    ws = ctypes.c_void_p(1 << 26)
    nv = _nv_layer()
    # the cluster GEMV path, T <= 8 and T * k <= 64 only
    for T in (1, 4, 8):
        assert L.elq_layer_kernel_count(ctypes.byref(nv), T) == 5
        assert L.elq_workspace_bytes(ctypes.byref(nv), T) > 0
    # beyond: the block-scaled tensor cores (D and U on the int8 ones, Q8_0 only)
    for T in (9, 16, 64, 2048):
        assert L.elq_layer_kernel_count(ctypes.byref(nv), T) == 11
        assert L.elq_workspace_bytes(ctypes.byref(nv), T) > 0
    nv4 = _nv_layer()
    nv4.D = _qm(2, 256, 512)
    nv4.U = _qm(2, 512, 256)
    assert L.elq_layer_kernel_count(ctypes.byref(nv4), 4) == 5
    for T in (9, 16, 64):
        assert L.elq_layer_kernel_count(ctypes.byref(nv4), T) == 0
        assert L.elq_moe_layer(ctypes.byref(nv4), x, 0, T, y, ws, 1 << 30, None) == -2
    # the fused flag does not apply: still the five-kernel sequence
    assert L.elq_layer_kernel_count(ctypes.byref(_nv_layer(flags=1)), 4) == 5
    # global scales: present, one per expert matrix; activation scales positive
    bad = _nv_layer()
    bad.gate_up.gs = None
    assert L.elq_moe_layer(ctypes.byref(bad), x, 0, 1, y, ws, 1 << 30, None) == -1
    bad = _nv_layer()
    bad.down.gs_rows = 128
    assert L.elq_moe_layer(ctypes.byref(bad), x, 0, 1, y, ws, 1 << 30, None) == -1
    bad = _nv_layer()
    bad.down.gs = (1 << 25) + 20482
    assert L.elq_moe_layer(ctypes.byref(bad), x, 0, 1, y, ws, 1 << 30, None) == -3
    for v in (0.0, -1.0, float("nan"), float("inf")):
        assert L.elq_moe_layer(ctypes.byref(_nv_layer(act_gh=v)), x, 0, 1, y, ws, 1 << 30, None) == -1
    # both expert matrices NVFP4 or neither; never D or U
    bad = _nv_layer()
    bad.down = _qm(8, 8 * 256, 256)
    assert L.elq_moe_layer(ctypes.byref(bad), x, 0, 1, y, ws, 1 << 30, None) == -2
    bad = _nv_layer()
    bad.D = elq.QMat(elq.NVFP4, 256, 512, 256, 1 << 20, 2 << 20, 3 << 20)
    assert L.elq_moe_layer(ctypes.byref(bad), x, 0, 1, y, ws, 1 << 30, None) == -2
    # whole 8-block chunks: L and I multiples of 256
    bad = _layer(L_=384, I=256)
    base = 1 << 25
    bad.gate_up = elq.QMat(elq.NVFP4, 8 * 512, 384, 512, base, base + 4096, base + 8192)
    bad.down = elq.QMat(elq.NVFP4, 8 * 384, 256, 384, base + 12288, base + 16384, base + 20480)
    bad.act_gz, bad.act_gh = 1.0, 1.0
    assert L.elq_moe_layer(ctypes.byref(bad), x, 0, 1, y, ws, 1 << 30, None) == -2
    # workspace still checked
    assert L.elq_moe_layer(ctypes.byref(nv), x, 0, 1, y, ws, 16, None) == -4


def test_nvfp4_arena_and_quantiser_validation(L):
    q, d = elq.SZ(), elq.SZ()
    # the Q4_0 byte geometry (16 code bytes and a 16-bit scale word per row and
    # block), the scales once more as the tensor cores' atoms
    assert L.elq_arena_bytes(elq.NVFP4, 2048, 1792, ctypes.byref(q), ctypes.byref(d)) == 2048 * 56 * 20
    assert q.value == 2048 * 56 * 16 and d.value == 2048 * 56 * 4
    assert L.elq_arena_bytes(elq.NVFP4, 128, 96, None, None) == 0              # whole 64-value pairs only
    x = ctypes.c_void_p(1 << 27)
    out = ctypes.c_void_p(1 << 28)
    assert L.elq_quantize_nvfp4(x, 0, 4, 64, 0.0, out, None) == -1
    assert L.elq_quantize_nvfp4(x, 0, 4, 64, float("inf"), out, None) == -1
    assert L.elq_quantize_nvfp4(x, 0, 4, 48, 1.0, out, None) == -2
    assert L.elq_quantize_nvfp4(x, 7, 4, 64, 1.0, out, None) == -2
    assert L.elq_quantize_nvfp4(x, 0, 4, 64, 1.0, ctypes.c_void_p((1 << 28) + 1), None) == -3
    assert L.elq_quantize_nvfp4(None, 0, 0, 64, 1.0, None, None) == 0        # no rows: nothing to do
    assert L.elq_quantize_weights(elq.NVFP4, x, 128, 64, out, out, None) == -2


def test_ext_format_layer_validation(L):
    """Q5_1 / Q4_K / Q5_K experts: the cluster GEMV path (T <= 8, T * k <= 64)
    only; gate/up and down in one format; K-quant matrices in whole
    256-value super-blocks."""
    x = ctypes.c_void_p(1 << 27)
    y = ctypes.c_void_p(1 << 28)
    ws = ctypes.c_void_p(1 << 26)
    q, d = elq.SZ(), elq.SZ()
    assert L.elq_arena_bytes(elq.Q5_1, 128, 64, ctypes.byref(q), ctypes.byref(d)) == 128 * 2 * (20 + 4)
    assert L.elq_arena_bytes(elq.Q4_K, 128, 256, ctypes.byref(q), ctypes.byref(d)) == 128 * 8 * (16 + 4)
    assert L.elq_arena_bytes(elq.Q5_K, 128, 256, ctypes.byref(q), ctypes.byref(d)) == 128 * 8 * (20 + 4)
    assert L.elq_arena_bytes(elq.Q4_K, 128, 128, None, None) == 0
    for fmt in (elq.Q5_1, elq.Q4_K, elq.Q5_K):
        ly = _layer(L_=256, I=256)
        ly.gate_up = _qm(fmt, 8 * 2 * 256, 256)
        ly.down = _qm(fmt, 8 * 256, 256)
        for T in (1, 4, 8):
            assert L.elq_layer_kernel_count(ctypes.byref(ly), T) == 5
        for T in (9, 64):
            assert L.elq_layer_kernel_count(ctypes.byref(ly), T) == 0
            assert L.elq_moe_layer(ctypes.byref(ly), x, 0, T, y, ws, 1 << 30, None) == -2
        mixed = _layer(L_=256, I=256)
        mixed.gate_up = _qm(fmt, 8 * 2 * 256, 256)
        assert L.elq_moe_layer(ctypes.byref(mixed), x, 0, 1, y, ws, 1 << 30, None) == -2
        bad = _layer(fmt=8)
        bad.D = _qm(fmt, 256, 512)
        assert L.elq_moe_layer(ctypes.byref(bad), x, 0, 1, y, ws, 1 << 30, None) == -2
    kq = _layer(L_=384, I=256)
    kq.gate_up = _qm(elq.Q4_K, 8 * 2 * 256, 384)
    kq.down = _qm(elq.Q4_K, 8 * 384, 256)
    assert L.elq_moe_layer(ctypes.byref(kq), x, 0, 1, y, ws, 1 << 30, None) == -2


def test_stack_validation(L):
    ws = ctypes.c_void_p(1 << 26)
    x = ctypes.c_void_p(1 << 27)
    h = ctypes.c_void_p(1 << 28)
    arr = (elq.LayerC * 2)(_layer(), _layer())
    # refused before any launch: bad counts, mixed shapes, unsupported T, input type, workspace
    assert L.elq_moe_stack(arr, 0, x, 0, 4, h, ws, 1 << 30, None) == -1
    assert L.elq_moe_stack(None, 2, x, 0, 4, h, ws, 1 << 30, None) == -1
    mixed = (elq.LayerC * 2)(_layer(), _layer(I=512))
    assert L.elq_moe_stack(mixed, 2, x, 0, 4, h, ws, 1 << 30, None) == -1
    assert L.elq_moe_stack(arr, 2, x, 0, 64, h, ws, 16, None) == -4           # tensor-core sizes too
    assert L.elq_moe_stack(arr, 2, x, 5, 4, h, ws, 1 << 30, None) == -2
    assert L.elq_moe_stack(arr, 2, x, 0, 4, h, ws, 16, None) == -4
    assert L.elq_moe_stack(arr, 2, ctypes.c_void_p((1 << 27) + 4), 0, 4, h, ws, 1 << 30, None) == -3
    assert L.elq_moe_stack(arr, 2, x, 0, 0, h, ws, 1 << 30, None) == 0         # nothing to do


def test_empty_inputs_return_ok_without_work(L):
    """T = 0 (no tokens): each entry point still validates its other arguments,
    then returns ELQ_OK without a launch (no GPU is touched here) and without
    reading its data pointers."""
    p = ctypes.c_void_p(1 << 24)
    good = _layer()
    assert L.elq_moe_layer(ctypes.byref(good), None, 0, 0, None, None, 0, None) == 0
    assert L.elq_moe_layer(ctypes.byref(good), None, 30, 0, None, None, 0, None) == 0     # bf16 input
    assert L.elq_moe_layer(ctypes.byref(good), None, 5, 0, None, None, 0, None) == -2     # input type still checked
    assert L.elq_moe_layer(ctypes.byref(_layer(k=9)), None, 0, 0, None, None, 0, None) == -1   # layer still checked
    assert L.elq_moe_experts_grouped(ctypes.byref(good), None, None, None, 0, None, None, 0, None) == 0
    assert L.elq_router_topk(None, None, None, 0, 64, 8, 2, None, None, None, None) == 0
    assert L.elq_router_topk(None, None, None, 0, 64, 8, 9, None, None, None, None) == -1  # k > E still checked
    assert L.elq_quantize_q8_1(None, 0, 0, 64, None, None) == 0
    qm = _qm(8, 256, 512)
    assert L.elq_latent_proj(ctypes.byref(qm), None, 0, None, None, 0, None) == 0
    assert L.elq_latent_proj_noalloc(ctypes.byref(qm), None, 0, None, None) == 0
    assert L.elq_latent_proj(ctypes.byref(qm), p, -1, p, p, 1 << 30, None) == -1
    # no tokens need no workspace
    assert L.elq_workspace_bytes(ctypes.byref(good), 0) == 0
    assert L.elq_latent_proj_workspace_bytes(ctypes.byref(qm), 0) == 0
    assert L.elq_layer_kernel_count(ctypes.byref(good), 0) == 0


def test_other_entry_validation(L):
    p = ctypes.c_void_p(1 << 24)
    assert L.elq_quantize_q8_1(p, 0, 4, 48, p, None) == -2          # cols % 32
    assert L.elq_quantize_q8_1(p, 7, 4, 64, p, None) == -2          # x type
    assert L.elq_quantize_q8_1(None, 0, 4, 64, p, None) == -1
    assert L.elq_quantize_q8_1(ctypes.c_void_p((1 << 24) + 1), 0, 4, 64, p, None) == -3
    assert L.elq_router_topk(p, p, None, 1, 64, 8, 9, p, p, p, None) == -1     # k > E
    assert L.elq_router_topk(p, p, None, 1, 64, 64, 33, p, p, p, None) == -2   # k > 32
    assert L.elq_router_topk(p, p, None, 1, 64, 8, 2, p, p, None, None) == -1  # logits required
    assert L.elq_router_topk(p, p, None, 1, 2080, 8, 2, p, p, p, None) == -2  # L > 2048
    assert L.elq_route_bucket(p, 4, 2, 8, None, p, p, p, None) == -1
    assert L.elq_route_bucket(p, 4, 9, 8, p, p, p, p, None) == -1
    qm = _qm(8, 256, 512)
    assert L.elq_latent_proj(ctypes.byref(qm), p, 2, p, None, 0, None) == -4
    assert L.elq_latent_proj(ctypes.byref(_qm(4, 256, 512)), p, 2, p, p, 1 << 30, None) == -2
    assert L.elq_latent_proj(ctypes.byref(_qm(8, 200, 512)), p, 2, p, p, 1 << 30, None) == -2
    assert L.elq_latent_proj(ctypes.byref(_qm(8, 256, 96)), p, 2, p, p, 1 << 30, None) == -2   # k % 128
    assert L.elq_arena_pack(8, p, 100, 64, p, p, None) == -2
    assert L.elq_arena_pack(8, p, 128, 64, ctypes.c_void_p((1 << 24) + 16), p, None) == -3
    assert L.elq_quantize_weights(2, p, 128, 40, p, p, None) == -2
    assert L.elq_quantize_gate_up(8, p, p, 2, 96, 64, p, p, None) == -2
    assert L.elq_test_block_isums(9, p, p, 4, p, p, None) == -2
    assert L.elq_workspace_status(None, None) == -1


def _with_q16(ly, names=("D", "U", "gate_up", "down"), base=1 << 29):
    for i, n in enumerate(names):
        m = getattr(ly, n)
        m.q16 = base + i * (1 << 24)
        setattr(ly, n, m)
    return ly


def test_f16_codes_validation(L):
    """The fp16 codes of a matrix: their size, the formats that may carry them,
    their alignment, and the workspace of a tensor-core call that uses them
    (the B operands' codes take twice the bytes)."""
    assert L.elq_f16_bytes(ctypes.byref(_qm(8, 256, 512))) == 256 * 512 * 2
    assert L.elq_f16_bytes(ctypes.byref(_qm(2, 256, 512))) == 0          # Q4_0 has none
    assert L.elq_f16_bytes(None) == 0
    q16 = ctypes.c_void_p(1 << 29)
    assert L.elq_pack_f16(ctypes.byref(_qm(2, 256, 512)), q16, None) == -2
    assert L.elq_pack_f16(ctypes.byref(_qm(8, 256, 512)), ctypes.c_void_p((1 << 29) + 16), None) == -3
    assert L.elq_pack_f16(ctypes.byref(_qm(8, 256, 512)), None, None) == -1
    assert L.elq_pack_f16(None, q16, None) == -1
    x = ctypes.c_void_p(1 << 27)
    y = ctypes.c_void_p(1 << 28)
    ws = ctypes.c_void_p(1 << 26)
    good = _with_q16(_layer())
    # the same launch sequence; a bigger workspace only where the tensor-core path runs
    assert L.elq_layer_kernel_count(ctypes.byref(good), 64) == 10
    assert L.elq_workspace_bytes(ctypes.byref(good), 64) > L.elq_workspace_bytes(ctypes.byref(_layer()), 64)
    assert L.elq_workspace_bytes(ctypes.byref(good), 4) == L.elq_workspace_bytes(ctypes.byref(_layer()), 4)
    # only some matrices with fp16 codes: the int8 GEMMs, the int8 workspace
    part = _with_q16(_layer(), names=("D", "U"))
    assert L.elq_workspace_bytes(ctypes.byref(part), 64) == L.elq_workspace_bytes(ctypes.byref(_layer()), 64)
    # fp16 codes on a Q4_0 matrix, or misaligned: refused before any launch
    bad = _with_q16(_layer(fmt=2), names=("D",))
    assert L.elq_moe_layer(ctypes.byref(bad), x, 0, 4, y, ws, 1 << 30, None) == -2
    bad = _with_q16(_layer(), names=("U",), base=(1 << 29) + 64)
    assert L.elq_moe_layer(ctypes.byref(bad), x, 0, 4, y, ws, 1 << 30, None) == -3


def test_bench_f16_choice():
    import sys
    sys.path.insert(0, ROOT)
    import bench
    from quantized_latent_moe_b200 import synth

    class A:
        f16 = "auto"
    a = A()
    assert bench.use_f16(a, synth.WORKLOADS["prefill"]) and not bench.use_f16(a, synth.WORKLOADS["decode"])
    a.f16 = "off"
    assert not bench.use_f16(a, synth.WORKLOADS["prefill"])
    a.f16 = "on"
    assert bench.use_f16(a, synth.WORKLOADS["decode"])
