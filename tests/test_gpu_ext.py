"""Parity of the Q5_1 / Q3_K / Q4_K / Q5_K expert path (through the C ABI)
with the CPU oracle: the packed arena byte for byte against the layout the
header states, and every intermediate and the output of layers with these
experts bit-exact (both sides take the same per-block integer sums, the same
fp32 factor products and the same chunk order, R22-R25)."""
import numpy as np
import pytest
import torch

from quantized_latent_moe_b200 import synth
from helpers import gpu_layer, oracle_forward, oracle_layer

pytestmark = pytest.mark.gpu
FMTS = ["q5_1", "q3_k", "q4_k", "q5_k"]


@pytest.fixture(scope="module")
def E():
    from quantized_latent_moe_b200 import build, elq
    build.build()
    elq.lib()
    assert torch.cuda.is_available()
    return elq


def _expected_arena(name, blocks, n_rows, k):
    """The header's arena layout, built here from the GGUF bytes."""
    import struct
    nb, tiles = k // 32, n_rows // 128
    qh5 = name in ("q5_1", "q5_k")
    piece = 640 if qh5 else 512
    q = np.zeros(tiles * nb * 4 * piece, np.uint8)
    d = np.zeros(tiles * nb * 128, np.uint32)
    for row in range(n_rows):
        rb = blocks[row]
        t, sl, r = row // 128, (row % 128) // 32, row % 32
        for kb in range(nb):
            if name == "q3_k":
                b = rb[110 * (kb // 8):110 * (kb // 8) + 110].astype(np.int64)
                j = kb % 8
                codes = []
                for l_ in range(32):
                    i = 32 * j + l_
                    n_, jj, ll = i // 128, (i % 128) // 32, i % 32
                    low = (b[32 + 32 * n_ + ll] >> (2 * jj)) & 3
                    high = (b[ll] >> (4 * n_ + jj)) & 1
                    codes.append(int(low - (0 if high else 4) + 8))
                sc6 = []
                for h in range(2):
                    s_ = 2 * j + h
                    low4 = (b[96 + s_] & 15) if s_ < 8 else (b[96 + s_ - 8] >> 4)
                    sc6.append(int(low4 | (((b[104 + s_ % 4] >> (2 * (s_ // 4))) & 3) << 4)))
                hi = int(b[108]) | int(b[109]) << 8 if j == 0 else 0
                sw = sc6[0] | sc6[1] << 8 | hi << 16
                qh = 0
            elif name == "q5_1":
                b = rb[24 * kb:24 * kb + 24]
                codes = [b[8 + i] & 15 for i in range(16)] + [b[8 + i] >> 4 for i in range(16)]
                qh = int(struct.unpack("<I", bytes(b[4:8]))[0])
                sw = int(struct.unpack("<I", bytes(b[0:4]))[0])
            else:
                bb = 176 if name == "q5_k" else 144
                b = rb[bb * (kb // 8):bb * (kb // 8) + bb]
                j = kb % 8
                sc = b[4:16]
                if j < 4:
                    s_, m_ = sc[j] & 63, sc[j + 4] & 63
                else:
                    s_, m_ = (sc[j + 4] & 15) | ((sc[j - 4] >> 6) << 4), (sc[j + 4] >> 4) | ((sc[j] >> 6) << 4)
                qs = b[bb - 128 + 32 * (j // 2):bb - 128 + 32 * (j // 2) + 32]
                codes = [(x >> 4) if j & 1 else (x & 15) for x in qs]
                qh = 0
                if name == "q5_k":
                    for l_ in range(32):
                        qh |= ((int(b[16 + l_]) >> j) & 1) << l_
                hi = int(b[0]) | int(b[1]) << 8 if j == 0 else (int(b[2]) | int(b[3]) << 8 if j == 1 else 0)
                sw = int(s_) | int(m_) << 8 | hi << 16
            base = (t * nb * 4 + sl * nb + kb) * piece
            for i in range(16):
                q[base + r * 16 + i] = codes[i] | (codes[i + 16] << 4)
            if qh5:
                q[base + 512 + r * 4:base + 512 + r * 4 + 4] = np.frombuffer(struct.pack("<I", qh), np.uint8)
            d[t * nb * 128 + sl * nb * 32 + kb * 32 + r] = sw
    return q, d.view(np.uint8)


@pytest.mark.parametrize("name", FMTS)
def test_arena_pack_ext(E, name):
    n_rows, k = 128, 512
    blocks = synth.ext_blocks(name, 13, 1, n_rows, k)
    m = E.QMatrix.from_aos(blocks.cuda(), E.FMT[name], n_rows, k)
    q, d = _expected_arena(name, blocks.numpy(), n_rows, k)
    assert np.array_equal(m.q.cpu().numpy(), q)
    assert np.array_equal(m.d.cpu().numpy(), d)


def _ext_tiny(name):
    return synth.Workload("ext_" + name, 14, 8, 512, 256, 8, 2, 256, synth.Q8_0, synth.F32, "normal",
                          ex_fmt=name)


@pytest.mark.parametrize("name", FMTS)
def test_ext_layer_exact(E, orc, name):
    wl = _ext_tiny(name)
    ly = gpu_layer(wl)
    ol = oracle_layer(orc, wl)
    for T in (1, 3, 8):
        assert ly.kernel_count(T) == 5
        x = synth.make_x(wl, T=T)
        y = E.moe_layer(ly, x.cuda()).cpu().numpy()
        assert E.workspace_status(ly.workspace(T)) == 0
        tr = ol.forward(x.float().numpy(), trace=True)
        v = lambda n: E.workspace_view(ly, T, n).cpu().numpy()
        assert np.array_equal(v("zq").reshape(T, -1), tr["zq"])
        assert np.array_equal(v("idx").reshape(T, -1), tr["idx"])
        pos = tr["pos"]
        assert np.array_equal(v("hq").reshape(T * ly.k, -1)[pos], tr["hq"])
        assert np.array_equal(v("o").reshape(T * ly.k, -1)[pos], tr["o"])
        assert np.array_equal(v("y_lat").reshape(T, -1), tr["y_lat"])
        assert np.array_equal(y, tr["y"]), T


@pytest.mark.parametrize("name", FMTS)
def test_ext_experts_grouped_exact(E, orc, name):
    wl = _ext_tiny(name)
    ly = gpu_layer(wl)
    ol = oracle_layer(orc, wl)
    tr = ol.forward(synth.make_x(wl).float().numpy(), trace=True)
    y_lat = E.moe_experts_grouped(ly, torch.from_numpy(tr["zq"]).cuda(), torch.from_numpy(tr["idx"]).cuda(),
                                  torch.from_numpy(tr["w"]).cuda()).cpu().numpy()
    assert np.array_equal(y_lat, tr["y_lat"])


@pytest.mark.parametrize("name,T", [("decode_q4_k", 1), ("decode_q4_k", 8), ("decode_q3_k", 1), ("decode_q3_k", 8)])
def test_kquant_decode_full_size(E, orc, name, T):
    """The decode shapes (128 experts, top-8, L = 1792 = 7 super-blocks, I =
    1024) with Q4_K and with Q3_K experts: the whole output equals the
    oracle's."""
    wl = synth.WORKLOADS[name]
    ly = gpu_layer(wl)
    x = synth.make_x(wl, T=T)
    y = E.moe_layer(ly, x.cuda()).cpu().numpy()
    assert E.workspace_status(ly.workspace(T)) == 0
    ol = oracle_layer(orc, wl, experts=[])
    tr = oracle_forward(orc, ol, wl, x.float().numpy(), trace=True)
    assert np.array_equal(E.workspace_view(ly, T, "y_lat").cpu().numpy().reshape(T, -1), tr["y_lat"])
    assert np.array_equal(y, tr["y"])
