// elq_kernels.cuh -- the layer's sm_100a kernels (decode/verify path):
//   k_quant_q8_1      a1/a4  activation quantiser
//   k_quant_nvfp4     NVFP4 quantiser (standalone entry point)
//   k_quant_weights   arena preparation from fp32 weights
//   k_arena_pack      arena preparation from GGUF-style AoS blocks
//   k_router          a3 (+a5)  logits, top-k, softmax, bucketing
//   k_topk, k_bucket  a3 / a5 standalone
//   k_wgemv           a2 (+a1, a4) / a6 + a7 / a8 + a9 / a10: grouped quantised
//                     GEMV over the arena, one warp per 32-row unit
#pragma once

#include "elq_device.cuh"

namespace elq {

constexpr unsigned kFull = 0xffffffffu;

// ============================================================================
// a1 / a4 -- Q8_1 activation quantiser: four lanes per 32-value block, eight
// values each (a warp reads 512 contiguous bytes of bf16): amax and the code
// sum over the four lanes, d = amax / 127, q = clamp(round(x / d)), s =
// fp16(d * sum q); the same operations as the warp quantiser.
// ============================================================================
template <bool kBF16>
__global__ void __launch_bounds__(256) k_quant_q8_1(const void* __restrict__ x, int64_t nblocks,
                                                    uint8_t* __restrict__ out) {
    pdl_wait();
    const int64_t tid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const int64_t blk = tid >> 2;      // four lanes per block, eight values each
    const int q4 = (int)(tid & 3);
    const bool on = blk < nblocks;
    float v[8];
    if (!on) {
#pragma unroll
        for (int i = 0; i < 8; ++i) v[i] = 0.0f;
    } else if ((reinterpret_cast<uintptr_t>(x) & 15) != 0) {
        // 4-byte aligned input: element loads
#pragma unroll
        for (int i = 0; i < 8; ++i)
            v[i] = kBF16 ? __bfloat162float(static_cast<const __nv_bfloat16*>(x)[blk * 32 + 8 * q4 + i])
                         : static_cast<const float*>(x)[blk * 32 + 8 * q4 + i];
    } else if (kBF16) {
        // a warp reads 512 contiguous bytes
        const uint4 w = __ldg(reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(x) + blk * 32) + q4);
        const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            v[2 * j] = __uint_as_float(ws[j] << 16);
            v[2 * j + 1] = __uint_as_float(ws[j] & 0xffff0000u);
        }
    } else {
        const float4* src = reinterpret_cast<const float4*>(static_cast<const float*>(x) + blk * 32) + 2 * q4;
        const float4 a = __ldg(src), b = __ldg(src + 1);
        v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
        v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
    }
    // the block's amax and code sum over its four lanes (order-free: a max and an integer sum)
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(v[i]));
    amax = fmaxf(amax, __shfl_xor_sync(kFull, amax, 1));
    amax = fmaxf(amax, __shfl_xor_sync(kFull, amax, 2));
    const float d = __fdiv_rn(amax, 127.0f);
    uint32_t w0 = 0, w1 = 0;
    int sum = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        int q = 0;
        if (d != 0.0f) q = (int)fminf(fmaxf(roundf(__fdiv_rn(v[i], d)), -127.0f), 127.0f);
        sum += q;
        if (i < 4) w0 |= (uint32_t)(q & 0xff) << (8 * i);
        else w1 |= (uint32_t)(q & 0xff) << (8 * (i - 4));
    }
    sum += __shfl_xor_sync(kFull, sum, 1);
    sum += __shfl_xor_sync(kFull, sum, 2);
    if (on) {
        uint32_t* o = reinterpret_cast<uint32_t*>(out + blk * 36);
        o[1 + 2 * q4] = w0;
        o[2 + 2 * q4] = w1;
        if (q4 == 0) o[0] = (uint32_t)f2h(d) | ((uint32_t)f2h(__fmul_rn(d, (float)sum)) << 16);
    }
    pdl_trigger();
}

// NVFP4 quantiser under global scale g: four lanes per 32-value block, eight
// values each (two lanes per 16-value micro-block), the same operations per
// value as warp_quant_nvfp4 (the layer's epilogues): s = e4m3(amax / 6 / g),
// den = s * g, codes e2m1(x / den) in pairs.
template <bool kBF16>
__global__ void __launch_bounds__(256) k_quant_nvfp4(const void* __restrict__ x, int64_t nblocks, float g,
                                                     uint8_t* __restrict__ out) {
    pdl_wait();
    const int64_t tid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const int64_t blk = tid >> 2;
    const int q4 = (int)(tid & 3);
    const bool on = blk < nblocks;
    float v[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] = 0.0f;
    if (on) {
        const int64_t e0 = blk * 32 + 8 * q4;
        if (!kBF16 && (reinterpret_cast<uintptr_t>(x) & 15) == 0) {
            const float4* src = reinterpret_cast<const float4*>(static_cast<const float*>(x) + e0);
            const float4 a = __ldg(src), b = __ldg(src + 1);
            v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
            v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
        } else {
#pragma unroll
            for (int i = 0; i < 8; ++i)
                v[i] = kBF16 ? __bfloat162float(static_cast<const __nv_bfloat16*>(x)[e0 + i])
                             : static_cast<const float*>(x)[e0 + i];
        }
    }
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(v[i]));
    amax = fmaxf(amax, __shfl_xor_sync(kFull, amax, 1));          // the micro-block's two lanes
    const uint32_t sc = f32_to_e4m3(__fdiv_rn(__fdiv_rn(amax, 6.0f), g));
    const float den = __fmul_rn(e4m3x2_to_f32(sc).x, g);
    uint32_t codes = 0;                                             // code bytes 4 q4 .. 4 q4 + 3
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const float xa = den != 0.0f ? __fdiv_rn(v[2 * j], den) : 0.0f;
        const float xb = den != 0.0f ? __fdiv_rn(v[2 * j + 1], den) : 0.0f;
        codes |= (f32x2_to_e2m1x2(xa, xb) & 0xffu) << (8 * j);
    }
    const uint32_t sc1 = __shfl_sync(kFull, sc, (threadIdx.x & 31 & ~3) | 2);   // micro-block 1's scale
    if (on) {
        uint16_t* dst = reinterpret_cast<uint16_t*>(out + blk * 18);            // 2-byte aligned
        dst[1 + 2 * q4] = (uint16_t)(codes & 0xffffu);
        dst[2 + 2 * q4] = (uint16_t)(codes >> 16);
        if (q4 == 0) dst[0] = (uint16_t)(sc | (sc1 << 8));
    }
    pdl_trigger();
}

// ============================================================================
// Arena preparation.  One thread per (row, block).
// src_mode 0: arena row = source row.  src_mode 1: gate/up interleave -- arena
// row R of expert e = R / (2I), local rr = R % (2I), tile j = rr / 128, r =
// rr % 128 takes gate[e][64 j + r] (r < 64) or up[e][64 j + r - 64].
// ============================================================================
__device__ __forceinline__ const float* weight_src_row(const float* w, const float* w2, int src_mode,
                                                       int64_t row, int k, int I) {
    if (src_mode == 0) return w + row * (int64_t)k;
    const int64_t e = row / (2 * I);
    const int rr = (int)(row % (2 * I));
    const int j = rr / 128, r = rr % 128;
    const float* base = (r < 64) ? w : w2;
    return base + (e * I + 64 * j + (r & 63)) * (int64_t)k;
}

template <int FMT>
__global__ void __launch_bounds__(256) k_quant_weights(const float* __restrict__ w, const float* __restrict__ w2,
                                                       int src_mode, int n_rows, int k, int I,
                                                       uint8_t* __restrict__ q, uint16_t* __restrict__ d) {
    const int nb = k / 32;
    const int64_t id = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (id >= (int64_t)n_rows * nb) return;
    const int64_t row = id / nb;
    const int kb = (int)(id % nb);
    const float* src = weight_src_row(w, w2, src_mode, row, k, I) + kb * 32;
    float x[32];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const float4 v = reinterpret_cast<const float4*>(src)[i];
        x[4 * i] = v.x; x[4 * i + 1] = v.y; x[4 * i + 2] = v.z; x[4 * i + 3] = v.w;
    }
    const int64_t tile = row / kTileRows;
    const int slice = (int)(row % kTileRows) / 32, r = (int)(row % 32);
    const int64_t sel = tile * nb * kTileRows + (int64_t)slice * nb * 32 + (int64_t)kb * 32 + r;
    if (FMT == 8) {
        float amax = 0.0f;
#pragma unroll
        for (int i = 0; i < 32; ++i) amax = fmaxf(amax, fabsf(x[i]));
        const float dd = __fdiv_rn(amax, 127.0f);
        uint32_t words[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) words[i] = 0;
#pragma unroll
        for (int i = 0; i < 32; ++i) {
            int v = 0;
            if (dd != 0.0f) v = (int)fminf(fmaxf(roundf(__fdiv_rn(x[i], dd)), -127.0f), 127.0f);
            words[i >> 2] |= (uint32_t)(v & 0xff) << (8 * (i & 3));
        }
        uint8_t* dst = q + tile * nb * kQ80Slab + (int64_t)slice * nb * 1024 + (int64_t)kb * 1024 + (r >> 3) * 256 +
                       (r & 7) * 16;
        *reinterpret_cast<uint4*>(dst) = make_uint4(words[0], words[1], words[2], words[3]);
        *reinterpret_cast<uint4*>(dst + 128) = make_uint4(words[4], words[5], words[6], words[7]);
        d[sel] = f2h(dd);
    } else {
        float amax = 0.0f, m = 0.0f;
#pragma unroll
        for (int i = 0; i < 32; ++i) {
            const float a = fabsf(x[i]);
            if (a > amax) { amax = a; m = x[i]; }
        }
        const float dd = __fdiv_rn(m, -8.0f);
        int qv[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) {
            int v = 8;
            if (dd != 0.0f) v = (int)fminf(fmaxf(__fadd_rn(roundf(__fdiv_rn(x[i], dd)), 8.0f), 0.0f), 15.0f);
            qv[i] = v;
        }
        uint32_t words[4] = {0, 0, 0, 0};
#pragma unroll
        for (int j = 0; j < 16; ++j)
            words[j >> 2] |= (uint32_t)(qv[j] | (qv[j + 16] << 4)) << (8 * (j & 3));
        uint8_t* dst = q + tile * nb * kQ40Slab + (int64_t)slice * nb * 512 + (int64_t)kb * 512 + r * 16;
        *reinterpret_cast<uint4*>(dst) = make_uint4(words[0], words[1], words[2], words[3]);
        d[sel] = f2h(dd);
    }
}

// NVFP4 scales of a tile: nb*128 16-bit words (each row's two micro-block
// scales per block, as Q4_0's fp16 scales), then the same bytes once more as
// the tensor cores' scale-factor atoms: per pair of blocks (64 values) one
// 512-byte atom, row m's four scales (blocks 2j, 2j+1, micro-blocks 0, 1) as
// one 32-bit word at byte (m % 32) * 16 + (m / 32) * 4.
// In 16-bit units; Q5_1 / K-quant tiles hold a 32-bit word per (row, block).
__host__ __device__ constexpr int64_t d_tile_elems(int fmt, int nb) {
    return (int64_t)nb * kTileRows * (fmt == kNV ? 2 : scale_units(fmt));
}

// Q5_1 / Q4_K / Q5_K arena from GGUF blocks, one thread per (row, 32-value
// block).  Per (tile, slice, block) piece: 32 rows of 16 code bytes (byte i:
// value i in the low nibble, value i + 16 in the high one -- Q4_0's order, 4-bit
// codes without an offset), then for Q5_1 / Q5_K 32 rows of a 32-bit word of
// the codes' fifth bits (bit i for value i).  Scale word per (row, block):
// Q5_1 fp16 d | fp16 m << 16; K-quants 6-bit scale | 6-bit min << 8 | (the
// super-block's fp16 d in sub-block 0, its fp16 dmin in sub-block 1) << 16.
template <int FMT>
__global__ void __launch_bounds__(256) k_arena_pack_ext(const uint8_t* __restrict__ aos, int n_rows, int k,
                                                        uint8_t* __restrict__ q, uint32_t* __restrict__ d) {
    const int nb = k / 32;
    const int64_t id = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (id >= (int64_t)n_rows * nb) return;
    const int64_t row = id / nb;
    const int kb = (int)(id % nb);
    const int64_t tile = row / kTileRows;
    const int slice = (int)(row % kTileRows) / 32, r = (int)(row % 32);
    constexpr int kPiece = fmt_has_qh(FMT) ? 640 : 512;
    uint8_t codes[32];
    uint32_t qh = 0, sw;
    if (FMT == kQ3K) {
        // codes q in -4 .. 3 stored as q + 8 (Q4_0's offset); the halves' scales
        const uint8_t* b = aos + (row * (nb / 8) + kb / 8) * 110;
        const int j = kb % 8;
        for (int l = 0; l < 32; ++l) {
            const int i = 32 * j + l, n = i / 128, jj = (i % 128) / 32, ll = i % 32;
            const int low = (b[32 + 32 * n + ll] >> (2 * jj)) & 3;
            const int high = (b[ll] >> (4 * n + jj)) & 1;
            codes[l] = (uint8_t)(low - (high ? 0 : 4) + 8);
        }
        uint32_t sc6[2];
        for (int h = 0; h < 2; ++h) {
            const int s = 2 * j + h;
            const int low4 = s < 8 ? (b[96 + s] & 15) : (b[96 + s - 8] >> 4);
            const int hi2 = (b[96 + 8 + s % 4] >> (2 * (s / 4))) & 3;
            sc6[h] = (uint32_t)(low4 | (hi2 << 4));
        }
        const uint32_t hi = j == 0 ? ((uint32_t)b[108] | ((uint32_t)b[109] << 8)) : 0u;
        sw = sc6[0] | (sc6[1] << 8) | (hi << 16);
    } else if (FMT == kQ51) {
        const uint8_t* b = aos + (row * nb + kb) * 24;
        for (int i = 0; i < 16; ++i) {
            codes[i] = b[8 + i] & 15;
            codes[i + 16] = b[8 + i] >> 4;
        }
        qh = (uint32_t)b[4] | ((uint32_t)b[5] << 8) | ((uint32_t)b[6] << 16) | ((uint32_t)b[7] << 24);
        sw = (uint32_t)b[0] | ((uint32_t)b[1] << 8) | ((uint32_t)b[2] << 16) | ((uint32_t)b[3] << 24);
    } else {
        constexpr int kBB = FMT == kQ5K ? 176 : 144;
        const uint8_t* b = aos + (row * (nb / 8) + kb / 8) * kBB;
        const int j = kb % 8;
        const uint8_t* sc = b + 4;
        int scale, mn;
        if (j < 4) {
            scale = sc[j] & 63;
            mn = sc[j + 4] & 63;
        } else {
            scale = (sc[j + 4] & 15) | ((sc[j - 4] >> 6) << 4);
            mn = (sc[j + 4] >> 4) | ((sc[j] >> 6) << 4);
        }
        const uint8_t* qs = b + (FMT == kQ5K ? 48 : 16) + 32 * (j / 2);
        for (int l = 0; l < 32; ++l) codes[l] = (j & 1) ? (qs[l] >> 4) : (qs[l] & 15);
        if (FMT == kQ5K)
            for (int l = 0; l < 32; ++l) qh |= (uint32_t)((b[16 + l] >> j) & 1) << l;
        uint32_t hi = 0;
        if (j == 0) hi = (uint32_t)b[0] | ((uint32_t)b[1] << 8);
        if (j == 1) hi = (uint32_t)b[2] | ((uint32_t)b[3] << 8);
        sw = (uint32_t)scale | ((uint32_t)mn << 8) | (hi << 16);
    }
    uint32_t words[4] = {0, 0, 0, 0};
    for (int i = 0; i < 16; ++i) words[i >> 2] |= (uint32_t)(codes[i] | (codes[i + 16] << 4)) << (8 * (i & 3));
    uint8_t* piece = q + tile * nb * (4 * kPiece) + (int64_t)slice * nb * kPiece + (int64_t)kb * kPiece;
    *reinterpret_cast<uint4*>(piece + r * 16) = make_uint4(words[0], words[1], words[2], words[3]);
    if (fmt_has_qh(FMT)) *reinterpret_cast<uint32_t*>(piece + 512 + r * 4) = qh;
    d[tile * nb * kTileRows + (int64_t)slice * nb * 32 + (int64_t)kb * 32 + r] = sw;
}

template <int FMT>
__global__ void __launch_bounds__(256) k_arena_pack(const uint8_t* __restrict__ aos, int n_rows, int k,
                                                    uint8_t* __restrict__ q, uint16_t* __restrict__ d) {
    const int nb = k / 32;
    const int bb = (FMT == 8) ? 34 : 18;
    const int64_t id = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (id >= (int64_t)n_rows * nb) return;
    const int64_t row = id / nb;
    const int kb = (int)(id % nb);
    const uint8_t* src = aos + id * bb;
    const int64_t tile = row / kTileRows;
    const int slice = (int)(row % kTileRows) / 32, r = (int)(row % 32);
    const uint16_t sw = (uint16_t)(src[0] | (src[1] << 8));
    d[tile * d_tile_elems(FMT, nb) + (int64_t)slice * nb * 32 + (int64_t)kb * 32 + r] = sw;
    if (FMT == kNV) {
        // the atom copy: row m = 32 slice + r, byte (kb % 2) * 2 of its word
        uint8_t* atoms = reinterpret_cast<uint8_t*>(d + tile * d_tile_elems(FMT, nb) + (int64_t)nb * kTileRows);
        *reinterpret_cast<uint16_t*>(atoms + (int64_t)(kb >> 1) * 512 + r * 16 + slice * 4 + (kb & 1) * 2) = sw;
    }
    uint32_t words[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    const int nq = (FMT == 8) ? 32 : 16;
    for (int i = 0; i < nq; ++i) words[i >> 2] |= (uint32_t)src[2 + i] << (8 * (i & 3));
    if (FMT == 8) {
        uint8_t* dst = q + tile * nb * kQ80Slab + (int64_t)slice * nb * 1024 + (int64_t)kb * 1024 + (r >> 3) * 256 +
                       (r & 7) * 16;
        *reinterpret_cast<uint4*>(dst) = make_uint4(words[0], words[1], words[2], words[3]);
        *reinterpret_cast<uint4*>(dst + 128) = make_uint4(words[4], words[5], words[6], words[7]);
    } else {
        *reinterpret_cast<uint4*>(q + tile * nb * kQ40Slab + (int64_t)slice * nb * 512 + (int64_t)kb * 512 + r * 16) =
            make_uint4(words[0], words[1], words[2], words[3]);
    }
}

// ============================================================================
// a5 -- bucketing by the warps of one CTA.  hist: shared [nwarps][E] ints.
// Pairs are split into one contiguous segment per warp; per-warp histograms
// give each warp's base position per expert; each warp then places its
// segment in order, ranking equal experts inside a 32-pair chunk with
// __match_any_sync, so perm is sorted by (expert, pair id).
// ============================================================================
__device__ void bucket_cta(const int32_t* idx, int P, int E, int32_t* counts, int32_t* offsets,
                           int32_t* perm, int32_t* pos, int32_t* act, int32_t* n_act, int* hist) {
    const int nw = blockDim.x >> 5;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int i = threadIdx.x; i < nw * E; i += blockDim.x) hist[i] = 0;
    __syncthreads();
    const int seg = (P + nw - 1) / nw;
    const int s0 = min(P, warp * seg), s1 = min(P, s0 + seg);
    // 8 chunks of 32 pairs loaded ahead of their updates
    for (int c0 = s0; c0 < s1; c0 += 256) {
        int ev[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const int p = c0 + 32 * u + lane;
            ev[u] = p < s1 ? __ldcg(idx + p) : -1;
        }
#pragma unroll
        for (int u = 0; u < 8; ++u)
            if (ev[u] >= 0) atomicAdd(&hist[warp * E + ev[u]], 1);
    }
    __syncthreads();
    if (warp == 0) {
        const int per = (E + 31) / 32;
        const int e0 = min(E, lane * per), e1 = min(E, e0 + per);
        int local = 0;
        for (int e = e0; e < e1; ++e) {
            int c = 0;
            for (int w = 0; w < nw; ++w) c += hist[w * E + e];
            counts[e] = c;
            local += c;
        }
        int incl = local;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int v = __shfl_up_sync(kFull, incl, o);
            if (lane >= o) incl += v;
        }
        int run = incl - local;
        for (int e = e0; e < e1; ++e) {
            offsets[e] = run;
            for (int w = 0; w < nw; ++w) {
                const int c = hist[w * E + e];
                hist[w * E + e] = run;
                run += c;
            }
        }
        if (lane == 31) offsets[E] = incl;
    }
    __syncthreads();
    for (int c0 = s0; c0 < s1; c0 += 256) {
        int ev[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const int p = c0 + 32 * u + lane;
            ev[u] = p < s1 ? __ldcg(idx + p) : -1 - lane;
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const int p = c0 + 32 * u + lane;
            const bool v = p < s1;
            const int e = ev[u];
            const unsigned m = __match_any_sync(kFull, e);
            if (v) {
                const int r = __popc(m & ((1u << lane) - 1u));
                const int posn = hist[warp * E + e] + r;
                perm[posn] = p;
                pos[p] = posn;
            }
            __syncwarp();
            if (v && lane == __ffs(m) - 1) hist[warp * E + e] += __popc(m);
            __syncwarp();
        }
    }
    __syncthreads();
    if (act && warp == 0) {
        int n = 0;
        for (int e0 = 0; e0 < E; e0 += 32) {
            const int e = e0 + lane;
            const bool on = e < E && counts[e] > 0;
            const unsigned b = __ballot_sync(kFull, on);
            if (on) act[n + __popc(b & ((1u << lane) - 1u))] = e;
            n += __popc(b);
        }
        if (lane == 0) *n_act = n;
    }
}

__global__ void k_bucket(const int32_t* idx, int P, int E, int32_t* counts, int32_t* offsets, int32_t* perm,
                         int32_t* pos, int32_t* act, int32_t* n_act) {
    extern __shared__ int hist_sm[];
    pdl_wait();
    bucket_cta(idx, P, E, counts, offsets, perm, pos, act, n_act, hist_sm);
    pdl_trigger();
}

// ============================================================================
// a3 -- router: logits (R9 order), top-k (lower id on ties), softmax over the
// k selected; optionally a5 by the last CTA.  A block of nw warps (4 or 16)
// holds nw experts, one per warp, each lane keeping its L/32 lane-strided
// router weights in registers (L <= 2048).  Grid (ceil(E/nw), gy): CTA (x, y)
// streams the token blocks y, y + gy, ... (8 tokens each) through a cp.async
// ring of one or two stages, so that a latent row is read once per CTA and
// reused by all its experts.  Each token block's top-k is done once all gx
// CTAs have finished it, normally by its owner CTA (rotating over x) after
// that CTA's stream; the last top-k buckets.
// ============================================================================
constexpr int kRouterTok = 8;
constexpr int kRouterJ = 64;          // register-held router weights per lane
constexpr int kRouterMaxL = 32 * kRouterJ;
constexpr int kRouterMaxWarps = 16;
constexpr int kRouterOwnWords = 32;   // deferred top-k list: the first 1024 blocks of a CTA

struct RouterArgs {
    const float* z;
    const float* w;
    const float* bias;
    int T, L, E, k;
    int32_t* idx;
    float* wts;
    float* logits;
    int* cnt_tok;     // [rblocks]: one per 8-token block; zero on entry and exit
    int* cnt_all;     // [1], right after cnt_tok (cnt_tok + rblocks); zero on entry and exit
    int do_bucket;
    int32_t *counts, *offsets, *perm, *pos, *act, *n_act;
};

// Top-k of one token's logits (in shared memory, lg[0..E)) by one warp, then
// the softmax over the k selected in rank order.  Lane j ends with rank j.
__device__ __forceinline__ void warp_topk_softmax(const float* lg, int E, int k, int32_t* idx_out,
                                                  float* w_out, int32_t* idx_sm = nullptr) {
    const int lane = threadIdx.x & 31;
    uint32_t taken = 0;
    float sel_v = 0.0f;
    int sel_e = 0;
    for (int j = 0; j < k; ++j) {
        float bv = -INFINITY;
        int be = 0x7fffffff;
        for (int i = 0, x = lane; x < E; ++i, x += 32) {
            if (taken & (1u << i)) continue;
            const float v0 = lg[x];
            const float v = (v0 != v0) ? -INFINITY : v0;   // R18: a NaN logit ranks as -inf
            if (v > bv || (v == bv && x < be)) { bv = v; be = x; }
        }
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) {
            const float ov = __shfl_xor_sync(kFull, bv, o);
            const int oe = __shfl_xor_sync(kFull, be, o);
            if (ov > bv || (ov == bv && oe < be)) { bv = ov; be = oe; }
        }
        if (be != 0x7fffffff && (be & 31) == lane) taken |= 1u << (be >> 5);
        if (lane == j) { sel_v = bv; sel_e = be; }
    }
    const float l0 = __shfl_sync(kFull, sel_v, 0);
    const float ex = (lane < k) ? exp_f32(__fsub_rn(sel_v, l0)) : 0.0f;
    float sum = 0.0f;
    for (int j = 0; j < k; ++j) sum = __fadd_rn(sum, __shfl_sync(kFull, ex, j));
    if (lane < k) {
        idx_out[lane] = sel_e;
        w_out[lane] = __fdiv_rn(ex, sum);
        if (idx_sm) idx_sm[lane] = sel_e;
    }
}

// a5 for at most 64 pairs by one warp: the rank of pair p is the number of
// pairs (e', p') before (e, p) in (expert, pair id) order; counts and offsets
// are direct counts.  idx_sm: the pairs' experts in shared memory.
// grp (optional): per active group a, (expert, first position, pairs).
__device__ void bucket_warp_small(const int32_t* idx_sm, int P, int E, int32_t* counts, int32_t* offsets,
                                  int32_t* perm, int32_t* pos, int32_t* act, int32_t* n_act,
                                  int4* grp = nullptr) {
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const int p = lane + 32 * h;
        if (p < P) {
            const int e = idx_sm[p];
            int r = 0;
            for (int q = 0; q < P; ++q) {
                const int eq = idx_sm[q];
                r += (eq < e) || (eq == e && q < p);
            }
            perm[r] = p;
            pos[p] = r;
        }
    }
    int n = 0;
    for (int e0 = 0; e0 < E; e0 += 32) {
        const int e = e0 + lane;
        int c = 0, lt = 0;
        for (int q = 0; q < P; ++q) {
            const int eq = idx_sm[q];
            c += (eq == e);
            lt += (eq < e);
        }
        if (e < E) {
            counts[e] = c;
            offsets[e] = lt;
        }
        const bool on = (e < E) && c > 0;
        const unsigned b = __ballot_sync(kFull, on);
        if (on && act) act[n + __popc(b & ((1u << lane) - 1u))] = e;
        if (on && grp) grp[n + __popc(b & ((1u << lane) - 1u))] = make_int4(e, lt, c, 0);
        n += __popc(b);
    }
    if (lane == 0) {
        offsets[E] = P;
        if (n_act) *n_act = n;
    }
}

// Warp sums of V values per lane (V a power of two, at most 32), each the same
// xor-butterfly tree as V separate butterflies over offsets 16, 8, 4, 2, 1
// (every level adds the two lanes' partials of the same value), but at each
// of the first log2(V) levels a lane keeps only half of its values and trades
// the other half with its partner: V - 1 + 5 - log2(V) shuffles instead of
// 5 V.  On return lane l holds the total of value l >> (5 - log2(V)).
template <int V>
__device__ __forceinline__ float warp_sum_scatter(float (&p)[V], int lane) {
    constexpr int LV = V >= 32 ? 5 : V >= 16 ? 4 : V >= 8 ? 3 : V >= 4 ? 2 : V >= 2 ? 1 : 0;
    static_assert((1 << LV) == V, "V is a power of two <= 32");
#pragma unroll
    for (int st = 0; st < LV; ++st) {
        const int o = 16 >> st, h = (V >> st) / 2;
        const bool up = (lane & o) != 0;
#pragma unroll
        for (int i = 0; i < h; ++i) {
            const float send = up ? p[i] : p[i + h];
            const float keep = up ? p[i + h] : p[i];
            p[i] = __fadd_rn(keep, __shfl_xor_sync(kFull, send, o));
        }
    }
    float r = p[0];
#pragma unroll
    for (int o = 16 >> LV; o >= 1; o >>= 1) r = __fadd_rn(r, __shfl_xor_sync(kFull, r, o));
    return r;
}

// EPW experts per warp (1 or 2): with 2, each latent value a lane reads from
// shared memory feeds two experts' chains (half the shared-memory traffic per
// logit, the bound of this loop), at twice the register-held weights.
template <int EPW>
__global__ void __launch_bounds__(EPW == 1 ? kRouterMaxWarps * 32 : kRouterMaxWarps * 16) k_router(RouterArgs a) {
    extern __shared__ __align__(128) float rsm[];   // [stages][<=8][L] latent rows, then [nw][E] scratch
    __shared__ int s_last, s_all;
    __shared__ int32_t s_idx[64];
    __shared__ uint32_t s_own[kRouterOwnWords];   // blocks of this CTA whose top-k it owns
    const int nw = blockDim.x >> 5;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int L = a.L, E = a.E;
    const int nj = L >> 5;
    const int rblocks = (a.T + kRouterTok - 1) / kRouterTok;
    const int gy = (int)gridDim.y;
    const int nmine = (rblocks - (int)blockIdx.y + gy - 1) / gy;   // >= 1: gridDim.y <= rblocks
    const int stages = (gy < rblocks) ? 2 : 1;
    const int rows = min(a.T, kRouterTok);
    const int Lp = (L + 255) & ~255;                // shared row stride: whole chunks of 8 lane-strided values
    float* scr = rsm + (size_t)stages * rows * Lp;
    const int e0 = ((int)blockIdx.x * nw + warp) * EPW;   // this warp's experts e0 .. e0 + EPW - 1
    const bool has_e = e0 < E;
    // the router rows do not depend on the upstream kernel: load them first
    float wr[EPW][kRouterJ];
    float bias[EPW];
#pragma unroll
    for (int x = 0; x < EPW; ++x) {
        const bool on = e0 + x < E;
        const float* wrow = a.w + (int64_t)(on ? e0 + x : 0) * L + lane;
#pragma unroll
        for (int j = 0; j < kRouterJ; ++j) wr[x][j] = (on && j < nj) ? __ldg(wrow + 32 * j) : 0.0f;
        bias[x] = (on && a.bias) ? __ldg(a.bias + e0 + x) : 0.0f;
    }
    pdl_wait();
    pdl_trigger();
    // token block number i of this CTA into stage i % stages: one cp.async
    // group per block (an empty group past the last block keeps the count)
    const int L4 = L >> 2;
    auto issue = [&](int i) {
        if (i < nmine) {
            const int t0 = ((int)blockIdx.y + i * gy) * kRouterTok;
            const int nr = min(kRouterTok, a.T - t0);
            const float* src = a.z + (int64_t)t0 * L;
            float* dst = rsm + (size_t)(i & (stages - 1)) * rows * Lp;
            int r = (int)threadIdx.x / L4, c = (int)threadIdx.x - r * L4;
            while (r < nr) {
                cp_async16(dst + r * Lp + 4 * c, src + (int64_t)r * L + 4 * c);
                c += (int)blockDim.x;
                while (c >= L4) {
                    c -= L4;
                    ++r;
                }
            }
        }
        cp_async_commit();
    };
    // the padding columns L .. Lp of every staged row are zeros (never copied into): a zero weight times
    // a zero adds +0 to a chain that, started at +0, is never -0, so it leaves the chain's bits alone
    if (Lp > L)
        for (int q = threadIdx.x; q < stages * rows * (Lp - L); q += blockDim.x)
            rsm[(q / (Lp - L)) * Lp + L + q % (Lp - L)] = 0.0f;
    issue(0);
    if (stages == 2) issue(1);
    const bool small = a.do_bucket && rblocks == 1 && a.T * a.k <= 64;
    const bool claims = stages == 2;                       // CTAs stream several blocks
    const int target = claims ? (int)gridDim.x : (int)gridDim.x - 1;   // counter before the last increment
    // top-k + softmax of token block b (all threads; its logits are complete),
    // then the arrival that makes the last token block's owner bucket
    auto topk_block = [&](int b) {
        const int t0 = b * kRouterTok;
        const int nt = min(kRouterTok, a.T - t0);
        __threadfence();
        float* lg = scr + (size_t)warp * E;
        for (int tt = warp; tt < nt; tt += nw) {
            const int t = t0 + tt;
            for (int x = lane; x < E; x += 32) lg[x] = __ldcg(a.logits + (int64_t)t * E + x);
            __syncwarp();
            warp_topk_softmax(lg, E, a.k, a.idx + (int64_t)t * a.k, a.wts + (int64_t)t * a.k,
                              small ? s_idx + t * a.k : nullptr);
            __syncwarp();
        }
        __syncthreads();
        if (threadIdx.x == 0) {
            a.cnt_tok[b] = 0;
            s_all = 0;
            if (a.do_bucket && !small) {
                __threadfence();
                s_all = (atomicAdd(a.cnt_all, 1) == rblocks - 1);
            }
        }
        __syncthreads();
        if (!a.do_bucket) return;
        if (small) {
            if (warp == 0)
                bucket_warp_small(s_idx, a.T * a.k, E, a.counts, a.offsets, a.perm, a.pos, a.act, a.n_act);
        } else if (s_all) {
            __threadfence();
            bucket_cta(a.idx, a.T * a.k, E, a.counts, a.offsets, a.perm, a.pos, a.act, a.n_act,
                       reinterpret_cast<int*>(scr));
            if (threadIdx.x == 0) *a.cnt_all = 0;
        }
        __syncthreads();
    };
    for (int i = threadIdx.x; i < kRouterOwnWords; i += blockDim.x) s_own[i] = 0u;
    for (int i = 0; i < nmine; ++i) {
        const int b = (int)blockIdx.y + i * gy;
        const int t0 = b * kRouterTok;
        const int nt = min(kRouterTok, a.T - t0);
        if (stages == 2)
            cp_async_wait<1>();
        else
            cp_async_wait<0>();
        __syncthreads();
        if (has_e) {
            // four tokens by EPW experts per pass; lane l keeps the chains of the lane-strided
            // values 32 j + l (R9), j in whole chunks of 8 (the rows are padded to 256)
            constexpr int kTq = 4, kV = kTq * EPW;
            const float* zs = rsm + (size_t)(i & (stages - 1)) * rows * Lp + lane;
            const int nc = Lp >> 8;
            for (int tt = 0; tt < nt; tt += kTq) {
                const float* zr[kTq];
#pragma unroll
                for (int q = 0; q < kTq; ++q) zr[q] = zs + min(tt + q, nt - 1) * Lp;
                float p[kV];
#pragma unroll
                for (int v = 0; v < kV; ++v) p[v] = 0.0f;
#pragma unroll
                for (int c = 0; c < kRouterJ / 8; ++c) {
                    if (c < nc) {
#pragma unroll
                        for (int u = 0; u < 8; ++u) {
                            const int j = 8 * c + u;
                            float zv[kTq];
#pragma unroll
                            for (int q = 0; q < kTq; ++q) zv[q] = zr[q][32 * j];
#pragma unroll
                            for (int q = 0; q < kTq; ++q)
#pragma unroll
                                for (int x = 0; x < EPW; ++x)
                                    p[q * EPW + x] = __fmaf_rn(zv[q], wr[x][j], p[q * EPW + x]);
                        }
                    }
                }
                // value v = q * EPW + x: token tt + q, expert e0 + x
                float r = warp_sum_scatter<kV>(p, lane);
                constexpr int kSh = 5 - (kV >= 32 ? 5 : kV >= 16 ? 4 : kV >= 8 ? 3 : kV >= 4 ? 2 : kV >= 2 ? 1 : 0);
                const int v = lane >> kSh, q = v / EPW, x = v - q * EPW;
                float bx = bias[0];
#pragma unroll
                for (int xx = 1; xx < EPW; ++xx)
                    if (x == xx) bx = bias[xx];
                if (a.bias) r = __fadd_rn(r, bx);
                if ((lane & ((1 << kSh) - 1)) == 0 && tt + q < nt && e0 + x < E)
                    a.logits[(int64_t)(t0 + tt + q) * E + e0 + x] = r;
            }
        }
        __syncthreads();                       // the stage is consumed: refill it
        if (stages == 2) issue(i + 2);
        if (!a.cnt_tok) continue;              // logits only; k_topk follows
        // arrival.  When CTAs stream several blocks, block b's counter takes
        // gx + 1 increments: one arrival per CTA of its token blocks, plus a
        // claim by its owner CTA (x = i % gx) after that CTA's stream, and
        // whoever makes the last increment does the top-k -- in practice the
        // owner, so that the top-k work is spread over the CTAs whatever order
        // they arrive in.  With one block per CTA the last arrival does it.
        // An arrival that completes the count defers its top-k to the end of
        // its own stream.
        if (threadIdx.x == 0) {
            __threadfence();
            const bool last = atomicAdd(&a.cnt_tok[b], 1) == target;
            if (i < 32 * kRouterOwnWords) {
                if (last) s_own[i >> 5] |= 1u << (i & 31);
            } else {
                s_last = last;
            }
        }
        if (i >= 32 * kRouterOwnWords) {       // past the deferred list: inline
            __syncthreads();
            if (s_last) topk_block(b);
            __syncthreads();
        }
    }
    if (!a.cnt_tok) return;
    if (claims) {
        for (int i = (int)blockIdx.x; i < nmine; i += (int)gridDim.x) {
            const int b = (int)blockIdx.y + i * gy;
            if (threadIdx.x == 0) {
                __threadfence();
                s_last = atomicAdd(&a.cnt_tok[b], 1) == target;
            }
            __syncthreads();
            if (s_last) topk_block(b);
            __syncthreads();
        }
    }
    __syncthreads();
    for (int i = 0; i < min(nmine, 32 * kRouterOwnWords); ++i)
        if ((s_own[i >> 5] >> (i & 31)) & 1u) topk_block((int)blockIdx.y + i * gy);
}

// Standalone top-k + softmax: one warp per token over logits [T][E].
__global__ void __launch_bounds__(128) k_topk(const float* __restrict__ logits, int T, int E, int k,
                                              int32_t* __restrict__ idx, float* __restrict__ wts) {
    extern __shared__ float tsm[];
    pdl_wait();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int t = blockIdx.x * 4 + warp;
    if (t >= T) return;
    float* lg = tsm + warp * E;
    for (int x = lane; x < E; x += 32) lg[x] = __ldcg(logits + (int64_t)t * E + x);
    __syncwarp();
    warp_topk_softmax(lg, E, k, idx + (int64_t)t * k, wts + (int64_t)t * k);
    pdl_trigger();
}

// ============================================================================
// Grouped quantised GEMV (dp4a) over the slice-major arena -- one warp per
// work unit.
//
// A unit is (group a, 128-row tile, chunk c of 8 blocks, 32-row slice s).  A
// group is one expert with the pairs the bucketing gave it, or the whole dense
// matrix with all T tokens.  Lane l owns row 32 s + l of the tile.
//
// Each warp runs its own ring of shared-memory stages: for a unit it issues
// bulk copies (completing on the stage's mbarrier) of the slice's codes for the
// chunk (8 KB Q8_0 / 4 KB Q4_0, contiguous), its fp16 scales (512 B) and, per
// token, the chunk's activation slice (8 Q8_1 blocks, or 256 raw values that
// it quantises itself).  The unit's weights are loaded into registers once and
// reused for every token.  The per-chunk partial sums go to a partial buffer;
// the warp completing the last of a tile's units (an atomic counter per tile)
// adds the chunks in order and runs the epilogue.  No block-wide barrier is
// taken after the start.  Work is dealt to the persistent CTAs in contiguous
// unit ranges; inside a CTA the warps take units from a shared counter.
// ============================================================================
constexpr int kTokMax = 32;        // tokens a unit stages at once

// OUT_F32_NV: fp32 rows and their NVFP4 blocks (the latent z of a layer with
// NVFP4 experts; the cluster GEMV only).
enum { OUT_F32 = 0, OUT_F32_Q81 = 1, OUT_SWIGLU = 2, OUT_F32_COMBINE = 3, OUT_F32_ADD = 4, OUT_F32_NV = 5 };
enum { X_Q81_TOKEN = 0, X_Q81_PAIR_TOKEN = 1, X_Q81_POSITION = 2, X_RAW_F32 = 3, X_RAW_BF16 = 4 };

struct WArgs {
    const uint8_t* q;           // arena codes of group 0
    const uint16_t* d;          // arena scales of group 0
    int64_t q_gstride;          // bytes between groups (experts)
    int64_t d_gstride;          // fp16 elements between groups
    int nb, tiles, nchunks;
    const int32_t* act;         // active experts, NULL for one dense group
    const int32_t* n_act;
    const int32_t* offsets;     // [E+1] pair offsets, NULL for dense
    const int32_t* perm;
    int kslots;                 // top-k: token of pair p is p / k
    int T;
    const void* x;
    int x_mode;
    int64_t x_row;              // elements per raw input row (X_RAW_*)
    int out_mode;
    float* y;                   // fp32 rows (token or pair position)
    int64_t y_ld;
    uint8_t* yq;                // Q8_1 rows
    int64_t yq_ld;              // blocks per Q8_1 row
    // OUT_F32_COMBINE: weighted combine of each token's k rows of y
    const float* wts;
    const int32_t* pos;
    int* cnt_comb;              // [T][tiles], zero on entry/exit
    float* ylat;
    uint8_t* ylq;
    int* comb_done;             // [tiles] tokens combined per latent tile, or NULL
    float* partial;             // [nchunks][part_tok][tiles*128]
    int64_t part_tok;
    int* counters;              // [groups][tiles], zero on entry/exit
    int dense_tg;               // dense: tokens per group (the token groups share the weights); 0 = all T
    int* err;
    uint64_t budget_ns;
    int stages, tokcap;
    int stage_bytes, act_off, act_bytes, scratch_bytes;
    // routing (act/offsets/perm) was complete before this grid was launched:
    // the prologue may read it before the grid dependency is resolved
    int routing_early;
};

template <int FMT>
struct WSlice {
    // bytes per (slice, block): Q8_0 codes; 4-bit codes (Q4_0, NVFP4, Q4_K);
    // 4-bit codes and a word of fifth bits per row (Q5_1, Q5_K)
    static constexpr int kCodes = (FMT == 8) ? 1024 : fmt_has_qh(FMT) ? 640 : 512;
};

struct WUnit {
    int a, tile, c, s, e, tok0, ntok, kbn;
};

// A warp's cache of the last group it decoded: its expert, first pair
// position and pair count, and (lane i < ntok) the token of its pair i.  The
// units a warp takes run in group order, so one L2 round trip per group
// replaces one per unit.
struct WGroupCache {
    int a, e, tok0, ntok, tok;
};

__device__ __forceinline__ WUnit wunit(const WArgs& g, int u) {
    WUnit r;
    const int per_tile = g.nchunks * 4;
    const int per_group = g.tiles * per_tile;
    r.a = u / per_group;
    int rem = u - r.a * per_group;
    r.tile = rem / per_tile;
    rem -= r.tile * per_tile;
    r.c = rem >> 2;
    r.s = rem & 3;
    r.e = g.act ? __ldcg(g.act + r.a) : 0;
    if (g.offsets) {
        r.tok0 = __ldcg(g.offsets + r.e);
        r.ntok = __ldcg(g.offsets + r.e + 1) - r.tok0;
    } else {
        const int tg = g.dense_tg > 0 ? g.dense_tg : g.T;
        r.tok0 = r.a * tg;
        r.ntok = min(tg, g.T - r.tok0);
    }
    r.kbn = min(kChunk, g.nb - r.c * kChunk);
    return r;
}

// wunit through the warp's group cache (all lanes call it with the same u).
template <int XM>
__device__ __forceinline__ WUnit wunit_c(const WArgs& g, int u, WGroupCache& c) {
    WUnit r;
    const int per_tile = g.nchunks * 4;
    const int per_group = g.tiles * per_tile;
    r.a = u / per_group;
    int rem = u - r.a * per_group;
    r.tile = rem / per_tile;
    rem -= r.tile * per_tile;
    r.c = rem >> 2;
    r.s = rem & 3;
    if (g.act) {
        if (c.a != r.a) {
            c.a = r.a;
            c.e = __ldcg(g.act + r.a);
            c.tok0 = __ldcg(g.offsets + c.e);
            c.ntok = __ldcg(g.offsets + c.e + 1) - c.tok0;
            c.tok = 0;
            if (XM == X_Q81_PAIR_TOKEN) {
                const int lane = threadIdx.x & 31;
                if (lane < c.ntok) c.tok = __ldcg(g.perm + c.tok0 + lane) / g.kslots;
            }
        }
        r.e = c.e;
        r.tok0 = c.tok0;
        r.ntok = c.ntok;
    } else {
        const int tg = g.dense_tg > 0 ? g.dense_tg : g.T;
        r.e = 0;
        r.tok0 = r.a * tg;
        r.ntok = min(tg, g.T - r.tok0);
    }
    r.kbn = min(kChunk, g.nb - r.c * kChunk);
    return r;
}

template <int XM>
__device__ __forceinline__ int64_t wunit_xrow(const WArgs& g, const WUnit& un, int i) {
    const int tp = un.tok0 + i;
    if (XM == X_Q81_PAIR_TOKEN) return __ldcg(g.perm + tp) / g.kslots;
    return tp;   // token (dense) or pair position
}

// Bytes of one token's activation slice for a chunk of kbn blocks.
template <int XM>
__device__ __forceinline__ uint32_t wact_bytes(int kbn) {
    if (XM == X_RAW_F32) return (uint32_t)kbn * 128u;
    if (XM == X_RAW_BF16) return (uint32_t)kbn * 64u;
    return (uint32_t)kbn * 36u;
}

template <int FMT, int XM>
__device__ __forceinline__ void wissue_weights(const WArgs& g, const WUnit& un, uint8_t* stage, uint64_t* bar,
                                               int ntok_pass) {
    using SL = WSlice<FMT>;
    const int lane = threadIdx.x & 31;
    const uint32_t cb = (uint32_t)(un.kbn * SL::kCodes), sb = (uint32_t)(un.kbn * 64);
    if (lane == 0) mbar_arrive_expect_tx(bar, cb + sb + (uint32_t)ntok_pass * wact_bytes<XM>(un.kbn));
    __syncwarp();
    if (lane == 0) {
        const uint8_t* src = g.q + un.e * g.q_gstride +
                             ((int64_t)un.tile * g.nb * 4 + (int64_t)un.s * g.nb + (int64_t)un.c * kChunk) * SL::kCodes;
        bulk_g2s(stage, src, cb, bar);
    } else if (lane == 1) {
        const uint16_t* src = g.d + un.e * g.d_gstride + (int64_t)un.tile * g.nb * kTileRows +
                              (int64_t)un.s * g.nb * 32 + (int64_t)un.c * kChunk * 32;
        bulk_g2s(stage + kChunk * SL::kCodes, src, sb, bar);
    }
}

template <int XM>
__device__ __forceinline__ void wissue_acts(const WArgs& g, const WUnit& un, uint8_t* act_area, uint64_t* bar,
                                            int first, int ntok_pass, const WGroupCache* c = nullptr) {
    const int lane = threadIdx.x & 31;
    const uint32_t ab = wact_bytes<XM>(un.kbn);
    for (int i = lane; i < ntok_pass; i += 32) {
        const int64_t row = (XM == X_Q81_PAIR_TOKEN && c && first == 0 && i < 32 && c->a == un.a)
                                ? (int64_t)c->tok
                                : wunit_xrow<XM>(g, un, first + i);
        const uint8_t* src;
        if (XM == X_RAW_F32)
            src = static_cast<const uint8_t*>(g.x) + (row * g.x_row + (int64_t)un.c * 256) * 4;
        else if (XM == X_RAW_BF16)
            src = static_cast<const uint8_t*>(g.x) + (row * g.x_row + (int64_t)un.c * 256) * 2;
        else
            src = static_cast<const uint8_t*>(g.x) + (row * g.nb + (int64_t)un.c * kChunk) * 36;
        bulk_g2s(act_area + i * g.act_bytes, src, ab, bar);
    }
}

// The unit's slice of weights (in its stage) into registers: w[kb][j] holds
// the signed 8-bit codes 4j..4j+3 of block kb of this lane's row, dw[kb] its
// scale; blocks past kbn are zero.
template <int FMT>
__device__ __forceinline__ void wload_regs(const uint8_t* stg, int kbn, int (&w)[kChunk][8], float (&dw)[kChunk]) {
    using SL = WSlice<FMT>;
    const int lane = threadIdx.x & 31;
    const uint16_t* sc = reinterpret_cast<const uint16_t*>(stg + kChunk * SL::kCodes);
#pragma unroll
    for (int kb = 0; kb < kChunk; ++kb) {
        if (kb < kbn) {
            dw[kb] = h2f(sc[kb * 32 + lane]);
            if (FMT == 8) {
                const uint8_t* cp = stg + kb * 1024 + (lane >> 3) * 256 + (lane & 7) * 16;
                const uint4 a = lds128(cp), b = lds128(cp + 128);
                w[kb][0] = (int)a.x; w[kb][1] = (int)a.y; w[kb][2] = (int)a.z; w[kb][3] = (int)a.w;
                w[kb][4] = (int)b.x; w[kb][5] = (int)b.y; w[kb][6] = (int)b.z; w[kb][7] = (int)b.w;
            } else {
                const uint4 a = lds128(stg + kb * 512 + lane * 16);
                const uint32_t v[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    // nibbles q (0..15) -> signed bytes q - 8, without borrows between bytes
                    const uint32_t lo = v[j] & 0x0F0F0F0Fu, hi = (v[j] >> 4) & 0x0F0F0F0Fu;
                    w[kb][j] = (int)(((lo | 0x80808080u) - 0x08080808u) ^ 0x80808080u);
                    w[kb][4 + j] = (int)(((hi | 0x80808080u) - 0x08080808u) ^ 0x80808080u);
                }
            }
        } else {
            dw[kb] = 0.0f;
#pragma unroll
            for (int j = 0; j < 8; ++j) w[kb][j] = 0;
        }
    }
}

// The row dot products of one unit with np staged tokens (the unit's tokens
// first .. first + np - 1), each chunk partial stored to the partial buffer.
// Raw activations are first quantised to Q8_1 in the warp's scratch.
template <int XM>
__device__ __forceinline__ void wdots(const WArgs& g, const WUnit& un, const int (&w)[kChunk][8],
                                      const float (&dw)[kChunk], const uint8_t* abase, int np, int first,
                                      uint8_t* scratch) {
    const int lane = threadIdx.x & 31;
    int astride = g.act_bytes;
    if (XM == X_RAW_F32 || XM == X_RAW_BF16) {
        for (int t = 0; t < np; ++t)
            for (int kb = 0; kb < un.kbn; ++kb) {
                float v;
                if (XM == X_RAW_F32)
                    v = reinterpret_cast<const float*>(abase + t * g.act_bytes)[kb * 32 + lane];
                else
                    v = __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(abase + t * g.act_bytes)[kb * 32 + lane]);
                warp_quant_q8_1(v, scratch + (t * kChunk + kb) * 36);
            }
        __syncwarp();
        abase = scratch;
        astride = kChunk * 36;
    }
    const int64_t rows_total = (int64_t)g.tiles * kTileRows;
    for (int t = 0; t < np; ++t) {
        const uint8_t* ab = abase + t * astride;
        float part = 0.0f;
#pragma unroll
        for (int kb = 0; kb < kChunk; ++kb) {
            if (kb < un.kbn) {
                const uint32_t* aw = reinterpret_cast<const uint32_t*>(ab + kb * 36 + 4);
                int isum = 0;
#pragma unroll
                for (int j = 0; j < 8; ++j) isum = __dp4a(w[kb][j], (int)aw[j], isum);
                const float da = h2f(*reinterpret_cast<const uint16_t*>(ab + kb * 36));
                part = __fmaf_rn(__int2float_rn(isum), __fmul_rn(dw[kb], da), part);
            }
        }
        const int64_t tokidx = (int64_t)un.tok0 + first + t;
        __stcg(g.partial + ((int64_t)un.c * g.part_tok + tokidx) * rows_total + (int64_t)un.tile * kTileRows +
                   un.s * 32 + lane,
               part);
    }
}

// Epilogue of a finished tile (all chunk partials present) by one warp.  The
// chunk partials of up to 16 chunks are loaded before any is added, so the
// L2 round trips overlap; the adds then run in chunk order.
template <int OM>
__device__ void wepilogue(const WArgs& g, const WUnit& un) {
    const int lane = threadIdx.x & 31;
    const int64_t rows_total = (int64_t)g.tiles * kTileRows;
    for (int i = 0; i < un.ntok; ++i) {
        const int64_t tokidx = (int64_t)un.tok0 + i;
        float v[4] = {0.0f, 0.0f, 0.0f, 0.0f};
        const float* pb = g.partial + tokidx * rows_total + (int64_t)un.tile * kTileRows + lane;
        const int64_t cstride = g.part_tok * rows_total;
        for (int c0 = 0; c0 < g.nchunks; c0 += 16) {
            float t[16][4];
#pragma unroll
            for (int c = 0; c < 16; ++c)
                if (c0 + c < g.nchunks) {
#pragma unroll
                    for (int q = 0; q < 4; ++q) t[c][q] = __ldcg(pb + (int64_t)(c0 + c) * cstride + 32 * q);
                }
#pragma unroll
            for (int c = 0; c < 16; ++c)
                if (c0 + c < g.nchunks) {
#pragma unroll
                    for (int q = 0; q < 4; ++q) v[q] = __fadd_rn(v[q], t[c][q]);
                }
        }
        if (OM == OUT_SWIGLU) {
#pragma unroll
            for (int hb = 0; hb < 2; ++hb) {
                const float h = __fmul_rn(silu_f32(v[hb]), v[2 + hb]);
                warp_quant_q8_1(h, g.yq + (tokidx * g.yq_ld + un.tile * 2 + hb) * 36);
            }
            continue;
        }
        float* yr = g.y + tokidx * g.y_ld + (int64_t)un.tile * kTileRows + lane;
        if (OM == OUT_F32_ADD) {
            // residual stream: y = y + the rows (fp32)
#pragma unroll
            for (int q = 0; q < 4; ++q) yr[32 * q] = __fadd_rn(yr[32 * q], v[q]);
            continue;
        }
#pragma unroll
        for (int q = 0; q < 4; ++q) yr[32 * q] = v[q];
        if (OM == OUT_F32_Q81) {
#pragma unroll
            for (int q = 0; q < 4; ++q)
                warp_quant_q8_1(v[q], g.yq + (tokidx * g.yq_ld + un.tile * 4 + q) * 36);
        } else if (OM == OUT_F32_COMBINE) {
            // the pair's rows of this tile are out: count them for the token
            __threadfence();
            __syncwarp();
            const int p = __ldcg(g.perm + tokidx);
            const int t = p / g.kslots;
            int last = 0;
            if (lane == 0) {
                int* cnt = g.cnt_comb + (int64_t)t * g.tiles + un.tile;
                last = (atomicAdd(cnt, 1) == g.kslots - 1);
                if (last) *cnt = 0;
            }
            last = __shfl_sync(kFull, last, 0);
            if (last) {
                __threadfence();
                const int L = g.tiles * kTileRows;
                float acc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
                for (int j0 = 0; j0 < g.kslots; j0 += 8) {
                    float ov[8][4], wv[8];
#pragma unroll
                    for (int j = 0; j < 8; ++j)
                        if (j0 + j < g.kslots) {
                            const int pj = t * g.kslots + j0 + j;
                            wv[j] = __ldcg(g.wts + pj);
                            const float* orow =
                                g.y + (int64_t)__ldcg(g.pos + pj) * g.y_ld + (int64_t)un.tile * kTileRows + lane;
#pragma unroll
                            for (int q = 0; q < 4; ++q) ov[j][q] = __ldcg(orow + 32 * q);
                        }
#pragma unroll
                    for (int j = 0; j < 8; ++j)
                        if (j0 + j < g.kslots) {
#pragma unroll
                            for (int q = 0; q < 4; ++q) acc[q] = __fmaf_rn(wv[j], ov[j][q], acc[q]);
                        }
                }
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    g.ylat[(int64_t)t * L + un.tile * kTileRows + 32 * q + lane] = acc[q];
                    warp_quant_q8_1(acc[q], g.ylq + ((int64_t)t * (L / 32) + un.tile * 4 + q) * 36);
                }
                if (g.comb_done) {
                    // consumers in this grid read ylq with bulk copies
                    fence_proxy_async_global();
                    __threadfence();
                    __syncwarp();
                    if (lane == 0) atomicAdd(g.comb_done + un.tile, 1);
                }
            }
        }
    }
}

// Completion of a batch of this warp's finished units (held one per lane in
// `pending`): one fence for all their partial stores, one atomic per unit;
// the warp then runs the epilogue of every tile it completed.
template <int OM>
__device__ __forceinline__ void wcomplete(const WArgs& g, int pending, int npend) {
    const int lane = threadIdx.x & 31;
    __threadfence();
    __syncwarp();
    int last = 0;
    if (lane < npend) {
        const WUnit un = wunit(g, pending);
        int* cnt = g.counters + (int64_t)un.a * g.tiles + un.tile;
        last = (atomicAdd(cnt, 1) == g.nchunks * 4 - 1);
        if (last) *cnt = 0;
    }
    unsigned m = __ballot_sync(kFull, last);
    if (m) __threadfence();
    while (m) {
        const int j = __ffs(m) - 1;
        m &= m - 1;
        const int u = __shfl_sync(kFull, pending, j);
        wepilogue<OM>(g, wunit(g, u));
    }
    __syncwarp();
}

template <int FMT, int XM, int OM>
__global__ void __launch_bounds__(256, 1) k_wgemv(WArgs g) {
    extern __shared__ __align__(128) uint8_t wsm[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int S = g.stages;
    uint64_t* bars = reinterpret_cast<uint64_t*>(wsm);                 // [nwarps][S]
    int* unit_of = reinterpret_cast<int*>(wsm + 8 * 8 * 4);             // [nwarps][S], S <= 4
    int* s_next = reinterpret_cast<int*>(wsm + 8 * 8 * 4 + 8 * 4 * 4);
    uint8_t* stages = wsm + 512 + (size_t)warp * (S * g.stage_bytes + g.scratch_bytes);
    uint8_t* scratch = stages + S * g.stage_bytes;
    uint64_t* mybar = bars + warp * 4;
    int* myunit = unit_of + warp * 4;

    if (threadIdx.x == 0) *s_next = 0;
    if (lane <= S) mbar_init(&mybar[lane], 1);     // S ring stages + one for extra token passes
    if (lane == 0) fence_barrier_init();
    __syncthreads();

    const bool dense = (g.act == nullptr);
    const bool early = dense || g.routing_early;
    int64_t n_units = 0, u0 = 0, u1 = 0;
    auto range = [&]() {
        const int64_t groups = dense ? (g.dense_tg > 0 ? (g.T + g.dense_tg - 1) / g.dense_tg : 1)
                                     : (int64_t)__ldcg(g.n_act);
        n_units = groups * g.tiles * g.nchunks * 4;
        u0 = n_units * blockIdx.x / gridDim.x;
        u1 = n_units * (blockIdx.x + 1) / gridDim.x;
    };
    auto grab = [&]() -> int {
        int u = 0;
        if (lane == 0) u = atomicAdd(s_next, 1);
        u = __shfl_sync(kFull, u, 0) + (int)u0;
        return (u < u1) ? u : -1;
    };
    const int tokcap = g.tokcap;
    WGroupCache gcache{-1, 0, 0, 0, 0};
    // completions are counted in batches; heavier units (more tokens each)
    // count sooner, so that tile epilogues spread over the warps
    const int cbatch = max(1, 32 / max(1, tokcap));

    // prologue: fill the ring.  Weights do not depend on the upstream kernel
    // (and the routing, when it was complete before this grid started), so
    // their copies start before the grid dependency is resolved.
    if (early) {
        range();
        for (int st = 0; st < S; ++st) {
            const int u = grab();
            if (lane == 0) myunit[st] = u;
            if (u >= 0) {
                const WUnit un = wunit_c<XM>(g, u, gcache);
                wissue_weights<FMT, XM>(g, un, stages + st * g.stage_bytes, &mybar[st], min(un.ntok, tokcap));
            }
        }
        pdl_wait();
        pdl_trigger();
        __syncwarp();
        for (int st = 0; st < S; ++st) {
            const int u = myunit[st];
            if (u >= 0) {
                const WUnit un = wunit_c<XM>(g, u, gcache);
                wissue_acts<XM>(g, un, stages + st * g.stage_bytes + g.act_off, &mybar[st], 0, min(un.ntok, tokcap), &gcache);
            }
        }
    } else {
        pdl_wait();
        pdl_trigger();
        range();
        for (int st = 0; st < S; ++st) {
            const int u = grab();
            if (lane == 0) myunit[st] = u;
            if (u >= 0) {
                const WUnit un = wunit_c<XM>(g, u, gcache);
                uint8_t* stg = stages + st * g.stage_bytes;
                wissue_weights<FMT, XM>(g, un, stg, &mybar[st], min(un.ntok, tokcap));
                wissue_acts<XM>(g, un, stg + g.act_off, &mybar[st], 0, min(un.ntok, tokcap), &gcache);
            }
        }
    }
    __syncwarp();

    uint32_t xuse = 0;          // uses of the extra barrier (its phase parity)
    bool ok = true;
    int it = 0;
    int pending = -1, npend = 0; // finished units awaiting their completion count (one per lane)
    for (;; ++it) {
        const int st = it % S;
        const int u = myunit[st];
        if (u < 0) break;
        if (!mbar_wait_bounded(&mybar[st], (uint32_t)((it / S) & 1), g.err, g.budget_ns)) {
            ok = false;
            break;
        }
        const WUnit un = wunit_c<XM>(g, u, gcache);
        uint8_t* stg = stages + st * g.stage_bytes;

        int w[kChunk][8];
        float dw[kChunk];
        wload_regs<FMT>(stg, un.kbn, w, dw);
        __syncwarp();

        for (int first = 0; first < un.ntok; first += tokcap) {
            const int np = min(tokcap, un.ntok - first);
            if (first > 0) {
                // more tokens than one staging holds: reload the activation area
                __syncwarp();
                fence_proxy_async();
                uint64_t* xb = &mybar[S];
                if (lane == 0) mbar_arrive_expect_tx(xb, (uint32_t)np * wact_bytes<XM>(un.kbn));
                __syncwarp();
                wissue_acts<XM>(g, un, stg + g.act_off, xb, first, np);
                const bool got = mbar_wait_bounded(xb, xuse & 1u, g.err, g.budget_ns);
                ++xuse;
                if (!got) {
                    ok = false;
                    break;
                }
            }
            wdots<XM>(g, un, w, dw, stg + g.act_off, np, first, scratch);
        }
        if (!ok) break;
        // stage consumed: refill it with this warp's next unit
        __syncwarp();
        fence_proxy_async();
        {
            const int nu = grab();
            if (lane == 0) myunit[st] = nu;
            if (nu >= 0) {
                const WUnit nn = wunit_c<XM>(g, nu, gcache);
                wissue_weights<FMT, XM>(g, nn, stg, &mybar[st], min(nn.ntok, tokcap));
                wissue_acts<XM>(g, nn, stg + g.act_off, &mybar[st], 0, min(nn.ntok, tokcap), &gcache);
            }
        }
        // completion of the tile (the last of its 4 * nchunks units runs the
        // epilogue), batched per warp so that one fence covers many units
        if (lane == npend) pending = u;
        if (++npend == cbatch) {
            wcomplete<OM>(g, pending, npend);
            npend = 0;
        }
    }
    if (ok && npend) wcomplete<OM>(g, pending, npend);
    if (!ok) {
        // drain: wait (bounded) for this warp's copies still in flight
        for (int k = 0; k < S; ++k) {
            const int j = it + k;
            if (myunit[j % S] >= 0) mbar_wait_bounded(&mybar[j % S], (uint32_t)((j / S) & 1), nullptr, g.budget_ns);
        }
        if (xuse) mbar_wait_bounded(&mybar[S], (xuse - 1) & 1u, nullptr, g.budget_ns);
    }
}

// RMS normalisation of each row of h (one warp per row): lane j sums h_i^2
// for i = j, j + 32, ... with fused multiply-adds, an xor butterfly (16 .. 1)
// of adds gives the total, ms = total / H, r = sqrt(ms + 1e-6), out_i =
// h_i / r (every operation IEEE round-to-nearest).
__global__ void __launch_bounds__(256) k_rmsnorm(const float* __restrict__ h, int T, int H, float* __restrict__ out) {
    const int lane = threadIdx.x & 31;
    const int t = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (t >= T) return;
    const float* hr = h + (int64_t)t * H;
    float p = 0.0f;
    for (int i = lane; i < H; i += 32) p = __fmaf_rn(hr[i], hr[i], p);
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) p = __fadd_rn(p, __shfl_xor_sync(0xffffffffu, p, o));
    const float ms = __fdiv_rn(p, (float)H);
    const float r = __fsqrt_rn(__fadd_rn(ms, 1e-6f));
    float* orow = out + (int64_t)t * H;
    for (int i = lane; i < H; i += 32) orow[i] = __fdiv_rn(hr[i], r);
}

// The residual stream's first value: fp32 copy of x (bf16 or fp32).
template <bool BF16>
__global__ void __launch_bounds__(256) k_to_f32(const void* __restrict__ x, int64_t n, float* __restrict__ h) {
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= n) return;
    h[i] = BF16 ? __bfloat162float(static_cast<const __nv_bfloat16*>(x)[i]) : static_cast<const float*>(x)[i];
}

// ============================================================================
// test kernels
// ============================================================================
__global__ void k_test_block_isums(int wfmt, const uint8_t* w, const uint8_t* x, int64_t n, int32_t* isum,
                                   float* term) {
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= n) return;
    const uint8_t* a = x + i * 36;
    int s = 0;
    if (wfmt == 8) {
        const uint8_t* b = w + i * 34;
        for (int j = 0; j < 32; ++j) s += (int)(int8_t)b[2 + j] * (int)(int8_t)a[4 + j];
        const float sc = __fmul_rn(h2f((uint16_t)(b[0] | (b[1] << 8))), h2f((uint16_t)(a[0] | (a[1] << 8))));
        isum[i] = s;
        term[i] = __fmul_rn(__int2float_rn(s), sc);
    } else {
        const uint8_t* b = w + i * 18;
        for (int j = 0; j < 16; ++j)
            s += ((b[2 + j] & 15) - 8) * (int)(int8_t)a[4 + j] + ((b[2 + j] >> 4) - 8) * (int)(int8_t)a[20 + j];
        const float sc = __fmul_rn(h2f((uint16_t)(b[0] | (b[1] << 8))), h2f((uint16_t)(a[0] | (a[1] << 8))));
        isum[i] = s;
        term[i] = __fmul_rn(__int2float_rn(s), sc);
    }
}

__global__ void k_test_expf(const float* in, float* out, int64_t n) {
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i < n) out[i] = exp_f32(in[i]);
}

}  // namespace elq
