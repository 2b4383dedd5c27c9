// elq_kernels.cuh -- the layer's sm_100a kernels (decode/verify path):
//   k_quant_q8_1      a1/a4  activation quantiser
//   k_quant_weights   arena preparation from fp32 weights
//   k_arena_pack      arena preparation from GGUF-style AoS blocks
//   k_router          a3 (+a5)  logits, top-k, softmax, bucketing
//   k_bucket          a5 standalone
//   k_qgemv           a2/a6/a7/a8/a10  grouped quantised GEMV over the arena
//   k_combine         a9  weighted combine + Q8_1
#pragma once

#include "elq_device.cuh"

namespace elq {

constexpr unsigned kFull = 0xffffffffu;

// ============================================================================
// a1 / a4 -- Q8_1 activation quantiser: one warp per 32-value block.
// ============================================================================
template <bool kBF16>
__global__ void __launch_bounds__(256) k_quant_q8_1(const void* __restrict__ x, int64_t nblocks,
                                                    uint8_t* __restrict__ out) {
    pdl_wait();
    const int64_t blk = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (blk >= nblocks) return;
    float v;
    if (kBF16)
        v = __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(x)[blk * 32 + lane]);
    else
        v = reinterpret_cast<const float*>(x)[blk * 32 + lane];
    warp_quant_q8_1(v, out + blk * 36);
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
    const int r = (int)(row % kTileRows);
    const int64_t slab = tile * nb + kb;
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
        uint8_t* dst = q + slab * kQ80Slab + (r >> 3) * 256 + (r & 7) * 16;
        *reinterpret_cast<uint4*>(dst) = make_uint4(words[0], words[1], words[2], words[3]);
        *reinterpret_cast<uint4*>(dst + 128) = make_uint4(words[4], words[5], words[6], words[7]);
        d[slab * kTileRows + r] = f2h(dd);
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
        uint8_t* dst = q + slab * kQ40Slab + r * 16;
        *reinterpret_cast<uint4*>(dst) = make_uint4(words[0], words[1], words[2], words[3]);
        d[slab * kTileRows + r] = f2h(dd);
    }
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
    const int r = (int)(row % kTileRows);
    const int64_t slab = tile * nb + kb;
    d[slab * kTileRows + r] = (uint16_t)(src[0] | (src[1] << 8));
    uint32_t words[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    const int nq = (FMT == 8) ? 32 : 16;
    for (int i = 0; i < nq; ++i) words[i >> 2] |= (uint32_t)src[2 + i] << (8 * (i & 3));
    if (FMT == 8) {
        uint8_t* dst = q + slab * kQ80Slab + (r >> 3) * 256 + (r & 7) * 16;
        *reinterpret_cast<uint4*>(dst) = make_uint4(words[0], words[1], words[2], words[3]);
        *reinterpret_cast<uint4*>(dst + 128) = make_uint4(words[4], words[5], words[6], words[7]);
    } else {
        *reinterpret_cast<uint4*>(q + slab * kQ40Slab + r * 16) = make_uint4(words[0], words[1], words[2], words[3]);
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
    for (int p = s0 + lane; p < s1; p += 32) atomicAdd(&hist[warp * E + __ldcg(idx + p)], 1);
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
    for (int c0 = s0; c0 < s1; c0 += 32) {
        const int p = c0 + lane;
        const bool v = p < s1;
        const int e = v ? __ldcg(idx + p) : -1 - lane;
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
// k selected; optionally a5 by the last CTA.  Grid (ceil(E/4), ceil(T/8)),
// 128 threads: one warp per expert, 8 tokens per CTA.  The last CTA of a
// token block does that block's top-k; the last token block buckets.
// ============================================================================
constexpr int kRouterWarps = 4;
constexpr int kRouterTok = 8;

struct RouterArgs {
    const float* z;
    const float* w;
    const float* bias;
    int T, L, E, k;
    int32_t* idx;
    float* wts;
    float* logits;
    int* cnt_tok;     // [gridDim.y], zero on entry, zero on exit
    int* cnt_all;     // [1]
    int do_bucket;
    int32_t *counts, *offsets, *perm, *pos, *act, *n_act;
};

// Top-k of one token's logits (in shared memory, lg[0..E)) by one warp, then
// the softmax over the k selected in rank order.  Lane j ends with rank j.
__device__ __forceinline__ void warp_topk_softmax(const float* lg, int E, int k, int32_t* idx_out,
                                                  float* w_out) {
    const int lane = threadIdx.x & 31;
    uint32_t taken = 0;
    float sel_v = 0.0f;
    int sel_e = 0;
    for (int j = 0; j < k; ++j) {
        float bv = -INFINITY;
        int be = 0x7fffffff;
        for (int i = 0, x = lane; x < E; ++i, x += 32) {
            if (taken & (1u << i)) continue;
            const float v = lg[x];
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
    }
}

__global__ void __launch_bounds__(128) k_router(RouterArgs a) {
    extern __shared__ float rsm[];
    __shared__ int s_last;
    pdl_wait();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int t0 = blockIdx.y * kRouterTok;
    const int nt = min(kRouterTok, a.T - t0);
    for (int i = threadIdx.x; i < nt * a.L; i += blockDim.x) rsm[i] = a.z[(int64_t)t0 * a.L + i];
    __syncthreads();
    const int e = blockIdx.x * kRouterWarps + warp;
    if (e < a.E) {
        const float* wr = a.w + (int64_t)e * a.L;
        const float b = a.bias ? a.bias[e] : 0.0f;
        for (int tt = 0; tt < nt; ++tt) {
            const float* zt = rsm + tt * a.L;
            float p = 0.0f;
            for (int l = lane; l < a.L; l += 32) p = __fmaf_rn(zt[l], __ldg(wr + l), p);
#pragma unroll
            for (int o = 16; o >= 1; o >>= 1) p = __fadd_rn(p, __shfl_xor_sync(kFull, p, o));
            if (a.bias) p = __fadd_rn(p, b);
            if (lane == 0) a.logits[(int64_t)(t0 + tt) * a.E + e] = p;
        }
    }
    if (!a.cnt_tok) {       // logits only; k_topk follows
        pdl_trigger();
        return;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        __threadfence();
        s_last = (atomicAdd(&a.cnt_tok[blockIdx.y], 1) == (int)gridDim.x - 1);
    }
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    float* lg = rsm + warp * a.E;
    for (int tt = warp; tt < nt; tt += kRouterWarps) {
        const int t = t0 + tt;
        for (int x = lane; x < a.E; x += 32) lg[x] = __ldcg(a.logits + (int64_t)t * a.E + x);
        __syncwarp();
        warp_topk_softmax(lg, a.E, a.k, a.idx + (int64_t)t * a.k, a.wts + (int64_t)t * a.k);
        __syncwarp();
    }
    __syncthreads();
    if (threadIdx.x == 0) a.cnt_tok[blockIdx.y] = 0;
    if (!a.do_bucket) {
        pdl_trigger();
        return;
    }
    if (threadIdx.x == 0) {
        __threadfence();
        s_last = (atomicAdd(a.cnt_all, 1) == (int)gridDim.y - 1);
    }
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    bucket_cta(a.idx, a.T * a.k, a.E, a.counts, a.offsets, a.perm, a.pos, a.act, a.n_act,
               reinterpret_cast<int*>(rsm));
    if (threadIdx.x == 0) *a.cnt_all = 0;
    pdl_trigger();
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
// Grouped quantised GEMV (dp4a) over the tile-slab arena.
//
// Work unit: (group a, tile, chunk range).  A group is one expert with its
// pairs (from the bucketing) or the whole dense matrix with all T tokens.
// split == 1: a unit is one chunk of 8 blocks; its per-chunk partial sums go
//   to a partial buffer and the last unit of a tile to arrive (atomic counter)
//   adds the chunks' partials in order and runs the epilogue.
// split == 0: a unit is a whole tile; chunk partials are added in order in
//   shared memory and the same CTA runs the epilogue.
// Units are dealt to the persistent CTAs in contiguous ranges.  Each step
// (unit, 32-token block, chunk) streams its weight slabs (<= 32 KB of codes +
// 2 KB of scales) into a ring of shared-memory stages with two bulk copies
// completing on an mbarrier; the activations of the step's tokens are staged
// next to them.  Warp w owns rows 16w .. 16w+15 of the tile.
// ============================================================================
constexpr int kGemvThreads = 256;
constexpr int kGemvStages = 4;
constexpr int kTokBlock = 32;      // tokens per token block
constexpr int kTokPass = 4;        // tokens per register pass

enum { OUT_F32 = 0, OUT_F32_Q81 = 1, OUT_SWIGLU = 2 };
enum { X_DENSE = 0, X_PAIR_TOKEN = 1, X_POSITION = 2 };

struct GemvArgs {
    const uint8_t* q;           // arena codes of group 0
    const uint16_t* d;          // arena scales of group 0
    int64_t q_gstride;          // bytes between groups
    int64_t d_gstride;          // fp16 elements between groups
    int nb, tiles, nchunks, split;
    const int32_t* act;         // active experts (NULL: one dense group)
    const int32_t* n_act;
    const int32_t* offsets;     // [E+1] pair offsets (NULL: dense)
    const int32_t* perm;
    int kslots;                 // k: token of pair p is p / k
    int T;
    const uint8_t* x;           // Q8_1 rows, nb blocks each
    int x_mode;
    int out_mode;
    float* y;                   // fp32 out rows (token or position), ld y_ld
    int64_t y_ld;
    uint8_t* yq;                // Q8_1 out rows, yq_ld blocks each
    int64_t yq_ld;
    float* partial;             // split: [nchunks][part_tok][tiles*128]
    int64_t part_tok;
    int* counters;              // split: per (group slot, tile), zero on entry/exit
    int* err;
    uint64_t budget_ns;
};

template <int FMT>
struct GemvSmem {
    static constexpr int kSlab = (FMT == 8) ? kQ80Slab : kQ40Slab;
    static constexpr int kStageQ = kSlab * kChunk;
    static constexpr int kStage = kStageQ + kScaleSlab * kChunk;
    static constexpr int kStagesBytes = kStage * kGemvStages;
    static constexpr int kAq = kStagesBytes;                           // int8 [32 tok][8 kb][32]
    static constexpr int kAd = kAq + kTokBlock * kChunk * 32;          // float [32][8]
    static constexpr int kAs = kAd + kTokBlock * kChunk * 4;           // int [32][8]
    static constexpr int kAcc = kAs + kTokBlock * kChunk * 4;          // float [32][128]
    static constexpr int kBar = kAcc + kTokBlock * kTileRows * 4;      // uint64 [stages]
    static constexpr int kTotal = kBar + 8 * kGemvStages + 16;
};

struct GemvUnit {
    int a, tile, c0, c1;
    int e, tok0, ntok;          // tok0: first pair position (experts) or 0
    bool valid;
};

__device__ __forceinline__ GemvUnit gemv_unit(const GemvArgs& g, int64_t u, int64_t u_end) {
    GemvUnit r;
    r.valid = u < u_end;
    if (!r.valid) return r;
    const int per_group = g.tiles * (g.split ? g.nchunks : 1);
    r.a = (int)(u / per_group);
    const int rem = (int)(u % per_group);
    r.tile = g.split ? rem / g.nchunks : rem;
    r.c0 = g.split ? rem % g.nchunks : 0;
    r.c1 = g.split ? r.c0 + 1 : g.nchunks;
    r.e = g.act ? __ldg(g.act + r.a) : 0;
    if (g.offsets) {
        r.tok0 = __ldg(g.offsets + r.e);
        r.ntok = __ldg(g.offsets + r.e + 1) - r.tok0;
    } else {
        r.tok0 = 0;
        r.ntok = g.T;
    }
    return r;
}

// Step cursor over (unit, token block, chunk) in order.
struct GemvCursor {
    GemvUnit un;
    int64_t u, u_end;
    int tb, c;
    __device__ __forceinline__ void start(const GemvArgs& g, int64_t u0, int64_t u1) {
        u = u0;
        u_end = u1;
        un = gemv_unit(g, u, u_end);
        tb = 0;
        c = un.valid ? un.c0 : 0;
    }
    __device__ __forceinline__ bool valid() const { return un.valid; }
    __device__ __forceinline__ void advance(const GemvArgs& g) {
        if (++c < un.c1) return;
        c = un.c0;
        if (++tb * kTokBlock < un.ntok) return;
        tb = 0;
        ++u;
        un = gemv_unit(g, u, u_end);
        c = un.valid ? un.c0 : 0;
    }
};

template <int FMT>
__device__ __forceinline__ void gemv_issue(const GemvArgs& g, const GemvCursor& cu, uint8_t* stage,
                                           uint64_t* bar) {
    using S = GemvSmem<FMT>;
    const int kbn = min(kChunk, g.nb - cu.c * kChunk);
    const int64_t slab0 = (int64_t)cu.un.tile * g.nb + (int64_t)cu.c * kChunk;
    const uint8_t* qs = g.q + cu.un.e * g.q_gstride + slab0 * S::kSlab;
    const uint16_t* ds = g.d + cu.un.e * g.d_gstride + slab0 * kTileRows;
    const uint32_t qb = (uint32_t)(kbn * S::kSlab), db = (uint32_t)(kbn * kScaleSlab);
    mbar_arrive_expect_tx(bar, qb + db);
    bulk_g2s(stage, qs, qb, bar);
    bulk_g2s(stage + S::kStageQ, ds, db, bar);
}

// Epilogue of one token block of a tile from acc[tok][row] in shared memory.
__device__ __forceinline__ void gemv_epilogue(const GemvArgs& g, const GemvUnit& un, int tb, int ntb,
                                              const float* acc) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t orow0 = (int64_t)un.tok0 + tb * kTokBlock;   // token (dense) or position (experts)
    if (g.out_mode == OUT_SWIGLU) {
        for (int i = warp; i < ntb * 2; i += kGemvThreads / 32) {
            const int tok = i >> 1, hb = i & 1;
            const float gv = acc[tok * kTileRows + hb * 32 + lane];
            const float uv = acc[tok * kTileRows + 64 + hb * 32 + lane];
            const float h = __fmul_rn(silu_f32(gv), uv);
            warp_quant_q8_1(h, g.yq + ((orow0 + tok) * g.yq_ld + un.tile * 2 + hb) * 36);
        }
        return;
    }
    for (int i = threadIdx.x; i < ntb * kTileRows; i += kGemvThreads) {
        const int tok = i / kTileRows, r = i % kTileRows;
        g.y[(orow0 + tok) * g.y_ld + (int64_t)un.tile * kTileRows + r] = acc[i];
    }
    if (g.out_mode == OUT_F32_Q81) {
        for (int i = warp; i < ntb * 4; i += kGemvThreads / 32) {
            const int tok = i >> 2, b = i & 3;
            warp_quant_q8_1(acc[tok * kTileRows + b * 32 + lane],
                            g.yq + ((orow0 + tok) * g.yq_ld + un.tile * 4 + b) * 36);
        }
    }
}

template <int FMT>
__global__ void __launch_bounds__(kGemvThreads, 1) k_qgemv(GemvArgs g) {
    using S = GemvSmem<FMT>;
    extern __shared__ __align__(128) uint8_t gsm[];
    uint8_t* stages = gsm;
    int8_t* aq = reinterpret_cast<int8_t*>(gsm + S::kAq);
    float* ad = reinterpret_cast<float*>(gsm + S::kAd);
    int* as = reinterpret_cast<int*>(gsm + S::kAs);
    float* acc = reinterpret_cast<float*>(gsm + S::kAcc);
    uint64_t* bars = reinterpret_cast<uint64_t*>(gsm + S::kBar);
    __shared__ int s_flag;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if (tid == 0) {
        for (int s = 0; s < kGemvStages; ++s) mbar_init(&bars[s], 1);
        fence_barrier_init();
    }
    __syncthreads();
    pdl_wait();

    // this CTA's unit range
    const int64_t n_groups = g.act ? (int64_t)__ldg(g.n_act) : 1;
    const int64_t n_units = n_groups * g.tiles * (g.split ? g.nchunks : 1);
    const int64_t u0 = n_units * blockIdx.x / gridDim.x;
    const int64_t u1 = n_units * (blockIdx.x + 1) / gridDim.x;
    if (u0 >= u1) return;

    GemvCursor prod, cons;
    int issued = 0;
    if (tid == 0) {
        prod.start(g, u0, u1);
        for (int s = 0; s < kGemvStages && prod.valid(); ++s) {
            gemv_issue<FMT>(g, prod, stages + s * S::kStage, &bars[s]);
            prod.advance(g);
            ++issued;
        }
    }
    cons.start(g, u0, u1);

    // lane -> (row, byte offset within a slab)
    int row, woff;
    if (FMT == 8) {
        const int r16 = lane & 15, kg = lane >> 4;
        row = warp * 16 + r16;
        woff = (row >> 3) * 256 + kg * 128 + (row & 7) * 16;
    } else {
        const int half = lane & 1;
        row = warp * 16 + (lane >> 1);
        woff = row * 16 + half * 8;
    }
    const bool owner = (FMT == 8) ? (lane < 16) : ((lane & 1) == 0);
    const int aoff = (FMT == 8) ? (lane >> 4) * 16 : (lane & 1) * 8;

    bool ok = true;
    for (int step = 0; cons.valid(); ++step) {
        const GemvUnit un = cons.un;
        const int tb = cons.tb, c = cons.c;
        const int ntb = min(kTokBlock, un.ntok - tb * kTokBlock);
        const int kbn = min(kChunk, g.nb - c * kChunk);
        const int stg = step % kGemvStages;

        // stage this step's activations: (token, block) -> codes, scale, code sum
        for (int i = tid; i < ntb * kbn; i += kGemvThreads) {
            const int tok = i / kbn, kb = i % kbn;
            const int tokpos = un.tok0 + tb * kTokBlock + tok;
            int64_t xrow;
            if (g.x_mode == X_DENSE) xrow = tokpos;
            else if (g.x_mode == X_PAIR_TOKEN) xrow = __ldg(g.perm + tokpos) / g.kslots;
            else xrow = tokpos;
            const uint32_t* src = reinterpret_cast<const uint32_t*>(
                g.x + (xrow * g.nb + (int64_t)c * kChunk + kb) * 36);
            const uint32_t dsw = __ldg(src);
            uint32_t* dst = reinterpret_cast<uint32_t*>(aq + (tok * kChunk + kb) * 32);
            int sum = 0;
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const uint32_t v = __ldg(src + 1 + j);
                dst[j] = v;
                sum = __dp4a((int)v, 0x01010101, sum);
            }
            ad[tok * kChunk + kb] = h2f((uint16_t)(dsw & 0xffff));
            as[tok * kChunk + kb] = sum;
        }
        if (tid == 0) s_flag = mbar_wait_bounded(&bars[stg], (step / kGemvStages) & 1, g.err, g.budget_ns);
        __syncthreads();
        if (!s_flag) { ok = false; break; }

        const uint8_t* sq = stages + stg * S::kStage;
        const uint16_t* sd = reinterpret_cast<const uint16_t*>(sq + S::kStageQ);
        for (int tp = 0; tp < ntb; tp += kTokPass) {
            float part[kTokPass];
#pragma unroll
            for (int t = 0; t < kTokPass; ++t) part[t] = 0.0f;
            for (int kb = 0; kb < kbn; ++kb) {
                const float dw = h2f(sd[kb * kTileRows + row]);
                if (FMT == 8) {
                    const uint4 w = lds128(sq + kb * kQ80Slab + woff);
#pragma unroll
                    for (int t = 0; t < kTokPass; ++t) {
                        if (tp + t < ntb) {
                            const int ai = (tp + t) * kChunk + kb;
                            const uint4 av = lds128(aq + ai * 32 + aoff);
                            int s = __dp4a((int)w.x, (int)av.x, 0);
                            s = __dp4a((int)w.y, (int)av.y, s);
                            s = __dp4a((int)w.z, (int)av.z, s);
                            s = __dp4a((int)w.w, (int)av.w, s);
                            s += __shfl_xor_sync(kFull, s, 16);
                            part[t] = __fmaf_rn(__int2float_rn(s), __fmul_rn(dw, ad[ai]), part[t]);
                        }
                    }
                } else {
                    const uint2 w = *reinterpret_cast<const uint2*>(sq + kb * kQ40Slab + woff);
                    const int lo0 = (int)(w.x & 0x0F0F0F0Fu), lo1 = (int)(w.y & 0x0F0F0F0Fu);
                    const int hi0 = (int)((w.x >> 4) & 0x0F0F0F0Fu), hi1 = (int)((w.y >> 4) & 0x0F0F0F0Fu);
#pragma unroll
                    for (int t = 0; t < kTokPass; ++t) {
                        if (tp + t < ntb) {
                            const int ai = (tp + t) * kChunk + kb;
                            const uint2 al = *reinterpret_cast<const uint2*>(aq + ai * 32 + aoff);
                            const uint2 ah = *reinterpret_cast<const uint2*>(aq + ai * 32 + 16 + aoff);
                            int s = __dp4a(lo0, (int)al.x, 0);
                            s = __dp4a(lo1, (int)al.y, s);
                            s = __dp4a(hi0, (int)ah.x, s);
                            s = __dp4a(hi1, (int)ah.y, s);
                            s += __shfl_xor_sync(kFull, s, 1);
                            s -= 8 * as[ai];
                            part[t] = __fmaf_rn(__int2float_rn(s), __fmul_rn(dw, ad[ai]), part[t]);
                        }
                    }
                }
            }
            if (owner) {
#pragma unroll
                for (int t = 0; t < kTokPass; ++t) {
                    if (tp + t < ntb) {
                        const int tok = tp + t;
                        if (g.split) {
                            const int64_t tokidx = (int64_t)un.tok0 + tb * kTokBlock + tok;
                            __stcg(g.partial + ((int64_t)c * g.part_tok + tokidx) * ((int64_t)g.tiles * kTileRows) +
                                       (int64_t)un.tile * kTileRows + row,
                                   part[t]);
                        } else {
                            float* ap = acc + tok * kTileRows + row;
                            *ap = (c == un.c0) ? __fadd_rn(0.0f, part[t]) : __fadd_rn(*ap, part[t]);
                        }
                    }
                }
            }
        }
        __syncthreads();   // stage and activations consumed
        if (tid == 0 && prod.valid()) {
            fence_proxy_async();
            gemv_issue<FMT>(g, prod, stages + stg * S::kStage, &bars[stg]);
            prod.advance(g);
            ++issued;
        }

        const bool last_chunk = (c + 1 == un.c1);
        const bool last_tb = ((tb + 1) * kTokBlock >= un.ntok);
        if (!g.split && last_chunk) {
            gemv_epilogue(g, un, tb, ntb, acc);
            __syncthreads();
        }
        if (g.split && last_chunk && last_tb) {
            // ordered completion of the tile: the last unit to arrive finishes it
            if (tid == 0) {
                __threadfence();
                int* cnt = g.counters + (int64_t)un.a * g.tiles + un.tile;
                const int old = atomicAdd(cnt, 1);
                s_flag = (old == g.nchunks - 1);
                if (s_flag) *cnt = 0;
            }
            __syncthreads();
            if (s_flag) {
                __threadfence();
                for (int tb2 = 0; tb2 * kTokBlock < un.ntok; ++tb2) {
                    const int n2 = min(kTokBlock, un.ntok - tb2 * kTokBlock);
                    for (int i = tid; i < n2 * kTileRows; i += kGemvThreads) {
                        const int tok = i / kTileRows, r = i % kTileRows;
                        const int64_t tokidx = (int64_t)un.tok0 + tb2 * kTokBlock + tok;
                        float s = 0.0f;
                        for (int cc = 0; cc < g.nchunks; ++cc)
                            s = __fadd_rn(s, __ldcg(g.partial + ((int64_t)cc * g.part_tok + tokidx) *
                                                                   ((int64_t)g.tiles * kTileRows) +
                                                    (int64_t)un.tile * kTileRows + r));
                        acc[i] = s;
                    }
                    __syncthreads();
                    gemv_epilogue(g, un, tb2, n2, acc);
                    __syncthreads();
                }
            }
        }
        cons.advance(g);
    }
    if (!ok && tid == 0) {
        // drain: wait (bounded) for every copy still in flight before exiting
        for (int s = 0; s < issued && s < kGemvStages; ++s) {
            const int st = issued - 1 - s;
            mbar_wait_bounded(&bars[st % kGemvStages], (st / kGemvStages) & 1, nullptr, g.budget_ns);
        }
    }
    pdl_trigger();
}

// ============================================================================
// a9 -- weighted combine in rank order, then Q8_1.  Grid (T, ceil(L/256)).
// ============================================================================
__global__ void __launch_bounds__(256) k_combine(const float* __restrict__ o, const int32_t* __restrict__ pos,
                                                 const float* __restrict__ w, int k, int L,
                                                 float* __restrict__ ylat, uint8_t* __restrict__ ylq) {
    pdl_wait();
    const int t = blockIdx.x;
    const int n = blockIdx.y * 256 + threadIdx.x;
    if (n >= L) return;   // L % 32 == 0: whole warps leave together
    float acc = 0.0f;
    for (int j = 0; j < k; ++j) {
        const int p = __ldg(pos + t * k + j);
        acc = __fmaf_rn(__ldg(w + t * k + j), __ldcg(o + (int64_t)p * L + n), acc);
    }
    ylat[(int64_t)t * L + n] = acc;
    warp_quant_q8_1(acc, ylq + ((int64_t)t * (L / 32) + n / 32) * 36);
    pdl_trigger();
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
