// elq_decode.cuh -- the whole layer for small token counts (T <= 8 and
// T * k <= 64: decode and short verification batches) as ONE persistent
// kernel, so that the steps of the layer overlap instead of paying a launch,
// a ramp-up and a tail each.
//
// Phases, in this order:
//   D  x -> z (fp32), zq (Q8_1).  Split-K units (128-row tile x chunk of 8
//      blocks x 32-row slice, as in k_wgemv) numbered chunk-major, so that a
//      CTA's share spans few chunks of x; the CTA quantises those chunks of x
//      once, in shared memory.  Chunk partials go to a partial buffer; the
//      warp completing a tile adds them in chunk order (R8) and writes z, zq.
//   R  router logit of (expert e, token t) in the R9 order, once every D tile
//      is out.  The warp finishing token t's last expert runs its top-k and
//      softmax; the warp finishing the last token's top-k buckets the pairs
//      and publishes the routing.
//   G  one unit per (routed expert, hq block): its 32 gate rows and 32 up rows
//      over the whole latent, chunk by chunk (R8 order, in registers), then
//      SwiGLU and the Q8_1 block of h for each of the expert's pairs.
//   N  one unit per (routed expert, 32 latent rows): the down rows over the
//      whole of I, chunk c as soon as the 8 hq blocks it reads are out; then
//      o, and the weighted combine of a token's 32 rows by the warp bringing
//      its last pair (one Q8_1 block of the latent output).
//   U  one unit per 32 output rows: chunk c as soon as the latent blocks it
//      reads are combined for every token; y.
//
// Every CTA (one per SM, cooperative launch, so all are resident) owns a
// contiguous share of every phase; its warps take units from one shared
// counter per phase, in phase order.  A warp keeps a ring of shared-memory
// stages, one chunk ("piece") of a unit each: a piece's weights are copied as
// soon as its unit is taken, its activations as soon as its input is out, and
// the warp blocks only on the piece at the head of its ring.  A warp that
// blocks has finished every unit it took from earlier phases, and every
// dependency points to an earlier phase, so all waits end; each is bounded by
// %globaltimer all the same and ends the warp's work with ELQ_ERR_TIMEOUT in
// the error word.  The last CTA to exit puts the flags and counters back to
// zero.
#pragma once

#include "elq_kernels.cuh"

namespace elq {

enum { PH_D = 0, PH_R = 1, PH_G = 2, PH_N = 3, PH_U = 4, PH_END = 5 };

constexpr int kDecWarps = 8;
constexpr int kDecMaxStages = 4;
constexpr int kDecPend = 8;          // finished D units a warp holds before counting them
constexpr int kDecMaxT = 8;
constexpr int kDecMaxPairs = 64;
constexpr int kDecHeader = 4096;     // bytes of shared memory before the x area and the rings
constexpr uint64_t kDecDrainNs = 2000000000ull;   // wait for own copies in flight on the error path

struct DecArgs {
    WArgs dproj;                     // D: split-K units, partials, tile epilogue into z, zq
    const uint8_t *gu_q, *dn_q, *u_q;        // arena codes of gate/up, down, U
    const uint16_t *gu_d, *dn_d, *u_d;       // their scales
    int64_t gu_qs, gu_ds, dn_qs, dn_ds;      // per-expert strides (bytes, fp16 elements)
    int T, H, L, E, k, I;
    const float* rw;                 // router weights [E][L] fp32
    const float* rb;                 // router bias [E] or NULL
    const float* z;                  // [T][L]
    float* logits;                   // [T][E]
    int32_t* idx;                    // [T][k]
    float* wts;                      // [T][k]
    int32_t *counts, *offsets, *perm, *pos, *act, *n_act;
    int4* grp;                       // [E] (expert, first pair position, pairs) per active group
    const uint8_t* zq;               // [T][L/32] Q8_1
    uint8_t* hq;                     // [T*k][I/32] Q8_1, by pair position
    float* o;                        // [T*k][L], by pair position
    float* ylat;                     // [T][L]
    uint8_t* ylq;                    // [T][L/32] Q8_1
    float* y;                        // [T][H]
    // sync words, zero on entry and on exit:
    //   [0] D tiles done  [1] tokens with top-k done  [2] routing out (n_act + 1)  [3] CTAs exited
    //   [4 .. 4+T)                experts done per token
    //   then [64][I/256 chunks]   hq blocks out per (group, chunk of I)
    //   then [L/256 chunks]       (token, latent block) combines out per chunk of L
    //   then [T][L/32]            pairs in per (token, latent block)
    int* sync;
    int* err;
    uint64_t budget_ns;
    const void* x;                   // [T][H] fp32 or bf16
    int x_bf16;
    int stages, stage_bytes;
    int xq_chunks;                   // chunks of x a CTA's D share may span (its Q8_1 area)
    int header;                      // bytes of shared memory before the x area (with the mirror)
    int withhold_routing;            // test hook: never publish the routing (its waits run out)
};

constexpr int kSyncD = 0, kSyncTopk = 1, kSyncRoute = 2, kSyncExit = 3, kSyncTok = 4;

inline int dec_nch(int n) { return (n / 32 + kChunk - 1) / kChunk; }   // chunks of a reduction length n
inline int dec_sync_ints(int T, int L, int I) {
    return kSyncTok + T + kDecMaxPairs * dec_nch(I) + dec_nch(L) + T * (L / 32);
}
// Words a CTA mirrors in shared memory: D tiles, routing, hq blocks per
// (group, chunk of I), latent combines per chunk of L.
inline int dec_mirror_words(int L, int I) { return 2 + kDecMaxPairs * dec_nch(I) + dec_nch(L); }
inline int dec_header_bytes(int L, int I) { return kDecHeader + (8 * dec_mirror_words(L, I) + 127) / 128 * 128; }

__device__ __forceinline__ int dnch(int n) { return (n / 32 + kChunk - 1) / kChunk; }
__device__ __forceinline__ int* dec_gu_cnt(const DecArgs& A) { return A.sync + kSyncTok + A.T; }
__device__ __forceinline__ int* dec_lat_cnt(const DecArgs& A) { return dec_gu_cnt(A) + kDecMaxPairs * dnch(A.I); }
__device__ __forceinline__ int* dec_comb(const DecArgs& A) { return dec_lat_cnt(A) + dnch(A.L); }

struct DecSlot {                     // one ring entry: a piece of a unit (written by lane 0)
    int ph, u, a, e;
    int tile, s, c, which;           // rows: 128-row tile, 32-row slice; chunk; G: 0 gate, 1 up
    int tok0, ntok, kbn, piece;
    int npieces, st, blk, pad;       // st: 1 weights issued, 2 activations too; blk: output block
};
static_assert(sizeof(DecSlot) == 64, "ring entry size");

// header layout (the mirror follows at kDecHeader: seen values, then poller flags)
constexpr int kDecNextOff = 256, kDecPendOff = 320, kDecLastOff = 640;
constexpr int kDecRingOff = 1024, kDecTokOff = 3072;
static_assert(kDecPendOff + kDecWarps * kDecPend * 4 <= kDecLastOff, "pending");
static_assert(kDecRingOff + kDecWarps * kDecMaxStages * 64 <= kDecTokOff, "ring");
static_assert(kDecTokOff + kDecWarps * kDecMaxStages * kDecMaxT * 4 <= kDecHeader, "header size");
constexpr int kMirD = 0, kMirRoute = 1, kMirGu = 2;
__device__ __forceinline__ int dec_mir_lat(const DecArgs& A) { return kMirGu + kDecMaxPairs * ((A.I / 32 + 7) / 8); }
__device__ __forceinline__ int dec_mir_words(const DecArgs& A) { return dec_mir_lat(A) + (A.L / 32 + 7) / 8; }

__device__ __forceinline__ int ld_acquire_gpu(const int* p) {
    int v;
    asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

// Has sync word p (mirror slot i) reached target?  One lane, non-blocking.
// The CTA keeps the last value it read of the word in shared memory; one
// warp of the CTA at a time reads the word itself (acquire).  The mirror is
// written after that acquire and read before the reader's own loads
// (block-scope fences), which carries the producer's release to every warp.
__device__ __forceinline__ bool dec_seen(int* seen, int* poll, int i, const int* p, int target) {
    if (*reinterpret_cast<volatile int*>(seen + i) >= target) {
        __threadfence_block();
        return true;
    }
    if (atomicCAS(poll + i, 0, 1) != 0) return false;    // another warp of the CTA is reading it
    const int v = ld_acquire_gpu(p);
    __threadfence_block();
    atomicMax(seen + i, v);
    atomicExch(poll + i, 0);
    return v >= target;
}

__device__ __forceinline__ int dec_units(const DecArgs& A, int ph, int n_act) {
    switch (ph) {
    case PH_D: return A.dproj.tiles * 4 * A.dproj.nchunks;
    case PH_R: return A.E * A.T;
    case PH_G: return n_act * (A.I / 32);
    case PH_N: return n_act * (A.L / 32);
    default: return A.H / 32;
    }
}

__device__ __forceinline__ int dec_npieces(const DecArgs& A, int ph) {
    switch (ph) {
    case PH_G: return 2 * dnch(A.L);
    case PH_N: return dnch(A.I);
    case PH_U: return dnch(A.L);
    default: return 1;
    }
}

struct GrpCache {
    int a, e, tok0, ntok;
};

// The unit-level fields of unit u (piece fields follow in dec_piece).
__device__ __forceinline__ DecSlot dec_unit(const DecArgs& A, int ph, int u, GrpCache& gc) {
    DecSlot r;
    r.ph = ph;
    r.u = u;
    r.a = r.e = r.tile = r.s = r.c = r.which = r.tok0 = r.kbn = r.piece = r.blk = r.pad = 0;
    r.ntok = A.T;
    r.npieces = dec_npieces(A, ph);
    r.st = 1;
    if (ph == PH_D) {
        const int per_chunk = A.dproj.tiles * 4;
        r.c = u / per_chunk;
        const int rem = u - r.c * per_chunk;
        r.tile = rem >> 2;
        r.s = rem & 3;
        r.kbn = min(kChunk, A.dproj.nb - r.c * kChunk);
        return r;
    }
    if (ph == PH_R) {
        r.e = u % A.E;
        r.tok0 = u / A.E;
        r.ntok = 1;
        return r;
    }
    if (ph == PH_U) {
        r.blk = u;
        return r;
    }
    const int per_group = (ph == PH_G) ? A.I / 32 : A.L / 32;
    r.a = u / per_group;
    r.blk = u - r.a * per_group;
    if (gc.a != r.a) {
        const int4 v = __ldcg(A.grp + r.a);
        gc.a = r.a;
        gc.e = v.x;
        gc.tok0 = v.y;
        gc.ntok = v.z;
    }
    r.e = gc.e;
    r.tok0 = gc.tok0;
    r.ntok = gc.ntok;
    return r;
}

// Piece p of a streaming unit: its chunk and the rows it covers.
__device__ __forceinline__ void dec_piece(const DecArgs& A, DecSlot& r, int p) {
    r.piece = p;
    if (r.ph == PH_G) {
        // hq block b = 2 * tile + half: gate rows in slice half, up rows in slice 2 + half
        r.which = p & 1;
        r.c = p >> 1;
        r.tile = r.blk >> 1;
        r.s = (r.blk & 1) + 2 * r.which;
        r.kbn = min(kChunk, A.L / 32 - r.c * kChunk);
    } else if (r.ph == PH_N || r.ph == PH_U) {
        r.c = p;
        r.tile = r.blk >> 2;
        r.s = r.blk & 3;
        r.kbn = min(kChunk, (r.ph == PH_N ? A.I : A.L) / 32 - r.c * kChunk);
    }
}

// Is the piece's input complete?  (one lane, non-blocking)
__device__ __forceinline__ bool dec_ready(const DecArgs& A, int* seen, int* poll, const DecSlot& r) {
    switch (r.ph) {
    case PH_R: return dec_seen(seen, poll, kMirD, A.sync + kSyncD, A.dproj.tiles);
    case PH_N: {
        const int w = r.a * dnch(A.I) + r.c;
        return dec_seen(seen, poll, kMirGu + w, dec_gu_cnt(A) + w, r.kbn);
    }
    case PH_U: return dec_seen(seen, poll, dec_mir_lat(A) + r.c, dec_lat_cnt(A) + r.c, A.T * r.kbn);
    default: return true;   // D: x is in shared memory; G: the routing was seen when the unit was taken
    }
}

// Bounded poll of `ready` by lane 0; the result is broadcast to the warp.
template <class F>
__device__ __forceinline__ bool dec_poll(const DecArgs& A, F ready) {
    int ok = 1;
    if ((threadIdx.x & 31) == 0 && !ready()) {
        ok = 0;
        const uint64_t t0 = global_timer_ns();
        for (uint32_t i = 0; i < (1u << 24); ++i) {
            __nanosleep(32);
            if (ready()) {
                ok = 1;
                break;
            }
            if ((i & 63) == 63 && global_timer_ns() - t0 > A.budget_ns) break;
        }
        if (!ok) atomicExch(A.err, kErrTimeout);
    }
    ok = __shfl_sync(kFull, ok, 0);
    __syncwarp();
    return ok != 0;
}

// Weights of one piece (32 rows x kbn blocks) into a stage, with expect_tx
// for them and for `extra` activation bytes that follow.
template <int FMT>
__device__ __forceinline__ void dec_issue_w(const uint8_t* q, const uint16_t* d, int nb, const DecSlot& r,
                                            uint8_t* stg, uint64_t* bar, uint32_t extra) {
    using SL = WSlice<FMT>;
    const int lane = threadIdx.x & 31;
    const uint32_t cb = (uint32_t)(r.kbn * SL::kCodes), sb = (uint32_t)(r.kbn * 64);
    if (lane == 0) {
        mbar_arrive_expect_tx(bar, cb + sb + extra);
        bulk_g2s(stg, q + ((int64_t)r.tile * nb * 4 + (int64_t)r.s * nb + (int64_t)r.c * kChunk) * SL::kCodes, cb,
                 bar);
        bulk_g2s(stg + kChunk * SL::kCodes,
                 d + (int64_t)r.tile * nb * kTileRows + (int64_t)r.s * nb * 32 + (int64_t)r.c * kChunk * 32, sb, bar);
    }
}

// One Q8_1 block from one value per lane, as a call: every site shares one
// copy of the code (the kernel's hot loop must stay in the instruction cache).
__device__ __noinline__ void dec_quant(float v, uint8_t* dst) { warp_quant_q8_1(v, dst); }

// Router unit (expert e, token t): the logit in the R9 order -- lane j sums
// l = j, j + 32, ... with fused multiply-adds, an xor butterfly of adds, then
// the bias.  wrow: the expert's weight row in shared memory.
__device__ __noinline__ void dec_router_unit(const DecArgs& A, int e, int t, const float* wrow) {
    const int lane = threadIdx.x & 31;
    const float* zt = A.z + (int64_t)t * A.L;
    float p = 0.0f;
    for (int l0 = 0; l0 < A.L; l0 += 1024) {
        float zv[32];
#pragma unroll
        for (int q = 0; q < 32; ++q) {
            const int l = l0 + 32 * q + lane;
            zv[q] = (l < A.L) ? __ldcg(zt + l) : 0.0f;
        }
#pragma unroll
        for (int q = 0; q < 32; ++q) {
            const int l = l0 + 32 * q + lane;
            if (l < A.L) p = __fmaf_rn(zv[q], wrow[l], p);
        }
    }
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) p = __fadd_rn(p, __shfl_xor_sync(kFull, p, o));
    if (A.rb) p = __fadd_rn(p, __ldg(A.rb + e));
    if (lane == 0) A.logits[(int64_t)t * A.E + e] = p;
}

// Top-k + softmax of token t (its logits complete); the warp finishing the
// last token then buckets all pairs and publishes the routing as n_act + 1.
// sm: a free stage of this warp (>= 4096 + 256 bytes).
__device__ __noinline__ void dec_topk(const DecArgs& A, int t, uint8_t* sm) {
    const int lane = threadIdx.x & 31;
    float* lg = reinterpret_cast<float*>(sm);
    int32_t* idx_sm = reinterpret_cast<int32_t*>(sm + 4096);
    for (int x = lane; x < A.E; x += 32) lg[x] = __ldcg(A.logits + (int64_t)t * A.E + x);
    __syncwarp();
    warp_topk_softmax(lg, A.E, A.k, A.idx + (int64_t)t * A.k, A.wts + (int64_t)t * A.k,
                      A.T == 1 ? idx_sm : nullptr);
    __syncwarp();
    const int P = A.T * A.k;
    if (A.T > 1) {
        __threadfence();
        __syncwarp();
        int last = 0;
        if (lane == 0) last = (atomicAdd(A.sync + kSyncTopk, 1) == A.T - 1);
        if (!__shfl_sync(kFull, last, 0)) return;
        __threadfence();
        for (int p = lane; p < P; p += 32) idx_sm[p] = __ldcg(A.idx + p);
        __syncwarp();
    }
    bucket_warp_small(idx_sm, P, A.E, A.counts, A.offsets, A.perm, A.pos, A.act, A.n_act, A.grp);
    __threadfence();
    __syncwarp();
    // lane 0 wrote n_act itself
    if (lane == 0 && !A.withhold_routing) atomicExch(A.sync + kSyncRoute, *A.n_act + 1);
}

// L2 prefetch of this CTA's share of the U weights (their addresses do not
// depend on the routing); warp w takes every 8th unit of the share.
template <int FMT>
__device__ __noinline__ void dec_prefetch_u(const DecArgs& A, int warp) {
    using SL = WSlice<FMT>;
    const int lane = threadIdx.x & 31;
    const int n = A.H / 32;
    const int u0 = (int)((int64_t)n * blockIdx.x / gridDim.x);
    const int u1 = (int)((int64_t)n * (blockIdx.x + 1) / gridDim.x);
    const int nb = A.L / 32;
    for (int u = u0 + warp; u < u1; u += kDecWarps) {
        const int tile = u >> 2, s = u & 3;
        if (lane == 0)
            bulk_prefetch_l2(A.u_q + ((int64_t)tile * nb * 4 + (int64_t)s * nb) * SL::kCodes,
                             (uint32_t)(nb * SL::kCodes));
        else if (lane == 1)
            bulk_prefetch_l2(A.u_d + (int64_t)tile * nb * kTileRows + (int64_t)s * nb * 32, (uint32_t)(nb * 64));
    }
    __syncwarp();
}

// First chunk of this CTA's D share and the number of chunks it spans.
__device__ __forceinline__ void dec_x_chunks(const DecArgs& A, int& c0, int& nc) {
    const WArgs& g = A.dproj;
    const int per_chunk = g.tiles * 4;
    const int n = per_chunk * g.nchunks;
    const int u0 = (int)((int64_t)n * blockIdx.x / gridDim.x);
    const int u1 = (int)((int64_t)n * (blockIdx.x + 1) / gridDim.x);
    c0 = u0 / per_chunk;
    nc = (u1 > u0) ? (u1 - 1) / per_chunk - c0 + 1 : 0;
}

// Q8_1 of the chunks of x this CTA's D units read: xq[(j * T + t) * 8 + kb]
// = block 8 (c0 + j) + kb of token t.  Items (chunk, token, block) are dealt
// to the warps eight at a time, their loads issued before any is quantised.
__device__ __noinline__ void dec_quant_x(const DecArgs& A, uint8_t* xq, int warp) {
    const int lane = threadIdx.x & 31;
    const int nbH = A.H / 32;
    int c0, nc;
    dec_x_chunks(A, c0, nc);
    const int per_chunk = A.T * kChunk;
    const int n = nc * per_chunk;
    for (int base = warp * 8; base < n; base += kDecWarps * 8) {
        float v[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int it = base + i;
            const int j = it / per_chunk, r = it - j * per_chunk, t = r / kChunk, kb = r - t * kChunk;
            const int blk = (c0 + j) * kChunk + kb;
            v[i] = 0.0f;
            if (it < n && blk < nbH) {
                const int64_t off = (int64_t)t * A.H + (int64_t)blk * 32 + lane;
                v[i] = A.x_bf16 ? __bfloat162float(static_cast<const __nv_bfloat16*>(A.x)[off])
                                : __ldg(static_cast<const float*>(A.x) + off);
            }
        }
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int it = base + i;
            const int j = it / per_chunk, r = it - j * per_chunk, t = r / kChunk, kb = r - t * kChunk;
            const int blk = (c0 + j) * kChunk + kb;
            if (it < n && blk < nbH) dec_quant(v[i], xq + ((j * A.T + t) * kChunk + kb) * 36);
        }
    }
}


// D tile epilogue: for each token, z rows 128 tile .. +127 = the chunk
// partials added in chunk order (R8), then their four Q8_1 blocks.  The
// partials of 8 chunks x 4 rows are loaded before any is added.
__device__ __noinline__ void dec_d_epilogue(const DecArgs& A, int tile) {
    const WArgs& g = A.dproj;
    const int lane = threadIdx.x & 31;
    const int64_t rows_total = (int64_t)g.tiles * kTileRows;
    const int64_t cstride = g.part_tok * rows_total;
#pragma unroll 1
    for (int t = 0; t < A.T; ++t) {
        const float* pb = g.partial + (int64_t)t * rows_total + (int64_t)tile * kTileRows + lane;
        float v0 = 0.0f, v1 = 0.0f, v2 = 0.0f, v3 = 0.0f;
#pragma unroll 1
        for (int c0 = 0; c0 < g.nchunks; c0 += 8) {
            float pv[8][4];
#pragma unroll
            for (int c = 0; c < 8; ++c)
#pragma unroll
                for (int q = 0; q < 4; ++q)
                    pv[c][q] = (c0 + c < g.nchunks) ? __ldcg(pb + (int64_t)(c0 + c) * cstride + 32 * q) : 0.0f;
#pragma unroll
            for (int c = 0; c < 8; ++c)
                if (c0 + c < g.nchunks) {
                    v0 = __fadd_rn(v0, pv[c][0]);
                    v1 = __fadd_rn(v1, pv[c][1]);
                    v2 = __fadd_rn(v2, pv[c][2]);
                    v3 = __fadd_rn(v3, pv[c][3]);
                }
        }
        float* zr = g.y + (int64_t)t * g.y_ld + (int64_t)tile * kTileRows + lane;
        zr[0] = v0;
        zr[32] = v1;
        zr[64] = v2;
        zr[96] = v3;
        uint8_t* qb = g.yq + ((int64_t)t * g.yq_ld + tile * 4) * 36;
        dec_quant(v0, qb);
        dec_quant(v1, qb + 36);
        dec_quant(v2, qb + 72);
        dec_quant(v3, qb + 108);
    }
}

// D unit: the chunk partial of its 32 rows for every token (x's Q8_1 slices
// in shared memory), stored to the partial buffer.
__device__ __forceinline__ void dec_d_dots(const DecArgs& A, const DecSlot& r, const int (&w)[kChunk][8],
                                           const float (&dw)[kChunk], const uint8_t* xs) {
    const WArgs& g = A.dproj;
    const int lane = threadIdx.x & 31;
    const int64_t rows_total = (int64_t)g.tiles * kTileRows;
#pragma unroll 1
    for (int t = 0; t < A.T; ++t) {
        const uint8_t* ab = xs + t * (kChunk * 36);
        float p = 0.0f;
#pragma unroll
        for (int kb = 0; kb < kChunk; ++kb) {
            if (kb < r.kbn) {
                const uint32_t* aw = reinterpret_cast<const uint32_t*>(ab + kb * 36 + 4);
                int isum = 0;
#pragma unroll
                for (int j = 0; j < 8; ++j) isum = __dp4a(w[kb][j], (int)aw[j], isum);
                const float da = h2f(*reinterpret_cast<const uint16_t*>(ab + kb * 36));
                p = __fmaf_rn(__int2float_rn(isum), __fmul_rn(dw[kb], da), p);
            }
        }
        __stcg(g.partial + ((int64_t)r.c * g.part_tok + t) * rows_total + (int64_t)r.tile * kTileRows + r.s * 32 + lane,
               p);
    }
}

// Chunk dot products of one piece, added to the unit's accumulators: for
// each of the piece's ntok staged Q8_1 activation slices, the chunk partial
// (R8: fused multiply-adds over the chunk's blocks in order) goes into
// acc0[t] or, for the up rows of a G unit, acc1[t] (acc = acc + part, chunk
// after chunk).
__device__ __forceinline__ void dec_accum(const int (&w)[kChunk][8], const float (&dw)[kChunk], const uint8_t* abase,
                                          int kbn, int ntok, int which, float (&acc0)[kDecMaxT],
                                          float (&acc1)[kDecMaxT]) {
#pragma unroll 1
    for (int t = 0; t < ntok; ++t) {
        const uint8_t* ab = abase + t * (kChunk * 36);
        float p = 0.0f;
#pragma unroll
        for (int kb = 0; kb < kChunk; ++kb) {
            if (kb < kbn) {
                const uint32_t* aw = reinterpret_cast<const uint32_t*>(ab + kb * 36 + 4);
                int isum = 0;
#pragma unroll
                for (int j = 0; j < 8; ++j) isum = __dp4a(w[kb][j], (int)aw[j], isum);
                const float da = h2f(*reinterpret_cast<const uint16_t*>(ab + kb * 36));
                p = __fmaf_rn(__int2float_rn(isum), __fmul_rn(dw[kb], da), p);
            }
        }
#pragma unroll
        for (int i = 0; i < kDecMaxT; ++i) {
            if (i == t) {
                if (which) acc1[i] = __fadd_rn(acc1[i], p);
                else acc0[i] = __fadd_rn(acc0[i], p);
            }
        }
    }
}

// a[t] of a register array, for a t known only at run time
__device__ __forceinline__ float dec_sel(const float (&a)[kDecMaxT], int t) {
    float v = a[0];
#pragma unroll
    for (int i = 1; i < kDecMaxT; ++i) v = (t == i) ? a[i] : v;
    return v;
}

__device__ __noinline__ float dec_swiglu(float g, float u) { return __fmul_rn(silu_f32(g), u); }

// End of a G unit: SwiGLU of the gate and up rows, the Q8_1 block of h of
// each pair, then one count for the (group, chunk of I) the block is in.
__device__ __forceinline__ void dec_finish_g(const DecArgs& A, const DecSlot& r, const float (&ag)[kDecMaxT],
                                             const float (&au)[kDecMaxT]) {
    const int lane = threadIdx.x & 31;
    const int nbI = A.I / 32;
#pragma unroll 1
    for (int t = 0; t < r.ntok; ++t) {
        const float h = dec_swiglu(dec_sel(ag, t), dec_sel(au, t));
        dec_quant(h, A.hq + ((int64_t)(r.tok0 + t) * nbI + r.blk) * 36);
    }
    fence_proxy_async_global();
    __threadfence();
    __syncwarp();
    if (lane == 0) atomicAdd(dec_gu_cnt(A) + r.a * dnch(A.I) + r.blk / kChunk, 1);
}

// End of an N unit: o for the group's pairs; the warp bringing a token's
// last pair for this latent block combines the token's k rows in rank order
// (R14) into y_lat and its Q8_1 block, and counts it for the U chunk.
__device__ __noinline__ void dec_combine(const DecArgs& A, const DecSlot& r, int tok, unsigned m);

__device__ __forceinline__ void dec_finish_n(const DecArgs& A, const DecSlot& r, const float (&acc)[kDecMaxT],
                                             const int32_t* toks) {
    const int lane = threadIdx.x & 31;
    const int L = A.L, nbL = A.L / 32;
#pragma unroll 1
    for (int t = 0; t < r.ntok; ++t) A.o[(int64_t)(r.tok0 + t) * L + r.blk * 32 + lane] = dec_sel(acc, t);
    __threadfence();
    __syncwarp();
    int last = 0, tok = 0;
    if (lane < r.ntok) {
        tok = toks[lane];
        int* cnt = dec_comb(A) + (int64_t)tok * nbL + r.blk;
        last = (atomicAdd(cnt, 1) == A.k - 1);
        if (last) *cnt = 0;
    }
    const unsigned m = __ballot_sync(kFull, last);
    if (m) dec_combine(A, r, tok, m);
}

// The weighted combines of the tokens in m (lane j holds token tok of its
// pair j) for the latent block of an N unit: y_lat = sum over the token's k
// pairs in rank order of fmaf(w_j, o_j, acc) (R14), its Q8_1 block, and one
// count for the U chunk that reads it.
__device__ __noinline__ void dec_combine(const DecArgs& A, const DecSlot& r, int tok, unsigned m) {
    const int lane = threadIdx.x & 31;
    const int L = A.L, nbL = A.L / 32;
    __threadfence();
    while (m) {
        const int j = __ffs(m) - 1;
        m &= m - 1;
        const int t = __shfl_sync(kFull, tok, j);
        int pj = 0;
        float wj = 0.0f;
        if (lane < A.k) {
            pj = __ldcg(A.pos + t * A.k + lane);
            wj = __ldcg(A.wts + t * A.k + lane);
        }
        float accv = 0.0f;
#pragma unroll 1
        for (int q0 = 0; q0 < A.k; q0 += 8) {
            float ov[8];
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                const int pq = __shfl_sync(kFull, pj, (q0 + q) & 31);
                ov[q] = (q0 + q < A.k) ? __ldcg(A.o + (int64_t)pq * L + r.blk * 32 + lane) : 0.0f;
            }
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                const float wq = __shfl_sync(kFull, wj, (q0 + q) & 31);
                if (q0 + q < A.k) accv = __fmaf_rn(wq, ov[q], accv);
            }
        }
        A.ylat[(int64_t)t * L + r.blk * 32 + lane] = accv;
        dec_quant(accv, A.ylq + ((int64_t)t * nbL + r.blk) * 36);
        fence_proxy_async_global();
        __threadfence();
        __syncwarp();
        if (lane == 0) atomicAdd(dec_lat_cnt(A) + r.blk / kChunk, 1);
    }
}

// Count this warp's finished D units (one fence, one atomic each); the warp
// completing a tile adds its chunk partials and writes z, zq, then counts the
// tile for the router.
__device__ __noinline__ void dec_flush_d(const DecArgs& A, const int* pend, int npend) {
    const WArgs& g = A.dproj;
    const int lane = threadIdx.x & 31;
    __threadfence();
    __syncwarp();
    int last = 0, tile = 0;
    if (lane < npend) {
        tile = pend[lane];
        int* cnt = g.counters + tile;
        last = (atomicAdd(cnt, 1) == g.nchunks * 4 - 1);
        if (last) *cnt = 0;
    }
    unsigned m = __ballot_sync(kFull, last);
    if (m) __threadfence();
    while (m) {
        const int j = __ffs(m) - 1;
        m &= m - 1;
        const int tl = __shfl_sync(kFull, tile, j);
        dec_d_epilogue(A, tl);
        fence_proxy_async_global();
        __threadfence();
        __syncwarp();
        if (lane == 0) atomicAdd(A.sync + kSyncD, 1);
    }
    __syncwarp();
}

template <int FDU, int FEX>
__global__ void __launch_bounds__(256, 1) k_decode_layer(const __grid_constant__ DecArgs A) {
    extern __shared__ __align__(128) uint8_t dsm[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int S = A.stages;
    uint64_t* mybar = reinterpret_cast<uint64_t*>(dsm) + warp * kDecMaxStages;
    int* s_next = reinterpret_cast<int*>(dsm + kDecNextOff);
    const int nmir = dec_mir_words(A);
    int* seen = reinterpret_cast<int*>(dsm + kDecHeader);
    int* poll = seen + nmir;
    int* pend = reinterpret_cast<int*>(dsm + kDecPendOff) + warp * kDecPend;   // tiles of finished D units
    int* s_last = reinterpret_cast<int*>(dsm + kDecLastOff);
    DecSlot* ring = reinterpret_cast<DecSlot*>(dsm + kDecRingOff) + warp * kDecMaxStages;
    int32_t* stok = reinterpret_cast<int32_t*>(dsm + kDecTokOff) + warp * kDecMaxStages * kDecMaxT;
    uint8_t* xq = dsm + A.header;
    const int xq_bytes = A.xq_chunks * A.T * kChunk * 36;
    uint8_t* mine = dsm + A.header + ((xq_bytes + 127) & ~127) + (size_t)warp * S * A.stage_bytes;
    const int act_off_ex = kChunk * WSlice<FEX>::kCodes + kChunk * 64;
    const int act_off_du = kChunk * WSlice<FDU>::kCodes + kChunk * 64;

    if (threadIdx.x < PH_END) s_next[threadIdx.x] = 0;
    for (int i = threadIdx.x; i < nmir; i += blockDim.x) {
        seen[i] = 0;
        poll[i] = 0;
    }
    if (lane < S) mbar_init(&mybar[lane], 1);
    if (lane == 0) fence_barrier_init();
    __syncthreads();
    pdl_wait();

    int cur = PH_D;                  // phase this warp takes units from
    int n_act = -1;                  // active groups, once the routing is out
    GrpCache gc{-1, 0, 0, 0};
    bool ok = true;
    bool prefetched = false;
    uint32_t parity = 0;             // bit s: phase parity of stage s's barrier
    int head = 0, filled = 0;        // ring slots head .. head + filled - 1 hold pieces
    int npend = 0;                   // finished D units not yet counted
    DecSlot fu;                      // the unit being put into the ring, piece by piece
    fu.npieces = 0;
    fu.piece = 0;
    int ftok = 0;                    // lane i < fu.ntok: token of the unit's pair i
    float acc0[kDecMaxT], acc1[kDecMaxT];
#pragma unroll
    for (int t = 0; t < kDecMaxT; ++t) acc0[t] = acc1[t] = 0.0f;
    int xc0, xnc;                    // chunks of x in the CTA's Q8_1 area
    dec_x_chunks(A, xc0, xnc);

    // Next unit of this CTA in phase order: >= 0; -1 when none is left (or on
    // a timeout, with ok false); -2 when the routing is not out and may_wait
    // is false.
    auto take = [&](bool may_wait, int& ph_out) -> int {
        while (cur < PH_END) {
            if ((cur == PH_G || cur == PH_N) && n_act < 0) {
                int r = 0;
                if (lane == 0) r = dec_seen(seen, poll, kMirRoute, A.sync + kSyncRoute, 1) ? 1 : 0;
                r = __shfl_sync(kFull, r, 0);
                if (!r) {
                    if (!may_wait) return -2;
                    if (!prefetched) {
                        dec_prefetch_u<FDU>(A, warp);
                        prefetched = true;
                    }
                    if (!dec_poll(A, [&]() { return dec_seen(seen, poll, kMirRoute, A.sync + kSyncRoute, 1); })) {
                        ok = false;
                        return -1;
                    }
                }
                __syncwarp();
                n_act = *reinterpret_cast<volatile int*>(seen + kMirRoute) - 1;
            }
            const int n = dec_units(A, cur, n_act);
            const int u0 = (int)((int64_t)n * blockIdx.x / gridDim.x);
            const int u1 = (int)((int64_t)n * (blockIdx.x + 1) / gridDim.x);
            int u = 0;
            if (lane == 0) u = atomicAdd(&s_next[cur], 1);
            u = __shfl_sync(kFull, u, 0) + u0;
            if (u < u1) {
                ph_out = cur;
                return u;
            }
            ++cur;
        }
        return -1;
    };

    // Put the next piece into the ring (taking a new unit when the current
    // one is exhausted) and start its weight copies.  False when no unit is
    // left, or the routing is not out and may_wait is false.
    auto put_next = [&](bool may_wait) -> bool {
        if (fu.piece >= fu.npieces) {
            int ph = 0;
            const int u = take(may_wait, ph);
            if (u < 0) return false;
            fu = dec_unit(A, ph, u, gc);
            fu.piece = 0;
            if (ph == PH_G || ph == PH_N) {
                // the token of each of the group's pairs
                ftok = 0;
                if (A.T > 1 && lane < fu.ntok) ftok = __ldcg(A.perm + fu.tok0 + lane) / A.k;
            }
        }
        const int slot = (head + filled) % S;
        DecSlot r = fu;
        dec_piece(A, r, fu.piece);
        r.st = (r.ph == PH_D) ? 2 : 1;   // D reads x from shared memory; the others wait for their input
        if (lane == 0) ring[slot] = r;
        if (lane < kDecMaxT) stok[slot * kDecMaxT + lane] = ftok;
        __syncwarp();
        uint8_t* stg = mine + slot * A.stage_bytes;
        const uint32_t acts = (uint32_t)(r.ntok * r.kbn * 36);
        switch (r.ph) {
        case PH_D:
            wissue_weights<FDU, X_Q81_TOKEN>(A.dproj, WUnit{0, r.tile, r.c, r.s, 0, 0, A.T, r.kbn}, stg, &mybar[slot], 0);
            break;
        case PH_R:
            if (lane == 0) {
                mbar_arrive_expect_tx(&mybar[slot], (uint32_t)A.L * 4u);
                bulk_g2s(stg, A.rw + (int64_t)r.e * A.L, (uint32_t)A.L * 4u, &mybar[slot]);
            }
            break;
        case PH_G:
            dec_issue_w<FEX>(A.gu_q + r.e * A.gu_qs, A.gu_d + r.e * A.gu_ds, A.L / 32, r, stg, &mybar[slot], acts);
            break;
        case PH_N:
            dec_issue_w<FEX>(A.dn_q + r.e * A.dn_qs, A.dn_d + r.e * A.dn_ds, A.I / 32, r, stg, &mybar[slot], acts);
            break;
        default: dec_issue_w<FDU>(A.u_q, A.u_d, A.L / 32, r, stg, &mybar[slot], acts); break;
        }
        __syncwarp();
        ++fu.piece;
        ++filled;
        return true;
    };

    // Activation copies of a held slot (its input is complete; R reads z
    // from global memory when it runs).
    auto put_acts = [&](int slot) {
        const DecSlot& r = ring[slot];
        if (r.st == 1 && r.ph != PH_R) {
            const int act_off = (r.ph == PH_U) ? act_off_du : act_off_ex;
            uint8_t* dst = mine + slot * A.stage_bytes + act_off;
            // the producers fenced their generic writes for the async proxy
            // before publishing them; the acquire that saw them orders these copies
            if (lane < r.ntok) {
                const uint8_t* src;
                if (r.ph == PH_G)
                    src = A.zq + ((int64_t)stok[slot * kDecMaxT + lane] * (A.L / 32) + r.c * kChunk) * 36;
                else if (r.ph == PH_N)
                    src = A.hq + ((int64_t)(r.tok0 + lane) * (A.I / 32) + r.c * kChunk) * 36;
                else
                    src = A.ylq + ((int64_t)lane * (A.L / 32) + r.c * kChunk) * 36;
                bulk_g2s(dst + lane * (kChunk * 36), src, (uint32_t)r.kbn * 36u, &mybar[slot]);
            }
        }
        __syncwarp();
        if (lane == 0) ring[slot].st = 2;
        __syncwarp();
    };

    auto flush = [&]() {
        if (npend) dec_flush_d(A, pend, npend);
        npend = 0;
    };

    bool first = true;
    while (ok) {
        // fill the ring; a warp holding nothing may wait for the routing
        while (filled < S) {
            if (!first && filled == 0) flush();
            if (!put_next(!first && filled == 0)) break;
        }
        if (first) {
            // prologue: the first weight copies are in flight; the CTA
            // quantises its chunks of x meanwhile
            first = false;
            dec_quant_x(A, xq, warp);
            __syncthreads();
            continue;
        }
        if (!ok || filled == 0) break;
        // activations of the held pieces, in order, while their inputs are complete
        for (int i = 0; i < filled; ++i) {
            const int slot = (head + i) % S;
            if (ring[slot].st == 2) continue;
            int rdy = 0;
            if (lane == 0) rdy = dec_ready(A, seen, poll, ring[slot]) ? 1 : 0;
            if (!__shfl_sync(kFull, rdy, 0)) break;
            __syncwarp();
            put_acts(slot);
        }
        const int slot = head;
        const DecSlot r = ring[slot];
        if (npend && (npend == kDecPend || r.ph != PH_D)) flush();
        if (r.st != 2) {
            // the head's input is not out: wait for it; the next pass issues its activations
            flush();
            if (!dec_poll(A, [&]() { return dec_ready(A, seen, poll, r); })) {
                ok = false;
                break;
            }
            continue;
        }
        if (!mbar_try_wait(&mybar[slot], (parity >> slot) & 1u)) {
            flush();
            if (!mbar_wait_bounded(&mybar[slot], (parity >> slot) & 1u, A.err, A.budget_ns)) {
                ok = false;
                break;
            }
        }
        parity ^= 1u << slot;
        uint8_t* stg = mine + slot * A.stage_bytes;
        if (r.ph == PH_R) {
            dec_router_unit(A, r.e, r.tok0, reinterpret_cast<const float*>(stg));
            __syncwarp();
            __threadfence();
            __syncwarp();
            int last = 0;
            if (lane == 0) last = (atomicAdd(A.sync + kSyncTok + r.tok0, 1) == A.E - 1);
            if (__shfl_sync(kFull, last, 0)) {
                __threadfence();
                dec_topk(A, r.tok0, stg);   // the router row is consumed: the stage is free
            }
        } else {
            int w[kChunk][8];
            float dw[kChunk];
            if (r.ph == PH_D || r.ph == PH_U) wload_regs<FDU>(stg, r.kbn, w, dw);
            else wload_regs<FEX>(stg, r.kbn, w, dw);
            __syncwarp();
            if (r.ph == PH_D) {
                dec_d_dots(A, r, w, dw, xq + (size_t)(r.c - xc0) * A.T * kChunk * 36);
                if (lane == 0) pend[npend] = r.tile;
                ++npend;
            } else {
                if (r.piece == 0) {
#pragma unroll
                    for (int t = 0; t < kDecMaxT; ++t) acc0[t] = acc1[t] = 0.0f;
                }
                dec_accum(w, dw, stg + (r.ph == PH_U ? act_off_du : act_off_ex), r.kbn, r.ntok, r.which, acc0, acc1);
                if (r.piece == r.npieces - 1) {
                    if (r.ph == PH_G) {
                        dec_finish_g(A, r, acc0, acc1);
                    } else if (r.ph == PH_N) {
                        dec_finish_n(A, r, acc0, stok + slot * kDecMaxT);
                    } else {
#pragma unroll 1
                        for (int t = 0; t < r.ntok; ++t) A.y[(int64_t)t * A.H + r.blk * 32 + lane] = dec_sel(acc0, t);
                    }
                }
            }
        }
        // the stage is free for the next piece's copies
        __syncwarp();
        fence_proxy_async();
        head = (head + 1 == S) ? 0 : head + 1;
        --filled;
    }
    if (ok) {
        flush();
    } else {
        // let this warp's copies in flight land: the slots holding only
        // weights get their activation copies too (in-bounds rows whatever
        // their contents), then each held stage's barrier is waited for
        for (int i = 0; i < filled; ++i) {
            const int slot = (head + i) % S;
            if (ring[slot].st == 1) put_acts(slot);
            if (lane == 0) mbar_wait_bounded(&mybar[slot], (parity >> slot) & 1u, nullptr, kDecDrainNs);
            __syncwarp();
        }
    }
    // the last CTA out puts the flags and counters back to zero for the next call
    __syncthreads();
    if (threadIdx.x == 0) {
        __threadfence();
        *s_last = (atomicAdd(A.sync + kSyncExit, 1) == (int)gridDim.x - 1);
    }
    __syncthreads();
    if (*s_last) {
        __threadfence();
        const int n = kSyncTok + A.T + kDecMaxPairs * dnch(A.I) + dnch(A.L) + A.T * (A.L / 32);
        for (int i = threadIdx.x; i < n; i += blockDim.x)
            if (i != kSyncExit) A.sync[i] = 0;
        __threadfence();
        __syncthreads();
        if (threadIdx.x == 0) A.sync[kSyncExit] = 0;
    }
}

}  // namespace elq
