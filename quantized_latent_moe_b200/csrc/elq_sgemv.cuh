// elq_sgemv.cuh -- grouped quantised GEMV for small token counts (T <= 8,
// T * k <= 64) with the split-K reduction inside a thread-block cluster.
//
// Work item: one 32-row slice of a group (the dense matrix, or one routed
// expert) over all of K -- or, for the gate/up projection, the gate slice and
// the up slice whose rows meet in one SwiGLU block.  A cluster of C CTAs
// takes an item; each CTA takes a contiguous run of the item's 8-block chunks,
// one chunk per warp.  A warp bulk-copies its chunk's codes and scales (one
// 8 KB / 4 KB contiguous piece of the arena plus 512 B) and its tokens'
// activation slices into its shared-memory stage, computes the chunk partial
// of each token (dp4a, then the chunk's ordered fused multiply-adds), and
// stores it into the partial buffer of the cluster's first CTA through
// distributed shared memory.  One cluster barrier later that CTA adds the
// chunk partials in chunk order and runs the epilogue.  No partial sum goes
// through global memory and no global counter is taken, except by the down
// projection's weighted combine, whose k pairs come from different items.
//
// Clusters are persistent: cluster i takes items i, i + n, i + 2n, ... and
// each warp keeps up to two items' copies in flight.  Weights that do not
// depend on the upstream kernel are requested before the grid dependency
// wait.  Each CTA also asks L2 to prefetch its share of weights a later
// kernel of the layer reads (the router rows and U during D), so that those
// kernels find them in L2.  (The routed experts' down matrices are not
// prefetched during gate/up: the down projection requests its weights before
// its own grid dependency wait, and the extra traffic only slowed gate/up.)
//
// Routing.  k_route_small (one cluster) computes the router logits, gathers
// them in its first CTA through distributed shared memory, and there takes
// the top-k, the softmax and the bucketing of the T * k <= 64 pairs, writing
// the routing arrays and a table of the routed groups (expert, first pair
// position, pairs, and each pair's token).  The expert kernels read that
// table (or build it from the bucketed arrays of the grouped-experts call)
// into shared memory once per CTA.
#pragma once

#include "elq_kernels.cuh"

namespace elq {

constexpr int kSMaxT = 8;            // tokens of a dense group / pairs of an expert group
constexpr int kSMaxPairs = 64;       // T * k
constexpr int kSMaxWarps = 16;
constexpr int kSMaxCluster = 8;
constexpr int kSHeader = 512;        // mbarriers [warps][2] and the routing scalars

enum { ROUTE_NONE = 0, ROUTE_ARRAYS = 1, ROUTE_GROUPS = 2 };

// ---- cluster primitives --------------------------------------------------------

__device__ __forceinline__ uint32_t cluster_rank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
// The shared-memory address in CTA `rank` of this cluster that corresponds to
// the local shared-memory address `a`.
__device__ __forceinline__ uint32_t dsmem_map(uint32_t a, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(rank));
    return r;
}
__device__ __forceinline__ void dsmem_st(uint32_t a, float v) {
    asm volatile("st.shared::cluster.f32 [%0], %1;" ::"r"(a), "f"(v) : "memory");
}
// Every thread of every CTA of the cluster: arrive (release), then wait (acquire).
__device__ __forceinline__ void cluster_barrier() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// The two halves of a cluster barrier that only has to establish that every
// CTA of the cluster is running (nothing to publish): arrive early, wait just
// before the first distributed shared-memory access.
__device__ __forceinline__ void cluster_arrive_relaxed() {
    asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait() {
    asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

struct SArgs {
    // weights: codes of slice s of tile t, blocks 8c .. 8c+7, of group e at
    // q + e*q_gstride + ((t*nb*4) + s*nb + 8c) * codes-per-block-slice
    const uint8_t* q;
    const uint16_t* d;
    int64_t q_gstride, d_gstride;
    int nb, nchunks;
    int items_per_group;     // slices (or slice pairs, SwiGLU) per group
    int groups_max;          // bound on the groups (dense: 1)
    int C, Cg, cpc, stages;  // cluster size, CTAs per slice, chunks (= warps) per CTA, ring depth
    // one stage of a CTA: codes [cpc][8 blocks], scales [cpc][8 blocks][32],
    // then per token its activations over the CTA's blocks (act_row bytes each)
    int stage_bytes, scales_off, acts_off, act_row, scratch_bytes, pbuf_off, route_off;
    // routing
    int route;
    int T, E, k;
    const int32_t *act, *n_act, *offsets, *perm, *pos;   // ROUTE_ARRAYS
    const int4* grp;                             // ROUTE_GROUPS: per group (expert, first position, pairs, 0)
    const int32_t* gtok;                         // ROUTE_GROUPS: [group][8] token of each pair
    const float* wts;                            // combine weights [T][k]
    // activations
    const void* x;
    int64_t x_row;                               // raw inputs: elements per row
    // outputs
    float* y;
    int64_t y_ld;
    uint8_t* yq;
    int64_t yq_ld;
    int* cnt_comb;                               // [T][L/32], zero on entry and exit
    float* ylat;
    uint8_t* ylq;
    int L;
    // L2 prefetch: up to three fixed ranges
    const uint8_t* pf[3];
    int64_t pf_bytes[3];
    int64_t pf_share[3];                         // bytes per CTA (a multiple of 256)
    // NVFP4: global scales of the weights (one per group's expert, indexed by
    // expert), of the input activations, and of the epilogue's NVFP4 output
    const float* wgs;
    float ags, ogs;
    int* err;
    uint64_t budget_ns;
    int early;               // weights and routing do not depend on the upstream grid
};

// Shared-memory table of the routed groups (expert modes): the count, then
// per group (expert, first pair position, pairs, 0) and the token of each of
// its pairs (a group holds at most one pair per token, so at most kSMaxT).
constexpr int kSRouteBytes = 16 + kSMaxPairs * 16 + kSMaxPairs * kSMaxT * 4;

__device__ __forceinline__ int* sr_nact(uint8_t* rs) { return reinterpret_cast<int*>(rs); }
__device__ __forceinline__ int4* sr_grp(uint8_t* rs) { return reinterpret_cast<int4*>(rs + 16); }
__device__ __forceinline__ int32_t* sr_tok(uint8_t* rs) { return reinterpret_cast<int32_t*>(rs + 16 + kSMaxPairs * 16); }

// Prefetch into L2 the part [lo, hi) of a byte range (lo, hi multiples of 16).
__device__ __forceinline__ void l2_prefetch_range(const uint8_t* base, int64_t lo, int64_t hi) {
    for (int64_t p = lo; p < hi; p += 65536) {
        const int64_t rem = hi - p;
        const uint32_t n = (uint32_t)(rem < 65536 ? rem : 65536);
        bulk_prefetch_l2(base + p, n);
    }
}

// This CTA's share of n bytes when every CTA of the grid takes `share`
// consecutive bytes (share: a multiple of 256, fixed by the host).
__device__ __forceinline__ void share_of(int64_t n, int64_t share, int64_t& lo, int64_t& hi) {
    lo = (int64_t)blockIdx.x * share;
    hi = lo + share < n ? lo + share : n;
}

// Fills the group table from global memory (all threads; ends with a
// CTA barrier).  ROUTE_GROUPS: the router's table; ROUTE_ARRAYS: built from
// the bucketed arrays (act, offsets, perm).
__device__ void s_load_groups(const SArgs& g, uint8_t* rs) {
    if (g.route == ROUTE_GROUPS) {
        const int na = __ldcg(g.n_act);
        for (int i = threadIdx.x; i < na; i += blockDim.x) sr_grp(rs)[i] = __ldcg(g.grp + i);
        for (int i = threadIdx.x; i < na * kSMaxT; i += blockDim.x) sr_tok(rs)[i] = __ldcg(g.gtok + i);
        if (threadIdx.x == 0) *sr_nact(rs) = na;
    } else {
        const int na = __ldcg(g.n_act);
        for (int a = threadIdx.x; a < na; a += blockDim.x) {
            const int e = __ldcg(g.act + a);
            const int o0 = __ldcg(g.offsets + e);
            const int n = __ldcg(g.offsets + e + 1) - o0;
            sr_grp(rs)[a] = make_int4(e, o0, n, 0);
            for (int i = 0; i < n && i < kSMaxT; ++i) sr_tok(rs)[a * kSMaxT + i] = __ldcg(g.perm + o0 + i) / g.k;
        }
        if (threadIdx.x == 0) *sr_nact(rs) = na;
    }
    __syncthreads();
}

// Group a: (expert, first pair position, pairs); dense: (0, 0, T).
__device__ __forceinline__ int4 sgroup(const SArgs& g, const uint8_t* rs, int a) {
    if (g.route == ROUTE_NONE) return make_int4(0, 0, g.T, 0);
    return reinterpret_cast<const int4*>(rs + 16)[a];
}

__device__ __forceinline__ int s_n_groups(const SArgs& g, const uint8_t* rs) {
    return g.route == ROUTE_NONE ? 1 : *reinterpret_cast<const int*>(rs);
}

// Token of pair i of group a.
__device__ __forceinline__ int s_tok(const uint8_t* rs, int a, int i) {
    return reinterpret_cast<const int32_t*>(rs + 16 + kSMaxPairs * 16)[a * kSMaxT + i];
}

// The unit of this warp in item `item`: slice, chunk and group.
struct SUnit {
    int a, tile, s, hb, c, kbn;
    int4 grp;                // expert, first position, pairs
    bool has;                // this warp has a chunk of the item
};

template <int OM>
__device__ __forceinline__ SUnit s_unit(const SArgs& g, const uint8_t* rs, int item, int rank, int warp) {
    SUnit u;
    u.a = item / g.items_per_group;
    const int ip = item - u.a * g.items_per_group;
    if (OM == OUT_SWIGLU) {
        u.tile = ip >> 1;
        u.hb = ip & 1;
        u.s = (rank / g.Cg) * 2 + u.hb;
    } else {
        u.tile = ip >> 2;
        u.s = ip & 3;
        u.hb = 0;
    }
    u.c = (rank % g.Cg) * g.cpc + warp;
    u.has = warp < g.cpc && u.c < g.nchunks;
    u.kbn = u.has ? min(kChunk, g.nb - u.c * kChunk) : 0;
    u.grp = sgroup(g, rs, u.a);
    return u;
}

// Bytes of one activation block (32 values) in the input's form: raw fp32 or
// bf16, or quantised (NVFP4 for NVFP4 weights, else Q8_1).
template <int FMT, int XM>
__device__ __forceinline__ uint32_t s_act_block() {
    return XM == X_RAW_F32 ? 128u : XM == X_RAW_BF16 ? 64u : FMT == kNV ? 18u : 36u;
}

// The CTA's blocks of an item: [kb0, kb0 + nblk) of slice (tile, s), the
// chunks (rank % Cg) * cpc .. +cpc-1 (clipped to the matrix).
struct SRange {
    int kb0, nblk;
};
__device__ __forceinline__ SRange s_range(const SArgs& g, int rank) {
    SRange r;
    r.kb0 = (rank % g.Cg) * g.cpc * kChunk;
    r.nblk = max(0, min(g.nb, r.kb0 + g.cpc * kChunk) - r.kb0);
    return r;
}

// One stage of a CTA in three kinds of bulk copies: the codes of all its
// chunks (contiguous in the arena), their scales, and per token its
// activations over the same blocks.  Thread 0 arms the stage's barrier with
// every byte and issues the weights; lanes 0 .. ntok-1 of warp 0 the
// activations (s_issue_acts).
template <int FMT, int XM>
__device__ __forceinline__ void s_issue_weights(const SArgs& g, const SUnit& u, const SRange& r, uint8_t* stg,
                                                uint64_t* bar) {
    using SL = WSlice<FMT>;
    constexpr int SU = scale_units(FMT);
    const uint32_t cb = (uint32_t)(r.nblk * SL::kCodes), sb = (uint32_t)(r.nblk * 64 * SU);
    mbar_arrive_expect_tx(bar, cb + sb + (uint32_t)u.grp.z * (uint32_t)r.nblk * s_act_block<FMT, XM>());
    bulk_g2s(stg, g.q + u.grp.x * g.q_gstride + ((int64_t)u.tile * g.nb * 4 + (int64_t)u.s * g.nb + r.kb0) * SL::kCodes,
             cb, bar);
    bulk_g2s(stg + g.scales_off,
             g.d + u.grp.x * g.d_gstride + u.tile * d_tile_elems(FMT, g.nb) +
                 ((int64_t)u.s * g.nb * 32 + (int64_t)r.kb0 * 32) * SU,
             sb, bar);
}

template <int FMT, int XM>
__device__ __forceinline__ void s_issue_acts(const SArgs& g, const uint8_t* rs, const SUnit& u, const SRange& r,
                                             uint8_t* stg, uint64_t* bar) {
    const int lane = threadIdx.x & 31;
    if (lane < u.grp.z) {
        int64_t row;
        if (XM == X_Q81_PAIR_TOKEN) row = s_tok(rs, u.a, lane);
        else if (XM == X_Q81_POSITION) row = u.grp.y + lane;
        else row = lane;
        const uint8_t* src;
        if (XM == X_RAW_F32)
            src = static_cast<const uint8_t*>(g.x) + (row * g.x_row + (int64_t)r.kb0 * 32) * 4;
        else if (XM == X_RAW_BF16)
            src = static_cast<const uint8_t*>(g.x) + (row * g.x_row + (int64_t)r.kb0 * 32) * 2;
        else
            src = static_cast<const uint8_t*>(g.x) + (row * g.nb + r.kb0) * (int64_t)s_act_block<FMT, XM>();
        bulk_g2s(stg + g.acts_off + lane * g.act_row, src, (uint32_t)r.nblk * s_act_block<FMT, XM>(), bar);
    }
}

// Q8_1 of one token's chunk of raw activations (kbn blocks of 32 values at
// src, fp32 or bf16) into kbn 36-byte blocks at dst, all blocks at once:
// lane l takes values 8 (l % 4) .. +7 of block l / 4.  Same arithmetic as
// the one-block warp quantiser: amax, d = amax / 127, q = clamp(round(x /
// d)), s = fp16(d * sum q).  The loops stay rolled: a short body keeps the
// code a warp runs once small (these kernels are bound by its fetch).
template <bool BF16>
__device__ __forceinline__ float raw_at(const uint8_t* src, int i) {
    return BF16 ? __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(src)[i])
                : reinterpret_cast<const float*>(src)[i];
}

template <bool BF16>
__device__ __noinline__ void warp_quant_chunk(const uint8_t* src, int kbn, uint8_t* dst) {
    const int lane = threadIdx.x & 31;
    const int b = lane >> 2, qd = lane & 3;
    const bool on = b < kbn;
    const int i0 = b * 32 + qd * 8;
    float amax = 0.0f;
#pragma unroll 1
    for (int i = 0; i < 8; ++i) amax = fmaxf(amax, on ? fabsf(raw_at<BF16>(src, i0 + i)) : 0.0f);
    amax = fmaxf(amax, __shfl_xor_sync(kFull, amax, 1));
    amax = fmaxf(amax, __shfl_xor_sync(kFull, amax, 2));
    const float d = __fdiv_rn(amax, 127.0f);
    uint32_t w0 = 0, w1 = 0;
    int sum = 0;
#pragma unroll 1
    for (int i = 0; i < 8; ++i) {
        int q = 0;
        if (on && d != 0.0f) q = (int)fminf(fmaxf(roundf(__fdiv_rn(raw_at<BF16>(src, i0 + i), d)), -127.0f), 127.0f);
        sum += q;
        const uint32_t bq = (uint32_t)(q & 0xff) << (8 * (i & 3));
        if (i < 4) w0 |= bq; else w1 |= bq;
    }
    sum += __shfl_xor_sync(kFull, sum, 1);
    sum += __shfl_xor_sync(kFull, sum, 2);
    if (on) {
        uint32_t* o = reinterpret_cast<uint32_t*>(dst + b * 36 + 4 + qd * 8);
        o[0] = w0;
        o[1] = w1;
        if (qd == 0) {
            const uint32_t dh = f2h(d);
            const uint32_t sh = f2h(__fmul_rn(d, (float)sum));
            *reinterpret_cast<uint32_t*>(dst + b * 36) = dh | (sh << 16);
        }
    }
}

// Block kb of this lane's row: signed 8-bit codes in w[0..7] (codes 4j ..
// 4j+3 in w[j]) from the chunk's codes, and its scale.
template <int FMT>
__device__ __forceinline__ void s_block(const uint8_t* codes, const uint16_t* scales, int kb, int (&w)[8], float& dw) {
    const int lane = threadIdx.x & 31;
    dw = h2f(scales[kb * 32 + lane]);
    if (FMT == 8) {
        const uint8_t* cp = codes + kb * 1024 + (lane >> 3) * 256 + (lane & 7) * 16;
        const uint4 a = lds128(cp), b = lds128(cp + 128);
        w[0] = (int)a.x; w[1] = (int)a.y; w[2] = (int)a.z; w[3] = (int)a.w;
        w[4] = (int)b.x; w[5] = (int)b.y; w[6] = (int)b.z; w[7] = (int)b.w;
    } else {
        const uint4 a = lds128(codes + kb * 512 + lane * 16);
        const uint32_t v[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            // nibbles q (0..15) -> signed bytes q - 8, without borrows between bytes
            const uint32_t lo = v[j] & 0x0F0F0F0Fu, hi = (v[j] >> 4) & 0x0F0F0F0Fu;
            w[j] = (int)(((lo | 0x80808080u) - 0x08080808u) ^ 0x80808080u);
            w[4 + j] = (int)(((hi | 0x80808080u) - 0x08080808u) ^ 0x80808080u);
        }
    }
}

// Chunk partials of the unit's tokens into the first CTA's partial buffer:
// token t's value of this lane's row goes to the shared-memory address
// `dst + (t * 32 + lane) * 4` of that CTA.  For each token the blocks are
// taken in order (part = fmaf(isum, d_w * d_a, part)), the block's codes read
// again from the stage per token.  Raw activations are first quantised to
// Q8_1 in the warp's scratch.
template <int FMT, int XM>
__device__ __forceinline__ void s_dots(const SArgs& g, const SUnit& u, const uint8_t* stg, uint8_t* scratch,
                                       uint32_t dst) {
    using SL = WSlice<FMT>;
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    // this warp's chunk inside the CTA's stage
    const uint8_t* codes = stg + warp * kChunk * SL::kCodes;
    const uint16_t* scales = reinterpret_cast<const uint16_t*>(stg + g.scales_off) + warp * kChunk * 32;
    const uint8_t* abase = stg + g.acts_off + warp * kChunk * s_act_block<FMT, XM>();
    int astride = g.act_row;
    const int nt = u.grp.z;
    if (XM == X_RAW_F32 || XM == X_RAW_BF16) {
#pragma unroll 1
        for (int t = 0; t < nt; ++t)
            warp_quant_chunk<XM == X_RAW_BF16>(abase + t * g.act_row, u.kbn, scratch + t * kChunk * 36);
        __syncwarp();
        abase = scratch;
        astride = kChunk * 36;
    }
#pragma unroll 1
    for (int t = 0; t < nt; ++t) {
        const uint8_t* ab = abase + t * astride;
        int isum[kChunk];
        float sc[kChunk];
        // the blocks' integer sums and scale products are independent: all
        // loads of the chunk are in flight together
#pragma unroll
        for (int kb = 0; kb < kChunk; ++kb) {
            isum[kb] = 0;
            sc[kb] = 0.0f;
            if (kb < u.kbn) {
                int w[8];
                float dw;
                s_block<FMT>(codes, scales, kb, w, dw);
                // a 36-byte Q8_1 block: 4-byte aligned only (d, s, then 8 words of codes)
                const uint32_t* aw = reinterpret_cast<const uint32_t*>(ab + kb * 36);
#pragma unroll
                for (int j = 0; j < 8; ++j) isum[kb] = __dp4a(w[j], (int)aw[1 + j], isum[kb]);
                sc[kb] = __fmul_rn(dw, h2f((uint16_t)(aw[0] & 0xffff)));
            }
        }
        // then the chunk's ordered chain of fused multiply-adds
        float part = 0.0f;
#pragma unroll
        for (int kb = 0; kb < kChunk; ++kb)
            if (kb < u.kbn) part = __fmaf_rn(__int2float_rn(isum[kb]), sc[kb], part);
        dsmem_st(dst + (uint32_t)((t * 32 + lane) * 4), part);
    }
}

// Sum over one 16-value micro-block of (2 w)(2 a): the row's 16 codes in
// w0, w1 (codes 0..7, 8..15) against the 16 doubled activation values as
// signed bytes in a (four per word, in order): the positive codes' doubled
// magnitudes and the negative codes' (byte permutes of the code nibbles)
// each in a dp4a chain, the second chain subtracted.
__device__ __forceinline__ int nv_dot16(uint32_t w0, uint32_t w1, const uint4& a) {
    const uint32_t n0 = w0 ^ 0x88888888u, n1 = w1 ^ 0x88888888u;
    int p = __dp4a((int)e2m1x4_pos(w0), (int)a.x, 0);
    int n = __dp4a((int)e2m1x4_pos(n0), (int)a.x, 0);
    p = __dp4a((int)e2m1x4_pos(w0 >> 16), (int)a.y, p);
    n = __dp4a((int)e2m1x4_pos(n0 >> 16), (int)a.y, n);
    p = __dp4a((int)e2m1x4_pos(w1), (int)a.z, p);
    n = __dp4a((int)e2m1x4_pos(n1), (int)a.z, n);
    p = __dp4a((int)e2m1x4_pos(w1 >> 16), (int)a.w, p);
    n = __dp4a((int)e2m1x4_pos(n1 >> 16), (int)a.w, n);
    return p - n;
}

// Bit 4 of each byte of a word from 4 bits of x (bit b -> bit 8 b + 4).
__device__ __forceinline__ uint32_t spread4_to_bit4(uint32_t x) {
    return ((x & 1u) | ((x & 2u) << 7) | ((x & 4u) << 14) | ((x & 8u) << 21)) << 4;
}

// The Q5_1 / Q4_K / Q5_K form of s_dots (Q8_1 activations): per block, the
// row's codes (4-bit, plus the fifth bits) as unsigned bytes, isum = sum q_w
// q_a and sumq = sum q_a (dp4a), and the block's two fp32 factors: Q5_1 sd =
// d_w d_a, sm = m_w d_a; K-quants sd = (d scale) d_a, sm = -((dmin min) d_a),
// d and dmin from the words of the chunk's (super-block's) first two blocks.
// Then part = fmaf(isum, sd, part), part = fmaf(sumq, sm, part) per block in
// order.
template <int FMT, int XM>
__device__ __forceinline__ void s_dots_ext(const SArgs& g, const SUnit& u, const uint8_t* stg, uint32_t dst) {
    using SL = WSlice<FMT>;
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const uint8_t* codes = stg + warp * kChunk * SL::kCodes;
    const uint32_t* sw = reinterpret_cast<const uint32_t*>(stg + g.scales_off) + warp * kChunk * 32;
    const uint8_t* abase = stg + g.acts_off + warp * kChunk * 36;
    const int nt = u.grp.z;
    float dk = 0.0f, dmk = 0.0f;
    if (FMT != kQ51) {
        dk = h2f((uint16_t)(sw[lane] >> 16));
        if (FMT != kQ3K) dmk = h2f((uint16_t)(sw[32 + lane] >> 16));
    }
#pragma unroll 1
    for (int t = 0; t < nt; ++t) {
        const uint8_t* ab = abase + t * g.act_row;
        float part = 0.0f;
        // four blocks' sums and factors at a time, then their ordered fmafs
#pragma unroll
        for (int h = 0; h < kChunk; h += 4) {
            int isum[4], sumq[4];
            float sd[4], sm[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int kb = h + i;
                isum[i] = sumq[i] = 0;
                sd[i] = sm[i] = 0.0f;
                if (kb < u.kbn) {
                    const uint4 c = lds128(codes + kb * SL::kCodes + lane * 16);
                    const uint32_t v[4] = {c.x, c.y, c.z, c.w};
                    uint32_t qh = 0;
                    if (fmt_has_qh(FMT))
                        qh = *reinterpret_cast<const uint32_t*>(codes + kb * SL::kCodes + 512 + lane * 4);
                    const uint32_t* aw = reinterpret_cast<const uint32_t*>(ab + kb * 36);
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        uint32_t lo = v[j] & 0x0F0F0F0Fu, hi = (v[j] >> 4) & 0x0F0F0F0Fu;
                        if (fmt_has_qh(FMT)) {
                            lo |= spread4_to_bit4((qh >> (4 * j)) & 15u);
                            hi |= spread4_to_bit4((qh >> (16 + 4 * j)) & 15u);
                        }
                        if (FMT == kQ3K) {
                            // q + 8 -> q (signed bytes, no borrow between bytes); the halves' sums
                            lo = ((lo | 0x80808080u) - 0x08080808u) ^ 0x80808080u;
                            hi = ((hi | 0x80808080u) - 0x08080808u) ^ 0x80808080u;
                            isum[i] = __dp4a((int)lo, (int)aw[1 + j], isum[i]);
                            sumq[i] = __dp4a((int)hi, (int)aw[5 + j], sumq[i]);
                            continue;
                        }
                        isum[i] = __dp4a((int)lo, (int)aw[1 + j], isum[i]);
                        isum[i] = __dp4a((int)hi, (int)aw[5 + j], isum[i]);
                        sumq[i] = __dp4a(0x01010101, (int)aw[1 + j], sumq[i]);
                        sumq[i] = __dp4a(0x01010101, (int)aw[5 + j], sumq[i]);
                    }
                    const float da = h2f((uint16_t)(aw[0] & 0xffff));
                    const uint32_t w = sw[kb * 32 + lane];
                    if (FMT == kQ3K) {
                        // Q3_K: (isum, sd) for values 0..15, (sumq, sm) for 16..31 (no min term)
                        sd[i] = __fmul_rn(__fmul_rn(dk, (float)((int)(w & 0xff) - 32)), da);
                        sm[i] = __fmul_rn(__fmul_rn(dk, (float)((int)((w >> 8) & 0xff) - 32)), da);
                    } else if (FMT == kQ51) {
                        sd[i] = __fmul_rn(h2f((uint16_t)(w & 0xffff)), da);
                        sm[i] = __fmul_rn(h2f((uint16_t)(w >> 16)), da);
                    } else {
                        sd[i] = __fmul_rn(__fmul_rn(dk, (float)(w & 0xff)), da);
                        sm[i] = -__fmul_rn(__fmul_rn(dmk, (float)((w >> 8) & 0xff)), da);
                    }
                }
            }
#pragma unroll
            for (int i = 0; i < 4; ++i)
                if (h + i < u.kbn) {
                    part = __fmaf_rn(__int2float_rn(isum[i]), sd[i], part);
                    part = __fmaf_rn(__int2float_rn(sumq[i]), sm[i], part);
                }
        }
        dsmem_st(dst + (uint32_t)((t * 32 + lane) * 4), part);
    }
}

// Scratch of the NVFP4 dot: per (token, block) of the chunk the activations'
// 32 doubled codes as signed bytes, then separately their two scales.
constexpr int kSNvScratch = kSMaxT * kChunk * 32 + kSMaxT * kChunk * 8;

// The NVFP4 form of s_dots.  The warp first expands its tokens' activation
// blocks (18-byte NVFP4) into signed doubled codes and fp32 scales in its
// scratch; then, token by token, each lane takes its row's 16 micro-block
// sums (nv_dot16) and scale products s_w * s_a, and part = fmaf(isum, sc,
// part) in micro-block order.  The global scales are applied in the epilogue.
template <int XM>
__device__ __forceinline__ void s_dots_nv(const SArgs& g, const SUnit& u, const uint8_t* stg, uint8_t* scratch,
                                          uint32_t dst) {
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const uint8_t* codes = stg + warp * kChunk * 512;
    const uint16_t* scales = reinterpret_cast<const uint16_t*>(stg + g.scales_off) + warp * kChunk * 32;
    const uint8_t* abase = stg + g.acts_off + warp * kChunk * 18;
    const int nt = u.grp.z, kbn = u.kbn;
    uint32_t* ap = reinterpret_cast<uint32_t*>(scratch);                          // [t][kb][8]
    float2* as = reinterpret_cast<float2*>(scratch + kSMaxT * kChunk * 32);       // [t][kb]
#pragma unroll 1
    for (int i = lane; i < nt * kChunk * 9; i += 32) {
        const int t = i / (kChunk * 9), r = i - t * (kChunk * 9);
        const int kb = r / 9, j = r - kb * 9;
        if (kb < kbn) {
            const uint8_t* blk = abase + t * g.act_row + kb * 18;
            const uint32_t v = *reinterpret_cast<const uint16_t*>(blk + (j < 8 ? 2 + 2 * j : 0));
            if (j < 8) ap[(t * kChunk + kb) * 8 + j] = e2m1x4_signed(v);
            else as[t * kChunk + kb] = e4m3x2_to_f32(v);
        }
    }
    __syncwarp();
#pragma unroll 1
    for (int t = 0; t < nt; ++t) {
        float part = 0.0f;
        // four blocks at a time: their 8 micro-block sums and scale products
        // are independent (their loads in flight together), then the ordered
        // chain of fused multiply-adds over them
#pragma unroll
        for (int h = 0; h < kChunk; h += 4) {
            int isum[8];
            float sc[8];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int kb = h + j;
                isum[2 * j] = isum[2 * j + 1] = 0;
                sc[2 * j] = sc[2 * j + 1] = 0.0f;
                if (kb < kbn) {
                    const uint4 q = lds128(codes + kb * 512 + lane * 16);
                    const float2 sw = e4m3x2_to_f32(scales[kb * 32 + lane]);
                    const uint32_t* at = ap + (t * kChunk + kb) * 8;
                    const uint4 a0 = lds128(at), a1 = lds128(at + 4);
                    const float2 sa = as[t * kChunk + kb];
                    isum[2 * j] = nv_dot16(q.x, q.y, a0);
                    isum[2 * j + 1] = nv_dot16(q.z, q.w, a1);
                    sc[2 * j] = __fmul_rn(sw.x, sa.x);
                    sc[2 * j + 1] = __fmul_rn(sw.y, sa.y);
                }
            }
#pragma unroll
            for (int i = 0; i < 8; ++i)
                if (h + i / 2 < kbn) part = __fmaf_rn(__int2float_rn(isum[i]), sc[i], part);
        }
        dsmem_st(dst + (uint32_t)((t * 32 + lane) * 4), part);
    }
}

// One out-of-line copy each of the epilogues' quantiser and SwiGLU.
__device__ __noinline__ void s_quant(float v, uint8_t* dst) { warp_quant_q8_1(v, dst); }
__device__ __noinline__ void s_quant_nv(float v, float g, uint8_t* dst) { warp_quant_nvfp4(v, g, dst); }
__device__ __noinline__ float s_swiglu(float g, float u) { return __fmul_rn(silu_f32(g), u); }

// The item's epilogue in the cluster's first CTA: per token (warps take
// tokens in turn) the chunk partials in chunk order, then (NVFP4 weights) the
// product of the global scales, then the output mode.
// pb: this item's partial buffer [units][T][32].
template <int FMT, int OM>
__device__ void s_epilogue(const SArgs& g, const uint8_t* rs, const SUnit& u, const float* pb) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nw = blockDim.x >> 5;
    const int T = g.T;
    const int nt = u.grp.z;
    const int row = u.tile * kTileRows + u.s * 32 + lane;      // row of the group's matrix
    // NVFP4: y = acc * ((g_w * g_a) * 0.25), the codes being doubled
    const float gq = FMT == kNV ? __fmul_rn(__fmul_rn(__ldg(g.wgs + u.grp.x), g.ags), 0.25f) : 1.0f;
    for (int t = warp; t < nt; t += nw) {
        float acc = 0.0f;
#pragma unroll 1
        for (int c = 0; c < g.nchunks; ++c) acc = __fadd_rn(acc, pb[(c * T + t) * 32 + lane]);
        if (FMT == kNV) acc = __fmul_rn(acc, gq);
        const int64_t pp = (int64_t)u.grp.y + t;                // token (dense) or pair position
        if (OM == OUT_SWIGLU) {
            // the up slice's partials follow the gate slice's
            float up = 0.0f;
#pragma unroll 1
            for (int c = 0; c < g.nchunks; ++c) up = __fadd_rn(up, pb[((g.nchunks + c) * T + t) * 32 + lane]);
            if (FMT == kNV) {
                up = __fmul_rn(up, gq);
                s_quant_nv(s_swiglu(acc, up), g.ogs, g.yq + (pp * g.yq_ld + u.tile * 2 + u.hb) * 18);
            } else {
                s_quant(s_swiglu(acc, up), g.yq + (pp * g.yq_ld + u.tile * 2 + u.hb) * 36);
            }
            continue;
        }
        float* yr = g.y + pp * g.y_ld + row;
        if (OM == OUT_F32_ADD) {
            *yr = __fadd_rn(*yr, acc);
            continue;
        }
        *yr = acc;
        if (OM == OUT_F32_Q81) {
            s_quant(acc, g.yq + (pp * g.yq_ld + u.tile * 4 + u.s) * 36);
        } else if (OM == OUT_F32_NV) {
            s_quant_nv(acc, g.ogs, g.yq + (pp * g.yq_ld + u.tile * 4 + u.s) * 18);
        } else if (OM == OUT_F32_COMBINE) {
            // this pair's 32 rows of o are out: count them for the token; the
            // last of the token's k pairs combines this 32-row block
            __threadfence();
            __syncwarp();
            const int tok = s_tok(rs, u.a, t);
            const int blk = u.tile * 4 + u.s;
            int last = 0;
            if (lane == 0) {
                int* cnt = g.cnt_comb + (int64_t)tok * (g.L / 32) + blk;
                last = (atomicAdd(cnt, 1) == g.k - 1);
                if (last) *cnt = 0;
            }
            last = __shfl_sync(kFull, last, 0);
            if (last) {
                __threadfence();
                float a2 = 0.0f;
                for (int j0 = 0; j0 < g.k; j0 += 8) {
                    float ov[8], wv[8];
#pragma unroll
                    for (int j = 0; j < 8; ++j)
                        if (j0 + j < g.k) {
                            const int pj = tok * g.k + j0 + j;
                            wv[j] = __ldcg(g.wts + pj);
                            const int pos = __ldcg(g.pos + pj);
                            ov[j] = __ldcg(g.y + (int64_t)pos * g.y_ld + row);
                        }
#pragma unroll
                    for (int j = 0; j < 8; ++j)
                        if (j0 + j < g.k) a2 = __fmaf_rn(wv[j], ov[j], a2);
                }
                g.ylat[(int64_t)tok * g.L + row] = a2;
                s_quant(a2, g.ylq + ((int64_t)tok * (g.L / 32) + blk) * 36);
            }
        }
    }
}

// Prefetch into L2 this CTA's weights in every item of its cluster from `m0`
// on (the items the ring has not requested yet), so that HBM streams them
// while the ring works through the earlier ones.  Thread 0.
template <int FMT, int OM>
__device__ __forceinline__ void s_prefetch_own(const SArgs& g, const uint8_t* rs, int n_items, int cid, int ncl,
                                               int m0, int rank) {
    using SL = WSlice<FMT>;
    const SRange r = s_range(g, rank);
    if (r.nblk <= 0) return;
    for (int item = cid + m0 * ncl; item < n_items; item += ncl) {
        const SUnit u = s_unit<OM>(g, rs, item, rank, 0);
        bulk_prefetch_l2(g.q + u.grp.x * g.q_gstride +
                             ((int64_t)u.tile * g.nb * 4 + (int64_t)u.s * g.nb + r.kb0) * SL::kCodes,
                         (uint32_t)(r.nblk * SL::kCodes));
        bulk_prefetch_l2(g.d + u.grp.x * g.d_gstride + u.tile * d_tile_elems(FMT, g.nb) +
                             ((int64_t)u.s * g.nb * 32 + (int64_t)r.kb0 * 32) * scale_units(FMT),
                         (uint32_t)(r.nblk * 64 * scale_units(FMT)));
    }
}

// ============================================================================
// a3 + a5 for T <= 8, T * k <= 64: the router as one cluster of C CTAs.
// CTA r holds experts r * epc .. +epc-1, one per warp, each lane keeping its
// L/32 lane-strided router weights in registers; a logit is that lane's fmaf
// chain over z, the xor butterfly of adds, plus the bias (the router's
// order).  The logits go to global memory and, through distributed shared
// memory, to the first CTA, which then ranks them (top-k, lower id first on
// ties, NaN as -inf), takes the softmax over the k in rank order, buckets the
// pairs, and writes the routing arrays and the group table.
// ============================================================================
struct RSArgs {
    const float* z;          // [T][L]
    const float* w;          // [E][L]
    const float* bias;       // [E] or NULL
    int T, L, E, k, C, epc;
    float* logits;           // [T][E]
    int32_t* idx;            // [T][k]
    float* wts;              // [T][k]
    int32_t *counts, *offsets, *perm, *pos, *act, *n_act;
    int4* grp;               // [groups]
    int32_t* gtok;           // [groups][8]
};

__host__ __device__ constexpr int rs_smem_bytes(int T, int L, int E) {
    // z rows, logits [T][E], top-k ids and values, bucket scratch
    return T * L * 4 + T * E * 4 + 64 * 4 * 2 + (2 * E + 1) * 4 + 64 * 4 * 2 + 64 * 16 + 16;
}

__global__ void __launch_bounds__(kSMaxWarps * 32, 1) k_route_small(RSArgs a) {
    extern __shared__ __align__(16) float rsm_small[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int T = a.T, L = a.L, E = a.E, k = a.k, P = T * k;
    const int rank = a.C > 1 ? (int)cluster_rank() : 0;
    float* zs = rsm_small;                          // [T][L]
    float* lg = zs + T * L;                         // [T][E] (first CTA)
    int32_t* sidx = reinterpret_cast<int32_t*>(lg + T * E);   // [64]
    float* sval = reinterpret_cast<float*>(sidx + 64);        // [64]
    int32_t* scount = reinterpret_cast<int32_t*>(sval + 64);  // [E], then offsets [E+1]
    int32_t* soff = scount + E;
    int32_t* sperm = soff + E + 1;                  // [64]
    int32_t* spos = sperm + 64;                     // [64]
    int4* sgrp = reinterpret_cast<int4*>(((uintptr_t)(spos + 64) + 15) & ~(uintptr_t)15);   // [64]
    int* snact = reinterpret_cast<int*>(sgrp + 64);
    const int e = rank * a.epc + warp;
    const bool has_e = warp < a.epc && e < E;
    const int nj = L >> 5;
    // the router rows do not depend on the upstream kernel
    float wr[kRouterJ];
    {
        const float* wrow = a.w + (int64_t)(has_e ? e : 0) * L + lane;
#pragma unroll
        for (int j = 0; j < kRouterJ; ++j) wr[j] = (has_e && j < nj) ? __ldg(wrow + 32 * j) : 0.0f;
    }
    const float bias = (has_e && a.bias) ? __ldg(a.bias + e) : 0.0f;
    // every CTA of the cluster is running before any distributed store: the
    // arrival goes out now, the wait comes after z is staged
    if (a.C > 1) cluster_arrive_relaxed();
    pdl_wait();
    pdl_trigger();
    for (int i = threadIdx.x; i < T * L / 4; i += blockDim.x)
        reinterpret_cast<float4*>(zs)[i] = __ldcg(reinterpret_cast<const float4*>(a.z) + i);
    __syncthreads();
    if (a.C > 1) cluster_wait();
    if (has_e) {
        const uint32_t lg_lead = a.C > 1 ? dsmem_map(smem_addr(lg), 0) : smem_addr(lg);
        for (int t = 0; t < T; ++t) {
            const float* zr = zs + t * L + lane;
            float p = 0.0f;
#pragma unroll
            for (int j = 0; j < kRouterJ; ++j)
                if (j < nj) p = __fmaf_rn(zr[32 * j], wr[j], p);
#pragma unroll
            for (int o = 16; o >= 1; o >>= 1) p = __fadd_rn(p, __shfl_xor_sync(kFull, p, o));
            if (a.bias) p = __fadd_rn(p, bias);
            if (lane == 0) {
                a.logits[(int64_t)t * E + e] = p;
                dsmem_st(lg_lead + (uint32_t)((t * E + e) * 4), p);
            }
        }
    }
    if (a.C > 1) cluster_barrier(); else __syncthreads();
    if (rank != 0) return;
    // ---- the first CTA: top-k by rank, softmax, bucketing ----
    for (int i = threadIdx.x; i < T * E; i += blockDim.x) {
        const float v0 = lg[i];
        lg[i] = (v0 != v0) ? -INFINITY : v0;          // a NaN logit ranks as -inf
    }
    __syncthreads();
    // rank of candidate (t, e): four lanes each count over a quarter of the
    // row, two shuffles add the quarters
    const int nq = (T * E + 7) / 8 * 8;             // candidates, padded so every lane quartet is whole
    for (int base = 0; base < nq * 4; base += (int)blockDim.x) {
        const int id = base + (int)threadIdx.x;
        const int c = id >> 2, qd = id & 3;
        int r = 0;
        float v = 0.0f;
        int ee = 0, t = 0;
        const bool live = c < T * E;
        if (live) {
            t = c / E;
            ee = c - t * E;
            const float* row = lg + t * E;
            v = row[ee];
            const int j0 = qd * ((E + 3) >> 2), j1 = min(E, j0 + ((E + 3) >> 2));
            for (int j = j0; j < j1; ++j) r += (row[j] > v) | ((row[j] == v) & (j < ee));
        }
        r += __shfl_xor_sync(kFull, r, 1);
        r += __shfl_xor_sync(kFull, r, 2);
        if (live && qd == 0 && r < k) {
            sidx[t * k + r] = ee;
            sval[t * k + r] = v;
        }
    }
    __syncthreads();
    for (int t = warp; t < T; t += (int)(blockDim.x >> 5)) {
        const float sel = lane < k ? sval[t * k + lane] : 0.0f;
        const float l0 = __shfl_sync(kFull, sel, 0);
        const float ex = lane < k ? exp_f32(__fsub_rn(sel, l0)) : 0.0f;
        float sum = 0.0f;
        for (int j = 0; j < k; ++j) sum = __fadd_rn(sum, __shfl_sync(kFull, ex, j));
        if (lane < k) {
            a.idx[t * k + lane] = sidx[t * k + lane];
            a.wts[t * k + lane] = __fdiv_rn(ex, sum);
        }
    }
    if (warp == 0) bucket_warp_small(sidx, P, E, scount, soff, sperm, spos, nullptr, snact, sgrp);
    __syncthreads();
    // the routing out to global memory: group table first (the expert
    // kernels wait for it), then the arrays of the bucketing
    const int na = *snact;
    for (int i = threadIdx.x; i < na * kSMaxT; i += blockDim.x) {
        const int ga = i / kSMaxT, j = i - ga * kSMaxT;
        const int4 gq = sgrp[ga];
        if (j == 0) {
            a.grp[ga] = gq;
            a.act[ga] = gq.x;
        }
        if (j < gq.z) a.gtok[i] = sperm[gq.y + j] / k;
    }
    if (threadIdx.x == 0) *a.n_act = na;
    for (int i = threadIdx.x; i <= E; i += blockDim.x) {
        if (i < P) {
            a.perm[i] = sperm[i];
            a.pos[i] = spos[i];
        }
        if (i < E) a.counts[i] = scount[i];
        a.offsets[i] = soff[i];
    }
    for (int i = threadIdx.x + E + 1; i < P; i += blockDim.x) {
        a.perm[i] = sperm[i];
        a.pos[i] = spos[i];
    }
}

template <int FMT, int XM, int OM>
__global__ void __launch_bounds__(kSMaxWarps * 32, 2) k_sgemv(SArgs g) {
    extern __shared__ __align__(128) uint8_t ssm[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int S = g.stages;
    const int rank = g.C > 1 ? (int)cluster_rank() : 0;
    const int cid = (int)blockIdx.x / g.C;
    const int ncl = (int)gridDim.x / g.C;
    uint64_t* bars = reinterpret_cast<uint64_t*>(ssm);            // [S] stage barriers
    volatile int* bad = reinterpret_cast<volatile int*>(ssm + 64);
    uint8_t* rs = ssm + g.route_off;
    uint8_t* stages = ssm + kSHeader;
    uint8_t* scratch = ssm + kSHeader + (size_t)S * g.stage_bytes + (size_t)warp * g.scratch_bytes;
    float* pbuf = reinterpret_cast<float*>(ssm + g.pbuf_off);
    const int units = (OM == OUT_SWIGLU ? 2 : 1) * g.nchunks;
    const uint32_t pb_local = smem_addr(pbuf);
    const uint32_t pb_lead = g.C > 1 ? dsmem_map(pb_local, 0) : pb_local;
    // this warp's unit index in the partial buffer
    const int uidx = (OM == OUT_SWIGLU ? (rank / g.Cg) * g.nchunks : 0) + (rank % g.Cg) * g.cpc + warp;
    const SRange rng = s_range(g, rank);
    const bool cta_has = rng.nblk > 0;

    if (threadIdx.x < S) mbar_init(&bars[threadIdx.x], 1);
    if (threadIdx.x == 0) {
        *bad = 0;
        fence_barrier_init();
    }
    __syncthreads();
    // every CTA of the cluster is running (its shared memory may be written
    // by the others) before the first distributed shared-memory store: the
    // arrival goes out now, the wait comes before the first item's dots
    if (g.C > 1) cluster_arrive_relaxed();
    bool cl_pending = g.C > 1;

    int n_items = 0;
    int issued = -1;                 // thread 0: the last item whose copies went out
    auto issue_w = [&](int m) {      // thread 0
        const int item = cid + m * ncl;
        if (item >= n_items || !cta_has) return;
        const SUnit u = s_unit<OM>(g, rs, item, rank, 0);
        s_issue_weights<FMT, XM>(g, u, rng, stages + (m % S) * g.stage_bytes, &bars[m % S]);
        issued = m;
    };
    auto issue_a = [&](int m) {      // warp 0
        const int item = cid + m * ncl;
        if (item >= n_items || !cta_has) return;
        const SUnit u = s_unit<OM>(g, rs, item, rank, 0);
        s_issue_acts<FMT, XM>(g, rs, u, rng, stages + (m % S) * g.stage_bytes, &bars[m % S]);
    };
    // L2 prefetch of the fixed ranges a later kernel reads (by the last warp)
    auto prefetch_fixed = [&]() {
        if (warp == (int)(blockDim.x >> 5) - 1 && lane < 3 && g.pf[lane]) {
            int64_t lo, hi;
            share_of(g.pf_bytes[lane], g.pf_share[lane], lo, hi);
            l2_prefetch_range(g.pf[lane], lo, hi);
        }
    };
    if (g.early) {
        // weights (and, for the down projection, the routing, complete
        // before the upstream gate/up started) do not depend on the upstream grid
        if (g.route != ROUTE_NONE) s_load_groups(g, rs);
        n_items = s_n_groups(g, rs) * g.items_per_group;
        if (threadIdx.x == 0)
            for (int m = 0; m < S; ++m) issue_w(m);
        pdl_wait();
        pdl_trigger();
        __syncwarp();
        if (warp == 0)
            for (int m = 0; m < S; ++m) issue_a(m);
        if (threadIdx.x == 0) s_prefetch_own<FMT, OM>(g, rs, n_items, cid, ncl, S, rank);
        prefetch_fixed();
    } else {
        pdl_wait();
        pdl_trigger();
        if (g.route != ROUTE_NONE) s_load_groups(g, rs);
        n_items = s_n_groups(g, rs) * g.items_per_group;
        if (warp == 0) {
            for (int m = 0; m < S; ++m) {
                if (lane == 0) issue_w(m);
                __syncwarp();
                issue_a(m);
            }
            if (lane == 0) s_prefetch_own<FMT, OM>(g, rs, n_items, cid, ncl, S, rank);
        }
        prefetch_fixed();
    }

    for (int m = 0;; ++m) {
        const int item = cid + m * ncl;
        if (item >= n_items) break;
        const int st = m % S;
        const SUnit u = s_unit<OM>(g, rs, item, rank, warp);
        const uint8_t* stg = stages + st * g.stage_bytes;
        if (cl_pending) {
            cluster_wait();
            cl_pending = false;
        }
        if (u.has && !*bad) {
            const bool got = mbar_wait_bounded(&bars[st], (uint32_t)((m / S) & 1), g.err, g.budget_ns);
            if (!__all_sync(kFull, got)) {
                if (lane == 0) *bad = 1;
            } else {
                const uint32_t dst = pb_lead + (uint32_t)(((m & 1) * units + uidx) * g.T * 128);
                if constexpr (FMT == kNV) s_dots_nv<XM>(g, u, stg, scratch, dst);
                else if constexpr (fmt_ext(FMT)) s_dots_ext<FMT, XM>(g, u, stg, dst);
                else s_dots<FMT, XM>(g, u, stg, scratch, dst);
            }
        }
        // every chunk partial of the item is in the first CTA, and every warp
        // of this CTA is done with the stage
        if (g.C > 1) cluster_barrier(); else __syncthreads();
        // refill the stage with this CTA's item m + S
        if (warp == 0 && !*bad) {
            if (lane == 0) {
                fence_proxy_async();
                issue_w(m + S);
            }
            __syncwarp();
            issue_a(m + S);
        }
        if (rank == 0) s_epilogue<FMT, OM>(g, rs, u, pbuf + (size_t)(m & 1) * units * g.T * 32);
    }
    if (cl_pending) cluster_wait();   // no item: the arrival is still matched
    if (*bad && threadIdx.x == 0) {
        // drain: wait (bounded) for the last copies of every stage
        for (int m = (issued - S + 1 > 0 ? issued - S + 1 : 0); m <= issued; ++m)
            mbar_wait_bounded(&bars[m % S], (uint32_t)((m / S) & 1), nullptr, g.budget_ns);
    }
}

}  // namespace elq
