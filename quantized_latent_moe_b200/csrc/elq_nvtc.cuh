// elq_nvtc.cuh -- NVFP4 expert projections for many tokens on the tensor
// cores: tcgen05.mma kind::mxf4nvf4 with block scales (E2M1 operands, one
// E4M3 scale per 16 values of each operand), fp32 accumulators in TMEM.
//
// The block-scaled MMA applies both operands' micro-block scales inside the
// tensor core and accumulates the whole K range in fp32, so the epilogue only
// multiplies by the two global scales: there is no per-block rescale.  The
// order of that fp32 accumulation is the hardware's, not the micro-block
// chain of the GEMV path, so these results agree with the GEMV's to rounding,
// not bit for bit.
//
// One MMA: M = 128 weight rows, N = up to 128 slots, K = 64 values (two
// 32-value blocks).  An MMA of this shape costs the same issue time whatever
// N, so token tiles are as wide as one scale atom (128 slots).  Shared-memory operands, K-major without swizzle:
//  A (weights): [block][slice][32 rows x 16 bytes], one tensor-map copy per
//    stage from the arena; for the MMA of blocks 2j, 2j+1: LBO = 2048 bytes
//    (the next 16-byte K chunk), SBO = 128 bytes (the next 8 rows).
//  B (activations): pre-packed per K step as [slot/8][2][8][16] bytes
//    (LBO = 128, SBO = 256), the Q8_1 B buffers' geometry.
// Scale factors go shared memory -> TMEM with tcgen05.cp (32 lanes x 128
// bits, repeated in all four lane quarters) from 512-byte atoms: row m's four
// scales of a K step as one 32-bit word at byte (m % 32) * 16 + (m / 32) * 4.
// The weights' atoms are stored in the arena; the activations' atoms are
// written by the packing kernel and the SwiGLU epilogue, per 128 slots.
//
// CTA: warp 0 issues the copies, warp 1 the scale copies and the MMAs, warps
// 2..17 drain the accumulators (4 TMEM lane quarters x 4 column quarters).
#pragma once

#include "elq_tc.cuh"

namespace elq {

// Instruction descriptor of kind::mxf4nvf4: E2M1 x E2M1 -> fp32, both
// K-major, UE4M3 scales, dense K = 64.
__host__ __device__ constexpr uint32_t umma_idesc_nvf4(int M, int N) {
    return (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

// D[tmem] (+)= (A x SFA) . (B x SFB)^T, scale factors in TMEM at sfa, sfb.
__device__ __forceinline__ void umma_nvf4(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                          uint32_t sfa, uint32_t sfb, uint32_t acc) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.scale_vec::4X [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(
            d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(acc), "r"(sfa), "r"(sfb)
        : "memory");
}

// Shared memory (a 512-byte atom: 32 rows of 16 bytes) -> TMEM columns
// taddr .. taddr+3 of all 128 lanes (each lane quarter gets the same rows).
__device__ __forceinline__ void tmem_cp_atom(uint32_t taddr, const void* atom) {
    const uint64_t desc = umma_desc(atom, 128, 128);
    asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(desc) : "memory");
}

// Untiled bulk copy global -> shared on an mbarrier (16-byte aligned, size a
// multiple of 16).  No multicast.
__device__ __forceinline__ void bulk_g2s_nv(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
    bulk_g2s(dst, src, bytes, bar);
}

constexpr int kNvKS = 4;                       // K steps (64 values each) per stage
constexpr int kNvN = 128;                      // slots per token tile (one whole scale atom)
constexpr int kNvStages = 4;
constexpr int kNvStageA = kNvKS * 4096;
constexpr int kNvStageB = kNvKS * kNvN * 32;
constexpr int kNvStageSfa = kNvKS * 512;
constexpr int kNvStageSfb = kNvKS * 512;
constexpr int kNvStage = kNvStageA + kNvStageB + kNvStageSfa + kNvStageSfb;
constexpr int kNvXld = 129;                    // SwiGLU exchange: [slot][128 rows], padded
constexpr int kNvXchg = kNvN * kNvXld * 4;
constexpr int kNvSmem = 1024 + kNvStages * kNvStage + kNvXchg + kUnitsBytes;
constexpr int kNvAccBufs = 2;                  // accumulators of kNvN columns
constexpr int kNvSfCol = kNvAccBufs * kNvN;    // scale-factor columns: kNvKS x (SFA 4, SFB 4)
constexpr int kNvTmemCols = 512;
constexpr int kNvEpiCols = 32;                 // accumulator columns per epilogue warp
static_assert(kNvSfCol + kNvKS * 8 <= kNvTmemCols, "TMEM plan");
static_assert(kTcEpiWarps / 4 * kNvEpiCols == kNvN, "the epilogue warps cover the 128 x 128 tile");
static_assert(kNvSmem <= 227 * 1024, "shared memory plan");

enum { NV_OUT_F32 = 0, NV_OUT_SWIGLU = 1 };

struct NvArgs {
    static constexpr int kN = kNvN;   // slots per token tile
    // tm_a: weight codes, uint32 [tiles][nb][4 slices][128] with strides
    //       (nb*2048, 512, nb*512) bytes; box [1][2 kNvKS][4][128] -> [block][slice][512 B]
    // tm_b: packed activation codes, uint32 [K steps][slots/8][64]; box [kNvKS][8][64]
    CUtensorMap tm_a, tm_b;
    const uint8_t* d;           // weight scales of the arena (the atoms follow each tile's per-row scales)
    int64_t d_tile_bytes;       // bytes of a tile's scales
    int nb, nks, rtiles;        // blocks, K steps, row tiles per group
    // groups: the routed experts (slot_off, offsets per expert, tt_off per active expert)
    const int32_t* act;
    const int32_t* n_act;
    const int32_t* slot_off;
    const int32_t* offsets;
    const int32_t* tt_off;
    int T;
    const uint8_t* sfb;         // activation atoms: [slot/128][nks][512]
    // global scales: weights (per expert) x the activations' static scale
    const float* wgs;
    float ags;
    // outputs
    float* y;                   // NV_OUT_F32: fp32 rows by slot
    int64_t y_ld;
    uint8_t* hq;                // NV_OUT_SWIGLU: the down projection's B codes
    uint8_t* hsf;               //   and its activation atoms
    int64_t sstride;            // slots of the B buffers (multiple of 128)
    int h_nks;                  // K steps of h (I / 64)
    float ogs;                  // the static scale of h
    int* err;
    uint64_t budget_ns;
};

__device__ __forceinline__ int nv_units(const NvArgs& g) { return __ldcg(g.tt_off + __ldcg(g.n_act)) * g.rtiles; }

// Unit u: row tile rt of the routed expert whose token tiles hold u / rtiles
// (the same order as the int8 path: a weight tile against all its expert's
// token tiles in turn).
__device__ __forceinline__ TcUnit tc_unit(const NvArgs& g, int u) {
    TcUnit r;
    const int q = u / g.rtiles;
    const int na = __ldcg(g.n_act);
    int lo = 0, hi = na;
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (__ldcg(g.tt_off + mid) <= q) lo = mid; else hi = mid;
    }
    r.e = __ldcg(g.act + lo);
    const int base = __ldcg(g.tt_off + lo);
    const int n_q = __ldcg(g.tt_off + lo + 1) - base;
    const int v = u - base * g.rtiles;
    r.rt = v / n_q;
    const int tt = v - r.rt * n_q;
    r.slot0 = __ldcg(g.slot_off + r.e) + tt * kNvN;
    const int cnt = __ldcg(g.offsets + r.e + 1) - __ldcg(g.offsets + r.e);
    r.nvalid = min(kNvN, cnt - tt * kNvN);
    r.ncols = (r.nvalid + 15) & ~15;
    r.valid = r.nvalid > 0;
    return r;
}

// ---- packing: NVFP4 rows (18-byte blocks) -> B codes and scale atoms ---------
// Pair p (row p / k) goes to slot pair_slot[p]: per K step its two blocks' 32
// code bytes to [K step][slot/8][2][8][16], their four scales as one word of
// the slot's atom.  One thread per (pair, K step); padding slots are left as
// they are (the GEMM's columns past a tile's pairs are unused).
struct NvPackArgs {
    const uint8_t* x;           // NVFP4 rows, nb blocks each
    int nb, nks;
    const int32_t* slot_off;    // the slots of expert e: slot_off[e] .. slot_off[e+1]-1; from slot_off[E] on unused
    const int32_t* offsets;     // its pairs: perm[offsets[e]] ..., row = pair / kslots; then zero slots
    const int32_t* perm;
    int E, kslots;
    uint8_t* bq;
    uint8_t* bsf;
    int64_t sstride;
};

// One thread per (K-step of 64, slot), slots fastest: the two 18-byte blocks
// of the slot's row (zeros for padding) into its codes and scale atom.
__global__ void __launch_bounds__(256) k_pack_nv(NvPackArgs a) {
    __shared__ int s_off[1025];
    pdl_wait();
    load_slot_off(s_off, a.slot_off, a.E);
    const int64_t id = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (id >= a.sstride * a.nks) return;
    const int ks = (int)(id / a.sstride);
    const int64_t slot = id - (int64_t)ks * a.sstride;
    if (slot >= s_off[a.E]) return;
    const int64_t row = slot_row_of(s_off, a.E, slot, a.offsets, a.perm, a.kslots);
    uint32_t c[8] = {0, 0, 0, 0, 0, 0, 0, 0}, sw = 0;
    if (row >= 0) {
        // two 18-byte blocks (2-byte aligned): scales, then 16 code bytes each
        const uint16_t* src = reinterpret_cast<const uint16_t*>(a.x + (row * a.nb + 2 * ks) * 18);
#pragma unroll
        for (int b = 0; b < 2; ++b) {
            const uint16_t* sb = src + 9 * b;
            sw |= (uint32_t)__ldg(sb) << (16 * b);
#pragma unroll
            for (int j = 0; j < 4; ++j)
                c[4 * b + j] = (uint32_t)__ldg(sb + 1 + 2 * j) | ((uint32_t)__ldg(sb + 2 + 2 * j) << 16);
        }
    }
    uint8_t* dst = a.bq + (int64_t)ks * a.sstride * 32 + (slot >> 3) * 256 + (slot & 7) * 16;
    *reinterpret_cast<uint4*>(dst) = make_uint4(c[0], c[1], c[2], c[3]);
    *reinterpret_cast<uint4*>(dst + 128) = make_uint4(c[4], c[5], c[6], c[7]);
    *reinterpret_cast<uint32_t*>(a.bsf + ((slot >> 7) * a.nks + ks) * 512 + (slot & 31) * 16 + ((slot >> 5) & 3) * 4) =
        sw;
    pdl_trigger();
}

// One micro-block of h (16 values held by one thread): NVFP4 under global
// scale gs (the rule of warp_quant_nvfp4), its 8 code bytes written into the
// down projection's B codes (half of the slot's 16-byte chunk of block kbh)
// and its scale byte into the slot's atom.
__device__ __forceinline__ void nv_quant_h16(const float (&h)[16], float gs, int64_t slot, int kbh, int mb,
                                             uint8_t* hq, uint8_t* hsf, int64_t sstride, int h_nks) {
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(h[i]));
    const uint32_t sb = f32_to_e4m3(__fdiv_rn(__fdiv_rn(amax, 6.0f), gs));
    const float den = __fmul_rn(e4m3x2_to_f32(sb).x, gs);
    uint32_t w[2] = {0u, 0u};
#pragma unroll
    for (int i = 0; i < 16; i += 2) {
        const float x0 = den != 0.0f ? __fdiv_rn(h[i], den) : 0.0f;
        const float x1 = den != 0.0f ? __fdiv_rn(h[i + 1], den) : 0.0f;
        w[i >> 3] |= f32x2_to_e2m1x2(x0, x1) << (4 * (i & 7));
    }
    const int ks = kbh >> 1;
    uint8_t* dst = hq + (int64_t)ks * sstride * 32 + (slot >> 3) * 256 + (kbh & 1) * 128 + (slot & 7) * 16 + mb * 8;
    *reinterpret_cast<uint2*>(dst) = make_uint2(w[0], w[1]);
    hsf[((slot >> 7) * h_nks + ks) * 512 + (slot & 31) * 16 + ((slot >> 5) & 3) * 4 + (kbh & 1) * 2 + mb] =
        (uint8_t)sb;
}

// ---- the GEMM ------------------------------------------------------------------

template <int OM>
__global__ void __launch_bounds__(kTcThreads, 1) k_nvgemm(const __grid_constant__ NvArgs g) {
    extern __shared__ __align__(1024) uint8_t nvsm[];
    uint64_t* full = reinterpret_cast<uint64_t*>(nvsm);            // [stages]: copies landed
    uint64_t* empty = full + kNvStages;                             // [stages]: MMAs done with them
    uint64_t* tfull = empty + kNvStages;                            // [2]: a unit's accumulator complete
    uint64_t* tempty = tfull + kNvAccBufs;                          // [2]: ... and drained
    uint64_t* xfull = tempty + kNvAccBufs;                          // SwiGLU: up rows handed over
    uint64_t* xempty = xfull + 1;                                   // ... and taken
    uint32_t* tmem_base_sm = reinterpret_cast<uint32_t*>(xempty + 1);
    int* abort_sm = reinterpret_cast<int*>(tmem_base_sm + 1);
    uint8_t* stages = nvsm + 1024;
    float* xchg = reinterpret_cast<float*>(nvsm + 1024 + kNvStages * kNvStage);   // [slot][128 rows]
    TcUnit* su = reinterpret_cast<TcUnit*>(nvsm + 1024 + kNvStages * kNvStage + kNvXchg);
    int* stt = reinterpret_cast<int*>(su + kUnitsSmem);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < kNvStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < kNvAccBufs; ++b) {
            mbar_init(&tfull[b], 1);
            mbar_init(&tempty[b], kTcEpiWarps);
        }
        mbar_init(xfull, kTcEpiWarps);
        mbar_init(xempty, kTcEpiWarps);
        *abort_sm = 0;
        fence_barrier_init();
    }
    if (warp == 0) {
        tmem_alloc(tmem_base_sm, kNvTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_base_sm;
    pdl_wait();

    const int n_units = nv_units(g);
    const int u0 = (int)((int64_t)n_units * blockIdx.x / gridDim.x);
    const int u1 = (int)((int64_t)n_units * (blockIdx.x + 1) / gridDim.x);
    const int kstages = g.nks / kNvKS;
    volatile int* abort_v = abort_sm;
    stage_units(g, u0, 1, u1 - u0, su, stt);
    auto unit_at = [&](int u) { return u - u0 < kUnitsSmem ? su[u - u0] : tc_unit(g, u); };

    if (warp == 0) {
        // ---------------- producer ----------------
        if (lane == 0) {
            int it = 0;
            for (int u = u0; u < u1 && !*abort_v; ++u) {
                const TcUnit un = unit_at(u);
                if (!un.valid) continue;
                const int tile = un.e * g.rtiles + un.rt;
                const uint8_t* sfa = g.d + (int64_t)tile * g.d_tile_bytes + (int64_t)g.nb * 256;
                const uint8_t* sfb = g.sfb + (int64_t)(un.slot0 >> 7) * g.nks * 512;
                for (int ks = 0; ks < kstages; ++ks, ++it) {
                    const int s = it % kNvStages;
                    if (it >= kNvStages &&
                        !mbar_wait_bounded(&empty[s], (uint32_t)((it / kNvStages - 1) & 1), g.err, g.budget_ns)) {
                        *abort_v = 1;
                        break;
                    }
                    uint8_t* st = stages + s * kNvStage;
                    mbar_arrive_expect_tx(&full[s], (uint32_t)kNvStage);
                    tma_load_4d(st, &g.tm_a, 0, 0, ks * 2 * kNvKS, tile, &full[s]);
                    tma_load_3d(st + kNvStageA, &g.tm_b, 0, un.slot0 >> 3, ks * kNvKS, &full[s]);
                    bulk_g2s(st + kNvStageA + kNvStageB, sfa + (int64_t)ks * kNvKS * 512, kNvStageSfa, &full[s]);
                    bulk_g2s(st + kNvStageA + kNvStageB + kNvStageSfa, sfb + (int64_t)ks * kNvKS * 512, kNvStageSfb,
                             &full[s]);
                }
            }
        }
    } else if (warp == 1) {
        // ---------------- scale copies and MMAs ----------------
        if (lane == 0) {
            int it = 0, uc = 0;
            const uint32_t sf = tmem + (uint32_t)kNvSfCol;
            for (int u = u0; u < u1 && !*abort_v; ++u) {
                const TcUnit un = unit_at(u);
                if (!un.valid) continue;
                const int ab = uc % kNvAccBufs;
                if (uc >= kNvAccBufs &&
                    !mbar_wait_bounded(&tempty[ab], (uint32_t)((uc / kNvAccBufs - 1) & 1), g.err, g.budget_ns)) {
                    *abort_v = 1;
                    break;
                }
                ++uc;
                tc_fence_after();
                const uint32_t idesc = umma_idesc_nvf4(128, un.ncols);
                const uint32_t dacc = tmem + (uint32_t)(ab * kNvN);
                for (int ks = 0; ks < kstages && !*abort_v; ++ks, ++it) {
                    const int s = it % kNvStages;
                    if (!mbar_wait_bounded(&full[s], (uint32_t)((it / kNvStages) & 1), g.err, g.budget_ns)) {
                        *abort_v = 1;
                        break;
                    }
                    tc_fence_after();
                    const uint8_t* st = stages + s * kNvStage;
                    for (int k = 0; k < kNvKS; ++k) {
                        const uint32_t sfa_t = sf + (uint32_t)(k * 8), sfb_t = sfa_t + 4u;
                        tmem_cp_atom(sfa_t, st + kNvStageA + kNvStageB + k * 512);
                        tmem_cp_atom(sfb_t, st + kNvStageA + kNvStageB + kNvStageSfa + k * 512);
                        const uint64_t adesc = umma_desc(st + k * 4096, 2048, 128);
                        const uint64_t bdesc = umma_desc(st + kNvStageA + k * kNvN * 32, 128, 256);
                        umma_nvf4(dacc, adesc, bdesc, idesc, sfa_t, sfb_t, (ks | k) != 0 ? 1u : 0u);
                    }
                    umma_commit(&empty[s]);
                }
                umma_commit(&tfull[ab]);
            }
            // let the last MMAs finish before the TMEM is freed
            if (uc > 0) {
                const int last = uc - 1;
                mbar_wait_bounded(&tfull[last % kNvAccBufs], (uint32_t)((last / kNvAccBufs) & 1), nullptr,
                                  g.budget_ns);
            }
        }
    } else {
        // ---------------- epilogue ----------------
        // warp: TMEM lane quarter sp (tile rows 32 sp ..), columns (slots) c0 .. c0 + 31
        const int ew = warp - 2;
        const int sp = warp & 3;
        const int c0 = (ew >> 2) * kNvEpiCols;
        const int row = sp * 32 + lane;
        int uc = 0, xc = 0;
        for (int u = u0; u < u1 && !*abort_v; ++u) {
            const TcUnit un = unit_at(u);
            if (!un.valid) continue;
            const int ab = uc % kNvAccBufs;
            if (!warp_wait_bounded(&tfull[ab], (uint32_t)((uc / kNvAccBufs) & 1), g.err, g.budget_ns)) {
                *abort_v = 1;
                break;
            }
            ++uc;
            tc_fence_after();
            float acc[kNvEpiCols];
            const bool active = c0 < un.ncols;
            if (active) {
                uint32_t rc[kNvEpiCols];
                tmem_ld32(tmem + ((uint32_t)(sp * 32) << 16) + (uint32_t)(ab * kNvN + c0), rc);
                tmem_ld_wait();
#pragma unroll
                for (int j = 0; j < kNvEpiCols; ++j) acc[j] = __uint_as_float(rc[j]);
            } else {
#pragma unroll
                for (int j = 0; j < kNvEpiCols; ++j) acc[j] = 0.0f;
            }
            tc_fence_before();
            __syncwarp();
            mbar_arrive_lane0(&tempty[ab], lane);
            const float gq = __fmul_rn(__ldg(g.wgs + un.e), g.ags);
#pragma unroll
            for (int j = 0; j < kNvEpiCols; ++j) acc[j] = __fmul_rn(acc[j], gq);
            const int nv = un.nvalid;
            const int64_t slot0 = un.slot0;
            if (OM == NV_OUT_SWIGLU) {
                // the tile through shared memory ([slot][row], padded), then two threads per
                // (slot, h block), one micro-block of 16 values each: h row 32 hb + i takes gate
                // row 32 hb + i and up row 64 + 32 hb + i of the tile
                if (xc > 0 && !warp_wait_bounded(xempty, (uint32_t)((xc - 1) & 1), g.err, g.budget_ns)) {
                    *abort_v = 1;
                    break;
                }
#pragma unroll
                for (int j = 0; j < kNvEpiCols; ++j) xchg[(c0 + j) * kNvXld + row] = acc[j];
                __syncwarp();
                mbar_arrive_lane0(xfull, lane);
                if (!warp_wait_bounded(xfull, (uint32_t)(xc & 1), g.err, g.budget_ns)) {
                    *abort_v = 1;
                    break;
                }
                {
                    const int task = ew * 32 + lane;          // 0 .. 511
                    const int mb = task & 1, b = task >> 1;
                    const int t = b >> 1, hb = b & 1;
                    if (t < nv) {
                        const float* gr = xchg + t * kNvXld + hb * 32 + mb * 16;
                        const float* ur = gr + 64;
                        float h[16];
#pragma unroll
                        for (int i = 0; i < 16; ++i) h[i] = __fmul_rn(silu_f32(gr[i]), ur[i]);
                        nv_quant_h16(h, g.ogs, slot0 + t, un.rt * 2 + hb, mb, g.hq, g.hsf, g.sstride, g.h_nks);
                    }
                }
                __syncwarp();
                mbar_arrive_lane0(xempty, lane);
                ++xc;
                continue;
            }
#pragma unroll
            for (int j = 0; j < kNvEpiCols; ++j) {
                const int t = c0 + j;
                if (t < nv) g.y[(slot0 + t) * g.y_ld + (int64_t)un.rt * kTileRows + row] = acc[j];
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) tmem_dealloc(tmem, kNvTmemCols);
    pdl_trigger();
}

// ---- measurement: the fp4 block-scaled tensor-core rate ------------------------
//
// One CTA per SM, one thread issuing n_mma tcgen05.mma kind::mxf4nvf4 (M = 128,
// N = n_cols, K = 64, 2 * 128 * n_cols * 64 operations each) from fixed
// shared-memory operands and scale atoms into one accumulator, then a bounded
// wait for them (ELQ_ERR_TIMEOUT's code 1 in *err if it runs out).  The atoms
// go to TMEM once, or (cp_each) before every MMA, as the GEMM's main loop
// does.
constexpr int kRateNvSmem = 1024 + (128 + kRateN) * 32 + 2 * 512;

__global__ void __launch_bounds__(128, 1) k_test_mma_nvf4_rate(int n_mma, int n_cols, int cp_each, int* sink, int* err,
                                                               uint64_t budget_ns) {
    extern __shared__ __align__(1024) uint8_t rnsm_[];
    uint64_t* done = reinterpret_cast<uint64_t*>(rnsm_);
    uint32_t* tbase = reinterpret_cast<uint32_t*>(rnsm_ + 8);
    uint8_t* a = rnsm_ + 1024;                // 128 x 32 bytes (64 E2M1 codes a row)
    uint8_t* b = a + 128 * 32;                // 256 x 32 bytes
    uint8_t* sf = b + kRateN * 32;            // two scale atoms (all 1.0)
    const int warp = threadIdx.x >> 5;
    for (int i = threadIdx.x; i < (128 + kRateN) * 32 / 4; i += blockDim.x)
        reinterpret_cast<uint32_t*>(a)[i] = 0x22222222u;                     // every value 1.0
    for (int i = threadIdx.x; i < 2 * 512 / 4; i += blockDim.x) reinterpret_cast<uint32_t*>(sf)[i] = 0x38383838u;
    if (threadIdx.x == 0) {
        mbar_init(done, 1);
        fence_barrier_init();
    }
    if (warp == 0) {
        tmem_alloc(tbase, 512);
        tmem_relinquish();
    }
    fence_proxy_async();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tbase;
    if (threadIdx.x == 0) {
        const uint32_t sfa = tmem + (uint32_t)kRateN, sfb = sfa + 4u;
        tmem_cp_atom(sfa, sf);
        tmem_cp_atom(sfb, sf + 512);
        const uint32_t idesc = umma_idesc_nvf4(128, n_cols);
        const uint64_t ad = umma_desc(a, 2048, 128), bd = umma_desc(b, 128, 256);
        for (int i = 0; i < n_mma; ++i) {
            if (cp_each) {
                tmem_cp_atom(sfa, sf);
                tmem_cp_atom(sfb, sf + 512);
            }
            umma_nvf4(tmem, ad, bd, idesc, sfa, sfb, i > 0 ? 1u : 0u);
        }
        umma_commit(done);
    }
    __syncwarp();
    const bool ok = warp_wait_bounded(done, 0, err, budget_ns);
    tc_fence_after();
    if (warp == 0) {
        uint32_t r[16];
        tmem_ld16(tmem, r);
        tmem_ld_wait();
        if (ok && threadIdx.x == 0) sink[blockIdx.x] = (int)r[0];
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) tmem_dealloc(tmem, 512);
}

}  // namespace elq
