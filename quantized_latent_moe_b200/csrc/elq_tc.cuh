// elq_tc.cuh -- the prefill path: grouped int8 GEMM on the 5th-generation
// tensor cores (tcgen05.mma kind::i8, accumulators in TMEM).
//
// A Q8_0 x Q8_1 row dot needs, for every 32-wide block, its exact int32 sum
// rescaled by f32(d_w) * f32(d_a) and added in a fixed order (8-block chunks,
// see elq.h).  One MMA with K = 32 is exactly one block, so each block's MMA
// writes a fresh TMEM accumulator (no accumulation inside the tensor core) and
// the epilogue warps drain it and apply the ordered fp32 rescale.
//
// CTA: warp 0 issues the bulk copies, warp 1 issues the MMAs (one elected
// thread each), warps 2..9 drain TMEM (warp w reads TMEM lanes 32*(w%4) ..
// +31, i.e. weight rows; warps 2..5 take tokens 0..31 of the tile, warps 6..9
// tokens 32..63).  Tile = 128 weight rows x up to 64 tokens x all K.
//
// Operands in shared memory use the K-major, no-swizzle canonical layout:
// 8-row x 16-byte core matrices, LBO = 128 B (next core matrix along K), SBO =
// 256 B (next 8 rows).  A weight tile's block kb is assembled from the four
// 1 KB slice pieces of the arena; the activations come pre-packed in the same
// layout ("B buffers": [kb][slot/8][2][8][16] codes and [kb][slot] fp32 scales).
#pragma once

#include <cuda.h>

#include "elq_kernels.cuh"

namespace elq {

// ---- tcgen05 primitives ----------------------------------------------------

__device__ __forceinline__ void tmem_alloc(uint32_t* dst_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_addr(dst_smem)),
                 "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// D[tmem] = A[smem] x B[smem]^T (int8 x int8 -> int32), accumulate if acc != 0.
__device__ __forceinline__ void umma_i8(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                        uint32_t acc) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, {%5, %6, %7, %8}, p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(acc), "r"(0u), "r"(0u), "r"(0u), "r"(0u)
        : "memory");
}
// D (fp32 in TMEM) = A * B (+ D when acc != 0), fp16 operands, K = 16.
__device__ __forceinline__ void umma_f16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                         uint32_t acc) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, {%5, %6, %7, %8}, p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(acc), "r"(0u), "r"(0u), "r"(0u), "r"(0u)
        : "memory");
}
// Arrive (once) on an mbarrier when all MMAs this thread issued so far are done.
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                     smem_addr(bar))
                 : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}
// One arrival for the warp, by lane 0, as a predicated instruction (no branch).
__device__ __forceinline__ void mbar_arrive_lane0(uint64_t* bar, int lane) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.eq.s32 p, %1, 0;\n\t@p mbarrier.arrive.shared::cta.b64 _, [%0];\n\t}" ::"r"(
            smem_addr(bar)),
        "r"(lane)
        : "memory");
}

// Tiled tensor copies global -> shared through a tensor map (a kernel
// parameter), completing on an mbarrier's transaction count.  No multicast.
// The innermost coordinate is always 0 or 16-byte aligned here.
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, int c0, int c1, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], "
        "[%4];" ::"r"(smem_addr(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(smem_addr(bar))
        : "memory");
}
__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* map, int c0, int c1, int c2, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], "
        "[%5];" ::"r"(smem_addr(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(smem_addr(bar))
        : "memory");
}
__device__ __forceinline__ void tma_load_4d(void* dst, const CUtensorMap* map, int c0, int c1, int c2, int c3,
                                            uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4, "
        "%5}], [%6];" ::"r"(smem_addr(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(smem_addr(bar))
        : "memory");
}

// 32 consecutive 32-bit TMEM columns of this thread's lane.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
        "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]),
          "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]),
          "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
}
// 16 consecutive TMEM columns of this thread's lane (32x32b shape).
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
        "%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr)
        : "memory");
}

__device__ __forceinline__ void tmem_ld_wait() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// Pairs of fp32 values in one 64-bit register and the packed two-wide fp32
// operations on them: each half is one IEEE round-to-nearest operation, the
// same result as the scalar instruction, at half the instruction count.
__device__ __forceinline__ uint64_t f2_pack(float lo, float hi) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}
__device__ __forceinline__ void f2_unpack(uint64_t v, float& lo, float& hi) {
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t f2_sub(uint64_t a, uint64_t b) {
    uint64_t r;
    asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}
__device__ __forceinline__ uint64_t f2_mul(uint64_t a, uint64_t b) {
    uint64_t r;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}
__device__ __forceinline__ uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t r;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
    return r;
}
__device__ __forceinline__ uint64_t f2_add(uint64_t a, uint64_t b) {
    uint64_t r;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}

// Two small integers (|q| <= 2048, exact in fp16) as an fp16 pair, q0 in the low half.
__device__ __forceinline__ uint32_t h2_pack_int(int q0, int q1) {
    return (uint32_t)__half_as_ushort(__int2half_rn(q0)) | ((uint32_t)__half_as_ushort(__int2half_rn(q1)) << 16);
}

// Eight signed 8-bit codes (w0 bytes 0..3, then w1) as eight fp16, in order.
__device__ __forceinline__ uint4 h8_from_i8(uint32_t w0, uint32_t w1) {
    auto b = [](uint32_t w, int i) { return (int)(int8_t)(uint8_t)(w >> (8 * i)); };
    return make_uint4(h2_pack_int(b(w0, 0), b(w0, 1)), h2_pack_int(b(w0, 2), b(w0, 3)),
                      h2_pack_int(b(w1, 0), b(w1, 1)), h2_pack_int(b(w1, 2), b(w1, 3)));
}

// Exact int32 -> fp32 for |s| < 2^22 without the (slow) conversion unit: the
// integer s + 0x4B400000 is the bit pattern of the float 1.5 * 2^23 + s, so
// one fp32 subtraction of 1.5 * 2^23 recovers s exactly.  Each block's MMA
// writes a fresh int32 accumulator; the epilogue adds the seed as it reads it.
constexpr uint32_t kAccSeed = 0x4B400000u;
constexpr float kAccSeedF = 12582912.0f;

// Bounded mbarrier wait of a whole warp: every lane polls (no divergent
// branch around the poll loop) and the warp agrees on the outcome, so
// warp-collective instructions after it stay converged.
__device__ __forceinline__ bool warp_wait_bounded(uint64_t* bar, uint32_t parity, int* err, uint64_t budget_ns) {
    return __all_sync(0xffffffffu, mbar_wait_bounded(bar, parity, err, budget_ns) ? 1 : 0) != 0;
}

// Shared-memory matrix descriptor: K-major, no swizzle, version 1.
__device__ __forceinline__ uint64_t umma_desc(const void* p, uint32_t lbo, uint32_t sbo) {
    const uint64_t a = smem_addr(p);
    return ((a >> 4) & 0x3FFFull) | ((uint64_t)((lbo >> 4) & 0x3FFF) << 16) |
           ((uint64_t)((sbo >> 4) & 0x3FFF) << 32) | (1ull << 46);
}

// Instruction descriptor: s8 x s8 -> s32, both K-major, M x N.
__host__ __device__ constexpr uint32_t umma_idesc_i8(int M, int N) {
    return (2u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}
// Instruction descriptor: f16 x f16 -> f32, both K-major, M x N.
__host__ __device__ constexpr uint32_t umma_idesc_f16(int M, int N) {
    return (1u << 4) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

// ---- B buffers: Q8_1 rows -> canonical slots ---------------------------------
//
// Slot s of a B buffer holds one activation row: for block kb its 32 codes at
// bq + kb*bstride*32 + (s/8)*256 + (c/16)*128 + (s%8)*16 + c%16, its scale at
// bd[kb*bstride + s].  Slots without a row hold zeros.

enum { PACK_DENSE = 0, PACK_SLOTS = 1 };

struct PackArgs {
    const uint8_t* x;           // Q8_1 AoS rows, nb blocks each
    int nb;
    int mode;
    int T;                      // PACK_DENSE: rows 0 .. T-1 -> slots 0 .. T-1
    // PACK_SLOTS: the slots of expert e are slot_off[e] .. slot_off[e+1]-1,
    // its pairs (perm[offsets[e]] ..., row = pair / kslots) then zeros; slots
    // from slot_off[E] on are past the routed tiles and stay as they are
    const int32_t* slot_off;
    const int32_t* offsets;
    const int32_t* perm;
    int E, kslots;
    uint8_t* bq;
    float* bd;
    int64_t bstride;            // slots in the buffer (multiple of 16)
    int f16;                    // codes widened to fp16 (the kind::f16 operand layout)
};

// Shared copy of slot_off[0 .. E] for slot_row_of (E <= 1024).
__device__ __forceinline__ void load_slot_off(int* s_off, const int32_t* slot_off, int E) {
    for (int i = threadIdx.x; i <= E; i += blockDim.x) s_off[i] = __ldcg(slot_off + i);
    __syncthreads();
}

// The token row of the pair in slot `slot` (< slot_off[E]), or -1 for a
// padding slot: the expert is the last e with slot_off[e] <= slot.
__device__ __forceinline__ int64_t slot_row_of(const int* s_off, int E, int64_t slot, const int32_t* offsets,
                                               const int32_t* perm, int kslots) {
    int lo = 0, hi = E;
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (s_off[mid] <= slot) lo = mid;
        else hi = mid;
    }
    const int r = (int)(slot - s_off[lo]);
    const int o0 = __ldg(offsets + lo), cnt = __ldg(offsets + lo + 1) - o0;
    return r < cnt ? __ldg(perm + o0 + r) / kslots : -1;
}

// PACK_SLOTS: one thread per (block, slot), slots fastest: a warp writes 32
// consecutive slots of one block (1 KB of codes and 128 B of scales,
// contiguous) and reads its rows' 36-byte blocks through L1.  PACK_DENSE: one
// thread per (slot, block), blocks fastest (a warp reads 32 consecutive blocks
// of a row).
__global__ void __launch_bounds__(256) k_pack_b(PackArgs a) {
    __shared__ int s_off[1025];
    pdl_wait();
    if (a.mode != PACK_DENSE) load_slot_off(s_off, a.slot_off, a.E);
    const int64_t id = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (id >= a.bstride * a.nb) return;
    int kb;
    int64_t slot, row;
    if (a.mode == PACK_DENSE) {
        slot = id / a.nb;
        kb = (int)(id - slot * a.nb);
        row = slot < a.T ? slot : -1;
    } else {
        kb = (int)(id / a.bstride);
        slot = id - (int64_t)kb * a.bstride;
        if (slot >= s_off[a.E]) return;
        row = slot_row_of(s_off, a.E, slot, a.offsets, a.perm, a.kslots);
    }
    uint4 lo4 = make_uint4(0, 0, 0, 0), hi4 = make_uint4(0, 0, 0, 0);
    float dd = 0.0f;
    if (row >= 0) {
        const uint32_t* src = reinterpret_cast<const uint32_t*>(a.x + (row * a.nb + kb) * 36);
        const uint32_t w0 = __ldg(src);
        lo4 = make_uint4(__ldg(src + 1), __ldg(src + 2), __ldg(src + 3), __ldg(src + 4));
        hi4 = make_uint4(__ldg(src + 5), __ldg(src + 6), __ldg(src + 7), __ldg(src + 8));
        dd = h2f((uint16_t)(w0 & 0xffff));
    }
    if (a.f16) {
        // half h (codes 16 h .. 16 h + 15) of the block: two 16-byte core-matrix rows of fp16
        uint8_t* dst = a.bq + (int64_t)kb * a.bstride * 64 + (slot >> 3) * 256 + (slot & 7) * 16;
        uint8_t* dst1 = dst + a.bstride * 32;
        *reinterpret_cast<uint4*>(dst) = h8_from_i8(lo4.x, lo4.y);
        *reinterpret_cast<uint4*>(dst + 128) = h8_from_i8(lo4.z, lo4.w);
        *reinterpret_cast<uint4*>(dst1) = h8_from_i8(hi4.x, hi4.y);
        *reinterpret_cast<uint4*>(dst1 + 128) = h8_from_i8(hi4.z, hi4.w);
    } else {
        uint8_t* dst = a.bq + (int64_t)kb * a.bstride * 32 + (slot >> 3) * 256 + (slot & 7) * 16;
        *reinterpret_cast<uint4*>(dst) = lo4;
        *reinterpret_cast<uint4*>(dst + 128) = hi4;
    }
    a.bd[(int64_t)kb * a.bstride + slot] = dd;
    pdl_trigger();
}

// fp16 copy of a Q8_0 arena's codes for the kind::f16 GEMM.  The int8 arena
// holds a 128-row tile slice-major -- [slice s][block][1 KB], the 1 KB of 32
// rows as [row/8][code/16][row%8][16] -- and the copy block-major: per (tile,
// block) 8 KB, [code/16][row/8][(code%16)/8][row%8][8 fp16] (per K = 16 half
// of the block, the no-swizzle K-major operand of one MMA).  One thread per
// 16-byte piece of the int8 arena.
__global__ void __launch_bounds__(256) k_arena_f16(const uint8_t* __restrict__ q, int64_t n_pieces, int nb,
                                                   uint8_t* __restrict__ q16) {
    const int64_t p = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (p >= n_pieces) return;
    const int64_t per_tile = (int64_t)nb * 256;     // pieces of a tile: 4 slices x nb blocks x 64
    const int64_t tile = p / per_tile;
    const int rem = (int)(p - tile * per_tile);
    const int sl = rem / (nb * 64), rem2 = rem - sl * nb * 64;
    const int kb = rem2 >> 6, pi = rem2 & 63;
    const int r8 = 4 * sl + (pi >> 4), hh = (pi >> 3) & 1, r = pi & 7;
    const uint4 w = __ldg(reinterpret_cast<const uint4*>(q) + p);
    uint8_t* dst = q16 + (tile * nb + kb) * 8192 + hh * 4096 + r8 * 256 + r * 16;
    *reinterpret_cast<uint4*>(dst) = h8_from_i8(w.x, w.y);
    *reinterpret_cast<uint4*>(dst + 128) = h8_from_i8(w.z, w.w);
}

constexpr int kTcN = 64;            // tokens per tile

// ---- routing -> padded slots -------------------------------------------------
// slot_off[e] = sum over e' < e of roundup(count(e'), align) (align 16, or 128
// for the NVFP4 path, whose token tiles start on whole scale atoms); tt_off[a]
// = sum over active experts a' < a of ceil(count / tile) (64, or 128 for
// NVFP4); pair_slot[p] = the slot of pair p.
// One CTA.
__global__ void __launch_bounds__(1024) k_tc_route(const int32_t* offsets, const int32_t* act, const int32_t* n_act,
                                                   const int32_t* idx, const int32_t* pos, int P, int E,
                                                   int32_t* slot_off, int32_t* tt_off, int32_t* pair_slot,
                                                   int align, int tile) {
    pdl_wait();
    __shared__ int s_slot[1025];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (warp == 0) {
        const int per = (E + 31) / 32;
        const int e0 = min(E, lane * per), e1 = min(E, e0 + per);
        int local = 0;
        for (int e = e0; e < e1; ++e) local += (__ldcg(offsets + e + 1) - __ldcg(offsets + e) + align - 1) & -align;
        int incl = local;
        for (int o = 1; o < 32; o <<= 1) {
            const int v = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += v;
        }
        int run = incl - local;
        for (int e = e0; e < e1; ++e) {
            s_slot[e] = run;
            slot_off[e] = run;
            run += (__ldcg(offsets + e + 1) - __ldcg(offsets + e) + align - 1) & -align;
        }
        if (lane == 31) {
            s_slot[E] = incl;
            slot_off[E] = incl;
        }
    } else if (warp == 1) {
        const int na = __ldcg(n_act);
        const int per = (na + 31) / 32;
        const int a0 = min(na, lane * per), a1 = min(na, a0 + per);
        int local = 0;
        for (int a = a0; a < a1; ++a) {
            const int e = __ldcg(act + a);
            local += (__ldcg(offsets + e + 1) - __ldcg(offsets + e) + tile - 1) / tile;
        }
        int incl = local;
        for (int o = 1; o < 32; o <<= 1) {
            const int v = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += v;
        }
        int run = incl - local;
        for (int a = a0; a < a1; ++a) {
            tt_off[a] = run;
            const int e = __ldcg(act + a);
            run += (__ldcg(offsets + e + 1) - __ldcg(offsets + e) + tile - 1) / tile;
        }
        if (lane == 31) tt_off[na] = incl;
    }
    __syncthreads();
    for (int p = threadIdx.x; p < P; p += blockDim.x) {
        const int e = __ldcg(idx + p);
        pair_slot[p] = s_slot[e] + __ldcg(pos + p) - __ldcg(offsets + e);
    }
    pdl_trigger();
}

// ---- the GEMM ------------------------------------------------------------------

constexpr int kTcKS = 4;            // blocks per pipeline stage (and per accumulator group)
constexpr int kTcTileRowsPad = 129; // padded row count of the SwiGLU transpose (no bank conflicts)
constexpr int kTcBufs = 8;          // TMEM accumulators of kTcN columns (all 512 columns), two groups of kTcKS
constexpr int kTcGroups = kTcBufs / kTcKS;
constexpr int kTcEpiWarps = 16;     // epilogue warps: 4 TMEM lane quarters x 4 column quarters
constexpr int kTcEpiCols = 16;      // accumulator columns (tokens) per epilogue warp
constexpr int kTcThreads = 32 * (2 + kTcEpiWarps);
constexpr int kTcStageDw = kTcKS * kTileRows * 2;
constexpr int kTcStageDa = kTcKS * kTcN * 4;
constexpr int kTcXld = kTcTileRowsPad;
constexpr int kTcXchg = kTcN * kTcXld * 4;                  // SwiGLU transpose: [token][row], padded rows
// One pipeline stage: weight codes (A), weight scales, activation codes (B),
// activation scales.  The codes are int8 (kind::i8 MMAs), or the same
// integers widened to fp16 (kind::f16 MMAs, fp32 accumulators that hold the
// block sums exactly: every product and partial sum is an integer below 2^24).
__host__ __device__ constexpr int tc_stage_a(bool f16) { return kTcKS * (f16 ? 8192 : 4096); }
__host__ __device__ constexpr int tc_stage_b(bool f16) { return kTcKS * kTcN * (f16 ? 64 : 32); }
__host__ __device__ constexpr int tc_stage(bool f16) {
    return tc_stage_a(f16) + kTcStageDw + tc_stage_b(f16) + kTcStageDa;
}
__host__ __device__ constexpr int tc_nstages(bool f16) { return f16 ? 3 : 6; }
__host__ __device__ constexpr int tc_smem(bool f16) {
    return 1024 + tc_nstages(f16) * tc_stage(f16) + kTcXchg + 6144 + 4100;   // + the staged units
}
static_assert(tc_smem(true) <= 227 * 1024 && tc_smem(false) <= 227 * 1024, "one CTA per SM");
static_assert(kTcEpiWarps * kTcEpiCols == 4 * kTcN, "the epilogue warps cover the 128 x 64 tile");

enum { TC_OUT_F32 = 0, TC_OUT_F32_Q81 = 1, TC_OUT_SWIGLU = 2, TC_OUT_F32_COMBINE = 3, TC_OUT_F32_ADD = 4 };

struct TcArgs {
    static constexpr int kN = kTcN;   // slots per token tile
    // tensor maps of one stage's four copies (host-encoded):
    //  tm_a : weight codes, uint32 [tiles][nb][4 slices][256] with strides
    //         (nb*4096, 1024, nb*1024) bytes; box [1][4][4][256] lands as
    //         [block][slice][1 KB], the MMA's A layout
    //  tm_d : weight scales, uint16 [tiles][nb][4][32]; box -> [block][slice][32]
    //  tm_b : packed activation codes, uint32 [nb][slots/8][64]; box [4][8][64]
    //         (fp16 codes: uint32 [nb][2][slots/8][64]; box [4][2][8][64])
    //  tm_bd: activation scales, fp32 [nb][slots]; box [4][64]
    // (fp16 codes: the weight codes come from q16 by one bulk copy a stage)
    CUtensorMap tm_a, tm_d, tm_b, tm_bd;
    const uint8_t* q;           // weight arena of group 0
    const uint16_t* d;
    int64_t q_gstride, d_gstride;
    const uint8_t* q16;         // fp16 codes (kind::f16 launches): [tiles][nb][2][16][2][8][8] fp16
    int64_t q16_gstride;
    int nb, rtiles;
    int n_groups;               // matrices in the arena (the experts, or 1)
    // groups: dense (act == NULL: one group of T tokens in slots 0 .. T-1) or
    // the routed experts (slot_off/counts per expert, tt_off per active expert)
    const int32_t* act;
    const int32_t* n_act;
    const int32_t* slot_off;    // [E+1]
    const int32_t* offsets;     // [E+1] pair offsets (tokens per expert = difference)
    const int32_t* tt_off;      // [E+1] token tiles before active expert a
    int T;
    // B operand
    const uint8_t* bq;
    const float* bd;
    int64_t bstride;
    // outputs
    int out_mode;
    float* y;                   // fp32 rows, by token (dense) or slot (experts)
    int64_t y_ld;
    uint8_t* yq;                // Q8_1 AoS rows (TC_OUT_F32_Q81)
    int64_t yq_ld;
    uint8_t* cq;                // canonical B buffer written by the epilogue (SWIGLU: hq; COMBINE: ylq)
    float* cd;
    int64_t cstride;
    // combine (down): weights, the slot of each pair, per (token, 32-row block) counters
    const float* wts;
    const int32_t* perm;        // pair of each position (experts)
    const int32_t* pair_slot;   // [T*k] slot of each pair
    int kslots;
    int* cnt_comb;              // [T][L/32]
    float* ylat;
    uint8_t* ylq;               // Q8_1 AoS of y_lat
    int* err;
    uint64_t budget_ns;
};

struct TcUnit {
    int rt, e, slot0, nvalid, ncols;
    bool valid;
};

// Units of a group (the dense matrix, or one routed expert with its n_q
// token tiles) run row tile by row tile, each row tile against all n_q token
// tiles in turn: a weight tile is read from HBM once and its next uses follow
// at once (from L2), while a group's token tiles (at most a few hundred KB)
// stay in L2 across its row tiles.
__device__ __forceinline__ TcUnit tc_unit(const TcArgs& g, int u) {
    TcUnit r;
    int tt;
    if (!g.act) {
        const int n_q = (g.T + kTcN - 1) / kTcN;
        r.rt = u / n_q;
        tt = u - r.rt * n_q;
        r.e = 0;
        r.slot0 = tt * kTcN;
        r.nvalid = min(kTcN, g.T - r.slot0);
    } else {
        const int q = u / g.rtiles;
        const int na = __ldcg(g.n_act);
        int lo = 0, hi = na;    // tt_off[lo] <= q < tt_off[hi]: the group's units are [tt_off[lo], tt_off[lo+1]) * rtiles
        while (hi - lo > 1) {
            const int mid = (lo + hi) >> 1;
            if (__ldcg(g.tt_off + mid) <= q) lo = mid; else hi = mid;
        }
        r.e = __ldcg(g.act + lo);
        const int base = __ldcg(g.tt_off + lo);
        const int n_q = __ldcg(g.tt_off + lo + 1) - base;
        const int v = u - base * g.rtiles;
        r.rt = v / n_q;
        tt = v - r.rt * n_q;
        r.slot0 = __ldcg(g.slot_off + r.e) + tt * kTcN;
        const int cnt = __ldcg(g.offsets + r.e + 1) - __ldcg(g.offsets + r.e);
        r.nvalid = min(kTcN, cnt - tt * kTcN);
    }
    r.ncols = (r.nvalid + 15) & ~15;
    r.valid = r.nvalid > 0;
    return r;
}

// A CTA's units staged once in shared memory: every role then reads a unit
// from there instead of repeating a binary search of dependent global loads
// per unit (each one an L2 round trip).
constexpr int kUnitsSmem = 256;
constexpr int kUnitTableInts = 1025;        // tt_off[0 .. na], na <= 1024
constexpr int kUnitsBytes = kUnitsSmem * (int)sizeof(TcUnit) + kUnitTableInts * 4;
static_assert(kUnitsBytes == 6144 + 4100, "tc_smem counts the staged units' bytes");

// Expert unit u with the token-tile offsets in shared memory (stt = tt_off[0
// .. na]): the search runs there; the expert, first slot and pair count take
// two dependent global loads.
template <class A>
__device__ __forceinline__ TcUnit unit_staged(const A& g, int u, const int* stt, int na) {
    TcUnit r;
    const int q = u / g.rtiles;
    int lo = 0, hi = na;
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (stt[mid] <= q) lo = mid; else hi = mid;
    }
    r.e = __ldcg(g.act + lo);
    const int base = stt[lo];
    const int n_q = stt[lo + 1] - base;
    const int v = u - base * g.rtiles;
    r.rt = v / n_q;
    const int tt = v - r.rt * n_q;
    r.slot0 = __ldcg(g.slot_off + r.e) + tt * A::kN;
    const int cnt = __ldcg(g.offsets + r.e + 1) - __ldcg(g.offsets + r.e);
    r.nvalid = min(A::kN, cnt - tt * A::kN);
    r.ncols = (r.nvalid + 15) & ~15;
    r.valid = r.nvalid > 0;
    return r;
}

// The CTA's units u0 + i * step, i < n (the first kUnitsSmem) into su, all
// threads; ends with a CTA barrier.  Dense launches (no routing) compute
// theirs directly.
template <class A>
__device__ void stage_units(const A& g, int u0, int step, int n_all, TcUnit* su, int* stt) {
    const int n = min(n_all, kUnitsSmem);
    const int na = g.act ? __ldcg(g.n_act) : 0;
    if (g.act && na + 1 <= kUnitTableInts) {
        for (int i = threadIdx.x; i <= na; i += blockDim.x) stt[i] = __ldcg(g.tt_off + i);
        __syncthreads();
        for (int i = threadIdx.x; i < n; i += blockDim.x) su[i] = unit_staged(g, u0 + i * step, stt, na);
    } else {
        for (int i = threadIdx.x; i < n; i += blockDim.x) su[i] = tc_unit(g, u0 + i * step);
    }
    __syncthreads();
}

__device__ __forceinline__ int tc_units(const TcArgs& g) {
    if (!g.act) return ((g.T + kTcN - 1) / kTcN) * g.rtiles;
    return __ldcg(g.tt_off + __ldcg(g.n_act)) * g.rtiles;
}


// Out-of-line pieces of the epilogues, called from unrolled loops: one copy
// of their code instead of one per column (the kernels' instruction
// footprint).
__device__ __noinline__ void tc_quant(float v, uint8_t* dst) { warp_quant_q8_1(v, dst); }


template <int OM, bool F16>
__global__ void __launch_bounds__(kTcThreads, 1) k_tcgemm(const __grid_constant__ TcArgs g) {
    constexpr int kTcStages = tc_nstages(F16), kTcStage = tc_stage(F16);
    constexpr int kTcStageA = tc_stage_a(F16), kTcStageB = tc_stage_b(F16);
    extern __shared__ __align__(1024) uint8_t tcsm[];
    uint64_t* full = reinterpret_cast<uint64_t*>(tcsm);            // [stages]
    uint64_t* empty = full + kTcStages;                             // [stages]
    uint64_t* tfull = empty + kTcStages;                            // [groups]: a stage's MMAs are done
    uint64_t* tempty = tfull + kTcGroups;                           // [groups]: its accumulators drained
    uint64_t* xfull = tempty + kTcGroups;                           // the tile handed over (epilogue warps)
    uint64_t* xempty = xfull + 1;                                   // ... and taken
    uint32_t* tmem_base_sm = reinterpret_cast<uint32_t*>(xempty + 1);
    int* abort_sm = reinterpret_cast<int*>(tmem_base_sm + 1);
    uint8_t* stages = tcsm + 1024;
    float* xchg = reinterpret_cast<float*>(tcsm + 1024 + kTcStages * kTcStage);
    TcUnit* su = reinterpret_cast<TcUnit*>(tcsm + 1024 + kTcStages * kTcStage + kTcXchg);
    int* stt = reinterpret_cast<int*>(su + kUnitsSmem);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < kTcStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1 + kTcEpiWarps);   // the MMA commit + the epilogue warps
        }
        for (int b = 0; b < kTcGroups; ++b) {
            mbar_init(&tfull[b], 1);
            mbar_init(&tempty[b], kTcEpiWarps);
        }
        mbar_init(xfull, kTcEpiWarps);
        mbar_init(xempty, kTcEpiWarps);
        *abort_sm = 0;
        fence_barrier_init();
    }
    if (warp == 0) {
        tmem_alloc(tmem_base_sm, kTcBufs * kTcN);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_base_sm;
    pdl_wait();

    const int n_units = tc_units(g);
    // CTA b takes units b, b + grid, b + 2 grid, ...: at any moment the CTAs work on neighbouring
    // units, so a weight row tile (the units of one row tile are consecutive) and an activation
    // tile are read by several CTAs together and come from L2 after the first (loop index u: the
    // CTA's i-th unit)
    const int n_mine = n_units > (int)blockIdx.x ? (n_units - (int)blockIdx.x + (int)gridDim.x - 1) / (int)gridDim.x
                                                 : 0;
    const int u0 = 0, u1 = n_mine;
    const int kstages = g.nb / kTcKS;
    volatile int* abort_v = abort_sm;
    stage_units(g, (int)blockIdx.x, (int)gridDim.x, n_mine, su, stt);
    auto unit_at = [&](int i) {
        return i < kUnitsSmem ? su[i] : tc_unit(g, (int)blockIdx.x + i * (int)gridDim.x);
    };

    if (warp == 0) {
        // ---------------- producer ----------------
        if (lane == 0) {
            int it = 0;
            for (int u = u0; u < u1 && !*abort_v; ++u) {
                const TcUnit un = unit_at(u);
                if (!un.valid) continue;
                const uint8_t* qa = g.q + un.e * g.q_gstride + (int64_t)un.rt * g.nb * 4096;
                const uint16_t* da = g.d + un.e * g.d_gstride + (int64_t)un.rt * g.nb * kTileRows;
                for (int ks = 0; ks < kstages; ++ks, ++it) {
                    const int s = it % kTcStages;
                    if (it >= kTcStages &&
                        !mbar_wait_bounded(&empty[s], (uint32_t)((it / kTcStages - 1) & 1), g.err, g.budget_ns)) {
                        *abort_v = 1;
                        break;
                    }
                    uint8_t* st = stages + s * kTcStage;
                    mbar_arrive_expect_tx(&full[s], (uint32_t)kTcStage);
                    const int kb0 = ks * kTcKS;
                    const int tile = un.e * g.rtiles + un.rt;
                    if constexpr (F16) {
                        bulk_g2s(st, g.q16 + un.e * g.q16_gstride + ((int64_t)un.rt * g.nb + kb0) * 8192,
                                 (uint32_t)kTcStageA, &full[s]);
                    } else {
                        tma_load_4d(st, &g.tm_a, 0, 0, kb0, tile, &full[s]);
                    }
                    tma_load_4d(st + kTcStageA, &g.tm_d, 0, 0, kb0, tile, &full[s]);
                    if constexpr (F16)
                        tma_load_4d(st + kTcStageA + kTcStageDw, &g.tm_b, 0, un.slot0 >> 3, 0, kb0, &full[s]);
                    else
                        tma_load_3d(st + kTcStageA + kTcStageDw, &g.tm_b, 0, un.slot0 >> 3, kb0, &full[s]);
                    tma_load_2d(st + kTcStageA + kTcStageDw + kTcStageB, &g.tm_bd, un.slot0, kb0, &full[s]);
                }
            }
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer ----------------
        // stage `it` goes to accumulator group it % 2 (kTcKS buffers, one per block)
        if (lane == 0) {
            int it = 0;
            for (int u = u0; u < u1 && !*abort_v; ++u) {
                const TcUnit un = unit_at(u);
                if (!un.valid) continue;
                const uint32_t idesc = F16 ? umma_idesc_f16(128, un.ncols) : umma_idesc_i8(128, un.ncols);
                for (int ks = 0; ks < kstages && !*abort_v; ++ks, ++it) {
                    const int s = it % kTcStages, gr = it % kTcGroups;
                    if (it >= kTcGroups &&
                        !mbar_wait_bounded(&tempty[gr], (uint32_t)((it / kTcGroups - 1) & 1), g.err, g.budget_ns)) {
                        *abort_v = 1;
                        break;
                    }
                    if (!mbar_wait_bounded(&full[s], (uint32_t)((it / kTcStages) & 1), g.err, g.budget_ns)) {
                        *abort_v = 1;
                        break;
                    }
                    tc_fence_after();
                    const uint8_t* st = stages + s * kTcStage;
                    for (int kl = 0; kl < kTcKS; ++kl) {
                        if constexpr (F16) {
                            // a block = two K = 16 halves, 4 KB of A and 2 KB of B each
                            for (int h = 0; h < 2; ++h) {
                                const uint64_t adesc = umma_desc(st + (kl * 2 + h) * 4096, 128, 256);
                                const uint64_t bdesc =
                                    umma_desc(st + kTcStageA + kTcStageDw + (kl * 2 + h) * kTcN * 32, 128, 256);
                                umma_f16(tmem + (uint32_t)((gr * kTcKS + kl) * kTcN), adesc, bdesc, idesc,
                                         (uint32_t)h);
                            }
                        } else {
                            const uint64_t adesc = umma_desc(st + kl * 4096, 128, 256);
                            const uint64_t bdesc = umma_desc(st + kTcStageA + kTcStageDw + kl * kTcN * 32, 128, 256);
                            umma_i8(tmem + (uint32_t)((gr * kTcKS + kl) * kTcN), adesc, bdesc, idesc, 0u);
                        }
                    }
                    umma_commit(&tfull[gr]);
                    umma_commit(&empty[s]);
                }
            }
            // let the last MMAs finish before the accumulators are freed
            if (it > 0) {
                const int last = it - 1;
                mbar_wait_bounded(&tfull[last % kTcGroups], (uint32_t)((last / kTcGroups) & 1), nullptr, g.budget_ns);
            }
        }
    } else {
        // ---------------- epilogue ----------------
        const int ew = warp - 2;              // 0 .. kTcEpiWarps-1
        const int sp = warp & 3;              // TMEM lane quarter this warp may read
        const int c0 = (ew >> 2) * kTcEpiCols;   // its accumulator columns (tokens) c0 .. c0+15
        const int row = sp * 32 + lane;       // weight row within the tile
        int it = 0, xc = 0;
        int s = 0;                            // it % kTcStages and the parity of it / kTcStages
        uint32_t sph = 0;
        for (int u = u0; u < u1 && !*abort_v; ++u) {
            const TcUnit un = unit_at(u);
            if (!un.valid) continue;
            // accumulator pairs (columns 2j, 2j+1)
            uint64_t acc2[kTcEpiCols / 2], part2[kTcEpiCols / 2];
#pragma unroll
            for (int j = 0; j < kTcEpiCols / 2; ++j) { acc2[j] = 0ull; part2[j] = 0ull; }
            bool ok = true;
            const bool active = c0 < un.ncols;
            const uint32_t tlane = (uint32_t)(sp * 32) << 16;
            const uint64_t seed2 = f2_pack(kAccSeedF, kAccSeedF);
            for (int ks = 0; ks < kstages; ++ks, ++it) {
                const int gr = it % kTcGroups;
                const uint8_t* st = stages + s * kTcStage;
                // the stage's scales (bulk copies) and its accumulators (MMAs)
                if (!warp_wait_bounded(&full[s], sph, g.err, g.budget_ns) ||
                    !warp_wait_bounded(&tfull[gr], (uint32_t)((it / kTcGroups) & 1), g.err, g.budget_ns)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint16_t* dws = reinterpret_cast<const uint16_t*>(st + kTcStageA);
                const float* das = reinterpret_cast<const float*>(st + kTcStageA + kTcStageDw + kTcStageB);
                const uint32_t tb = tmem + tlane + (uint32_t)(gr * kTcKS * kTcN + c0);
                // column groups past the tile's tokens hold no MMA result
                if (active) {
#pragma unroll
                    for (int kp = 0; kp < kTcKS; kp += 2) {
                        // two blocks' accumulators per wait
                        uint32_t rc[2][kTcEpiCols];
                        tmem_ld16(tb + (uint32_t)(kp * kTcN), rc[0]);
                        tmem_ld16(tb + (uint32_t)((kp + 1) * kTcN), rc[1]);
                        tmem_ld_wait();
#pragma unroll
                        for (int h = 0; h < 2; ++h) {
                            const int kl = kp + h;
                            // block kl of the stage: part = fmaf(isum, d_w * d_a, part) per column, two at a time
                            const float dw = h2f(dws[kl * kTileRows + sp * 32 + lane]);
                            const uint64_t dw2 = f2_pack(dw, dw);
                            const float4* dak = reinterpret_cast<const float4*>(das + kl * kTcN + c0);
#pragma unroll
                            for (int j4 = 0; j4 < kTcEpiCols / 4; ++j4) {
                                const float4 dv = dak[j4];
                                uint64_t i0, i1;
                                if constexpr (F16) {
                                    // fp32 accumulators: the block sums themselves
                                    i0 = f2_pack(__uint_as_float(rc[h][4 * j4]), __uint_as_float(rc[h][4 * j4 + 1]));
                                    i1 = f2_pack(__uint_as_float(rc[h][4 * j4 + 2]),
                                                 __uint_as_float(rc[h][4 * j4 + 3]));
                                } else {
                                    i0 = f2_sub(f2_pack(__uint_as_float(rc[h][4 * j4] + kAccSeed),
                                                        __uint_as_float(rc[h][4 * j4 + 1] + kAccSeed)),
                                                seed2);
                                    i1 = f2_sub(f2_pack(__uint_as_float(rc[h][4 * j4 + 2] + kAccSeed),
                                                        __uint_as_float(rc[h][4 * j4 + 3] + kAccSeed)),
                                                seed2);
                                }
                                part2[2 * j4] = f2_fma(i0, f2_mul(dw2, f2_pack(dv.x, dv.y)), part2[2 * j4]);
                                part2[2 * j4 + 1] = f2_fma(i1, f2_mul(dw2, f2_pack(dv.z, dv.w)), part2[2 * j4 + 1]);
                            }
                        }
                    }
                }
                // a run of 8 blocks ends with every (8 / kTcKS)-th stage (and with the last)
                if ((ks + 1) % (kChunk / kTcKS) == 0 || ks == kstages - 1) {
#pragma unroll
                    for (int j = 0; j < kTcEpiCols / 2; ++j) {
                        acc2[j] = f2_add(acc2[j], part2[j]);
                        part2[j] = 0ull;
                    }
                }
                tc_fence_before();
                __syncwarp();
                mbar_arrive_lane0(&tempty[gr], lane);
                mbar_arrive_lane0(&empty[s], lane);
                if (++s == kTcStages) {
                    s = 0;
                    sph ^= 1u;
                }
            }
            float acc[kTcEpiCols];
#pragma unroll
            for (int j = 0; j < kTcEpiCols / 2; ++j) f2_unpack(acc2[j], acc[2 * j], acc[2 * j + 1]);
            if (!ok) {
                *abort_v = 1;
                break;
            }
            // ---- outputs of the tile ----
            const int nv = un.nvalid;
            const int64_t slot0 = un.slot0;
            if (OM == TC_OUT_SWIGLU) {
                // transpose the tile's accumulators through shared memory ([token][row], padded), then
                // the epilogue threads build the Q8_1 blocks of h = silu(gate) * up, four per block:
                // h row 32*hb + i of token t takes gate row 32*hb + i and up row 64 + 32*hb + i
                if (xc > 0 && !warp_wait_bounded(xempty, (uint32_t)((xc - 1) & 1), g.err, g.budget_ns)) {
                    *abort_v = 1;
                    break;
                }
#pragma unroll
                for (int j = 0; j < kTcEpiCols; ++j) xchg[(c0 + j) * kTcXld + row] = acc[j];
                __syncwarp();
                mbar_arrive_lane0(xfull, lane);
                if (!warp_wait_bounded(xfull, (uint32_t)(xc & 1), g.err, g.budget_ns)) {
                    *abort_v = 1;
                    break;
                }
                // all 512 epilogue threads: four lanes per (token, h block),
                // eight values each; amax and the code sum by two shuffles
                {
                    const int task = ew * 32 + lane;        // 0 .. 511
                    const int b = task >> 2, qd = task & 3;  // block (token t, half hb), quarter
                    const int t = b >> 1, hb = b & 1;
                    const bool on = t < nv;
                    float h[8];
                    float amax = 0.0f;
                    if (on) {
                        const float* gr = xchg + t * kTcXld + hb * 32 + qd * 8;
                        const float* ur = gr + 64;
#pragma unroll
                        for (int i = 0; i < 8; ++i) {
                            h[i] = __fmul_rn(silu_f32(gr[i]), ur[i]);
                            amax = fmaxf(amax, fabsf(h[i]));
                        }
                    } else {
#pragma unroll
                        for (int i = 0; i < 8; ++i) h[i] = 0.0f;
                    }
                    amax = fmaxf(amax, __shfl_xor_sync(kFull, amax, 1));
                    amax = fmaxf(amax, __shfl_xor_sync(kFull, amax, 2));
                    const float d = __fdiv_rn(amax, 127.0f);
                    uint32_t w0 = 0, w1 = 0;
                    int qv[8];
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        int q = 0;
                        if (d != 0.0f) q = (int)fminf(fmaxf(roundf(__fdiv_rn(h[i], d)), -127.0f), 127.0f);
                        qv[i] = q;
                        if (i < 4) w0 |= (uint32_t)(q & 0xff) << (8 * i);
                        else w1 |= (uint32_t)(q & 0xff) << (8 * (i - 4));
                    }
                    if (on) {
                        const int64_t slot = slot0 + t;
                        const int kbh = un.rt * 2 + hb;
                        if constexpr (F16) {
                            // codes 8 qd .. 8 qd + 7 as fp16: half qd / 2 of the block, core matrix qd % 2
                            uint8_t* dst = g.cq + (int64_t)kbh * g.cstride * 64 + (int64_t)(qd >> 1) * g.cstride * 32 +
                                           (slot >> 3) * 256 + (qd & 1) * 128 + (slot & 7) * 16;
                            *reinterpret_cast<uint4*>(dst) = make_uint4(h2_pack_int(qv[0], qv[1]), h2_pack_int(qv[2], qv[3]),
                                                                        h2_pack_int(qv[4], qv[5]), h2_pack_int(qv[6], qv[7]));
                        } else {
                            // codes 8 qd .. 8 qd + 7 of the slot's 32: first or second 16-byte half, low or high 8 bytes
                            uint8_t* dst = g.cq + (int64_t)kbh * g.cstride * 32 + (slot >> 3) * 256 + (qd >> 1) * 128 +
                                           (slot & 7) * 16 + (qd & 1) * 8;
                            *reinterpret_cast<uint2*>(dst) = make_uint2(w0, w1);
                        }
                        // the activation scale as the down projection reads it: fp32 of the stored fp16
                        if (qd == 0) g.cd[(int64_t)kbh * g.cstride + slot] = __half2float(__float2half_rn(d));
                    }
                }
                __syncwarp();
                mbar_arrive_lane0(xempty, lane);
                ++xc;
                continue;
            }
#pragma unroll
            for (int j = 0; j < kTcEpiCols; ++j) {
                const int t = c0 + j;
                if (t < nv) {
                    const int64_t orow = slot0 + t;
                    float* yp = g.y + orow * g.y_ld + (int64_t)un.rt * kTileRows + row;
                    // TC_OUT_F32_ADD: the residual stream, y = y + the rows (fp32)
                    *yp = (OM == TC_OUT_F32_ADD) ? __fadd_rn(*yp, acc[j]) : acc[j];
                    if (OM == TC_OUT_F32_Q81)
                        tc_quant(acc[j], g.yq + (orow * g.yq_ld + un.rt * 4 + sp) * 36);
                }
            }
            if (OM == TC_OUT_F32_COMBINE) {
                // each (token, 32-row block) is combined by the warp that writes its last expert row
                // block: lane j < 16 counts token c0 + j, all counters of the warp at once
                __threadfence();
                __syncwarp();
                const int L = g.rtiles * kTileRows;
                const int blk = un.rt * 4 + sp;
                const int tj = c0 + lane;
                int tok = 0, last = 0;
                if (lane < kTcEpiCols && tj < nv) {
                    const int i = (int)(slot0 + tj - __ldcg(g.slot_off + un.e));
                    const int p = __ldcg(g.perm + __ldcg(g.offsets + un.e) + i);
                    tok = p / g.kslots;
                    int* cnt = g.cnt_comb + (int64_t)tok * (L / 32) + blk;
                    last = (atomicAdd(cnt, 1) == g.kslots - 1);
                    if (last) *cnt = 0;
                }
                unsigned m = __ballot_sync(kFull, last);
                if (m) __threadfence();
                while (m) {
                    const int j = __ffs(m) - 1;
                    m &= m - 1;
                    const int tk = __shfl_sync(kFull, tok, j);
                    float a2 = 0.0f;
                    for (int j0 = 0; j0 < g.kslots; j0 += 8) {
                        float ov[8], wv[8];
#pragma unroll
                        for (int q = 0; q < 8; ++q)
                            if (j0 + q < g.kslots) {
                                const int pj = tk * g.kslots + j0 + q;
                                wv[q] = __ldcg(g.wts + pj);
                                ov[q] = __ldcg(g.y + (int64_t)__ldcg(g.pair_slot + pj) * g.y_ld + blk * 32 + lane);
                            }
#pragma unroll
                        for (int q = 0; q < 8; ++q)
                            if (j0 + q < g.kslots) a2 = __fmaf_rn(wv[q], ov[q], a2);
                    }
                    g.ylat[(int64_t)tk * L + blk * 32 + lane] = a2;
                    warp_quant_q8_1(a2, g.ylq + ((int64_t)tk * (L / 32) + blk) * 36);
                    __syncwarp();
                    if (g.cq) {
                        // the same block, packed for the U projection (slot = token)
                        uint8_t* dst = g.cq + (int64_t)blk * g.cstride * 32 + ((int64_t)tk >> 3) * 256 + (tk & 7) * 16;
                        const uint8_t* srcb = g.ylq + ((int64_t)tk * (L / 32) + blk) * 36;
                        if (lane < 8)
                            reinterpret_cast<uint32_t*>(dst + (lane >> 2) * 128)[lane & 3] =
                                reinterpret_cast<const uint32_t*>(srcb + 4)[lane];
                        if (lane == 0)
                            g.cd[(int64_t)blk * g.cstride + tk] = h2f(*reinterpret_cast<const uint16_t*>(srcb));
                    }
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) tmem_dealloc(tmem, kTcBufs * kTcN);
    pdl_trigger();
}

// ---- a9 on the tensor-core path: the weighted combine --------------------------
//
// One warp per (token, 4 consecutive 32-row latent blocks): lane l keeps the 4
// rows 4 (l % 8) .. +3 of block l / 8, so each read of a pair's o row is 512
// contiguous bytes for the warp.  Every row is y_lat = fmaf(w_j, o_j, y_lat)
// over the token's k pairs in rank order (o read by the pair's slot), then
// the Q8_1 block of each 8-lane group (amax and code sum by three shuffles),
// written both row-major (ylq) and into the packed buffer the U projection
// reads (slot = token).
struct CombArgs {
    const float* o;             // [slots][L] by slot
    const float* wts;           // [T][k]
    const int32_t* pair_slot;   // [T*k]
    int T, L, k;
    float* ylat;                // [T][L]
    uint8_t* ylq;               // [T][L/32] Q8_1
    uint8_t* cq;                // packed codes [L/32][cstride] (fp16 codes: [L/32][2][cstride] x 32 B)
    float* cd;                  // packed scales [L/32][cstride]
    int64_t cstride;
    int f16;                    // codes widened to fp16 (the kind::f16 operand layout)
};

__global__ void __launch_bounds__(256) k_tc_combine(CombArgs a) {
    pdl_wait();
    pdl_trigger();
    const int lane = threadIdx.x & 31;
    const int64_t task = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int nbl = a.L / 32, nch = (nbl + 3) / 4;
    if (task >= (int64_t)a.T * nch) return;          // whole warps
    const int t = (int)(task / nch), c = (int)(task - (int64_t)t * nch);
    const int blk = 4 * c + (lane >> 3), m = lane & 7;
    const bool on = blk < nbl;
    const int64_t col = (int64_t)blk * 32 + 4 * m;   // this lane's first row
    float4 acc = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
#pragma unroll 4
    for (int j = 0; j < a.k; ++j) {
        const int pj = t * a.k + j;
        const float wj = __ldg(a.wts + pj);
        const int64_t slot = __ldg(a.pair_slot + pj);
        if (on) {
            const float4 v = __ldcg(reinterpret_cast<const float4*>(a.o + slot * a.L + col));
            acc.x = __fmaf_rn(wj, v.x, acc.x);
            acc.y = __fmaf_rn(wj, v.y, acc.y);
            acc.z = __fmaf_rn(wj, v.z, acc.z);
            acc.w = __fmaf_rn(wj, v.w, acc.w);
        }
    }
    if (on) *reinterpret_cast<float4*>(a.ylat + (int64_t)t * a.L + col) = acc;
    // the block's Q8_1 (the quantiser's rule) over its 8-lane group
    float amax = fmaxf(fmaxf(fabsf(acc.x), fabsf(acc.y)), fmaxf(fabsf(acc.z), fabsf(acc.w)));
#pragma unroll
    for (int o = 1; o < 8; o <<= 1) amax = fmaxf(amax, __shfl_xor_sync(kFull, amax, o));
    const float d = __fdiv_rn(amax, 127.0f);
    const float av[4] = {acc.x, acc.y, acc.z, acc.w};
    uint32_t wv = 0;
    int sum = 0;
    int qv[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        int q = 0;
        if (d != 0.0f) q = (int)fminf(fmaxf(roundf(__fdiv_rn(av[i], d)), -127.0f), 127.0f);
        qv[i] = q;
        sum += q;
        wv |= (uint32_t)(q & 0xff) << (8 * i);
    }
#pragma unroll
    for (int o = 1; o < 8; o <<= 1) sum += __shfl_xor_sync(kFull, sum, o);
    if (!on) return;
    const uint16_t dh = f2h(d);
    uint32_t* qb = reinterpret_cast<uint32_t*>(a.ylq + ((int64_t)t * nbl + blk) * 36);
    qb[1 + m] = wv;
    if (a.f16) {
        // codes 4 m .. 4 m + 3 as fp16: half m / 4 of the block, core matrix (m / 2) % 2, its 8-byte half m % 2
        uint8_t* dst = a.cq + (int64_t)blk * a.cstride * 64 + (int64_t)(m >> 2) * a.cstride * 32 +
                       ((int64_t)t >> 3) * 256 + ((m >> 1) & 1) * 128 + (t & 7) * 16 + (m & 1) * 8;
        *reinterpret_cast<uint2*>(dst) = make_uint2(h2_pack_int(qv[0], qv[1]), h2_pack_int(qv[2], qv[3]));
    } else {
        uint8_t* dst = a.cq + (int64_t)blk * a.cstride * 32 + ((int64_t)t >> 3) * 256 + (t & 7) * 16;
        *reinterpret_cast<uint32_t*>(dst + (m < 4 ? 4 * m : 128 + 4 * (m - 4))) = wv;
    }
    if (m == 0) {
        qb[0] = (uint32_t)dh | ((uint32_t)f2h(__fmul_rn(d, (float)sum)) << 16);
        a.cd[(int64_t)blk * a.cstride + t] = h2f(dh);
    }
}

// ---- measurement: the int8 tensor-core rate ------------------------------------
//
// One CTA per SM (the launch asks for enough shared memory to keep it alone),
// one thread issuing n_mma back-to-back tcgen05.mma kind::i8 of M=128, N=256,
// K=32 (one int8 block of 128 x 256 outputs, 2 * 128 * 256 * 32 operations)
// from two fixed shared-memory operand tiles into two alternating TMEM
// accumulators, then one commit.  The operands' values do not matter for the
// rate; the sink receives one accumulator word per CTA so the work is
// observable.  Every wait is bounded.
constexpr int kRateN = 256;
constexpr int kRateSmem = 150 * 1024;

__global__ void __launch_bounds__(128, 1) k_test_mma_i8_rate(int n_mma, int* sink, int* err, uint64_t budget_ns) {
    extern __shared__ __align__(1024) uint8_t rsm_[];
    uint64_t* done = reinterpret_cast<uint64_t*>(rsm_);
    uint32_t* tbase = reinterpret_cast<uint32_t*>(rsm_ + 8);
    uint8_t* a = rsm_ + 1024;                 // 128 x 32 codes
    uint8_t* b = a + 128 * 32;                // 256 x 32 codes
    const int warp = threadIdx.x >> 5;
    for (int i = threadIdx.x; i < (128 + kRateN) * 32 / 4; i += blockDim.x)
        reinterpret_cast<uint32_t*>(a)[i] = 0x01010101u * (uint32_t)((i & 7) + 1);
    if (threadIdx.x == 0) {
        mbar_init(done, 1);
        fence_barrier_init();
    }
    if (warp == 0) {
        tmem_alloc(tbase, 2 * kRateN);
        tmem_relinquish();
    }
    fence_proxy_async();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tbase;
    if (threadIdx.x == 0) {
        const uint32_t idesc = umma_idesc_i8(128, kRateN);
        const uint64_t ad = umma_desc(a, 128, 256), bd = umma_desc(b, 128, 256);
        for (int i = 0; i < n_mma; ++i)
            umma_i8(tmem + (uint32_t)((i & 1) * kRateN), ad, bd, idesc, i >= 2 ? 1u : 0u);
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
    if (warp == 0) tmem_dealloc(tmem, 2 * kRateN);
}

// ---- measurement: the fp16 tensor-core rate ------------------------------------
//
// As k_test_mma_i8_rate, with tcgen05.mma kind::f16 of M=128, N=256, K=16
// (fp16 operands holding small integers, fp32 accumulators): the peak of the
// fp16-operand GEMMs.
__global__ void __launch_bounds__(128, 1) k_test_mma_f16_rate(int n_mma, int* sink, int* err, uint64_t budget_ns) {
    extern __shared__ __align__(1024) uint8_t rsm16_[];
    uint64_t* done = reinterpret_cast<uint64_t*>(rsm16_);
    uint32_t* tbase = reinterpret_cast<uint32_t*>(rsm16_ + 8);
    uint8_t* a = rsm16_ + 1024;               // 128 x 16 fp16 (4 KB)
    uint8_t* b = a + 128 * 32;                // 256 x 16 fp16 (8 KB)
    const int warp = threadIdx.x >> 5;
    for (int i = threadIdx.x; i < (128 + kRateN) * 32 / 4; i += blockDim.x)
        reinterpret_cast<uint32_t*>(a)[i] = h2_pack_int((i & 7) + 1, (i & 3) - 2);
    if (threadIdx.x == 0) {
        mbar_init(done, 1);
        fence_barrier_init();
    }
    if (warp == 0) {
        tmem_alloc(tbase, 2 * kRateN);
        tmem_relinquish();
    }
    fence_proxy_async();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tbase;
    if (threadIdx.x == 0) {
        const uint32_t idesc = umma_idesc_f16(128, kRateN);
        const uint64_t ad = umma_desc(a, 128, 256), bd = umma_desc(b, 128, 256);
        for (int i = 0; i < n_mma; ++i)
            umma_f16(tmem + (uint32_t)((i & 1) * kRateN), ad, bd, idesc, i >= 2 ? 1u : 0u);
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
    if (warp == 0) tmem_dealloc(tmem, 2 * kRateN);
}

// ---- measurement: the packed fp32 rate --------------------------------------
//
// Every thread runs n iterations of 8 independent chains of fma.rn.f32x2
// (each instruction two fused multiply-adds); one word per thread lands in
// sink so that the work is observable.  The caller times the launch and
// divides threads * n * 8 instructions by the time: the epilogue bound of the
// tensor-core GEMM is counted in these instructions.
__global__ void __launch_bounds__(1024) k_test_f32x2_rate(int n, float* sink) {
    uint64_t a[8], b = f2_pack(1.0000001f, 0.9999999f), c = f2_pack(1e-7f, -1e-7f);
#pragma unroll
    for (int j = 0; j < 8; ++j) a[j] = f2_pack((float)threadIdx.x + j, (float)blockIdx.x - j);
    for (int i = 0; i < n; ++i) {
#pragma unroll
        for (int j = 0; j < 8; ++j) a[j] = f2_fma(a[j], b, c);
    }
    float lo, hi, acc = 0.0f;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        f2_unpack(a[j], lo, hi);
        acc = __fadd_rn(acc, __fadd_rn(lo, hi));
    }
    sink[(int64_t)blockIdx.x * blockDim.x + threadIdx.x] = acc;
}

}  // namespace elq
