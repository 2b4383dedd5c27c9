// elq_device.cuh -- device helpers of the sm_100a kernels: number formats,
// the library's own exp, block quantisation of one warp's 32 values, and the
// bulk-copy / mbarrier primitives (inline PTX) with bounded waits.
//
// Every fp32 operation whose rounding is part of the layer's definition is
// written with an explicit round-to-nearest intrinsic (__fmul_rn, __fadd_rn,
// __fdiv_rn, __fmaf_rn); the library is also compiled with -fmad=false so no
// other multiply-add is contracted.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace elq {

constexpr int kTileRows = 128;     // rows per arena tile
constexpr int kChunk = 8;          // blocks per ordered accumulation chunk
constexpr int kQ80Slab = 4096;     // bytes of one Q8_0 (tile, block) slab
constexpr int kQ40Slab = 2048;     // bytes of one Q4_0 (tile, block) slab
constexpr int kScaleSlab = 256;    // bytes of one slab's 128 fp16 scales

// Device error word codes (first int32 of a workspace).
constexpr int kErrTimeout = 1;

__device__ __forceinline__ float h2f(uint16_t h) { return __half2float(__ushort_as_half(h)); }
__device__ __forceinline__ uint16_t f2h(float f) { return __half_as_ushort(__float2half_rn(f)); }

// exp(x): Cody-Waite reduction x = n ln2 + r (ln2 as a 16-bit high part and
// an fp32 low part), e^r by its Taylor series to degree 7 in Horner form with
// fused multiply-adds, then an exact scaling by 2^n, split in two where the
// result is subnormal or near overflow.
__device__ __forceinline__ float exp_f32(float x) {
    if (x != x) return x;
    if (x > 88.72283935546875f) return __int_as_float(0x7f800000);
    if (x < -103.972076416015625f) return 0.0f;
    const float n = rintf(__fmul_rn(x, 1.44269502162933349609375f));
    float r = __fmaf_rn(-n, 0.693145751953125f, x);
    r = __fmaf_rn(-n, 1.428606765330187045037746429443359375e-06f, r);
    float p = 1.98412701138295233249664306640625e-04f;
    p = __fmaf_rn(p, r, 1.388888922519981861114501953125e-03f);
    p = __fmaf_rn(p, r, 8.333333767950534820556640625e-03f);
    p = __fmaf_rn(p, r, 4.16666679084300994873046875e-02f);
    p = __fmaf_rn(p, r, 1.6666667163372039794921875e-01f);
    p = __fmaf_rn(p, r, 0.5f);
    p = __fmaf_rn(p, r, 1.0f);
    p = __fmaf_rn(p, r, 1.0f);
    const int ni = (int)n;
    if (ni > 127)
        return __fmul_rn(__fmul_rn(p, __int_as_float(254 << 23)), __int_as_float((ni - 127 + 127) << 23));
    if (ni < -125)
        return __fmul_rn(__fmul_rn(p, __int_as_float((ni + 100 + 127) << 23)), __int_as_float(27 << 23));
    return __fmul_rn(p, __int_as_float((ni + 127) << 23));
}

__device__ __forceinline__ float silu_f32(float g) {
    const float e = exp_f32(-g);
    return __fdiv_rn(g, __fadd_rn(1.0f, e));
}

// Quantise one 32-value block held one value per lane (lane i = element i)
// into a Q8_1 block at dst (4-byte aligned): fp16 d, fp16 s, int8 q[32].
__device__ __forceinline__ void warp_quant_q8_1(float v, uint8_t* dst) {
    const int lane = threadIdx.x & 31;
    float amax = fabsf(v);
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    const float d = __fdiv_rn(amax, 127.0f);
    int q = 0;
    if (d != 0.0f) {
        float r = roundf(__fdiv_rn(v, d));
        r = fminf(fmaxf(r, -127.0f), 127.0f);
        q = (int)r;
    }
    int s = q;
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    // gather 4 codes per lane into one word: lane j (< 8) writes codes 4j..4j+3
    const uint32_t b = (uint32_t)(q & 0xff);
    const uint32_t b0 = __shfl_sync(0xffffffffu, b, (lane * 4 + 0) & 31);
    const uint32_t b1 = __shfl_sync(0xffffffffu, b, (lane * 4 + 1) & 31);
    const uint32_t b2 = __shfl_sync(0xffffffffu, b, (lane * 4 + 2) & 31);
    const uint32_t b3 = __shfl_sync(0xffffffffu, b, (lane * 4 + 3) & 31);
    if (lane < 8)
        reinterpret_cast<uint32_t*>(dst + 4)[lane] = b0 | (b1 << 8) | (b2 << 16) | (b3 << 24);
    if (lane == 0) {
        const uint32_t dh = f2h(d);
        const uint32_t sh = f2h(__fmul_rn(d, (float)s));
        reinterpret_cast<uint32_t*>(dst)[0] = dh | (sh << 16);
    }
}

// ---- NVFP4: E2M1 codes under E4M3 micro-block scales ---------------------------

constexpr int kNV = 100;           // format id of NVFP4 (ELQ_NVFP4)
constexpr int kQ51 = 7, kQ3K = 11, kQ4K = 12, kQ5K = 13;   // Q5_1, Q3_K, Q4_K, Q5_K (GGUF ids)

// Formats whose arena scale word per (row, 32-value block) is 32 bits (two
// 16-bit units): Q5_1 (fp16 d, fp16 m), Q4_K / Q5_K (6-bit scale and min,
// and the super-block's fp16 d or dmin in sub-blocks 0 and 1), Q3_K (the two
// 16-value halves' 6-bit scales, and d in sub-block 0).
__host__ __device__ constexpr bool fmt_ext(int fmt) {
    return fmt == kQ51 || fmt == kQ3K || fmt == kQ4K || fmt == kQ5K;
}
__host__ __device__ constexpr bool fmt_has_qh(int fmt) { return fmt == kQ51 || fmt == kQ5K; }
__host__ __device__ constexpr int scale_units(int fmt) { return fmt_ext(fmt) ? 2 : 1; }

// The two E4M3 bytes of s (s[0] the low byte) as fp32, exactly (every E4M3
// value is an fp16 value): the hardware conversion to fp16x2, then widening.
__device__ __forceinline__ float2 e4m3x2_to_f32(uint32_t s) {
    uint32_t h2;
    const uint16_t s16 = (uint16_t)s;
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(s16));
    return make_float2(h2f((uint16_t)(h2 & 0xffffu)), h2f((uint16_t)(h2 >> 16)));
}

// fp32 -> E4M3 byte: round to nearest even, finite results saturating at 448
// (the hardware's satfinite conversion); NaN and non-positive inputs give 0.
__device__ __forceinline__ uint32_t f32_to_e4m3(float x) {
    if (!(x > 0.0f)) return 0u;
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(0.0f), "f"(x));
    return (uint32_t)(r & 0xffu);
}

// E2M1 codes of lo (low nibble) and hi (high nibble): round to nearest even,
// saturating at 6.  -0 counts as +0 and a negative input that rounds to zero
// keeps its sign bit, whatever the conversion does with signed zeros.
__device__ __forceinline__ uint32_t f32x2_to_e2m1x2(float lo, float hi) {
    lo = __fadd_rn(lo, 0.0f);
    hi = __fadd_rn(hi, 0.0f);
    uint32_t r;
    asm("{\n\t.reg .b8 t;\n\tcvt.rn.satfinite.e2m1x2.f32 t, %1, %2;\n\tcvt.u32.u8 %0, t;\n\t}"
        : "=r"(r)
        : "f"(hi), "f"(lo));
    return (r & 0x77u) | (lo < 0.0f ? 0x08u : 0u) | (hi < 0.0f ? 0x80u : 0u);
}

// Doubled magnitudes (0, 1, 2, 3, 4, 6, 8, 12) of the four E2M1 codes in the
// low 16 bits of c (code i in bits 4i .. 4i+3), one byte each, in order; a
// code whose sign bit is set gives 0 (the byte permute's sign-replicating
// selectors pick a table byte whose top bit is clear).
__device__ __forceinline__ uint32_t e2m1x4_pos(uint32_t c) {
    uint32_t r;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(0x03020100u), "r"(0x0C080604u), "r"(c));
    return r;
}

// Signed doubled values (2 * e2m1) of the four codes in the low 16 bits of c.
__device__ __forceinline__ uint32_t e2m1x4_signed(uint32_t c) {
    return __vsub4(e2m1x4_pos(c), e2m1x4_pos(c ^ 0x8888u));
}

// Quantise one 32-value block held one value per lane (lane i = element i)
// into an NVFP4 block at dst (2-byte aligned) under global scale g: per
// 16-lane half s = e4m3(amax / 6 / g), code = e2m1(x / (e4m3(s) * g)), zero
// codes for a zero scale.
__device__ __forceinline__ void warp_quant_nvfp4(float v, float g, uint8_t* dst) {
    const int lane = threadIdx.x & 31;
    float amax = fabsf(v);
#pragma unroll
    for (int o = 8; o >= 1; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    const uint32_t s = f32_to_e4m3(__fdiv_rn(__fdiv_rn(amax, 6.0f), g));
    const float den = __fmul_rn(e4m3x2_to_f32(s).x, g);
    const float x = den != 0.0f ? __fdiv_rn(v, den) : 0.0f;
    const float xo = __shfl_down_sync(0xffffffffu, x, 1);     // value 2j+1, on lane 2j
    const uint32_t byte = f32x2_to_e2m1x2(x, xo);             // code byte j, on lane 2j
    const uint32_t b2 = __shfl_down_sync(0xffffffffu, byte, 2);
    const uint32_t s1 = __shfl_sync(0xffffffffu, s, 16);
    if ((lane & 3) == 0)
        reinterpret_cast<uint16_t*>(dst + 2)[lane >> 2] = (uint16_t)((byte & 0xffu) | ((b2 & 0xffu) << 8));
    if (lane == 0) *reinterpret_cast<uint16_t*>(dst) = (uint16_t)(s | (s1 << 8));
}

// ---- bulk copies and mbarriers (sm_90+ PTX, used on sm_100a) ------------------

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
    return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_barrier_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void fence_proxy_async() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Orders this thread's generic-proxy global writes before later async-proxy
// (bulk copy) reads of them, also by other CTAs after a release/acquire.
__device__ __forceinline__ void fence_proxy_async_global() {
    asm volatile("fence.proxy.async.global;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)), "r"(bytes)
                 : "memory");
}

// Global -> shared bulk copy completing on an mbarrier's transaction count.
// dst, src 16-byte aligned, bytes a multiple of 16.  No multicast.
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_addr(dst)),
        "l"(src), "r"(bytes), "r"(smem_addr(bar))
        : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_addr(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

__device__ __forceinline__ uint64_t global_timer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// try_wait with a suspend-time hint: the thread sleeps until the phase
// completes or about hint_ns pass, instead of spinning on issue slots.
__device__ __forceinline__ bool mbar_try_wait_hint(uint64_t* bar, uint32_t parity, uint32_t hint_ns) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_addr(bar)), "r"(parity), "r"(hint_ns)
        : "memory");
    return ok != 0;
}

// Bounded wait for an mbarrier phase: gives up after budget_ns of wall time
// (and a hard cap on polls), records kErrTimeout in *err and returns false.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity, int* err,
                                                  uint64_t budget_ns) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_timer_ns();
    for (uint32_t i = 0; i < (1u << 26); ++i) {
        if (mbar_try_wait_hint(bar, parity, 20000u)) return true;
        if ((i & 15) == 15 && global_timer_ns() - t0 > budget_ns) break;
    }
    if (err) atomicExch(err, kErrTimeout);
    return false;
}

// Programmatic dependent launch: wait for the upstream grid's memory, and let
// the downstream grid start launching.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// L2 prefetch of a global range (16-byte aligned, size a multiple of 16).
__device__ __forceinline__ void bulk_prefetch_l2(const void* src, uint32_t bytes) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
}

// 16-byte asynchronous global -> shared copy (both addresses 16-byte aligned),
// in commit groups that cp_async_wait<N> retires down to N pending.
__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_addr(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

__device__ __forceinline__ uint4 lds128(const void* p) {
    return *reinterpret_cast<const uint4*>(p);
}

}  // namespace elq
