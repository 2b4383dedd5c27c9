/*
 * elq_oracle.c -- scalar CPU oracle of the quantized latent-MoE expert layer.
 *
 * TEST INFRASTRUCTURE ONLY (tests, the package smoke check and the benchmark's
 * CPU-baseline leg).  Plain loops, one element at a time, in the order the
 * definitions state.  Build flags: -O2 -ffp-contract=off -fno-fast-math, so
 * that every fp32 operation below is one IEEE round-to-nearest operation and
 * fmaf is the only fused one.  Readings R1-R14 are listed in elq_oracle.h.
 */
#include "elq_oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------------ */
/* formats                                                                  */

int orc_block_bytes(int fmt)
{
    switch (fmt) {
    case ORC_Q4_0: return 18;
    case ORC_Q8_0: return 34;
    case ORC_Q8_1: return 36;
    case ORC_NVFP4: return 18;
    case ORC_Q5_1: return 24;
    default: return 0;
    }
}

/* bytes of a row of k values (K-quants: super-blocks of 256) */
int64_t orc_row_bytes(int fmt, int64_t k)
{
    if (fmt == ORC_Q3_K) return (k / 256) * 110;
    if (fmt == ORC_Q4_K) return (k / 256) * 144;
    if (fmt == ORC_Q5_K) return (k / 256) * 176;
    return (k / 32) * (int64_t)orc_block_bytes(fmt);
}

int64_t orc_matrix_bytes(int fmt, int64_t rows, int64_t k)
{
    return rows * orc_row_bytes(fmt, k);
}

/* fp32 -> fp16, round to nearest, ties to even (the loader's narrowing rule in
 * "Q8 0 support", CONV1D).  Written from the IEEE 754 binary16 definition:
 * 1 sign bit, 5 exponent bits (bias 15), 10 fraction bits, subnormals below
 * 2^-14 with quantum 2^-24. */
uint16_t orc_f32_to_f16(float f)
{
    uint32_t x;
    memcpy(&x, &f, 4);
    uint16_t sign = (uint16_t)((x >> 16) & 0x8000u);
    uint32_t bexp = (x >> 23) & 0xFFu;
    uint32_t frac = x & 0x7FFFFFu;
    if (bexp == 0xFFu)                       /* inf or nan */
        return (uint16_t)(sign | 0x7C00u | (frac ? 0x200u : 0u));
    if (bexp == 0u)                          /* fp32 zero/subnormal < 2^-126 */
        return sign;
    int e = (int)bexp - 127;                 /* value = m * 2^(e-23) */
    uint32_t m = frac | 0x800000u;           /* 24-bit significand */
    if (e < -25)
        return sign;                         /* below half the smallest subnormal */
    int shift = (e >= -14) ? 13 : (-1 - e);  /* bits dropped from m */
    uint32_t q = m >> shift;
    uint32_t rem = m & ((1u << shift) - 1u);
    uint32_t half = 1u << (shift - 1);
    if (rem > half || (rem == half && (q & 1u)))
        q += 1u;
    if (e >= -14) {                          /* normal result */
        if (q == 0x800u) { q >>= 1; e += 1; }
        int he = e + 15;
        if (he >= 31)
            return (uint16_t)(sign | 0x7C00u);
        return (uint16_t)(sign | ((uint32_t)he << 10) | (q & 0x3FFu));
    }
    /* subnormal result; q == 0x400 is the smallest normal, encoded the same */
    return (uint16_t)(sign | q);
}

float orc_f16_to_f32(uint16_t h)
{
    uint32_t sign = (uint32_t)(h & 0x8000u) << 16;
    uint32_t he = (h >> 10) & 0x1Fu;
    uint32_t hf = h & 0x3FFu;
    float v;
    if (he == 0u) {
        v = (float)hf * 5.9604644775390625e-08f;   /* hf * 2^-24, exact */
    } else if (he == 31u) {
        uint32_t bits = 0x7F800000u | (hf << 13);
        memcpy(&v, &bits, 4);
    } else {
        uint32_t bits = ((he - 15u + 127u) << 23) | (hf << 13);
        memcpy(&v, &bits, 4);
    }
    uint32_t out;
    memcpy(&out, &v, 4);
    out |= sign;
    memcpy(&v, &out, 4);
    return v;
}

float orc_bf16_to_f32(uint16_t b)
{
    uint32_t bits = (uint32_t)b << 16;
    float v;
    memcpy(&v, &bits, 4);
    return v;
}

/* R12: exp(x) by Cody and Waite's argument reduction (x = n ln2 + r with
 * |r| <= ln2/2, ln2 carried as a high and a low fp32 part), the Taylor series
 * of e^r to degree 7 evaluated by Horner's rule with fmaf, and an exact scaling
 * by 2^n (two steps where the result is subnormal). */
float orc_expf(float x)
{
    if (x != x) return x;
    if (x > 88.72283935546875f) return INFINITY;          /* > ln(FLT_MAX) */
    if (x < -103.972076416015625f) return 0.0f;           /* < ln(2^-150) */
    const float log2e = 1.44269502162933349609375f;       /* fp32(1/ln 2) */
    const float ln2_hi = 0.693145751953125f;              /* ln2, 16 significant bits */
    const float ln2_lo = 1.428606765330187045037746429443359375e-06f; /* fp32(ln2 - ln2_hi) */
    float n = rintf(x * log2e);
    float r = fmaf(-n, ln2_hi, x);
    r = fmaf(-n, ln2_lo, r);
    /* 1/k! for k = 7 .. 2, each rounded to fp32 */
    float p = 1.98412701138295233249664306640625e-04f;     /* 1/5040 */
    p = fmaf(p, r, 1.388888922519981861114501953125e-03f); /* 1/720 */
    p = fmaf(p, r, 8.333333767950534820556640625e-03f);    /* 1/120 */
    p = fmaf(p, r, 4.16666679084300994873046875e-02f);     /* 1/24 */
    p = fmaf(p, r, 1.6666667163372039794921875e-01f);      /* 1/6 */
    p = fmaf(p, r, 0.5f);
    p = fmaf(p, r, 1.0f);
    p = fmaf(p, r, 1.0f);
    int ni = (int)n;
    if (ni > 127) {                                        /* p * 2^127 * 2^(n-127) */
        uint32_t b1 = 254u << 23, b2 = (uint32_t)(ni - 127 + 127) << 23;
        float s1, s2;
        memcpy(&s1, &b1, 4);
        memcpy(&s2, &b2, 4);
        return (p * s1) * s2;
    }
    if (ni < -125) {                                       /* p * 2^(n+100) * 2^-100 */
        uint32_t b1 = (uint32_t)(ni + 100 + 127) << 23, b2 = (uint32_t)(-100 + 127) << 23;
        float s1, s2;
        memcpy(&s1, &b1, 4);
        memcpy(&s2, &b2, 4);
        return (p * s1) * s2;
    }
    uint32_t b = (uint32_t)(ni + 127) << 23;
    float s;
    memcpy(&s, &b, 4);
    return p * s;
}

/* R13: silu(g) = g / (1 + exp(-g)) */
float orc_silu(float g)
{
    float e = orc_expf(-g);
    float den = 1.0f + e;
    return g / den;
}

/* ------------------------------------------------------------------------ */
/* quantisers                                                               */

static void put16(uint8_t* p, uint16_t v) { p[0] = (uint8_t)(v & 0xFF); p[1] = (uint8_t)(v >> 8); }
static uint16_t get16(const uint8_t* p) { return (uint16_t)(p[0] | (p[1] << 8)); }

/* R1-R3: q = clamp(round(x / d), -127, 127) with d = amax / 127 (fp32) */
static void quant_sym8(const float* xb, float* d_out, int8_t* q, int* sumq)
{
    float amax = 0.0f;
    for (int i = 0; i < 32; ++i) {
        float a = fabsf(xb[i]);
        if (a > amax) amax = a;
    }
    float d = amax / 127.0f;
    int s = 0;
    for (int i = 0; i < 32; ++i) {
        int v = 0;
        if (d != 0.0f) {
            float r = roundf(xb[i] / d);
            if (r > 127.0f) r = 127.0f;
            if (r < -127.0f) r = -127.0f;
            v = (int)r;
        }
        q[i] = (int8_t)v;
        s += v;
    }
    *d_out = d;
    *sumq = s;
}

/* Q8_1 activation block: fp16 d, fp16 s = d * sum(q) (R4), int8 q[32] */
void orc_quantize_q8_1(const float* x, int64_t n, uint8_t* out)
{
    for (int64_t b = 0; b < n / 32; ++b) {
        float d;
        int8_t q[32];
        int sumq;
        quant_sym8(x + 32 * b, &d, q, &sumq);
        uint8_t* o = out + 36 * b;
        put16(o, orc_f32_to_f16(d));
        put16(o + 2, orc_f32_to_f16(d * (float)sumq));
        memcpy(o + 4, q, 32);
    }
}

/* Q8_0 weight block: fp16 d, int8 q[32] */
void orc_quantize_q8_0(const float* x, int64_t n, uint8_t* out)
{
    for (int64_t b = 0; b < n / 32; ++b) {
        float d;
        int8_t q[32];
        int sumq;
        quant_sym8(x + 32 * b, &d, q, &sumq);
        uint8_t* o = out + 34 * b;
        put16(o, orc_f32_to_f16(d));
        memcpy(o + 2, q, 32);
    }
}

/* Q4_0 weight block (R5, R6): fp16 d = m / -8, nibbles q in [0, 15] */
void orc_quantize_q4_0(const float* x, int64_t n, uint8_t* out)
{
    for (int64_t b = 0; b < n / 32; ++b) {
        const float* xb = x + 32 * b;
        float amax = 0.0f, m = 0.0f;
        for (int i = 0; i < 32; ++i) {
            float a = fabsf(xb[i]);
            if (a > amax) { amax = a; m = xb[i]; }
        }
        float d = m / -8.0f;
        uint8_t q[32];
        for (int i = 0; i < 32; ++i) {
            int v = 8;
            if (d != 0.0f) {
                float r = roundf(xb[i] / d) + 8.0f;
                if (r < 0.0f) r = 0.0f;
                if (r > 15.0f) r = 15.0f;
                v = (int)r;
            }
            q[i] = (uint8_t)v;
        }
        uint8_t* o = out + 18 * b;
        put16(o, orc_f32_to_f16(d));
        for (int j = 0; j < 16; ++j)
            o[2 + j] = (uint8_t)(q[j] | (q[j + 16] << 4));
    }
}

void orc_dequantize(int fmt, const uint8_t* blocks, int64_t n, double* out)
{
    for (int64_t b = 0; b < n / 32; ++b) {
        double* ob = out + 32 * b;
        if (fmt == ORC_Q8_0 || fmt == ORC_Q8_1) {
            const uint8_t* p = blocks + (int64_t)orc_block_bytes(fmt) * b;
            double d = (double)orc_f16_to_f32(get16(p));
            const int8_t* q = (const int8_t*)(p + (fmt == ORC_Q8_0 ? 2 : 4));
            for (int i = 0; i < 32; ++i) ob[i] = d * (double)q[i];
        } else if (fmt == ORC_Q4_0) {
            const uint8_t* p = blocks + 18 * b;
            double d = (double)orc_f16_to_f32(get16(p));
            for (int j = 0; j < 16; ++j) {
                ob[j] = d * (double)((p[2 + j] & 0x0F) - 8);
                ob[j + 16] = d * (double)((p[2 + j] >> 4) - 8);
            }
        }
    }
}

/* ------------------------------------------------------------------------ */
/* Q5_1 and the K-quants Q4_K, Q5_K ("Q8 0 support - Pull Request #255",    */
/* follow-up commit "per-role format lists": the Q4_K / Q5_K / Q5_1 expert  */
/* dots, Q5_1's min term on the sum of the quantised activations).  The     */
/* block layouts are the GGUF formats the pages name (R22-R24 in            */
/* elq_oracle.h).                                                            */

/* Q5_1, 24-byte blocks of 32: fp16 d, fp16 m, uint32 qh, 16 code bytes.
 * Value i: code q = (low nibble of byte i for i < 16, high nibble of byte
 * i - 16 otherwise) + 16 * bit i of qh; x = d * q + m. */
static int q51_code(const uint8_t* b, int i)
{
    uint32_t qh = (uint32_t)b[4] | ((uint32_t)b[5] << 8) | ((uint32_t)b[6] << 16) | ((uint32_t)b[7] << 24);
    int lo = i < 16 ? (b[8 + i] & 0x0F) : (b[8 + i - 16] >> 4);
    return lo | (int)(((qh >> i) & 1u) << 4);
}

/* K-quant super-block (256 values, 8 sub-blocks of 32): fp16 d, fp16 dmin,
 * 12 bytes of 6-bit sub-block scales and mins, [Q5_K: 32 bytes qh], 128
 * code bytes.  Sub-block j < 4: scale = byte j & 63, min = byte j+4 & 63;
 * j >= 4: scale = (byte j+4 & 15) | (byte j-4 >> 6) << 4, min = (byte j+4 >>
 * 4) | (byte j >> 6) << 4. */
static void kq_scale_min(const uint8_t* sc, int j, int* scale, int* min)
{
    if (j < 4) {
        *scale = sc[j] & 63;
        *min = sc[j + 4] & 63;
    } else {
        *scale = (sc[j + 4] & 15) | ((sc[j - 4] >> 6) << 4);
        *min = (sc[j + 4] >> 4) | ((sc[j] >> 6) << 4);
    }
}

/* value i (0..255) of a super-block: code bytes 32p .. 32p+31 hold sub-block
 * 2p (low nibbles) and 2p+1 (high nibbles), value l of each at byte 32p + l;
 * Q5_K adds 16 * bit j of qh[l] for value l of sub-block j. */
static int kq_code(int fmt, const uint8_t* b, int i)
{
    int j = i / 32, l = i % 32;
    const uint8_t* qs = b + (fmt == ORC_Q5_K ? 48 : 16);
    int q = (j & 1) ? (qs[32 * (j / 2) + l] >> 4) : (qs[32 * (j / 2) + l] & 0x0F);
    if (fmt == ORC_Q5_K) q |= ((b[16 + l] >> j) & 1) << 4;
    return q;
}

int orc_is_kquant(int fmt) { return fmt == ORC_Q3_K || fmt == ORC_Q4_K || fmt == ORC_Q5_K; }

/* Q3_K super-block (110 bytes, 256 values): hmask[32], qs[64], 12 bytes of
 * 16 packed 6-bit scales, fp16 d last.  Value i = 128 n + 32 j + l (half n,
 * bit pair j, l < 32): low two bits (qs[32 n + l] >> 2 j) & 3, high bit =
 * bit (4 n + j) of hmask[l]; q = low - (high ? 0 : 4) in -4 .. 3.  Scale of
 * the 16-value sub-block s = i / 16: four low bits from byte s (s < 8, low
 * nibble) or byte s - 8 (high nibble), two high bits (byte 8 + s % 4 >> 2 (s /
 * 4)) & 3; scale = that 6-bit value - 32.  x = d * scale * q. */
static int q3k_code(const uint8_t* b, int i)
{
    int n = i / 128, j = (i % 128) / 32, l = i % 32;
    int low = (b[32 + 32 * n + l] >> (2 * j)) & 3;
    int high = (b[l] >> (4 * n + j)) & 1;
    return low - (high ? 0 : 4);
}

static int q3k_scale(const uint8_t* b, int s)
{
    const uint8_t* sc = b + 96;
    int low4 = s < 8 ? (sc[s] & 15) : (sc[s - 8] >> 4);
    int hi2 = (sc[8 + s % 4] >> (2 * (s / 4))) & 3;
    return (low4 | (hi2 << 4)) - 32;
}

/* x of value i of a row (fp64) */
static double ext_value(int fmt, const uint8_t* row, int64_t i)
{
    if (fmt == ORC_Q3_K) {
        const uint8_t* b = row + 110 * (i / 256);
        int v = (int)(i % 256);
        return (double)orc_f16_to_f32(get16(b + 108)) * q3k_scale(b, v / 16) * q3k_code(b, v);
    }
    if (fmt == ORC_Q5_1) {
        const uint8_t* b = row + 24 * (i / 32);
        return (double)orc_f16_to_f32(get16(b)) * (double)q51_code(b, (int)(i % 32)) +
               (double)orc_f16_to_f32(get16(b + 2));
    }
    const uint8_t* b = row + (fmt == ORC_Q5_K ? 176 : 144) * (i / 256);
    int sc, mn;
    kq_scale_min(b + 4, (int)(i % 256) / 32, &sc, &mn);
    return (double)orc_f16_to_f32(get16(b)) * sc * kq_code(fmt, b, (int)(i % 256)) -
           (double)orc_f16_to_f32(get16(b + 2)) * mn;
}

void orc_dequantize_ext(int fmt, const uint8_t* W, int N, int K, double* out)
{
    int64_t rb = orc_row_bytes(fmt, K);
    for (int n = 0; n < N; ++n)
        for (int64_t i = 0; i < K; ++i) out[(int64_t)n * K + i] = ext_value(fmt, W + n * rb, i);
}

/* R22-R24: per 32-value block kb of a row against Q8_1 block kb: isum = sum
 * q_w q_a, sumq = sum q_a (exact integers); sd = fp32 scale product, sm = the
 * min product; part = fmaf((float)isum, sd, part) then part = fmaf((float)sumq,
 * sm, part), blocks in order within chunks of 8 (= one K-quant super-block),
 * acc = acc + part over chunks.  Q5_1: sd = d_w * d_a, sm = m_w * d_a.
 * K-quants: sd = (d * scale_j) * d_a, sm = -((dmin * min_j) * d_a). */
void orc_block_ext(int fmt, const uint8_t* row, int kb, const uint8_t* a, int32_t* isum, int32_t* sumq,
                   float* sd, float* sm)
{
    const int8_t* qa = (const int8_t*)(a + 4);
    float da = orc_f16_to_f32(get16(a));
    int32_t s = 0, z = 0;
    if (fmt == ORC_Q3_K) {
        /* two 16-value sub-blocks: (isum, sd) of the first as (isum, sd),
         * of the second as (sumq, sm), so that the R24 chain takes them in
         * order (R25) */
        const uint8_t* b = row + 110 * (kb / 8);
        int j = kb % 8;
        int32_t s0 = 0, s1 = 0;
        for (int i = 0; i < 16; ++i) s0 += q3k_code(b, 32 * j + i) * (int32_t)qa[i];
        for (int i = 16; i < 32; ++i) s1 += q3k_code(b, 32 * j + i) * (int32_t)qa[i];
        float d = orc_f16_to_f32(get16(b + 108));
        *isum = s0;
        *sumq = s1;
        *sd = (d * (float)q3k_scale(b, 2 * j)) * da;
        *sm = (d * (float)q3k_scale(b, 2 * j + 1)) * da;
        return;
    }
    if (fmt == ORC_Q5_1) {
        const uint8_t* b = row + 24 * kb;
        for (int i = 0; i < 32; ++i) {
            s += q51_code(b, i) * (int32_t)qa[i];
            z += qa[i];
        }
        *sd = orc_f16_to_f32(get16(b)) * da;
        *sm = orc_f16_to_f32(get16(b + 2)) * da;
    } else {
        const uint8_t* b = row + (fmt == ORC_Q5_K ? 176 : 144) * (kb / 8);
        int j = kb % 8, sc, mn;
        kq_scale_min(b + 4, j, &sc, &mn);
        for (int i = 0; i < 32; ++i) {
            s += kq_code(fmt, b, 32 * j + i) * (int32_t)qa[i];
            z += qa[i];
        }
        float dsc = orc_f16_to_f32(get16(b)) * (float)sc;
        float dmn = orc_f16_to_f32(get16(b + 2)) * (float)mn;
        *sd = dsc * da;
        *sm = -(dmn * da);
    }
    *isum = s;
    *sumq = z;
}

void orc_qmatmul_ext(int fmt, const uint8_t* W, int N, int K, const uint8_t* Xq, int T, float* Y)
{
    int nb = K / 32;
    int64_t rb = orc_row_bytes(fmt, K);
    for (int t = 0; t < T; ++t) {
        const uint8_t* xr = Xq + (int64_t)t * nb * 36;
        for (int n = 0; n < N; ++n) {
            const uint8_t* wr = W + (int64_t)n * rb;
            float acc = 0.0f;
            for (int c = 0; c < nb; c += 8) {
                float part = 0.0f;
                for (int kb = c; kb < c + 8 && kb < nb; ++kb) {
                    int32_t isum, sumq;
                    float sd, sm;
                    orc_block_ext(fmt, wr, kb, xr + (int64_t)kb * 36, &isum, &sumq, &sd, &sm);
                    part = fmaf((float)isum, sd, part);
                    part = fmaf((float)sumq, sm, part);
                }
                acc = acc + part;
            }
            Y[(int64_t)t * N + n] = acc;
        }
    }
}

/* ------------------------------------------------------------------------ */
/* block dots ("Q8 0 support", GPU EXPERT KERNELS; R7 for Q4_0)              */

int32_t orc_block_isum(int wfmt, const uint8_t* w, const uint8_t* a)
{
    const int8_t* qa = (const int8_t*)(a + 4);
    int32_t s = 0;
    if (wfmt == ORC_Q8_0) {
        const int8_t* qw = (const int8_t*)(w + 2);
        for (int i = 0; i < 32; ++i) s += (int32_t)qw[i] * (int32_t)qa[i];
    } else if (wfmt == ORC_Q4_0) {
        for (int j = 0; j < 16; ++j) {
            int lo = (w[2 + j] & 0x0F) - 8;
            int hi = (w[2 + j] >> 4) - 8;
            s += lo * (int32_t)qa[j] + hi * (int32_t)qa[j + 16];
        }
    }
    return s;
}

float orc_block_term(int wfmt, const uint8_t* w, const uint8_t* a)
{
    float sc = orc_f16_to_f32(get16(w)) * orc_f16_to_f32(get16(a));
    return (float)orc_block_isum(wfmt, w, a) * sc;
}

/* R8 */
void orc_qmatmul(int wfmt, const uint8_t* W, int N, int K,
                 const uint8_t* Xq, int T, float* Y)
{
    int nb = K / 32;
    int wb = orc_block_bytes(wfmt);
    for (int t = 0; t < T; ++t) {
        const uint8_t* xr = Xq + (int64_t)t * nb * 36;
        for (int n = 0; n < N; ++n) {
            const uint8_t* wr = W + (int64_t)n * nb * wb;
            float acc = 0.0f;
            for (int c = 0; c < nb; c += 8) {
                float part = 0.0f;
                for (int kb = c; kb < c + 8 && kb < nb; ++kb) {
                    const uint8_t* wk = wr + (int64_t)kb * wb;
                    const uint8_t* ak = xr + (int64_t)kb * 36;
                    int32_t isum = orc_block_isum(wfmt, wk, ak);
                    float sc = orc_f16_to_f32(get16(wk)) * orc_f16_to_f32(get16(ak));
                    part = fmaf((float)isum, sc, part);
                }
                acc = acc + part;
            }
            Y[(int64_t)t * N + n] = acc;
        }
    }
}

/* ------------------------------------------------------------------------ */
/* NVFP4 (page "edge0-strata", section "Changes from upstream Strata": the  */
/* Edge0 latent experts are NVFP4).  The pages name the format only; the    */
/* readings R19-R21 in elq_oracle.h fix the rest.                           */

/* E2M1 magnitudes by code 0..7 (sign in bit 3). */
static const float kE2M1[8] = {0.0f, 0.5f, 1.0f, 1.5f, 2.0f, 3.0f, 4.0f, 6.0f};

/* R19: fp32 -> E2M1, round to nearest with ties to the even code, finite
 * values saturate at 6, the sign kept (a negative value rounding to 0 gives
 * code 8, -0).  Written as the intervals of the grid's midpoints. */
uint8_t orc_f32_to_e2m1(float v)
{
    uint8_t sign = (v < 0.0f) ? 8u : 0u;
    float a = fabsf(v);
    uint8_t c;
    if (!(a > 0.25f)) c = 0;           /* also NaN */
    else if (a < 0.75f) c = 1;
    else if (a <= 1.25f) c = 2;
    else if (a < 1.75f) c = 3;
    else if (a <= 2.5f) c = 4;
    else if (a < 3.5f) c = 5;
    else if (a <= 5.0f) c = 6;
    else c = 7;
    return (uint8_t)(sign | c);
}

float orc_e2m1_to_f32(uint8_t c)
{
    float m = kE2M1[c & 7u];
    return (c & 8u) ? -m : m;
}

/* R19: unsigned fp32 -> E4M3 (1 sign bit, 4 exponent bits with bias 7, 3
 * fraction bits; no infinity, 0x7F is NaN), round to nearest even, finite
 * values saturate at 448 (0x7E); NaN and non-positive values give 0.
 * Written from the format's definition: normals 2^(e-7) * (1 + f/8) for
 * e = 1..15, subnormals f * 2^-9. */
uint8_t orc_f32_to_e4m3(float v)
{
    if (!(v > 0.0f)) return 0;
    if (v >= 448.0f) return 0x7E;
    uint32_t x;
    memcpy(&x, &v, 4);
    int e = (int)((x >> 23) & 0xFFu) - 127;       /* v = m * 2^(e-23), m 24 bits */
    uint32_t m = (x & 0x7FFFFFu) | (((x >> 23) & 0xFFu) ? 0x800000u : 0u);
    if (((x >> 23) & 0xFFu) == 0u) e = -126;       /* fp32 subnormal (underflows to 0 below) */
    /* the quantum is 2^-9 below 2^-6 and 2^(e-3) above: drop bits of m */
    int shift = (e >= -6) ? 20 : 20 + (-6 - e);    /* fraction bits kept: 3, fewer when subnormal */
    if (shift > 24) return 0;                      /* below half the smallest subnormal */
    uint32_t q = m >> shift;
    uint32_t rem = m & ((1u << shift) - 1u);
    uint32_t half = 1u << (shift - 1);
    if (rem > half || (rem == half && (q & 1u))) q += 1u;
    /* q is the significand on the grid: 8..16 for normals (16 = next exponent),
     * 0..8 for subnormals (8 = the smallest normal) */
    int ee;
    uint32_t f;
    if (e >= -6) {
        ee = e + 7;
        if (q == 16u) { ee += 1; q = 8u; }
        f = q - 8u;
    } else {
        if (q == 8u) { ee = 1; f = 0u; }
        else { ee = 0; f = q; }
    }
    if (ee > 15 || (ee == 15 && f == 7u)) return 0x7E;   /* saturate */
    return (uint8_t)((ee << 3) | f);
}

float orc_e4m3_to_f32(uint8_t b)
{
    int e = (b >> 3) & 15, f = b & 7;
    if (e == 15 && f == 7) return NAN;
    if (e == 0) return ldexpf((float)f, -9);
    return ldexpf(1.0f + (float)f / 8.0f, e - 7);
}

/* R20: global scale of a weight matrix: amax / (6 * 448) (fp32 divide), 1 for
 * an all-zero matrix.  Activations take 1. */
float orc_nvfp4_global(const float* x, int64_t n)
{
    float amax = 0.0f;
    for (int64_t i = 0; i < n; ++i) {
        float a = fabsf(x[i]);
        if (a > amax) amax = a;
    }
    return amax > 0.0f ? amax / 2688.0f : 1.0f;
}

/* R20: blocks of 32 values (two 16-value micro-blocks), 18 bytes each: the
 * two E4M3 scales, then 16 bytes of codes, value 2j in the low nibble of
 * byte j and value 2j+1 in its high nibble.  Micro-block scale s =
 * e4m3(amax / 6 / g) (fp32 divides), code = e2m1(x / (dec(s) * g)) (fp32
 * product and divide); a zero scale gives zero codes. */
void orc_quantize_nvfp4(const float* x, int64_t n, float g, uint8_t* out)
{
    for (int64_t b = 0; b < n / 32; ++b) {
        const float* xb = x + 32 * b;
        uint8_t* o = out + 18 * b;
        uint8_t codes[32];
        for (int mb = 0; mb < 2; ++mb) {
            float amax = 0.0f;
            for (int i = 0; i < 16; ++i) {
                float a = fabsf(xb[16 * mb + i]);
                if (a > amax) amax = a;
            }
            uint8_t sb = orc_f32_to_e4m3((amax / 6.0f) / g);
            o[mb] = sb;
            float ds = orc_e4m3_to_f32(sb);
            float den = ds * g;
            for (int i = 0; i < 16; ++i)
                codes[16 * mb + i] = (den != 0.0f) ? orc_f32_to_e2m1(xb[16 * mb + i] / den) : 0u;
        }
        for (int j = 0; j < 16; ++j)
            o[2 + j] = (uint8_t)(codes[2 * j] | (codes[2 * j + 1] << 4));
    }
}

/* value i of an NVFP4 block, as the doubled integer 2 * e2m1 (exact) */
static int nv_code2(const uint8_t* blk, int i)
{
    uint8_t c = (uint8_t)((blk[2 + i / 2] >> ((i & 1) * 4)) & 0x0Fu);
    static const int mag2[8] = {0, 1, 2, 3, 4, 6, 8, 12};
    return (c & 8u) ? -mag2[c & 7u] : mag2[c & 7u];
}

void orc_dequantize_nvfp4(const uint8_t* blocks, int64_t n, float g, double* out)
{
    for (int64_t b = 0; b < n / 32; ++b) {
        const uint8_t* p = blocks + 18 * b;
        for (int i = 0; i < 32; ++i)
            out[32 * b + i] = (double)nv_code2(p, i) * 0.5 * (double)orc_e4m3_to_f32(p[i / 16]) * (double)g;
    }
}

/* R21: Y[t][n] = row n of W (NVFP4, global gw) . X[t] (NVFP4, global ga).
 * Per 16-value micro-block m: isum = sum (2 w)(2 a) exact, sc = dec(sw) *
 * dec(sa); part = fmaf((float)isum, sc, part) over the micro-blocks of a
 * chunk of 8 blocks (16 micro-blocks) in order from 0; acc = acc + part over
 * the chunks in order from 0; y = acc * ((gw * ga) * 0.25). */
void orc_qmatmul_nvfp4(const uint8_t* W, float gw, int N, int K, const uint8_t* X, float ga,
                       int T, float* Y)
{
    int nb = K / 32;
    float gq = (gw * ga) * 0.25f;
    for (int t = 0; t < T; ++t) {
        const uint8_t* xr = X + (int64_t)t * nb * 18;
        for (int n = 0; n < N; ++n) {
            const uint8_t* wr = W + (int64_t)n * nb * 18;
            float acc = 0.0f;
            for (int c = 0; c < nb; c += 8) {
                float part = 0.0f;
                for (int kb = c; kb < c + 8 && kb < nb; ++kb)
                    for (int mb = 0; mb < 2; ++mb) {
                        const uint8_t* wk = wr + (int64_t)kb * 18;
                        const uint8_t* ak = xr + (int64_t)kb * 18;
                        int32_t isum = 0;
                        for (int i = 16 * mb; i < 16 * mb + 16; ++i) isum += nv_code2(wk, i) * nv_code2(ak, i);
                        float sc = orc_e4m3_to_f32(wk[mb]) * orc_e4m3_to_f32(ak[mb]);
                        part = fmaf((float)isum, sc, part);
                    }
                acc = acc + part;
            }
            Y[(int64_t)t * N + n] = acc * gq;
        }
    }
}

/* ------------------------------------------------------------------------ */
/* router (R9-R11)                                                          */

void orc_router_topk(const float* z, const float* Wr, const float* bias,
                     int T, int L, int E, int k,
                     int32_t* idx, float* w, float* logits)
{
    float* lg = (float*)malloc(sizeof(float) * (size_t)E);
    char* taken = (char*)malloc((size_t)E);
    for (int t = 0; t < T; ++t) {
        const float* zt = z + (int64_t)t * L;
        for (int e = 0; e < E; ++e) {
            const float* we = Wr + (int64_t)e * L;
            float part[32];
            for (int j = 0; j < 32; ++j) {
                float p = 0.0f;
                for (int l = j; l < L; l += 32) p = fmaf(zt[l], we[l], p);
                part[j] = p;
            }
            for (int off = 16; off >= 1; off /= 2) {
                float nxt[32];
                for (int j = 0; j < 32; ++j) nxt[j] = part[j] + part[j ^ off];
                memcpy(part, nxt, sizeof(part));
            }
            float v = part[0];
            if (bias) v = v + bias[e];
            lg[e] = v;
            if (logits) logits[(int64_t)t * E + e] = v;
        }
        /* R18: a NaN logit ranks as -infinity (in the selection and in the
         * softmax), so the k chosen ids are always valid and distinct */
        for (int e = 0; e < E; ++e)
            if (isnan(lg[e])) lg[e] = -INFINITY;
        memset(taken, 0, (size_t)E);
        for (int j = 0; j < k; ++j) {          /* k largest, lower id on ties */
            int best = -1;
            for (int e = 0; e < E; ++e) {
                if (taken[e]) continue;
                if (best < 0 || lg[e] > lg[best]) best = e;
            }
            taken[best] = 1;
            idx[(int64_t)t * k + j] = best;
        }
        float l0 = lg[idx[(int64_t)t * k]];
        float ex[64];
        float sum = 0.0f;
        for (int j = 0; j < k; ++j) {
            ex[j] = orc_expf(lg[idx[(int64_t)t * k + j]] - l0);
            sum = sum + ex[j];
        }
        for (int j = 0; j < k; ++j) w[(int64_t)t * k + j] = ex[j] / sum;
    }
    free(lg);
    free(taken);
}

/* ------------------------------------------------------------------------ */
/* bucketing                                                                */

void orc_bucket(const int32_t* idx, int T, int k, int E,
                int32_t* counts, int32_t* offsets, int32_t* perm, int32_t* pos)
{
    int P = T * k;
    for (int e = 0; e < E; ++e) counts[e] = 0;
    for (int p = 0; p < P; ++p) counts[idx[p]] += 1;
    offsets[0] = 0;
    for (int e = 0; e < E; ++e) offsets[e + 1] = offsets[e] + counts[e];
    int n = 0;
    for (int e = 0; e < E; ++e)
        for (int p = 0; p < P; ++p)
            if (idx[p] == e) { perm[n] = p; pos[p] = n; ++n; }
}

/* ------------------------------------------------------------------------ */
/* the layer                                                                */

static int check_layer(const orc_layer* ly)
{
    if (ly->H % 32 || ly->L % 32 || ly->I % 32 || ly->E < 1 || ly->k < 1 ||
        ly->k > ly->E || ly->k > 64)
        return -2;
    if (!orc_row_bytes(ly->du_fmt, 256) || !orc_row_bytes(ly->ex_fmt, 256) ||
        ly->du_fmt == ORC_Q8_1 || ly->ex_fmt == ORC_Q8_1 || ly->du_fmt == ORC_NVFP4 ||
        ly->du_fmt == ORC_Q5_1 || orc_is_kquant(ly->du_fmt))
        return -2;
    if (orc_is_kquant(ly->ex_fmt) && (ly->L % 256 || ly->I % 256)) return -2;
    if (ly->ex_fmt == ORC_NVFP4 && (!ly->gate_g || !ly->up_g || !ly->down_g ||
                                    !(ly->act_gz > 0.0f) || !(ly->act_gh > 0.0f)))
        return -2;
    return 0;
}

int orc_route(const orc_layer* ly, const float* x, int T, int32_t* idx, float* w)
{
    if (check_layer(ly)) return -2;
    int H = ly->H, L = ly->L;
    uint8_t* xq = (uint8_t*)malloc((size_t)T * (H / 32) * 36 + 1);
    float* z = (float*)malloc(sizeof(float) * (size_t)T * L + 1);
    orc_quantize_q8_1(x, (int64_t)T * H, xq);
    orc_qmatmul(ly->du_fmt, ly->D, L, H, xq, T, z);
    orc_router_topk(z, ly->router_w, ly->router_bias, T, L, ly->E, ly->k, idx, w, NULL);
    free(xq);
    free(z);
    return 0;
}

int orc_moe_layer(const orc_layer* ly, const float* x, int T, float* y, orc_trace* tr)
{
    if (check_layer(ly)) return -2;
    int H = ly->H, L = ly->L, E = ly->E, k = ly->k, I = ly->I;
    int P = T * k;
    size_t xqb = (size_t)T * (H / 32) * 36, zqb = (size_t)T * (L / 32) * 36;
    uint8_t* xq = (uint8_t*)malloc(xqb + 1);
    float* z = (float*)malloc(sizeof(float) * (size_t)T * L + 1);
    float* lg = (float*)malloc(sizeof(float) * (size_t)T * E + 1);
    int32_t* idx = (int32_t*)malloc(sizeof(int32_t) * (size_t)P + 1);
    float* w = (float*)malloc(sizeof(float) * (size_t)P + 1);
    uint8_t* zq = (uint8_t*)malloc(zqb + 1);
    int32_t* counts = (int32_t*)malloc(sizeof(int32_t) * (size_t)E);
    int32_t* offsets = (int32_t*)malloc(sizeof(int32_t) * (size_t)(E + 1));
    int32_t* perm = (int32_t*)malloc(sizeof(int32_t) * (size_t)P + 1);
    int32_t* pos = (int32_t*)malloc(sizeof(int32_t) * (size_t)P + 1);
    float* g = (float*)malloc(sizeof(float) * (size_t)I);
    float* u = (float*)malloc(sizeof(float) * (size_t)I);
    float* h = (float*)malloc(sizeof(float) * (size_t)I);
    uint8_t* hq = (uint8_t*)malloc((size_t)(I / 32) * 36);
    float* o = (float*)malloc(sizeof(float) * (size_t)P * L + 1);
    float* ylat = (float*)malloc(sizeof(float) * (size_t)T * L + 1);
    uint8_t* ylq = (uint8_t*)malloc(zqb + 1);
    int rc = 0;

    /* a1, a2: x -> xq -> z */
    orc_quantize_q8_1(x, (int64_t)T * H, xq);
    orc_qmatmul(ly->du_fmt, ly->D, L, H, xq, T, z);
    /* a3: router on the fp32 latent */
    orc_router_topk(z, ly->router_w, ly->router_bias, T, L, E, k, idx, w, lg);
    /* a4: latent activations for the experts (NVFP4 experts: NVFP4
     * activations under the layer's static scale act_gz, R20) */
    int nv = ly->ex_fmt == ORC_NVFP4;
    int ext = ly->ex_fmt == ORC_Q5_1 || orc_is_kquant(ly->ex_fmt);
    if (nv) orc_quantize_nvfp4(z, (int64_t)T * L, ly->act_gz, zq);
    else orc_quantize_q8_1(z, (int64_t)T * L, zq);
    /* a5 */
    orc_bucket(idx, T, k, E, counts, offsets, perm, pos);
    /* a6-a8, one (token, slot) pair at a time, in pair order */
    for (int p = 0; p < P && rc == 0; ++p) {
        int t = p / k, e = idx[p];
        if (!ly->gate[e] || !ly->up[e] || !ly->down[e]) { rc = -1; break; }
        if (nv) {
            const uint8_t* zt = zq + (size_t)t * (L / 32) * 18;
            orc_qmatmul_nvfp4(ly->gate[e], ly->gate_g[e], I, L, zt, ly->act_gz, 1, g);
            orc_qmatmul_nvfp4(ly->up[e], ly->up_g[e], I, L, zt, ly->act_gz, 1, u);
            for (int i = 0; i < I; ++i) h[i] = orc_silu(g[i]) * u[i];
            orc_quantize_nvfp4(h, I, ly->act_gh, hq);
            orc_qmatmul_nvfp4(ly->down[e], ly->down_g[e], L, I, hq, ly->act_gh, 1, o + (size_t)p * L);
        } else if (ext) {
            const uint8_t* zt = zq + (size_t)t * (L / 32) * 36;
            orc_qmatmul_ext(ly->ex_fmt, ly->gate[e], I, L, zt, 1, g);
            orc_qmatmul_ext(ly->ex_fmt, ly->up[e], I, L, zt, 1, u);
            for (int i = 0; i < I; ++i) h[i] = orc_silu(g[i]) * u[i];
            orc_quantize_q8_1(h, I, hq);
            orc_qmatmul_ext(ly->ex_fmt, ly->down[e], L, I, hq, 1, o + (size_t)p * L);
        } else {
            const uint8_t* zt = zq + (size_t)t * (L / 32) * 36;
            orc_qmatmul(ly->ex_fmt, ly->gate[e], I, L, zt, 1, g);
            orc_qmatmul(ly->ex_fmt, ly->up[e], I, L, zt, 1, u);
            for (int i = 0; i < I; ++i) h[i] = orc_silu(g[i]) * u[i];
            orc_quantize_q8_1(h, I, hq);
            orc_qmatmul(ly->ex_fmt, ly->down[e], L, I, hq, 1, o + (size_t)p * L);
        }
        const size_t hqb = (size_t)(I / 32) * (nv ? 18 : 36);
        if (tr && tr->g) memcpy(tr->g + (size_t)p * I, g, sizeof(float) * (size_t)I);
        if (tr && tr->u) memcpy(tr->u + (size_t)p * I, u, sizeof(float) * (size_t)I);
        if (tr && tr->hq) memcpy(tr->hq + (size_t)p * hqb, hq, hqb);
    }
    if (rc == 0) {
        /* a9: weighted combine in rank order, then Q8_1 */
        for (int t = 0; t < T; ++t)
            for (int n = 0; n < L; ++n) {
                float acc = 0.0f;
                for (int j = 0; j < k; ++j)
                    acc = fmaf(w[t * k + j], o[(size_t)(t * k + j) * L + n], acc);
                ylat[(size_t)t * L + n] = acc;
            }
        orc_quantize_q8_1(ylat, (int64_t)T * L, ylq);
        /* a10 */
        orc_qmatmul(ly->du_fmt, ly->U, H, L, ylq, T, y);
    }
    if (tr) {
        if (tr->xq) memcpy(tr->xq, xq, xqb);
        if (tr->z) memcpy(tr->z, z, sizeof(float) * (size_t)T * L);
        if (tr->logits) memcpy(tr->logits, lg, sizeof(float) * (size_t)T * E);
        if (tr->idx) memcpy(tr->idx, idx, sizeof(int32_t) * (size_t)P);
        if (tr->w) memcpy(tr->w, w, sizeof(float) * (size_t)P);
        if (tr->zq) memcpy(tr->zq, zq, nv ? (size_t)T * (L / 32) * 18 : zqb);
        if (tr->counts) memcpy(tr->counts, counts, sizeof(int32_t) * (size_t)E);
        if (tr->offsets) memcpy(tr->offsets, offsets, sizeof(int32_t) * (size_t)(E + 1));
        if (tr->perm) memcpy(tr->perm, perm, sizeof(int32_t) * (size_t)P);
        if (tr->pos) memcpy(tr->pos, pos, sizeof(int32_t) * (size_t)P);
        if (rc == 0) {
            if (tr->o) memcpy(tr->o, o, sizeof(float) * (size_t)P * L);
            if (tr->y_lat) memcpy(tr->y_lat, ylat, sizeof(float) * (size_t)T * L);
            if (tr->ylq) memcpy(tr->ylq, ylq, zqb);
        }
    }
    free(xq); free(z); free(lg); free(idx); free(w); free(zq); free(counts);
    free(offsets); free(perm); free(pos); free(g); free(u); free(h); free(hq);
    free(o); free(ylat); free(ylq);
    return rc;
}

/* ------------------------------------------------------------------------ */
/* device arena layout, written out element by element.
 * Rows in tiles of 128, each tile in four slices of 32 rows; per (tile,
 * slice) the blocks kb = 0 .. nb-1 follow one another:
 *   Q8_0 codes: 1024 bytes per (tile, slice, kb) at
 *       tile*nb*4096 + slice*nb*1024 + kb*1024 + (r/8)*256 + (i/16)*128 + (r%8)*16 + (i%16)
 *       for local row r (0..31) of the slice and code i (0..31) of the block;
 *   Q4_0 codes: 512 bytes per (tile, slice, kb) at
 *       tile*nb*2048 + slice*nb*512 + kb*512 + r*16 + j (the block's 16 nibble bytes);
 *   scales: fp16 element tile*nb*128 + slice*nb*32 + kb*32 + r. */

void orc_arena_pack(int fmt, const uint8_t* aos, int n_rows, int k,
                    uint8_t* q_out, uint8_t* d_out)
{
    int nb = k / 32;
    int wb = orc_block_bytes(fmt);
    for (int row = 0; row < n_rows; ++row) {
        int tile = row / 128, slice = (row % 128) / 32, r = row % 32;
        for (int kb = 0; kb < nb; ++kb) {
            const uint8_t* blk = aos + ((int64_t)row * nb + kb) * wb;
            int64_t sel = (int64_t)tile * nb * 128 + (int64_t)slice * nb * 32 + (int64_t)kb * 32 + r;
            d_out[sel * 2] = blk[0];
            d_out[sel * 2 + 1] = blk[1];
            if (fmt == ORC_Q8_0) {
                int64_t base = (int64_t)tile * nb * 4096 + (int64_t)slice * nb * 1024 + (int64_t)kb * 1024;
                for (int i = 0; i < 32; ++i)
                    q_out[base + (r / 8) * 256 + (i / 16) * 128 + (r % 8) * 16 + (i % 16)] = blk[2 + i];
            } else {
                int64_t base = (int64_t)tile * nb * 2048 + (int64_t)slice * nb * 512 + (int64_t)kb * 512;
                for (int j = 0; j < 16; ++j)
                    q_out[base + r * 16 + j] = blk[2 + j];
            }
        }
    }
}

/* RMS normalisation of the rows of h [T][H] (the stack's reading): the sum of
 * squares as 32 partials (partial j takes i = j, j+32, ... with fmaf), an xor
 * butterfly (16, 8, 4, 2, 1) of adds, ms = sum / H, r = sqrtf(ms + 1e-6f),
 * out_i = h_i / r. */
void orc_rmsnorm(const float* h, int T, int H, float* out)
{
    for (int t = 0; t < T; ++t) {
        const float* hr = h + (int64_t)t * H;
        float part[32];
        for (int j = 0; j < 32; ++j) {
            float p = 0.0f;
            for (int i = j; i < H; i += 32) p = fmaf(hr[i], hr[i], p);
            part[j] = p;
        }
        for (int off = 16; off >= 1; off /= 2) {
            float nxt[32];
            for (int j = 0; j < 32; ++j) nxt[j] = part[j] + part[j ^ off];
            memcpy(part, nxt, sizeof(part));
        }
        const float ms = part[0] / (float)H;
        const float r = sqrtf(ms + 1e-6f);
        for (int i = 0; i < H; ++i) out[(int64_t)t * H + i] = hr[i] / r;
    }
}
