/*
 * elq_oracle.h -- scalar CPU oracle of the quantized latent-MoE expert layer.
 *
 * TEST INFRASTRUCTURE ONLY.  This is the slow, plain statement of what the
 * layer computes, used by the test-suite, by the package's smoke check and by
 * the benchmark's CPU-baseline leg.  It shares no code, header, table or
 * constant with the CUDA library (quantized_latent_moe_b200/csrc); the two are
 * written independently from the same definitions and compared element by
 * element.
 *
 * Sources (page title, section):
 *  - "edge0-strata/EDGE0.md", section "Changes from upstream Strata": latent-MoE
 *    layers with dense D (hidden->latent) and U (latent->hidden) projections in
 *    Q8 or Q4, latent sizes 1792 / 1280.
 *  - "Q8 0 support - Pull Request #255 - Niko1221/Strata", section "GPU EXPERT
 *    KERNELS": the Q8_0 block (qk 32) and the Q8_0 x Q8_1 block dot; section
 *    "VERIFIED AGAINST AN ORACLE": GPU experts quantize activations to Q8_1.
 *    Follow-up commit "per-role format lists": a min/offset term multiplies the
 *    sum of the QUANTIZED activations, not the stored s.
 *  - "Sync upstream Strata v0.1.39 into Lanes" (Strata-Lanes PR #24), SYCL-port
 *    commit: the activation quantiser is byte-exact only with a correctly
 *    rounded fp32 divide.  Q8_0 PR #255, "CONV1D": fp32 -> fp16 narrowing is
 *    round-to-nearest-even.
 *
 * Block byte layouts (little endian):
 *   Q8_0 : fp16 d, int8 q[32]                       34 B
 *   Q4_0 : fp16 d, uint8 nib[16] (q[j] | q[j+16]<<4) 18 B
 *   Q8_1 : fp16 d, fp16 s, int8 q[32]               36 B
 *
 * Readings where the pages are silent (each is the plainest one the rest
 * supports):
 *   R1 round(.) is round-half-away-from-zero (C roundf).
 *   R2 d = amax / 127 and q = round(x / d) use an IEEE round-to-nearest fp32
 *      divide; d == 0 gives q = 0; q is clamped to [-127, 127] (only reachable
 *      when d is a tiny subnormal).
 *   R3 q is computed with the fp32 d; the stored d is fp16(d) (RNE).
 *   R4 Q8_1 s = fp16(d * (float)sum(q)).
 *   R5 Q4_0: m = the element of largest |x| (lowest index on ties),
 *      d = m / -8, q = clamp(round(x / d) + 8, 0, 15); d == 0 gives q = 8.
 *   R6 Q4_0 nibble order: byte j = q[j] | q[j+16] << 4.
 *   R7 Q4_0 x Q8_1: isum = sum (q4 - 8) * q8 (exact integer); s is unused.
 *   R8 a row dot product accumulates in fp32 over chunks of 8 blocks:
 *      sc = f32(d_w) * f32(d_a); part = fmaf((float)isum, sc, part) over the
 *      blocks of a chunk in order from 0; acc = acc + part over the chunks in
 *      order from 0.
 *   R9 router logit = 32 strided fp32 partials (partial j takes l = j, j+32,
 *      ... with fmaf), then an xor butterfly (16, 8, 4, 2, 1) of fp32 adds,
 *      then + bias.  The router reads the unquantised fp32 latent z.
 *   R10 bias takes part in selection and weights; top-k by logit descending,
 *      lower expert id first on equal logits.
 *   R11 weights = softmax over the k selected logits, in rank order.
 *   R12 exp is this file's own orc_expf (Cody-Waite reduction, degree-7 Taylor
 *      polynomial by fmaf, scaling by 2^n).
 *   R13 SwiGLU: h = (g / (1 + exp(-g))) * u.
 *   R14 combine: y_lat = sum_j fmaf(w_j, o_j, acc) over the k slots in rank
 *      order from 0.
 *   R18 a NaN router logit ranks as -infinity, in the selection and in the
 *       softmax (ties still by lower id), so the chosen ids are always valid.
 *
 * NVFP4 latent experts (page "edge0-strata", section "Changes from upstream
 * Strata": NVFP4 and Q3_K latent experts).  The pages name the format and
 * nothing more; readings:
 *   R19 E2M1 values (codes 0..7: 0, 0.5, 1, 1.5, 2, 3, 4, 6; bit 3 the
 *       sign) and E4M3 scales; conversions round to nearest with ties to the
 *       even code and saturate finite values (6 and 448); a NaN or
 *       non-positive scale input gives scale 0.
 *   R20 a weight matrix (an expert's interleaved gate/up, or its down) has
 *       one fp32 global scale g = amax / (6 * 448), 1 if all zero; the
 *       experts' activations (the latent z and the SwiGLU output h) are NVFP4
 *       too, each under a static fp32 global scale of the layer (act_gz for
 *       z, act_gh for h), given with the weights as a calibrated checkpoint
 *       carries it.  Per 16 values: s = e4m3(amax / 6 / g), code =
 *       e2m1(x / (dec(s) * g)).  An 18-byte block holds 32 values: two
 *       scales, then 16 bytes of codes (value 2j low nibble of byte j, 2j+1
 *       high).
 *   R21 row dot: per 16-value micro-block isum = sum (2w)(2a) (exact), sc =
 *       dec(sw) * dec(sa), part = fmaf((float)isum, sc, part) over the 16
 *       micro-blocks of a chunk of 8 blocks in order, acc = acc + part over
 *       chunks, y = acc * ((g_w * g_a) * 0.25).
 *
 * Q5_1, Q4_K and Q5_K experts ("Q8 0 support - Pull Request #255 -
 * Niko1221/Strata", follow-up commit "per-role format lists": the Q4_K, Q5_K
 * and Q5_1 expert dots; Q5_1's min term multiplies the sum of the quantised
 * activations, not the stored s).  The blocks are the GGUF layouts those
 * names stand for; readings:
 *   R22 Q5_1: x = d q + m, q = 4-bit code + 16 * its qh bit (q in 0..31).
 *       Q4_K, Q5_K: super-blocks of 256 in 8 sub-blocks of 32 with 6-bit
 *       scale_j and min_j; x = d scale_j q - dmin min_j.
 *   R23 per 32-value block (a K-quant sub-block) against a Q8_1 block:
 *       isum = sum q_w q_a and sumq = sum q_a, exact integers (the min term
 *       takes the quantised sum for every one of these formats).
 *   R24 order: part = fmaf((float)isum, sd, part), then part =
 *       fmaf((float)sumq, sm, part), blocks in order within chunks of 8 (one
 *       super-block), acc = acc + part over chunks.  Q5_1: sd = d_w d_a, sm =
 *       m_w d_a; K-quants: sd = (d scale_j) d_a, sm = -((dmin min_j) d_a),
 *       each product one fp32 multiply (d scale_j and dmin min_j are exact).
 *
 * Q3_K experts ("edge0-strata/EDGE0.md", "Changes from upstream Strata":
 * "NVFP4 and Q3_K latent experts"):
 *   R25 the GGUF Q3_K super-block (256 values, 16 sub-blocks of 16 with
 *       6-bit scales stored offset by 32, 3-bit codes as two low bits and a
 *       high-bit mask, q = low - 4 when the high bit is clear); x = d scale q.
 *       Per 32-value block the two 16-value halves: isum_h = sum q_w q_a
 *       (exact), sd_h = (d scale_h) d_a; part = fmaf(isum_0, sd_0, part), then
 *       part = fmaf(isum_1, sd_1, part), in the R8 chunk order (no min term).
 *       orc_block_ext returns (isum_0, isum_1, sd_0, sd_1) in (isum, sumq,
 *       sd, sm).
 */
#ifndef ELQ_ORACLE_H
#define ELQ_ORACLE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

enum { ORC_Q4_0 = 2, ORC_Q5_1 = 7, ORC_Q8_0 = 8, ORC_Q8_1 = 9, ORC_Q3_K = 11, ORC_Q4_K = 12, ORC_Q5_K = 13,
       ORC_NVFP4 = 100 };

int      orc_block_bytes(int fmt);                /* 18, 34, 36; 0 if unknown */
int64_t  orc_matrix_bytes(int fmt, int64_t rows, int64_t k);

/* number formats */
uint16_t orc_f32_to_f16(float x);                 /* round to nearest even */
float    orc_f16_to_f32(uint16_t h);
float    orc_bf16_to_f32(uint16_t b);
float    orc_expf(float x);                       /* R12 */
float    orc_silu(float g);                       /* R13 first factor */

/* quantisers: n % 32 == 0, out holds n/32 blocks */
void orc_quantize_q8_1(const float* x, int64_t n, uint8_t* out);
void orc_quantize_q8_0(const float* x, int64_t n, uint8_t* out);
void orc_quantize_q4_0(const float* x, int64_t n, uint8_t* out);
/* fp64 dequantisers (self-checks) */
void orc_dequantize(int fmt, const uint8_t* blocks, int64_t n, double* out);

/* one weight block (Q8_0 or Q4_0) against one Q8_1 block */
int32_t orc_block_isum(int wfmt, const uint8_t* wblk, const uint8_t* ablk);
float   orc_block_term(int wfmt, const uint8_t* wblk, const uint8_t* ablk);

/* Y[t][n] = row n of W (row-major AoS blocks, N rows x K) . Xq[t] (Q8_1, K)
 * under R8; chunk = blocks per ordered chunk (8 in the layer). */
void orc_qmatmul(int wfmt, const uint8_t* W, int N, int K,
                 const uint8_t* Xq, int T, float* Y);

/* router, R9-R11 and R18 (a NaN logit ranks as -infinity): idx [T][k],
 * w [T][k], logits [T][E] (may be NULL; raw values) */
void orc_router_topk(const float* z, const float* Wr, const float* bias,
                     int T, int L, int E, int k,
                     int32_t* idx, float* w, float* logits);

/* token -> expert bucketing: counts [E], offsets [E+1] (exclusive scan),
 * perm [T*k] pair ids sorted by (expert, pair id), pos [T*k] inverse. */
void orc_bucket(const int32_t* idx, int T, int k, int E,
                int32_t* counts, int32_t* offsets, int32_t* perm, int32_t* pos);

/* NVFP4 (R19-R21) */
uint8_t  orc_f32_to_e2m1(float v);
float    orc_e2m1_to_f32(uint8_t c);
uint8_t  orc_f32_to_e4m3(float v);
float    orc_e4m3_to_f32(uint8_t b);
float    orc_nvfp4_global(const float* x, int64_t n);
void     orc_quantize_nvfp4(const float* x, int64_t n, float g, uint8_t* out);
void     orc_dequantize_nvfp4(const uint8_t* blocks, int64_t n, float g, double* out);
void     orc_qmatmul_nvfp4(const uint8_t* W, float gw, int N, int K, const uint8_t* X, float ga,
                           int T, float* Y);

/* Q5_1 / Q4_K / Q5_K (R22-R24) */
int64_t  orc_row_bytes(int fmt, int64_t k);
int      orc_is_kquant(int fmt);
void     orc_dequantize_ext(int fmt, const uint8_t* W, int N, int K, double* out);
void     orc_block_ext(int fmt, const uint8_t* row, int kb, const uint8_t* a, int32_t* isum, int32_t* sumq,
                       float* sd, float* sm);
void     orc_qmatmul_ext(int fmt, const uint8_t* W, int N, int K, const uint8_t* Xq, int T, float* Y);

/* One latent-MoE layer.  Weight matrices are row-major AoS blocks.
 * gate/up/down are arrays of E pointers; an expert no token selects may be
 * NULL. */
typedef struct {
    int H, L, E, k, I;
    int du_fmt;                 /* format of D and U */
    int ex_fmt;                 /* format of gate, up, down */
    const uint8_t* D;           /* [L rows][H] */
    const uint8_t* U;           /* [H rows][L] */
    const float* router_w;      /* [E][L] fp32 */
    const float* router_bias;   /* [E] or NULL */
    const uint8_t* const* gate; /* E x [I rows][L] */
    const uint8_t* const* up;   /* E x [I rows][L] */
    const uint8_t* const* down; /* E x [L rows][I] */
    /* NVFP4 experts: each matrix's global scale (E entries each); gate and
     * up of an expert share one (they are one interleaved matrix, R20) */
    const float* gate_g;
    const float* up_g;
    const float* down_g;
    float act_gz;               /* static global scales of the NVFP4 expert inputs */
    float act_gh;
} orc_layer;

/* Optional intermediates; any pointer may be NULL. */
typedef struct {
    uint8_t* xq;        /* [T][H/32] Q8_1 */
    float*   z;         /* [T][L] */
    float*   logits;    /* [T][E] */
    int32_t* idx;       /* [T][k] */
    float*   w;         /* [T][k] */
    uint8_t* zq;        /* [T][L/32] Q8_1 */
    int32_t* counts;    /* [E] */
    int32_t* offsets;   /* [E+1] */
    int32_t* perm;      /* [T*k] */
    int32_t* pos;       /* [T*k] */
    float*   g;         /* [T*k][I], pair order p = t*k + j */
    float*   u;         /* [T*k][I] */
    uint8_t* hq;        /* [T*k][I/32] Q8_1 */
    float*   o;         /* [T*k][L] */
    float*   y_lat;     /* [T][L] */
    uint8_t* ylq;       /* [T][L/32] Q8_1 */
} orc_trace;

/* Returns 0, or -1 if a selected expert's weights are NULL, -2 on bad sizes. */
int orc_moe_layer(const orc_layer* ly, const float* x, int T, float* y,
                  orc_trace* tr);

/* Only the routing half of the layer (x -> xq -> z -> idx, w), so that a caller
 * can learn which experts a token set needs before supplying them. */
int orc_route(const orc_layer* ly, const float* x, int T, int32_t* idx, float* w);

/* The stack's layer input: each row of h divided by sqrt(mean(h^2) + 1e-6),
 * the sum of squares in the R9 order (32 strided fmaf partials, xor
 * butterfly of adds). */
void orc_rmsnorm(const float* h, int T, int H, float* out);

/* The device arena layout, stated plainly (the definition is written out in
 * elq_oracle.c): tiles of 128 rows, four 32-row slices per tile, per slice
 * its blocks one after another (1024-byte Q8_0 or 512-byte Q4_0 pieces) and a
 * parallel array of fp16 scales.  aos is row-major AoS blocks; n_rows % 128
 * == 0. */
void orc_arena_pack(int fmt, const uint8_t* aos, int n_rows, int k,
                    uint8_t* q_out, uint8_t* d_out);

#ifdef __cplusplus
}
#endif
#endif
