/*
 * elq.h -- C ABI of the quantized latent-MoE expert layer for B200 (sm_100a).
 *
 * The layer (page "edge0-strata/EDGE0.md", section "Changes from upstream
 * Strata"): a dense D projection (hidden H -> latent L, L = 1792 or 1280), a
 * router with top-k over E experts, per-expert gate/up -> SwiGLU -> down in the
 * latent space, and a dense U projection (latent -> hidden).  Weights are
 * Q8_0 or Q4_0 blocks of 32 values; activations are quantised to Q8_1 ("Q8 0
 * support - Pull Request #255 - Niko1221/Strata", section "VERIFIED AGAINST AN
 * ORACLE": the GPU experts quantise activations to Q8_1; section "GPU EXPERT
 * KERNELS": the Q8_0 x Q8_1 block dot).
 *
 * Conventions shared by every call
 *  - Pointers named as device pointers are CUDA device memory owned by the
 *    caller.  The library allocates no memory and never synchronises the
 *    stream (elq_workspace_status and elq_latent_proj_noalloc_status are the
 *    documented blocking exceptions).  The state it keeps between calls is
 *    per device and read-only after the first call there: the SM count, the
 *    kernels' shared-memory opt-ins, and, for elq_latent_proj_noalloc only,
 *    the address of its file-scope 4 MiB scratch array (below).  `stream` is
 *    a cudaStream_t (NULL = legacy default stream).
 *  - Device pointers must be 16-byte aligned unless stated otherwise.
 *  - Every call validates its arguments on the host before it enqueues any
 *    work, and returns ELQ_OK or a negative elq_status.  On an error nothing is
 *    enqueued and no output is written.  Launch failures return ELQ_ERR_CUDA.
 *    Faults inside kernels surface at the caller's next synchronisation.
 *  - No tokens (T = 0, or rows = 0) is a valid call: it checks its other
 *    arguments, then returns ELQ_OK without enqueuing anything or reading its
 *    data pointers, which may then be NULL; the *_workspace_bytes calls return
 *    0.  elq_route_bucket is the exception: it still writes zero counts and
 *    offsets.
 *  - Calls that take a workspace `ws` use it for intermediates.  It must be at
 *    least the size the matching *_workspace_bytes call returns, 256-byte
 *    aligned, and ZERO-FILLED before its first use; every call leaves its
 *    counters at zero again, so a workspace can be reused without clearing.
 *    Two calls that share a workspace must not overlap on the GPU.
 *  - Floating-point results follow a fixed accumulation order (below), so the
 *    same inputs always give the same bits, whatever the launch shape.
 *
 * Block formats (little endian)
 *   Q8_0 : fp16 d, int8 q[32]                    x = d * q            34 B
 *   Q4_0 : fp16 d, uint8 nib[16]                 x = d * (q - 8)      18 B
 *          byte j holds q[j] (low nibble) and q[j+16] (high nibble)
 *   Q8_1 : fp16 d, fp16 s, int8 q[32]            s = d * sum(q)       36 B
 *   NVFP4: uint8 s[2], uint8 nib[16]          32 values as two micro-blocks  18 B
 *          of 16; s[m] the E4M3 scale of micro-block m; byte j holds the
 *          E2M1 code of value 2j (low nibble) and 2j+1 (high nibble); code
 *          c (bit 3 the sign) stands for +-(0, 0.5, 1, 1.5, 2, 3, 4, 6)[c & 7];
 *          x = e2m1(c) * e4m3(s[m]) * g, g the fp32 global scale of the
 *          tensor ("edge0-strata/EDGE0.md", section "Changes from upstream
 *          Strata": NVFP4 latent experts; the pages give no more, the layout
 *          and the rules below are this library's reading)
 *   Quantisation of a block: amax = max |x|; Q8: d = amax / 127 (fp32,
 *   correctly rounded), q = round-half-away(x / d) (correctly rounded divide),
 *   d stored as fp16 (round to nearest even); Q4_0: m = the element of largest
 *   |x| (lowest index on ties), d = m / -8, q = clamp(round(x / d) + 8, 0, 15).
 *   A zero scale gives all-zero codes (Q4_0: 8).  NVFP4 under global scale
 *   g: per micro-block s = e4m3(amax / 6 / g) (fp32 divides; round to nearest
 *   even, saturating at 448), code = e2m1(x / (e4m3(s) * g)) (round to nearest
 *   even, saturating at 6; a result that rounds to zero keeps the sign of a
 *   negative input, -0 counts as +0); s = 0 gives zero codes.
 *
 * Arithmetic
 *   Block dot of a weight block with a Q8_1 block: isum = sum q_w * q_a (Q4_0:
 *   sum (q_w - 8) * q_a, with the quantised activations' own sum, not s), an
 *   exact int32.  A row dot over K = 32 * nb accumulates, for each run of 8
 *   blocks in order, part = fmaf((float)isum, f32(d_w) * f32(d_a), part) from
 *   0, and adds the runs' parts in order into an fp32 sum from 0.
 *   Router logit: 32 lane-strided fp32 fmaf partials, an xor butterfly of adds
 *   (16, 8, 4, 2, 1), plus the bias.  Top-k by logit, lower expert id first on
 *   ties; weights are the softmax over the k selected logits.  exp() is the
 *   library's own (Cody-Waite reduction, degree-7 Taylor polynomial).
 *   NVFP4 experts: the activations they read (z, and h of SwiGLU) are
 *   NVFP4 under the layer's static global scales act_gz and act_gh.  Per
 *   micro-block isum = sum (2 c_w)(2 c_a) over the 16 doubled codes (exact),
 *   part = fmaf((float)isum, e4m3(s_w) * e4m3(s_a), part) over the chunk's 16
 *   micro-blocks in order, the chunks added as above, and the row's result is
 *   acc * ((g_w * g_a) * 0.25).
 *   SwiGLU h = (g / (1 + exp(-g))) * u; the weighted combine sums
 *   fmaf(w_j, o_j, acc) over the k slots in rank order.
 *
 * Device weight arena ("tile-slab" layout)
 *   A matrix of n_rows x k (n_rows % 128 == 0, k % 32 == 0, nb = k / 32) is
 *   stored as tiles of 128 rows, each tile as four slices of 32 rows, and each
 *   slice as its nb blocks one after another.  For tile t, slice s (rows
 *   128 t + 32 s .. +31), block kb and local row r (0..31):
 *     q : Q8_0 -- a 1024-byte piece at q + t*nb*4096 + s*nb*1024 + kb*1024;
 *         code i of row r sits at byte (r/8)*256 + (i/16)*128 + (r%8)*16 +
 *         (i%16) of the piece: 8-row x 16-byte core matrices, the K-major
 *         no-swizzle operand layout of the tcgen05 tensor cores.
 *         Q4_0 -- a 512-byte piece at q + t*nb*2048 + s*nb*512 + kb*512; row
 *         r's 16 nibble bytes at byte 16 r of the piece, in the block's order.
 *         NVFP4 -- as Q4_0: row r's 16 code bytes at byte 16 r of a
 *         512-byte piece.
 *     d : fp16 scale at element t*nb*128 + s*nb*32 + kb*32 + r.
 *         NVFP4 (k % 64 == 0): tile t's scales start at element t*nb*256;
 *         its first nb*128 elements hold the block's two scale bytes (s[0]
 *         the low byte) in the order above, the next nb*256 bytes the same
 *         bytes again as the tensor cores' scale-factor atoms: for blocks 2j
 *         and 2j+1 one 512-byte atom, tile row m = 32 s + r's four scales
 *         (block 2j s[0], s[1], block 2j+1 s[0], s[1]) at byte 16 r + 4 s.
 *   So the 8 blocks of a 32-row slice that one warp of the decode kernels
 *   reads are one contiguous bulk copy.  q and d must be 256-byte aligned.
 *   The layer's matrices (and elq_latent_proj's) need k % 128 == 0.
 *
 * Layer weights
 *   D      : L rows x H;   U : H rows x L  (any weight format each)
 *   router : fp32 [E][L], optional fp32 bias [E]; L <= 2048
 *   gate_up: E * 2I rows x L; expert e owns rows [2I e, 2I (e+1)); its tile j
 *            holds gate rows 64j .. 64j+63 then up rows 64j .. 64j+63.
 *            I % 64 == 0.
 *   down   : E * L rows x I; expert e owns rows [L e, L (e+1)).
 *   NVFP4 experts (gate_up and down both ELQ_NVFP4; D and U Q8_0 or Q4_0):
 *            gate_up.gs holds one global scale per expert (gs_rows = 2I),
 *            down.gs one per expert (gs_rows = L); L % 256 == 0 and
 *            I % 256 == 0; act_gz, act_gh > 0.  Such layers run for T <= 8
 *            tokens (T * k <= 64) only; other T return ELQ_ERR_UNSUPPORTED.
 */
#ifndef ELQ_H
#define ELQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    ELQ_OK = 0,
    ELQ_ERR_INVALID_ARG = -1,   /* null pointer, bad size, k > E, ... */
    ELQ_ERR_UNSUPPORTED = -2,   /* format or shape the kernels do not take */
    ELQ_ERR_ALIGNMENT = -3,     /* a pointer is not aligned as required */
    ELQ_ERR_WORKSPACE = -4,     /* workspace missing or too small */
    ELQ_ERR_CUDA = -5,          /* a CUDA runtime call failed */
    ELQ_ERR_TIMEOUT = -6        /* a bounded device wait ran out */
} elq_status;

typedef enum {                  /* GGUF type ids */
    ELQ_F32 = 0,
    ELQ_Q4_0 = 2,
    ELQ_Q8_0 = 8,
    ELQ_Q8_1 = 9,
    ELQ_Q5_1 = 7,
    ELQ_Q3_K = 11,
    ELQ_Q4_K = 12,
    ELQ_Q5_K = 13,
    ELQ_BF16 = 30,
    ELQ_NVFP4 = 100             /* not a GGUF id: this library's own */
} elq_type;

/* One quantised matrix in the tile-slab arena (device pointers q, d). */
typedef struct {
    int32_t fmt;                /* ELQ_Q8_0, ELQ_Q4_0, or ELQ_NVFP4 (expert matrices) */
    int32_t n_rows;             /* multiple of 128 */
    int32_t k;                  /* multiple of 32 */
    int32_t gs_rows;            /* NVFP4: rows that share one global scale; else 0 */
    const void* q;
    const void* d;
    const float* gs;            /* NVFP4: device fp32 [n_rows / gs_rows], 4-byte aligned; else NULL */
    const void* q16;            /* optional, Q8_0 only: the codes widened to fp16 (elq_pack_f16), 256-byte
                                 * aligned.  When every int8 tensor-core matrix of a layer call carries
                                 * it, the T >= 16 path multiplies fp16 operands (tcgen05 kind::f16,
                                 * fp32 accumulators that hold each block's integer sum exactly) instead
                                 * of int8 ones; the results are the same bits.  NULL: int8. */
} elq_qmat;

/* elq_layer.flags bits. */
enum {
    /* Run small token counts (T <= 8, T * k <= 64) as one cooperative
     * persistent kernel instead of the separate-kernel sequence (same
     * results, bit for bit).  Off by default: on B200 it measures slower
     * than the sequence (its phase-to-phase handoffs through global memory
     * cost more than the launches they replace). */
    ELQ_LAYER_FUSED = 1
};

/* One latent-MoE layer.  The struct lives in host memory; every pointer in it
 * is device memory. */
typedef struct {
    int32_t H, L, E, k, I;
    int32_t flags;              /* ELQ_LAYER_* bits, 0 by default */
    elq_qmat D;                 /* L x H  */
    elq_qmat U;                 /* H x L  */
    const float* router_w;      /* [E][L] */
    const float* router_bias;   /* [E] or NULL */
    elq_qmat gate_up;           /* E*2I x L, interleaved by 64-row halves */
    elq_qmat down;              /* E*L x I */
    float act_gz, act_gh;       /* NVFP4 experts: global scales of z and h; else unused */
} elq_layer;

/* ---- status ------------------------------------------------------------ */

/* Static English text of a status code. */
const char* elq_status_string(int32_t status);

/* ABI version (increments on any change of this header). */
int32_t elq_version(void);

/* ---- arena preparation (not part of a layer call) ------------------------ */

/* Bytes of the arena arrays of an n_rows x k matrix in format fmt.  Returns
 * q_bytes + d_bytes, or 0 for an unsupported format/shape.  Either out
 * pointer may be NULL. */
size_t elq_arena_bytes(int32_t fmt, int32_t n_rows, int32_t k,
                       size_t* q_bytes, size_t* d_bytes);

/* Repack row-major GGUF-style AoS blocks (device, n_rows x k/32 blocks of
 * 34 B (Q8_0) or 18 B (Q4_0, NVFP4), no alignment requirement) into the
 * arena.  NVFP4 global scales stay with the caller (elq_qmat.gs). */
elq_status elq_arena_pack(int32_t fmt, const void* aos, int32_t n_rows, int32_t k,
                          void* q_out, void* d_out, void* stream);

/* The fp16 codes of a Q8_0 arena matrix (elq_qmat.q16): 2 * n_rows * k bytes,
 * or 0 for another format.  Block-major: per (128-row tile, 32-value block),
 * tile-major then block, 8 KB laid out [code / 16][row / 8][(code % 16) / 8]
 * [row % 8][8 fp16] -- per 16-value half of the block the no-swizzle K-major
 * operand of one fp16 MMA (experts: each expert's 2x its code bytes). */
size_t elq_f16_bytes(const elq_qmat* w);

/* Fill q16 (device, elq_f16_bytes(w) bytes, 256-byte aligned) from w's
 * arena codes: every code c becomes the fp16 value c (exact).  Stream order;
 * w->q16 is not read. */
elq_status elq_pack_f16(const elq_qmat* w, void* q16, void* stream);

/* Quantise fp32 weights (device, row-major n_rows x k) into the arena with the
 * format's own quantiser (block rules above).  Q8_0 and Q4_0; NVFP4 weights
 * go through elq_quantize_nvfp4 and elq_arena_pack. */
elq_status elq_quantize_weights(int32_t fmt, const float* w, int32_t n_rows, int32_t k,
                                void* q_out, void* d_out, void* stream);

/* Quantise E experts' fp32 gate and up matrices (device, [E][I][L] each) into
 * one gate_up arena (E*2I rows x L, interleaved as described above). */
elq_status elq_quantize_gate_up(int32_t fmt, const float* gate, const float* up,
                                int32_t E, int32_t I, int32_t L,
                                void* q_out, void* d_out, void* stream);

/* ---- the hot path --------------------------------------------------------- */

/* Q8_1 activation quantiser (a1, a4).  x: device [rows][cols] fp32 (x_type
 * ELQ_F32) or bf16 (ELQ_BF16), cols % 32 == 0, 4-byte aligned.  out: device
 * rows*cols/32 Q8_1 blocks (36 B each, row-major, 4-byte aligned). */
elq_status elq_quantize_q8_1(const void* x, int32_t x_type, int64_t rows, int64_t cols,
                             void* out_q8_1, void* stream);

/* NVFP4 quantiser under global scale g (> 0, finite): x device [rows][cols]
 * fp32 (ELQ_F32) or bf16 (ELQ_BF16), cols % 32 == 0, 4-byte aligned; out
 * device rows*cols/32 18-byte blocks, row-major, 2-byte aligned.  The
 * layer's own NVFP4 activations are quantised by the same warp routine. */
elq_status elq_quantize_nvfp4(const void* x, int32_t x_type, int64_t rows, int64_t cols, float g,
                              void* out, void* stream);

/* Router (a3): logits = W_r z + bias, top-k, softmax over the k.  z: device fp32
 * [T][L] (unquantised latent), w_router [E][L], bias [E] or NULL.  idx: device
 * int32 [T][k] in rank order; weights fp32 [T][k]; logits fp32 [T][E] or NULL.
 * 1 <= k <= min(E, 32), E <= 1024, L % 32 == 0, L <= 2048 (each lane of the
 * router kernel holds its L/32 weights of a router row in registers). */
elq_status elq_router_topk(const float* z, const float* w_router, const float* bias,
                           int32_t T, int32_t L, int32_t E, int32_t k,
                           int32_t* idx, float* weights, float* logits, void* stream);

/* Token -> expert bucketing (a5): counts [E], offsets [E+1] (exclusive scan),
 * perm [T*k] = pair ids p = t*k + j sorted by (expert, p), pos [T*k] its
 * inverse.  All device int32. */
elq_status elq_route_bucket(const int32_t* idx, int32_t T, int32_t k, int32_t E,
                            int32_t* counts, int32_t* offsets, int32_t* perm,
                            int32_t* pos, void* stream);

/* Latent projection (a2 with D, a10 with U): y[t][n] = row n of w . x[t].
 * x_q8_1: device T rows of w->k/32 Q8_1 blocks; y: device fp32 [T][w->n_rows]. */
size_t elq_latent_proj_workspace_bytes(const elq_qmat* w, int32_t T);
elq_status elq_latent_proj(const elq_qmat* w, const void* x_q8_1, int32_t T, float* y,
                           void* ws, size_t ws_bytes, void* stream);

/* elq_latent_proj without a workspace, for callers that cannot allocate
 * device memory: code embedded in a host engine whose plugin interface hands
 * over only input and output pointers, engines that reserve all of HBM up
 * front for the resident expert arena and forbid allocation afterwards, and
 * callers that may not call cudaMalloc between setting up and running their
 * decode loop.  The paper has no counterpart; this is a calling convention of
 * this library.
 *  - It always runs the GEMV kernel, whatever T.  Its scratch (error word,
 *    tile counters, and the chunk partial sums: k/256 chunks x T x n_rows x 4
 *    bytes) is one file-scope device array of 4 MiB (4,194,304 bytes) that
 *    every GPU which loads the library holds until the process exits.  A
 *    shape whose scratch exceeds it returns ELQ_ERR_WORKSPACE; e.g. a
 *    1792 x 4096 Q8_0 matrix fits up to 36 tokens.
 *  - The first call on a device looks up the array's device address
 *    (cudaGetSymbolAddress, with that device current) and caches it; make
 *    that first call before any stream capture.
 *  - Every call clears the error word and the counters on its stream (a
 *    cudaMemsetAsync) before its kernel; nothing is allocated or freed.
 *  - All calls share the one array: calls that overlap on the GPU (different
 *    streams, or several host threads) race and give wrong results.  Order
 *    them on one stream.
 *  - A bounded device wait that runs out (2 s) leaves y undefined and sets the
 *    array's error word, which elq_latent_proj_noalloc_status reads; the next
 *    call clears it. */
elq_status elq_latent_proj_noalloc(const elq_qmat* w, const void* x_q8_1, int32_t T, float* y,
                                   void* stream);

/* Outcome of the last elq_latent_proj_noalloc call on the current device:
 * copies the static array's error word to the host (blocking: it
 * synchronises `stream`, which must be the stream of that call) and returns
 * ELQ_OK, or ELQ_ERR_TIMEOUT if one of that call's bounded waits ran out.
 * Allocates nothing; the word is cleared by the next noalloc call. */
elq_status elq_latent_proj_noalloc_status(void* stream);

/* Grouped experts (a5-a9): bucketing, gate/up with SwiGLU and Q8_1 requant,
 * down, and the weighted combine.  z_q8_1: device T rows of L/32 Q8_1 blocks;
 * idx, weights: device [T][k] as elq_router_topk writes them; y_lat: device
 * fp32 [T][L].  Uses layer->L, E, k, I, gate_up and down.  NVFP4 experts
 * (T <= 8, T * k <= 64): z is T rows of L/32 NVFP4 blocks under act_gz. */
elq_status elq_moe_experts_grouped(const elq_layer* layer, const void* z_q8_1,
                                   const int32_t* idx, const float* weights, int32_t T,
                                   float* y_lat, void* ws, size_t ws_bytes, void* stream);

/* The whole layer (a1-a10): x device [T][H] fp32 or bf16 -> y device fp32
 * [T][H]. */
size_t elq_workspace_bytes(const elq_layer* layer, int32_t T);
elq_status elq_moe_layer(const elq_layer* layer, const void* x, int32_t x_type, int32_t T,
                         float* y, void* ws, size_t ws_bytes, void* stream);

/* A stack of layers on one residual stream.  The pages give no rule for it;
 * the reading taken: h = fp32(x), then for l = 0 .. n_layers-1,
 * h = h + layer_l(rms(h)), where rms(h) is each row divided by
 * sqrt(mean(h^2) + 1e-6) (no learned scale; the sum of squares by 32
 * lane-strided fused multiply-adds and an xor butterfly of adds, every step
 * IEEE round-to-nearest fp32).  Without the normalisation the stack diverges:
 * a layer's output grows with the square of its input.
 * layers: host array of n_layers layers of identical shapes and formats (their
 * pointers device memory); x: device [T][H] fp32 or bf16 (the new tokens);
 * h: device [T][H] fp32 output.  ws: one workspace of
 * elq_stack_workspace_bytes(&layers[0], T) bytes, shared by the layers in
 * turn (the layer workspace, then the normalised input).  Each layer takes
 * the path elq_moe_layer would (ELQ_LAYER_FUSED is ignored here); the last
 * projection adds into h.  Launches 1 + n_layers * (1 + the layer's kernel
 * count without ELQ_LAYER_FUSED) kernels.
 * Validation as elq_moe_layer, before anything is enqueued. */
elq_status elq_moe_stack(const elq_layer* layers, int32_t n_layers, const void* x, int32_t x_type,
                         int32_t T, float* h, void* ws, size_t ws_bytes, void* stream);
size_t elq_stack_workspace_bytes(const elq_layer* layer, int32_t T);

/* Number of kernels one elq_moe_layer call launches at this T (0 if the
 * layer is invalid).  Fused small-T path (ELQ_LAYER_FUSED set, T <= 8,
 * T * k <= 64, D and U in one format, gate/up and down in one format, the
 * shared-memory plan fits): 1, a cooperative persistent kernel running the
 * whole layer.  Decode/verify path otherwise, in order: [activation
 * quantiser, for T > 8], D projection (quantising x itself for T <= 8; +
 * latent Q8_1), router (+ top-k, bucketing), gate/up (+ SwiGLU, Q8_1), down
 * (+ weighted combine, Q8_1), U projection.  Tensor-core path (T >= 16 and
 * every matrix Q8_0): activation quantiser, x packing, D, router, slot map, z
 * packing, gate/up, down, weighted combine, U. */
int32_t elq_layer_kernel_count(const elq_layer* layer, int32_t T);

/* elq_moe_layer that also records CUDA events on the stream: events[0] before
 * the first kernel and events[i] after kernel i (i = 1 .. kernel count), so
 * that elapsed times between consecutive events give each kernel's device
 * time.  events: host array of n_events >= kernel count + 1 cudaEvent_t.
 * Kernels launched this way do not overlap their prologues with the previous
 * kernel (no programmatic dependent launch). */
elq_status elq_moe_layer_profiled(const elq_layer* layer, const void* x, int32_t x_type, int32_t T,
                                  float* y, void* ws, size_t ws_bytes, void* const* events,
                                  int32_t n_events, void* stream);

/* Intermediates of an elq_moe_layer call inside its workspace, for tests and
 * measurement.  `which`: 0 xq (Q8_1 of x), 1 z (fp32 [T][L]), 2 zq, 3 logits
 * (fp32 [T][E]), 4 idx (int32 [T][k]), 5 weights (fp32 [T][k]), 6 counts
 * (int32 [E]), 7 offsets (int32 [E+1]), 8 perm (int32 [T*k]), 9 pos, 10 hq
 * (Q8_1 [T*k][I/32], by pair position), 11 o (fp32 [T*k][L], by position),
 * 12 y_lat (fp32 [T][L]), 13 ylq (Q8_1), 14 number of routed experts (int32).
 * With NVFP4 experts zq and hq hold NVFP4 blocks (18 B) instead of Q8_1.
 * On the tensor-core path (T >= 16, all matrices Q8_0) hq and o are kept in
 * padded per-expert slots instead, and their views return ELQ_ERR_INVALID_ARG.
 * Sets *offset (bytes from the workspace start) and *bytes; returns ELQ_OK or
 * ELQ_ERR_INVALID_ARG.  The values are those of the last call on that
 * workspace once the stream has reached its end. */
elq_status elq_workspace_view(const elq_layer* layer, int32_t T, int32_t which,
                              size_t* offset, size_t* bytes);

/* Reads the workspace's device error word after the stream has been
 * synchronised by the caller (blocking copy of 4 bytes); returns ELQ_OK or
 * ELQ_ERR_TIMEOUT, and clears the word. */
elq_status elq_workspace_status(void* ws, void* stream);

/* ---- test entry points ----------------------------------------------------- */

/* Failure detection of the fused small-T kernel: runs the layer exactly as
 * elq_moe_layer's fused path would, except that the routing is never
 * published, so every wait for it runs out after budget_ns (1 ms .. 2 s) of
 * device time.  The kernel then lets its own copies in flight land and
 * returns; the workspace error word reads ELQ_ERR_TIMEOUT afterwards (see
 * elq_workspace_status) and the workspace must be zero-filled again before
 * its next use.  y is left undefined.  ELQ_ERR_UNSUPPORTED when the layer at
 * this T does not take the fused path. */
elq_status elq_test_fused_timeout(const elq_layer* layer, const void* x, int32_t x_type, int32_t T,
                                  float* y, void* ws, size_t ws_bytes, uint64_t budget_ns,
                                  void* stream);

/* Single-block dots ("Q8 0 support", GPU EXPERT KERNELS: block-dot parity to
 * 1e-7): for i < nblocks, isum[i] and term[i] = (float)isum * (f32(d_w) *
 * f32(d_a)) of AoS weight block i (wfmt Q8_0 or Q4_0) against Q8_1 block i.
 * All device pointers, no alignment requirement. */
elq_status elq_test_block_isums(int32_t wfmt, const void* w_aos, const void* x_q8_1,
                                int64_t nblocks, int32_t* isum, float* term, void* stream);

/* The int8 tensor-core rate, for the roofline's peak: one CTA per SM, each
 * issuing n_mma (>= 2) tcgen05.mma kind::i8 instructions of M = 128, N = 256,
 * K = 32 back to back (2 * 128 * 256 * 32 integer operations each) from fixed
 * shared-memory operands into TMEM, then waiting (bounded, 2 s) for them.
 * The caller times the launch on `stream` (CUDA events) and divides the
 * operations, n_mma * elq_sm_count() * 2097152, by the time.  sink: device
 * int32 [elq_sm_count()], one accumulator word per CTA; err: device int32,
 * zero before the call, ELQ_ERR_TIMEOUT's code 1 if a wait ran out. */
elq_status elq_test_mma_i8_rate(int32_t n_mma, int32_t* sink, int32_t* err, void* stream);

/* The fp16 tensor-core rate, for the roofline of the fp16-operand GEMMs: as
 * elq_test_mma_i8_rate with tcgen05.mma kind::f16 of M = 128, N = 256, K = 16
 * (2 * 128 * 256 * 16 = 1048576 operations each, fp32 accumulators). */
elq_status elq_test_mma_f16_rate(int32_t n_mma, int32_t* sink, int32_t* err, void* stream);

/* The fp4 block-scaled tensor-core rate, for the NVFP4 experts' roofline: as
 * elq_test_mma_i8_rate with n_mma (>= 1) tcgen05.mma kind::mxf4nvf4 of M =
 * 128, N = n_cols (16 .. 256, a multiple of 16), K = 64 (2 * 128 * n_cols * 64
 * operations each) into one accumulator; the scale factors are copied to TMEM
 * once, or before every MMA when cp_each is nonzero. */
elq_status elq_test_mma_nvf4_rate(int32_t n_mma, int32_t n_cols, int32_t cp_each, int32_t* sink, int32_t* err,
                                  void* stream);

/* The packed fp32 rate, for the tensor-core epilogue's bound: 2 * SM count
 * CTAs of 1024 threads, each thread running n iterations of 8 independent
 * fma.rn.f32x2 instructions.  The caller times the launch on `stream` and
 * divides 2 * elq_sm_count() * 1024 * n * 8 instructions by the time.  sink:
 * device fp32 [2 * elq_sm_count() * 1024]. */
elq_status elq_test_f32x2_rate(int32_t n, float* sink, void* stream);

/* Streaming multiprocessors of the current device (the grid the persistent
 * kernels use). */
int32_t elq_sm_count(void);

/* Runs the library's own exp on n fp32 values (device in -> out). */
elq_status elq_test_expf(const float* in, float* out, int64_t n, void* stream);

#ifdef __cplusplus
}
#endif
#endif /* ELQ_H */
