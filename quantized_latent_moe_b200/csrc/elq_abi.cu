// elq_abi.cu -- the C ABI declared in include/elq.h: host-side validation,
// workspace layout and kernel launches.  No allocation, no synchronisation
// (except elq_workspace_status, which is documented as blocking).
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>
#include <cstring>
#include <functional>

#include "../../include/elq.h"
#include "elq_kernels.cuh"

using namespace elq;

namespace {

constexpr uint64_t kWaitBudgetNs = 2000000000ull;   // 2 s per bounded device wait
constexpr int kMaxDevices = 64;
constexpr int kLayerKernels = 7;   // quant, D, router, gate/up, down, combine, U

inline bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }
inline size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

int sm_count() {
    static int cache[kMaxDevices] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 148;
    if (dev < 0 || dev >= kMaxDevices) return 148;
    if (!cache[dev]) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
        cache[dev] = n;
    }
    return cache[dev];
}

// Opt a kernel in to large dynamic shared memory once per device.
template <typename K>
cudaError_t smem_optin(K kern, int bytes, uint64_t* done_mask_per_dev) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < kMaxDevices && (done_mask_per_dev[dev] >> 0 & 1ull)) return cudaSuccess;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e == cudaSuccess && dev >= 0 && dev < kMaxDevices) done_mask_per_dev[dev] |= 1ull;
    return e;
}

template <typename... KArgs, typename... Args>
cudaError_t launch(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s, bool pdl,
                   Args... args) {
    cudaLaunchConfig_t cfg;
    std::memset(&cfg, 0, sizeof(cfg));
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = pdl ? attr : nullptr;
    cfg.numAttrs = pdl ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
}

inline elq_status cuda_status(cudaError_t e) { return e == cudaSuccess ? ELQ_OK : ELQ_ERR_CUDA; }

bool fmt_ok(int32_t f) { return f == ELQ_Q8_0 || f == ELQ_Q4_0; }
int slab_bytes(int32_t f) { return f == ELQ_Q8_0 ? kQ80Slab : kQ40Slab; }

elq_status check_qmat(const elq_qmat* w, int32_t rows, int32_t k) {
    if (!w) return ELQ_ERR_INVALID_ARG;
    if (!fmt_ok(w->fmt)) return ELQ_ERR_UNSUPPORTED;
    if (w->n_rows != rows || w->k != k || rows <= 0 || k <= 0) return ELQ_ERR_INVALID_ARG;
    if (rows % kTileRows || k % 32) return ELQ_ERR_UNSUPPORTED;
    if (!w->q || !w->d) return ELQ_ERR_INVALID_ARG;
    if (!aligned(w->q, 256) || !aligned(w->d, 256)) return ELQ_ERR_ALIGNMENT;
    return ELQ_OK;
}

// ---------------------------------------------------------------------------
// GEMV planning

struct GemvPlan {
    int split;      // 1: per-chunk units with ordered partial completion
    int grid;
    size_t partial_bytes;
    size_t counter_ints;
};

// groups_max: upper bound on active groups (1 for dense); tok_rows: rows of
// the partial buffer's token dimension (T or P).
GemvPlan plan_gemv(int n_rows_per_group, int k, int groups_max, int64_t tok_rows) {
    GemvPlan p;
    const int sms = sm_count();
    const int tiles = n_rows_per_group / kTileRows;
    const int nchunks = (k / 32 + kChunk - 1) / kChunk;
    const int64_t units_whole = (int64_t)groups_max * tiles;
    p.split = (units_whole < 2 * sms && nchunks > 1) ? 1 : 0;
    p.grid = sms;
    p.partial_bytes = p.split ? (size_t)nchunks * tok_rows * tiles * kTileRows * sizeof(float) : 0;
    p.counter_ints = p.split ? (size_t)groups_max * tiles : 0;
    return p;
}

uint64_t g_smem_done_q80[kMaxDevices], g_smem_done_q40[kMaxDevices], g_smem_done_router[kMaxDevices],
    g_smem_done_bucket[kMaxDevices];

cudaError_t launch_gemv(const GemvArgs& g, int fmt, int grid, cudaStream_t s, bool pdl) {
    if (fmt == ELQ_Q8_0) {
        cudaError_t e = smem_optin(k_qgemv<8>, GemvSmem<8>::kTotal, g_smem_done_q80);
        if (e != cudaSuccess) return e;
        return launch(k_qgemv<8>, dim3(grid), dim3(kGemvThreads), GemvSmem<8>::kTotal, s, pdl, g);
    }
    cudaError_t e = smem_optin(k_qgemv<2>, GemvSmem<2>::kTotal, g_smem_done_q40);
    if (e != cudaSuccess) return e;
    return launch(k_qgemv<2>, dim3(grid), dim3(kGemvThreads), GemvSmem<2>::kTotal, s, pdl, g);
}

GemvArgs dense_args(const elq_qmat* w, int T, const void* x, int out_mode, float* y, uint8_t* yq,
                    const GemvPlan& pl, float* partial, int* counters, int* err) {
    GemvArgs g;
    std::memset(&g, 0, sizeof(g));
    g.q = static_cast<const uint8_t*>(w->q);
    g.d = static_cast<const uint16_t*>(w->d);
    g.nb = w->k / 32;
    g.tiles = w->n_rows / kTileRows;
    g.nchunks = (g.nb + kChunk - 1) / kChunk;
    g.split = pl.split;
    g.T = T;
    g.kslots = 1;
    g.x = static_cast<const uint8_t*>(x);
    g.x_mode = X_DENSE;
    g.out_mode = out_mode;
    g.y = y;
    g.y_ld = w->n_rows;
    g.yq = yq;
    g.yq_ld = w->n_rows / 32;
    g.partial = partial;
    g.part_tok = T;
    g.counters = counters;
    g.err = err;
    g.budget_ns = kWaitBudgetNs;
    return g;
}

// ---------------------------------------------------------------------------
// Workspace layouts

struct Carve {
    size_t off = 0;
    template <typename T>
    T* take(void* base, size_t bytes) {
        T* p = base ? reinterpret_cast<T*>(static_cast<char*>(base) + off) : nullptr;
        off = round_up(off + bytes, 256);
        return p;
    }
};

struct ProjWs {
    int* err;
    int* counters;
    float* partial;
    size_t total;
};

ProjWs proj_layout(const elq_qmat* w, int T, void* base, GemvPlan* plan_out) {
    GemvPlan pl = plan_gemv(w->n_rows, w->k, 1, T);
    Carve c;
    ProjWs ws;
    ws.err = c.take<int>(base, 256 + pl.counter_ints * sizeof(int));
    ws.counters = ws.err ? ws.err + 64 : nullptr;
    ws.partial = c.take<float>(base, pl.partial_bytes);
    ws.total = c.off;
    if (plan_out) *plan_out = pl;
    return ws;
}

struct LayerWs {
    int* err;               // error word, then counters
    int* cnt_router;        // ceil(T/8) + 1
    int* cnt_d;             // D projection tiles
    int* cnt_gu;            // gate/up (group, tile)
    int* cnt_dn;            // down
    int* cnt_u;             // U projection
    uint8_t* xq;
    float* z;
    uint8_t* zq;
    float* logits;
    int32_t* idx;
    float* wts;
    int32_t *counts, *offsets, *perm, *pos, *act, *n_act;
    uint8_t* hq;
    float* o;
    float* ylat;
    uint8_t* ylq;
    float* partial;
    GemvPlan pd, pgu, pdn, pu;
    size_t total;
};

LayerWs layer_layout(const elq_layer* ly, int T, void* base) {
    LayerWs w;
    const int H = ly->H, L = ly->L, E = ly->E, k = ly->k, I = ly->I;
    const int64_t P = (int64_t)T * k;
    const int gmax = (int)std::min<int64_t>(E, P);
    w.pd = plan_gemv(L, H, 1, T);
    w.pgu = plan_gemv(2 * I, L, gmax, P);
    w.pdn = plan_gemv(L, I, gmax, P);
    w.pu = plan_gemv(H, L, 1, T);
    const int rblocks = (T + kRouterTok - 1) / kRouterTok;
    const size_t n_cnt = 64 + (rblocks + 1) + w.pd.counter_ints + w.pgu.counter_ints + w.pdn.counter_ints +
                         w.pu.counter_ints;
    Carve c;
    w.err = c.take<int>(base, n_cnt * sizeof(int));
    int* cur = w.err ? w.err + 64 : nullptr;
    auto adv = [&](size_t n) { int* r = cur; if (cur) cur += n; return r; };
    w.cnt_router = adv(rblocks + 1);
    w.cnt_d = adv(w.pd.counter_ints);
    w.cnt_gu = adv(w.pgu.counter_ints);
    w.cnt_dn = adv(w.pdn.counter_ints);
    w.cnt_u = adv(w.pu.counter_ints);
    w.xq = c.take<uint8_t>(base, (size_t)T * (H / 32) * 36);
    w.z = c.take<float>(base, (size_t)T * L * 4);
    w.zq = c.take<uint8_t>(base, (size_t)T * (L / 32) * 36);
    w.logits = c.take<float>(base, (size_t)T * E * 4);
    w.idx = c.take<int32_t>(base, (size_t)P * 4);
    w.wts = c.take<float>(base, (size_t)P * 4);
    w.counts = c.take<int32_t>(base, (size_t)E * 4);
    w.offsets = c.take<int32_t>(base, (size_t)(E + 1) * 4);
    w.perm = c.take<int32_t>(base, (size_t)P * 4);
    w.pos = c.take<int32_t>(base, (size_t)P * 4);
    w.act = c.take<int32_t>(base, (size_t)E * 4);
    w.n_act = c.take<int32_t>(base, 4);
    w.hq = c.take<uint8_t>(base, (size_t)P * (I / 32) * 36);
    w.o = c.take<float>(base, (size_t)P * L * 4);
    w.ylat = c.take<float>(base, (size_t)T * L * 4);
    w.ylq = c.take<uint8_t>(base, (size_t)T * (L / 32) * 36);
    const size_t part = std::max(std::max(w.pd.partial_bytes, w.pgu.partial_bytes),
                                 std::max(w.pdn.partial_bytes, w.pu.partial_bytes));
    w.partial = c.take<float>(base, part);
    w.total = c.off;
    return w;
}

elq_status check_layer(const elq_layer* ly, int32_t T) {
    if (!ly) return ELQ_ERR_INVALID_ARG;
    if (T < 0) return ELQ_ERR_INVALID_ARG;
    const int H = ly->H, L = ly->L, E = ly->E, k = ly->k, I = ly->I;
    if (H <= 0 || L <= 0 || E <= 0 || k <= 0 || I <= 0) return ELQ_ERR_INVALID_ARG;
    if (k > E) return ELQ_ERR_INVALID_ARG;
    if (k > 32 || E > 1024) return ELQ_ERR_UNSUPPORTED;
    if (H % kTileRows || L % kTileRows || I % 64) return ELQ_ERR_UNSUPPORTED;
    if ((int64_t)T * k > (int64_t)1 << 30) return ELQ_ERR_UNSUPPORTED;
    elq_status s;
    if ((s = check_qmat(&ly->D, L, H)) != ELQ_OK) return s;
    if ((s = check_qmat(&ly->U, H, L)) != ELQ_OK) return s;
    if ((int64_t)E * 2 * I > INT32_MAX || (int64_t)E * L > INT32_MAX) return ELQ_ERR_UNSUPPORTED;
    if ((s = check_qmat(&ly->gate_up, E * 2 * I, L)) != ELQ_OK) return s;
    if ((s = check_qmat(&ly->down, E * L, I)) != ELQ_OK) return s;
    if (!ly->router_w) return ELQ_ERR_INVALID_ARG;
    if (!aligned(ly->router_w, 16) || (ly->router_bias && !aligned(ly->router_bias, 4))) return ELQ_ERR_ALIGNMENT;
    return ELQ_OK;
}

size_t router_smem(int T, int L, int E) {
    const int nt = std::min(T, kRouterTok);
    size_t a = (size_t)nt * L * 4;
    size_t b = (size_t)kRouterWarps * E * 4;
    return std::max(a, b);
}

cudaError_t launch_router(const float* z, const float* w, const float* bias, int T, int L, int E, int k,
                          int32_t* idx, float* wts, float* logits, int* cnt, bool do_bucket, int32_t* counts,
                          int32_t* offsets, int32_t* perm, int32_t* pos, int32_t* act, int32_t* n_act,
                          cudaStream_t s, bool pdl) {
    RouterArgs a;
    a.z = z; a.w = w; a.bias = bias; a.T = T; a.L = L; a.E = E; a.k = k;
    a.idx = idx; a.wts = wts; a.logits = logits;
    const int rblocks = (T + kRouterTok - 1) / kRouterTok;
    a.cnt_tok = cnt;
    a.cnt_all = cnt ? cnt + rblocks : nullptr;
    a.do_bucket = do_bucket ? 1 : 0;
    a.counts = counts; a.offsets = offsets; a.perm = perm; a.pos = pos; a.act = act; a.n_act = n_act;
    const size_t sm = router_smem(T, L, E);
    cudaError_t e = smem_optin(k_router, 227 * 1024, g_smem_done_router);
    if (e != cudaSuccess) return e;
    dim3 grid((E + kRouterWarps - 1) / kRouterWarps, rblocks);
    return launch(k_router, grid, dim3(kRouterWarps * 32), sm, s, pdl, a);
}

bool router_shape_ok(int T, int L, int E) { return router_smem(T, L, E) <= 227 * 1024; }

}  // namespace

// ===========================================================================
extern "C" {

const char* elq_status_string(int32_t status) {
    switch (status) {
    case ELQ_OK: return "ok";
    case ELQ_ERR_INVALID_ARG: return "invalid argument";
    case ELQ_ERR_UNSUPPORTED: return "unsupported format or shape";
    case ELQ_ERR_ALIGNMENT: return "misaligned pointer";
    case ELQ_ERR_WORKSPACE: return "workspace missing or too small";
    case ELQ_ERR_CUDA: return "CUDA runtime error";
    case ELQ_ERR_TIMEOUT: return "bounded device wait timed out";
    default: return "unknown status";
    }
}

int32_t elq_version(void) { return 1; }

size_t elq_arena_bytes(int32_t fmt, int32_t n_rows, int32_t k, size_t* q_bytes, size_t* d_bytes) {
    if (!fmt_ok(fmt) || n_rows <= 0 || k <= 0 || n_rows % kTileRows || k % 32) {
        if (q_bytes) *q_bytes = 0;
        if (d_bytes) *d_bytes = 0;
        return 0;
    }
    const size_t slabs = (size_t)(n_rows / kTileRows) * (k / 32);
    const size_t q = slabs * slab_bytes(fmt), d = slabs * kScaleSlab;
    if (q_bytes) *q_bytes = q;
    if (d_bytes) *d_bytes = d;
    return q + d;
}

elq_status elq_arena_pack(int32_t fmt, const void* aos, int32_t n_rows, int32_t k, void* q_out, void* d_out,
                          void* stream) {
    if (!fmt_ok(fmt)) return ELQ_ERR_UNSUPPORTED;
    if (!aos || !q_out || !d_out || n_rows <= 0 || k <= 0) return ELQ_ERR_INVALID_ARG;
    if (n_rows % kTileRows || k % 32) return ELQ_ERR_UNSUPPORTED;
    if (!aligned(q_out, 256) || !aligned(d_out, 256)) return ELQ_ERR_ALIGNMENT;
    const int64_t n = (int64_t)n_rows * (k / 32);
    const dim3 grid((unsigned)((n + 255) / 256));
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (fmt == ELQ_Q8_0)
        k_arena_pack<8><<<grid, 256, 0, s>>>(static_cast<const uint8_t*>(aos), n_rows, k,
                                             static_cast<uint8_t*>(q_out), static_cast<uint16_t*>(d_out));
    else
        k_arena_pack<2><<<grid, 256, 0, s>>>(static_cast<const uint8_t*>(aos), n_rows, k,
                                             static_cast<uint8_t*>(q_out), static_cast<uint16_t*>(d_out));
    return cuda_status(cudaGetLastError());
}

static elq_status quant_weights_impl(int32_t fmt, const float* w, const float* w2, int mode, int32_t n_rows,
                                     int32_t k, int32_t I, void* q_out, void* d_out, void* stream) {
    const int64_t n = (int64_t)n_rows * (k / 32);
    const dim3 grid((unsigned)((n + 255) / 256));
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (fmt == ELQ_Q8_0)
        k_quant_weights<8><<<grid, 256, 0, s>>>(w, w2, mode, n_rows, k, I, static_cast<uint8_t*>(q_out),
                                                static_cast<uint16_t*>(d_out));
    else
        k_quant_weights<2><<<grid, 256, 0, s>>>(w, w2, mode, n_rows, k, I, static_cast<uint8_t*>(q_out),
                                                static_cast<uint16_t*>(d_out));
    return cuda_status(cudaGetLastError());
}

elq_status elq_quantize_weights(int32_t fmt, const float* w, int32_t n_rows, int32_t k, void* q_out,
                                void* d_out, void* stream) {
    if (!fmt_ok(fmt)) return ELQ_ERR_UNSUPPORTED;
    if (!w || !q_out || !d_out || n_rows <= 0 || k <= 0) return ELQ_ERR_INVALID_ARG;
    if (n_rows % kTileRows || k % 32) return ELQ_ERR_UNSUPPORTED;
    if (!aligned(w, 16)) return ELQ_ERR_ALIGNMENT;
    if (!aligned(q_out, 256) || !aligned(d_out, 256)) return ELQ_ERR_ALIGNMENT;
    return quant_weights_impl(fmt, w, nullptr, 0, n_rows, k, 0, q_out, d_out, stream);
}

elq_status elq_quantize_gate_up(int32_t fmt, const float* gate, const float* up, int32_t E, int32_t I,
                                int32_t L, void* q_out, void* d_out, void* stream) {
    if (!fmt_ok(fmt)) return ELQ_ERR_UNSUPPORTED;
    if (!gate || !up || !q_out || !d_out || E <= 0 || I <= 0 || L <= 0) return ELQ_ERR_INVALID_ARG;
    if (I % 64 || L % 32) return ELQ_ERR_UNSUPPORTED;
    if ((int64_t)E * 2 * I > INT32_MAX) return ELQ_ERR_UNSUPPORTED;
    if (!aligned(gate, 16) || !aligned(up, 16)) return ELQ_ERR_ALIGNMENT;
    if (!aligned(q_out, 256) || !aligned(d_out, 256)) return ELQ_ERR_ALIGNMENT;
    return quant_weights_impl(fmt, gate, up, 1, E * 2 * I, L, I, q_out, d_out, stream);
}

elq_status elq_quantize_q8_1(const void* x, int32_t x_type, int64_t rows, int64_t cols, void* out_q8_1,
                             void* stream) {
    if (x_type != ELQ_F32 && x_type != ELQ_BF16) return ELQ_ERR_UNSUPPORTED;
    if (rows < 0 || cols <= 0) return ELQ_ERR_INVALID_ARG;
    if (cols % 32) return ELQ_ERR_UNSUPPORTED;
    if (rows == 0) return ELQ_OK;
    if (!x || !out_q8_1) return ELQ_ERR_INVALID_ARG;
    if (!aligned(x, 4) || !aligned(out_q8_1, 4)) return ELQ_ERR_ALIGNMENT;
    const int64_t nblk = rows * (cols / 32);
    const dim3 grid((unsigned)((nblk * 32 + 255) / 256));
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (x_type == ELQ_BF16)
        return cuda_status(launch(k_quant_q8_1<true>, grid, dim3(256), 0, s, false, x, nblk,
                                  static_cast<uint8_t*>(out_q8_1)));
    return cuda_status(launch(k_quant_q8_1<false>, grid, dim3(256), 0, s, false, x, nblk,
                              static_cast<uint8_t*>(out_q8_1)));
}

elq_status elq_router_topk(const float* z, const float* w_router, const float* bias, int32_t T, int32_t L,
                           int32_t E, int32_t k, int32_t* idx, float* weights, float* logits, void* stream) {
    if (T < 0 || L <= 0 || E <= 0 || k <= 0 || k > E) return ELQ_ERR_INVALID_ARG;
    if (k > 32 || E > 1024 || L % 32) return ELQ_ERR_UNSUPPORTED;
    if (T == 0) return ELQ_OK;
    if (!z || !w_router || !idx || !weights || !logits) return ELQ_ERR_INVALID_ARG;
    if (!aligned(z, 4) || !aligned(w_router, 4) || (bias && !aligned(bias, 4)) || !aligned(idx, 4) ||
        !aligned(weights, 4) || !aligned(logits, 4))
        return ELQ_ERR_ALIGNMENT;
    if (!router_shape_ok(T, L, E)) return ELQ_ERR_UNSUPPORTED;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaError_t e = launch_router(z, w_router, bias, T, L, E, k, idx, weights, logits, nullptr, false, nullptr,
                                  nullptr, nullptr, nullptr, nullptr, nullptr, s, false);
    if (e != cudaSuccess) return ELQ_ERR_CUDA;
    e = launch(k_topk, dim3((T + 3) / 4), dim3(128), (size_t)4 * E * 4, s, true, (const float*)logits, (int)T,
               (int)E, (int)k, idx, weights);
    return cuda_status(e);
}

elq_status elq_route_bucket(const int32_t* idx, int32_t T, int32_t k, int32_t E, int32_t* counts,
                            int32_t* offsets, int32_t* perm, int32_t* pos, void* stream) {
    if (T < 0 || k <= 0 || E <= 0 || k > E) return ELQ_ERR_INVALID_ARG;
    if (E > 1024 || (int64_t)T * k > (int64_t)1 << 30) return ELQ_ERR_UNSUPPORTED;
    if (!counts || !offsets) return ELQ_ERR_INVALID_ARG;
    if (T > 0 && (!idx || !perm || !pos)) return ELQ_ERR_INVALID_ARG;
    if (!aligned(counts, 4) || !aligned(offsets, 4) || (idx && !aligned(idx, 4)) || (perm && !aligned(perm, 4)) ||
        (pos && !aligned(pos, 4)))
        return ELQ_ERR_ALIGNMENT;
    const int nw = 32;
    cudaError_t e = smem_optin(k_bucket, 227 * 1024, g_smem_done_bucket);
    if (e != cudaSuccess) return ELQ_ERR_CUDA;
    e = launch(k_bucket, dim3(1), dim3(nw * 32), (size_t)nw * E * 4, static_cast<cudaStream_t>(stream), false, idx,
               (int)(T * k), (int)E, counts, offsets, perm, pos, (int32_t*)nullptr, (int32_t*)nullptr);
    return cuda_status(e);
}

size_t elq_latent_proj_workspace_bytes(const elq_qmat* w, int32_t T) {
    if (!w || T <= 0 || check_qmat(w, w->n_rows, w->k) == ELQ_ERR_UNSUPPORTED) return 0;
    if (!fmt_ok(w->fmt) || w->n_rows <= 0 || w->k <= 0 || w->n_rows % kTileRows || w->k % 32) return 0;
    return proj_layout(w, T, nullptr, nullptr).total;
}

elq_status elq_latent_proj(const elq_qmat* w, const void* x_q8_1, int32_t T, float* y, void* ws, size_t ws_bytes,
                           void* stream) {
    if (!w) return ELQ_ERR_INVALID_ARG;
    elq_status st = check_qmat(w, w->n_rows, w->k);
    if (st != ELQ_OK) return st;
    if (T < 0) return ELQ_ERR_INVALID_ARG;
    if (T == 0) return ELQ_OK;
    if (!x_q8_1 || !y) return ELQ_ERR_INVALID_ARG;
    if (!aligned(x_q8_1, 4) || !aligned(y, 16)) return ELQ_ERR_ALIGNMENT;
    GemvPlan pl;
    ProjWs lay = proj_layout(w, T, ws, &pl);
    if (!ws || ws_bytes < lay.total) return ELQ_ERR_WORKSPACE;
    if (!aligned(ws, 256)) return ELQ_ERR_ALIGNMENT;
    GemvArgs g = dense_args(w, T, x_q8_1, OUT_F32, y, nullptr, pl, lay.partial, lay.counters, lay.err);
    return cuda_status(launch_gemv(g, w->fmt, pl.grid, static_cast<cudaStream_t>(stream), false));
}

size_t elq_workspace_bytes(const elq_layer* layer, int32_t T) {
    if (check_layer(layer, T) != ELQ_OK || T <= 0) return 0;
    return layer_layout(layer, T, nullptr).total;
}

static elq_status run_experts(const elq_layer* ly, const LayerWs& w, int T, const uint8_t* zq, float* y_lat,
                              cudaStream_t s, bool pdl, std::function<bool()> mark = std::function<bool()>()) {
    auto marked = [&]() { return !mark || mark(); };
    const int L = ly->L, k = ly->k, I = ly->I;
    const int64_t P = (int64_t)T * k;
    // a6 + a7: gate/up with SwiGLU and Q8_1 requant -> hq by pair position
    GemvArgs g;
    std::memset(&g, 0, sizeof(g));
    g.q = static_cast<const uint8_t*>(ly->gate_up.q);
    g.d = static_cast<const uint16_t*>(ly->gate_up.d);
    g.nb = L / 32;
    g.tiles = 2 * I / kTileRows;
    g.nchunks = (g.nb + kChunk - 1) / kChunk;
    g.q_gstride = (int64_t)g.tiles * g.nb * slab_bytes(ly->gate_up.fmt);
    g.d_gstride = (int64_t)g.tiles * g.nb * kTileRows;
    g.split = w.pgu.split;
    g.act = w.act; g.n_act = w.n_act; g.offsets = w.offsets; g.perm = w.perm; g.kslots = k; g.T = T;
    g.x = zq; g.x_mode = X_PAIR_TOKEN;
    g.out_mode = OUT_SWIGLU;
    g.yq = w.hq; g.yq_ld = I / 32;
    g.partial = w.partial; g.part_tok = P; g.counters = w.cnt_gu; g.err = w.err; g.budget_ns = kWaitBudgetNs;
    cudaError_t e = launch_gemv(g, ly->gate_up.fmt, w.pgu.grid, s, pdl);
    if (e != cudaSuccess || !marked()) return ELQ_ERR_CUDA;
    // a8: down -> o by pair position
    GemvArgs h;
    std::memset(&h, 0, sizeof(h));
    h.q = static_cast<const uint8_t*>(ly->down.q);
    h.d = static_cast<const uint16_t*>(ly->down.d);
    h.nb = I / 32;
    h.tiles = L / kTileRows;
    h.nchunks = (h.nb + kChunk - 1) / kChunk;
    h.q_gstride = (int64_t)h.tiles * h.nb * slab_bytes(ly->down.fmt);
    h.d_gstride = (int64_t)h.tiles * h.nb * kTileRows;
    h.split = w.pdn.split;
    h.act = w.act; h.n_act = w.n_act; h.offsets = w.offsets; h.perm = w.perm; h.kslots = k; h.T = T;
    h.x = w.hq; h.x_mode = X_POSITION;
    h.out_mode = OUT_F32;
    h.y = w.o; h.y_ld = L;
    h.partial = w.partial; h.part_tok = P; h.counters = w.cnt_dn; h.err = w.err; h.budget_ns = kWaitBudgetNs;
    e = launch_gemv(h, ly->down.fmt, w.pdn.grid, s, pdl);
    if (e != cudaSuccess || !marked()) return ELQ_ERR_CUDA;
    // a9: combine + Q8_1
    e = launch(k_combine, dim3(T, (L + 255) / 256), dim3(256), 0, s, pdl, (const float*)w.o,
               (const int32_t*)w.pos, (const float*)w.wts, k, L, y_lat, w.ylq);
    if (e != cudaSuccess || !marked()) return ELQ_ERR_CUDA;
    return ELQ_OK;
}

elq_status elq_moe_experts_grouped(const elq_layer* layer, const void* z_q8_1, const int32_t* idx,
                                   const float* weights, int32_t T, float* y_lat, void* ws, size_t ws_bytes,
                                   void* stream) {
    elq_status st = check_layer(layer, T);
    if (st != ELQ_OK) return st;
    if (T == 0) return ELQ_OK;
    if (!z_q8_1 || !idx || !weights || !y_lat) return ELQ_ERR_INVALID_ARG;
    if (!aligned(z_q8_1, 4) || !aligned(idx, 4) || !aligned(weights, 4) || !aligned(y_lat, 16))
        return ELQ_ERR_ALIGNMENT;
    LayerWs w = layer_layout(layer, T, ws);
    if (!ws || ws_bytes < w.total) return ELQ_ERR_WORKSPACE;
    if (!aligned(ws, 256)) return ELQ_ERR_ALIGNMENT;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const int E = layer->E, k = layer->k;
    const int64_t P = (int64_t)T * k;
    // bucketing on one CTA; the combine reads the caller's weights
    const int nw = 32;
    cudaError_t e = smem_optin(k_bucket, 227 * 1024, g_smem_done_bucket);
    if (e != cudaSuccess) return ELQ_ERR_CUDA;
    e = launch(k_bucket, dim3(1), dim3(nw * 32), (size_t)nw * E * 4, s, false, idx, (int)P, E, w.counts,
               w.offsets, w.perm, w.pos, w.act, w.n_act);
    if (e != cudaSuccess) return ELQ_ERR_CUDA;
    LayerWs w2 = w;
    w2.wts = const_cast<float*>(weights);
    return run_experts(layer, w2, T, static_cast<const uint8_t*>(z_q8_1), y_lat, s, true);
}

static elq_status run_layer(const elq_layer* layer, const void* x, int32_t x_type, int32_t T, float* y, void* ws,
                            size_t ws_bytes, void* stream, void* const* events, int32_t n_events) {
    elq_status st = check_layer(layer, T);
    if (st != ELQ_OK) return st;
    if (x_type != ELQ_F32 && x_type != ELQ_BF16) return ELQ_ERR_UNSUPPORTED;
    if (T == 0) return ELQ_OK;
    if (!x || !y) return ELQ_ERR_INVALID_ARG;
    if (!aligned(x, 4) || !aligned(y, 16)) return ELQ_ERR_ALIGNMENT;
    if (events && n_events < kLayerKernels + 1) return ELQ_ERR_INVALID_ARG;
    if (!router_shape_ok(T, layer->L, layer->E)) return ELQ_ERR_UNSUPPORTED;
    LayerWs w = layer_layout(layer, T, ws);
    if (!ws || ws_bytes < w.total) return ELQ_ERR_WORKSPACE;
    if (!aligned(ws, 256)) return ELQ_ERR_ALIGNMENT;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const int H = layer->H, L = layer->L, E = layer->E, k = layer->k;
    int ev = 0;
    auto mark = [&]() -> bool {
        if (!events) return true;
        return cudaEventRecord(static_cast<cudaEvent_t>(events[ev++]), s) == cudaSuccess;
    };
    const bool pdl = (events == nullptr);
    cudaError_t e;
    if (!mark()) return ELQ_ERR_CUDA;
    // a1
    const int64_t nblk = (int64_t)T * (H / 32);
    if (x_type == ELQ_BF16)
        e = launch(k_quant_q8_1<true>, dim3((unsigned)((nblk * 32 + 255) / 256)), dim3(256), 0, s, false, x, nblk,
                   w.xq);
    else
        e = launch(k_quant_q8_1<false>, dim3((unsigned)((nblk * 32 + 255) / 256)), dim3(256), 0, s, false, x,
                   nblk, w.xq);
    if (e != cudaSuccess || !mark()) return ELQ_ERR_CUDA;
    // a2 + a4: z and zq
    GemvArgs gd = dense_args(&layer->D, T, w.xq, OUT_F32_Q81, w.z, w.zq, w.pd, w.partial, w.cnt_d, w.err);
    if (launch_gemv(gd, layer->D.fmt, w.pd.grid, s, pdl) != cudaSuccess || !mark()) return ELQ_ERR_CUDA;
    // a3 + a5
    e = launch_router(w.z, layer->router_w, layer->router_bias, T, L, E, k, w.idx, w.wts, w.logits, w.cnt_router,
                      true, w.counts, w.offsets, w.perm, w.pos, w.act, w.n_act, s, pdl);
    if (e != cudaSuccess || !mark()) return ELQ_ERR_CUDA;
    // a6 - a9
    st = run_experts(layer, w, T, w.zq, w.ylat, s, pdl, events ? [&]() { return mark(); } : std::function<bool()>());
    if (st != ELQ_OK) return st;
    // a10
    GemvArgs gu = dense_args(&layer->U, T, w.ylq, OUT_F32, y, nullptr, w.pu, w.partial, w.cnt_u, w.err);
    if (launch_gemv(gu, layer->U.fmt, w.pu.grid, s, pdl) != cudaSuccess || !mark()) return ELQ_ERR_CUDA;
    return ELQ_OK;
}

elq_status elq_moe_layer(const elq_layer* layer, const void* x, int32_t x_type, int32_t T, float* y, void* ws,
                         size_t ws_bytes, void* stream) {
    return run_layer(layer, x, x_type, T, y, ws, ws_bytes, stream, nullptr, 0);
}

int32_t elq_layer_kernel_count(void) { return kLayerKernels; }

elq_status elq_moe_layer_profiled(const elq_layer* layer, const void* x, int32_t x_type, int32_t T, float* y,
                                  void* ws, size_t ws_bytes, void* const* events, int32_t n_events, void* stream) {
    if (!events) return ELQ_ERR_INVALID_ARG;
    for (int i = 0; i < n_events && i < kLayerKernels + 1; ++i)
        if (!events[i]) return ELQ_ERR_INVALID_ARG;
    return run_layer(layer, x, x_type, T, y, ws, ws_bytes, stream, events, n_events);
}

elq_status elq_workspace_view(const elq_layer* layer, int32_t T, int32_t which, size_t* offset, size_t* bytes) {
    if (check_layer(layer, T) != ELQ_OK || T <= 0 || !offset || !bytes) return ELQ_ERR_INVALID_ARG;
    char* const base = reinterpret_cast<char*>((uintptr_t)1 << 40);   // only offsets are taken
    LayerWs w = layer_layout(layer, T, base);
    const size_t Tz = (size_t)T, P = (size_t)T * layer->k, L = layer->L, H = layer->H, E = layer->E,
                 I = layer->I;
    const void* p = nullptr;
    size_t n = 0;
    switch (which) {
    case 0: p = w.xq; n = Tz * (H / 32) * 36; break;
    case 1: p = w.z; n = Tz * L * 4; break;
    case 2: p = w.zq; n = Tz * (L / 32) * 36; break;
    case 3: p = w.logits; n = Tz * E * 4; break;
    case 4: p = w.idx; n = P * 4; break;
    case 5: p = w.wts; n = P * 4; break;
    case 6: p = w.counts; n = E * 4; break;
    case 7: p = w.offsets; n = (E + 1) * 4; break;
    case 8: p = w.perm; n = P * 4; break;
    case 9: p = w.pos; n = P * 4; break;
    case 10: p = w.hq; n = P * (I / 32) * 36; break;
    case 11: p = w.o; n = P * L * 4; break;
    case 12: p = w.ylat; n = Tz * L * 4; break;
    case 13: p = w.ylq; n = Tz * (L / 32) * 36; break;
    case 14: p = w.n_act; n = 4; break;
    default: return ELQ_ERR_INVALID_ARG;
    }
    *offset = (size_t)(static_cast<const char*>(p) - base);
    *bytes = n;
    return ELQ_OK;
}

elq_status elq_workspace_status(void* ws, void* stream) {
    if (!ws) return ELQ_ERR_INVALID_ARG;
    int v = 0;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (cudaMemcpyAsync(&v, ws, sizeof(int), cudaMemcpyDeviceToHost, s) != cudaSuccess) return ELQ_ERR_CUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess) return ELQ_ERR_CUDA;
    if (v == 0) return ELQ_OK;
    if (cudaMemsetAsync(ws, 0, sizeof(int), s) != cudaSuccess) return ELQ_ERR_CUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess) return ELQ_ERR_CUDA;
    return ELQ_ERR_TIMEOUT;
}

elq_status elq_test_block_isums(int32_t wfmt, const void* w_aos, const void* x_q8_1, int64_t nblocks,
                                int32_t* isum, float* term, void* stream) {
    if (!fmt_ok(wfmt)) return ELQ_ERR_UNSUPPORTED;
    if (nblocks < 0) return ELQ_ERR_INVALID_ARG;
    if (nblocks == 0) return ELQ_OK;
    if (!w_aos || !x_q8_1 || !isum || !term) return ELQ_ERR_INVALID_ARG;
    k_test_block_isums<<<(unsigned)((nblocks + 255) / 256), 256, 0, static_cast<cudaStream_t>(stream)>>>(
        wfmt, static_cast<const uint8_t*>(w_aos), static_cast<const uint8_t*>(x_q8_1), nblocks, isum, term);
    return cuda_status(cudaGetLastError());
}

elq_status elq_test_expf(const float* in, float* out, int64_t n, void* stream) {
    if (n < 0) return ELQ_ERR_INVALID_ARG;
    if (n == 0) return ELQ_OK;
    if (!in || !out) return ELQ_ERR_INVALID_ARG;
    k_test_expf<<<(unsigned)((n + 255) / 256), 256, 0, static_cast<cudaStream_t>(stream)>>>(in, out, n);
    return cuda_status(cudaGetLastError());
}

}  // extern "C"
