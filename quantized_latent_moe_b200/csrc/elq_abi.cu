// elq_abi.cu -- the C ABI declared in include/elq.h: host-side validation,
// workspace layout and kernel launches.  No allocation, no synchronisation
// (except elq_workspace_status, which is documented as blocking).
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <functional>
#include <mutex>

#include "../../include/elq.h"
#include "elq_decode.cuh"
#include "elq_sgemv.cuh"
#include "elq_nvtc.cuh"

using namespace elq;

namespace {

constexpr uint64_t kWaitBudgetNs = 2000000000ull;   // 2 s per bounded device wait
constexpr int kMaxDevices = 64;
constexpr int kRouterSmemMax = 200 * 1024;           // dynamic shared memory cap of router/bucket
constexpr int kGemvSmemMax = 225 * 1024;             // dynamic shared memory cap of the GEMV
constexpr int kRawMaxT = 8;                          // D quantises x itself up to this many tokens
constexpr int kTcMinT = 16;                          // tensor-core path from this many tokens (Q8_0 weights)

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
cudaError_t smem_optin(K kern, int bytes, bool* done_per_dev) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < kMaxDevices && done_per_dev[dev]) return cudaSuccess;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e == cudaSuccess && dev >= 0 && dev < kMaxDevices) done_per_dev[dev] = true;
    return e;
}

bool g_optin_router[kMaxDevices], g_optin_router2[kMaxDevices], g_optin_bucket[kMaxDevices],
    g_optin_topk[kMaxDevices], g_optin_dec[4][kMaxDevices];

// Cooperative launch: every CTA of the grid is resident at once.
template <typename... KArgs, typename... Args>
cudaError_t launch_coop(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                        Args... args) {
    cudaLaunchConfig_t cfg;
    std::memset(&cfg, 0, sizeof(cfg));
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
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
// formats the arena holds (NVFP4 in the Q4_0 geometry: 16 code bytes and a
// 16-bit scale word per row and block)
bool ext_fmt(int32_t f) { return f == ELQ_Q5_1 || f == ELQ_Q3_K || f == ELQ_Q4_K || f == ELQ_Q5_K; }
bool arena_fmt_ok(int32_t f) { return fmt_ok(f) || f == ELQ_NVFP4 || ext_fmt(f); }
// codes per (tile, block): four slices' pieces (WSlice::kCodes each)
int slab_bytes(int32_t f) { return f == ELQ_Q8_0 ? kQ80Slab : fmt_has_qh(f) ? 4 * 640 : kQ40Slab; }
// k granularity of an arena matrix
int arena_k_unit(int32_t f) {
    return f == ELQ_NVFP4 ? 64 : (f == ELQ_Q3_K || f == ELQ_Q4_K || f == ELQ_Q5_K) ? 256 : 32;
}

// expert: the matrix may also be NVFP4 (with a global scale per gs_rows
// rows), Q5_1, Q4_K or Q5_K (a layer's expert matrices).
elq_status check_qmat(const elq_qmat* w, int32_t rows, int32_t k, bool expert = false) {
    if (!w) return ELQ_ERR_INVALID_ARG;
    if (!(fmt_ok(w->fmt) || (expert && (w->fmt == ELQ_NVFP4 || ext_fmt(w->fmt))))) return ELQ_ERR_UNSUPPORTED;
    if (w->n_rows != rows || w->k != k || rows <= 0 || k <= 0) return ELQ_ERR_INVALID_ARG;
    if (rows % kTileRows || k % 128) return ELQ_ERR_UNSUPPORTED;
    if (!w->q || !w->d) return ELQ_ERR_INVALID_ARG;
    if (!aligned(w->q, 256) || !aligned(w->d, 256)) return ELQ_ERR_ALIGNMENT;
    if ((w->fmt == ELQ_Q3_K || w->fmt == ELQ_Q4_K || w->fmt == ELQ_Q5_K) && k % 256)
        return ELQ_ERR_UNSUPPORTED;   // whole super-blocks
    if (w->fmt == ELQ_NVFP4) {
        if (k % 256) return ELQ_ERR_UNSUPPORTED;   // whole 8-block chunks of 18-byte activation blocks
        if (!w->gs || w->gs_rows <= 0 || rows % w->gs_rows) return ELQ_ERR_INVALID_ARG;
        if (!aligned(w->gs, 4)) return ELQ_ERR_ALIGNMENT;
    }
    if (w->q16) {
        if (w->fmt != ELQ_Q8_0) return ELQ_ERR_UNSUPPORTED;
        if (!aligned(w->q16, 256)) return ELQ_ERR_ALIGNMENT;
    }
    return ELQ_OK;
}

// ---------------------------------------------------------------------------
// GEMV planning

struct WPlan {
    int warps, stages, tokcap, stage_bytes, act_off, act_bytes, scratch_bytes, smem, grid;
    int nchunks, tiles;
    size_t partial_bytes, counter_ints;
};

// rows_per_group: matrix rows of one group; k: reduction length; groups_max:
// bound on active groups; tok_rows: rows of the partial buffer's token
// dimension (T or T*k); tokmax: most tokens one group can hold.
constexpr int kDenseTg = 8;   // tokens per group of a dense projection (the groups share the weights)
constexpr int kGroupTok = 8;  // tokens staged per unit for an expert group (more take extra passes)

int dense_groups(int T) { return (T + kDenseTg - 1) / kDenseTg; }

WPlan plan_w(int fmt, int x_mode, int rows_per_group, int k, int groups_max, int64_t tok_rows, int tokmax) {
    WPlan p;
    p.tiles = rows_per_group / kTileRows;
    p.nchunks = (k / 32 + kChunk - 1) / kChunk;
    p.tokcap = std::max(1, std::min(tokmax, kTokMax));
    p.act_bytes = (x_mode == X_RAW_F32) ? 1024 : (x_mode == X_RAW_BF16) ? 512 : kChunk * 36;
    const int codes = kChunk * (fmt == ELQ_Q8_0 ? 1024 : 512);
    p.act_off = codes + kChunk * 64;
    p.stage_bytes = (int)round_up((size_t)p.act_off + (size_t)p.tokcap * p.act_bytes, 128);
    p.scratch_bytes = (x_mode == X_RAW_F32 || x_mode == X_RAW_BF16) ? (int)round_up((size_t)p.tokcap * 288, 128) : 0;
    static const int cand[][2] = {{8, 3}, {8, 2}, {4, 2}, {2, 2}, {1, 2}};
    p.warps = 0;
    for (const auto& c : cand) {
        const long need = 512 + (long)c[0] * (c[1] * p.stage_bytes + p.scratch_bytes);
        if (need <= kGemvSmemMax) {
            p.warps = c[0];
            p.stages = c[1];
            p.smem = (int)need;
            break;
        }
    }
    p.grid = sm_count();
    p.partial_bytes = (size_t)p.nchunks * tok_rows * p.tiles * kTileRows * sizeof(float);
    p.counter_ints = (size_t)groups_max * p.tiles;
    return p;
}

// One kernel per (format, activation mode, output mode): each launch runs
// only its own code paths, which keeps its instruction footprint small.
template <int FMT, int XM, int OM>
cudaError_t launch_w_t(const WArgs& g, const WPlan& p, cudaStream_t s, bool pdl) {
    static bool optin[kMaxDevices];
    cudaError_t e = smem_optin(k_wgemv<FMT, XM, OM>, kGemvSmemMax, optin);
    if (e != cudaSuccess) return e;
    return launch(k_wgemv<FMT, XM, OM>, dim3(p.grid), dim3(32 * p.warps), p.smem, s, pdl, g);
}

template <int FMT>
cudaError_t launch_w_f(const WArgs& g, const WPlan& p, cudaStream_t s, bool pdl) {
    switch (g.x_mode * 16 + g.out_mode) {
    case X_RAW_BF16 * 16 + OUT_F32_Q81: return launch_w_t<FMT, X_RAW_BF16, OUT_F32_Q81>(g, p, s, pdl);
    case X_RAW_F32 * 16 + OUT_F32_Q81: return launch_w_t<FMT, X_RAW_F32, OUT_F32_Q81>(g, p, s, pdl);
    case X_Q81_TOKEN * 16 + OUT_F32_Q81: return launch_w_t<FMT, X_Q81_TOKEN, OUT_F32_Q81>(g, p, s, pdl);
    case X_Q81_TOKEN * 16 + OUT_F32: return launch_w_t<FMT, X_Q81_TOKEN, OUT_F32>(g, p, s, pdl);
    case X_Q81_TOKEN * 16 + OUT_F32_ADD: return launch_w_t<FMT, X_Q81_TOKEN, OUT_F32_ADD>(g, p, s, pdl);
    case X_Q81_PAIR_TOKEN * 16 + OUT_SWIGLU: return launch_w_t<FMT, X_Q81_PAIR_TOKEN, OUT_SWIGLU>(g, p, s, pdl);
    case X_Q81_POSITION * 16 + OUT_F32_COMBINE: return launch_w_t<FMT, X_Q81_POSITION, OUT_F32_COMBINE>(g, p, s, pdl);
    default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_w(WArgs g, int fmt, const WPlan& p, cudaStream_t s, bool pdl) {
    g.stages = p.stages;
    g.tokcap = p.tokcap;
    g.stage_bytes = p.stage_bytes;
    g.act_off = p.act_off;
    g.act_bytes = p.act_bytes;
    g.scratch_bytes = p.scratch_bytes;
    g.nchunks = p.nchunks;
    g.tiles = p.tiles;
    g.budget_ns = kWaitBudgetNs;
    if (p.warps == 0) return cudaErrorInvalidConfiguration;
    return fmt == ELQ_Q8_0 ? launch_w_f<8>(g, p, s, pdl) : launch_w_f<2>(g, p, s, pdl);
}

WArgs dense_w(const elq_qmat* w, int T, const void* x, int x_mode, int64_t x_row, int out_mode, float* y,
              uint8_t* yq, float* partial, int* counters, int* err) {
    WArgs g;
    std::memset(&g, 0, sizeof(g));
    g.q = static_cast<const uint8_t*>(w->q);
    g.d = static_cast<const uint16_t*>(w->d);
    g.nb = w->k / 32;
    g.kslots = 1;
    g.T = T;
    g.x = x;
    g.x_mode = x_mode;
    g.x_row = x_row;
    g.out_mode = out_mode;
    g.y = y;
    g.y_ld = w->n_rows;
    g.yq = yq;
    g.yq_ld = w->n_rows / 32;
    g.partial = partial;
    g.part_tok = T;
    g.counters = counters;
    g.err = err;
    g.dense_tg = kDenseTg;
    return g;
}

// ---------------------------------------------------------------------------
// Small-T cluster GEMV planning (k_sgemv)

struct SPlan {
    bool ok;
    int C, Cg, cpc, stages, stage_bytes, scales_off, acts_off, act_row, scratch_bytes, pbuf_off, route_off, smem,
        clusters;
    int nchunks, ipg;
};

constexpr int kSSmemMax = 227 * 1024;

// rows_per_group: matrix rows of one group; K: reduction length; groups_max:
// bound on the groups; routed: an expert projection (a group table in shared
// memory).
SPlan plan_s(int fmt, int x_mode, bool swiglu, int rows_per_group, int K, int groups_max, int T, bool routed) {
    SPlan p;
    std::memset(&p, 0, sizeof(p));
    if (T < 1 || T > kSMaxT || groups_max < 1 || groups_max > kSMaxPairs) return p;
    const int nb = K / 32;
    p.nchunks = (nb + kChunk - 1) / kChunk;
    p.ipg = swiglu ? rows_per_group / 64 : rows_per_group / 32;
    const int64_t n_items = (int64_t)groups_max * p.ipg;
    const int sms = sm_count();
    const int halves = swiglu ? 2 : 1;
    // split an item's chunks over Cg CTAs until there are CTAs for every SM
    // (and at most 16 chunks, one per warp, per CTA)
    int Cg = 1;
    while (Cg < p.nchunks && halves * Cg * 2 <= kSMaxCluster &&
           ((p.nchunks + Cg - 1) / Cg > kSMaxWarps || n_items * halves * Cg < sms))
        Cg *= 2;
    if ((p.nchunks + Cg - 1) / Cg > kSMaxWarps) return p;
    p.Cg = Cg;
    p.C = Cg * halves;
    p.cpc = (p.nchunks + Cg - 1) / Cg;
    // one stage of a CTA: the codes and scales of its cpc chunks, then each
    // token's activations over the same blocks
    const int codes = p.cpc * kChunk * (slab_bytes(fmt) / 4);
    const int ablock = x_mode == X_RAW_F32 ? 128 : x_mode == X_RAW_BF16 ? 64 : fmt == ELQ_NVFP4 ? 18 : 36;
    p.scales_off = codes;
    p.acts_off = (int)round_up((size_t)codes + (size_t)p.cpc * kChunk * 64 * scale_units(fmt), 128);
    p.act_row = p.cpc * kChunk * ablock;
    p.stage_bytes = (int)round_up((size_t)p.acts_off + (size_t)T * p.act_row, 128);
    p.scratch_bytes = (x_mode == X_RAW_F32 || x_mode == X_RAW_BF16) ? (int)round_up((size_t)T * kChunk * 36, 128)
                      : fmt == ELQ_NVFP4                        ? (int)round_up((size_t)kSNvScratch, 128)
                                                                : 0;
    const int pbuf = 2 * halves * p.nchunks * T * 128;
    const int route = routed ? (int)round_up((size_t)kSRouteBytes, 128) : 0;
    auto smem_for = [&](int st) { return kSHeader + st * p.stage_bytes + p.cpc * p.scratch_bytes + pbuf + route; };
    // resident CTAs per SM: shared memory (1 KB reserved per CTA), warps, and
    // registers at the launch bound's 64 per thread
    auto per_sm = [&](int smem) {
        const int a = (228 * 1024) / (smem + 1024);
        const int b = 32 / p.cpc, c = 64 / p.cpc;
        return std::max(0, std::min(std::min(a, b), std::min(c, 32)));
    };
    auto clusters_for = [&](int st) {
        const int64_t cap = std::max<int64_t>(1, (int64_t)per_sm(smem_for(st)) * sms / p.C);
        return (int)std::min<int64_t>(n_items, cap);
    };
    if (smem_for(1) > kSSmemMax) return p;
    // rounds of items per cluster: one stage exposes the latency of each
    // round (later rounds' weights come from L2, prefetched at the start),
    // two stages hide every other round but fit fewer CTAs
    const int64_t r1 = (n_items + clusters_for(1) - 1) / clusters_for(1);
    p.stages = 1;
    if (smem_for(2) <= kSSmemMax) {
        const int64_t r2 = (n_items + clusters_for(2) - 1) / clusters_for(2);
        if (r2 + 1 < 2 * r1) p.stages = 2;
    }
    p.clusters = clusters_for(p.stages);
    p.pbuf_off = kSHeader + p.stages * p.stage_bytes + p.cpc * p.scratch_bytes;
    p.route_off = p.pbuf_off + pbuf;
    p.smem = smem_for(p.stages);
    p.ok = true;
    return p;
}

template <int FMT, int XM, int OM>
cudaError_t launch_s_t(const SArgs& g, const SPlan& p, cudaStream_t s, bool pdl) {
    static bool optin[kMaxDevices];
    cudaError_t e = smem_optin(k_sgemv<FMT, XM, OM>, kSSmemMax, optin);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg;
    std::memset(&cfg, 0, sizeof(cfg));
    cfg.gridDim = dim3((unsigned)(p.clusters * p.C));
    cfg.blockDim = dim3((unsigned)(32 * p.cpc));
    cfg.dynamicSmemBytes = (size_t)p.smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[2];
    int na = 0;
    if (p.C > 1) {
        attr[na].id = cudaLaunchAttributeClusterDimension;
        attr[na].val.clusterDim.x = (unsigned)p.C;
        attr[na].val.clusterDim.y = 1;
        attr[na].val.clusterDim.z = 1;
        ++na;
    }
    if (pdl) {
        attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[na].val.programmaticStreamSerializationAllowed = 1;
        ++na;
    }
    cfg.attrs = na ? attr : nullptr;
    cfg.numAttrs = na;
    return cudaLaunchKernelEx(&cfg, k_sgemv<FMT, XM, OM>, g);
}

template <int FMT>
cudaError_t launch_s_f(const SArgs& g, int x_mode, int out_mode, const SPlan& p, cudaStream_t s, bool pdl) {
    switch (x_mode * 16 + out_mode) {
    case X_RAW_BF16 * 16 + OUT_F32_Q81: return launch_s_t<FMT, X_RAW_BF16, OUT_F32_Q81>(g, p, s, pdl);
    case X_RAW_F32 * 16 + OUT_F32_Q81: return launch_s_t<FMT, X_RAW_F32, OUT_F32_Q81>(g, p, s, pdl);
    case X_RAW_BF16 * 16 + OUT_F32_NV: return launch_s_t<FMT, X_RAW_BF16, OUT_F32_NV>(g, p, s, pdl);
    case X_RAW_F32 * 16 + OUT_F32_NV: return launch_s_t<FMT, X_RAW_F32, OUT_F32_NV>(g, p, s, pdl);
    case X_Q81_TOKEN * 16 + OUT_F32: return launch_s_t<FMT, X_Q81_TOKEN, OUT_F32>(g, p, s, pdl);
    case X_Q81_TOKEN * 16 + OUT_F32_ADD: return launch_s_t<FMT, X_Q81_TOKEN, OUT_F32_ADD>(g, p, s, pdl);
    case X_Q81_PAIR_TOKEN * 16 + OUT_SWIGLU: return launch_s_t<FMT, X_Q81_PAIR_TOKEN, OUT_SWIGLU>(g, p, s, pdl);
    case X_Q81_POSITION * 16 + OUT_F32_COMBINE: return launch_s_t<FMT, X_Q81_POSITION, OUT_F32_COMBINE>(g, p, s, pdl);
    default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_s(SArgs g, int fmt, int x_mode, int out_mode, const SPlan& p, cudaStream_t s, bool pdl) {
    if (!p.ok) return cudaErrorInvalidConfiguration;
    g.nchunks = p.nchunks;
    g.items_per_group = p.ipg;
    g.C = p.C;
    g.Cg = p.Cg;
    g.cpc = p.cpc;
    g.stages = p.stages;
    g.stage_bytes = p.stage_bytes;
    g.scales_off = p.scales_off;
    g.acts_off = p.acts_off;
    g.act_row = p.act_row;
    g.scratch_bytes = p.scratch_bytes;
    g.pbuf_off = p.pbuf_off;
    g.route_off = p.route_off;
    g.budget_ns = kWaitBudgetNs;
    const int64_t ctas = (int64_t)p.clusters * p.C;
    for (int r = 0; r < 3; ++r)
        g.pf_share[r] = g.pf[r] ? (int64_t)round_up((size_t)((g.pf_bytes[r] + ctas - 1) / ctas), 256) : 0;
    if (ext_fmt(fmt)) {
        // Q5_1 / Q4_K / Q5_K expert projections only
        const int sel = x_mode * 16 + out_mode;
        if (sel != X_Q81_PAIR_TOKEN * 16 + OUT_SWIGLU && sel != X_Q81_POSITION * 16 + OUT_F32_COMBINE)
            return cudaErrorInvalidValue;
        const bool gu = sel == X_Q81_PAIR_TOKEN * 16 + OUT_SWIGLU;
        switch (fmt) {
        case ELQ_Q5_1:
            return gu ? launch_s_t<kQ51, X_Q81_PAIR_TOKEN, OUT_SWIGLU>(g, p, s, pdl)
                      : launch_s_t<kQ51, X_Q81_POSITION, OUT_F32_COMBINE>(g, p, s, pdl);
        case ELQ_Q3_K:
            return gu ? launch_s_t<kQ3K, X_Q81_PAIR_TOKEN, OUT_SWIGLU>(g, p, s, pdl)
                      : launch_s_t<kQ3K, X_Q81_POSITION, OUT_F32_COMBINE>(g, p, s, pdl);
        case ELQ_Q4_K:
            return gu ? launch_s_t<kQ4K, X_Q81_PAIR_TOKEN, OUT_SWIGLU>(g, p, s, pdl)
                      : launch_s_t<kQ4K, X_Q81_POSITION, OUT_F32_COMBINE>(g, p, s, pdl);
        default:
            return gu ? launch_s_t<kQ5K, X_Q81_PAIR_TOKEN, OUT_SWIGLU>(g, p, s, pdl)
                      : launch_s_t<kQ5K, X_Q81_POSITION, OUT_F32_COMBINE>(g, p, s, pdl);
        }
    }
    if (fmt == ELQ_NVFP4) {
        // NVFP4 expert projections only
        switch (x_mode * 16 + out_mode) {
        case X_Q81_PAIR_TOKEN * 16 + OUT_SWIGLU: return launch_s_t<kNV, X_Q81_PAIR_TOKEN, OUT_SWIGLU>(g, p, s, pdl);
        case X_Q81_POSITION * 16 + OUT_F32_COMBINE:
            return launch_s_t<kNV, X_Q81_POSITION, OUT_F32_COMBINE>(g, p, s, pdl);
        default: return cudaErrorInvalidValue;
        }
    }
    return fmt == ELQ_Q8_0 ? launch_s_f<8>(g, x_mode, out_mode, p, s, pdl) : launch_s_f<2>(g, x_mode, out_mode, p, s, pdl);
}

// A dense projection of T <= 8 tokens on k_sgemv.
SArgs dense_s(const elq_qmat* w, int T, const void* x, int64_t x_row, float* y, uint8_t* yq, int* err) {
    SArgs g;
    std::memset(&g, 0, sizeof(g));
    g.q = static_cast<const uint8_t*>(w->q);
    g.d = static_cast<const uint16_t*>(w->d);
    g.nb = w->k / 32;
    g.groups_max = 1;
    g.route = ROUTE_NONE;
    g.T = T;
    g.k = 1;
    g.x = x;
    g.x_row = x_row;
    g.y = y;
    g.y_ld = w->n_rows;
    g.yq = yq;
    g.yq_ld = w->n_rows / 32;
    g.err = err;
    g.early = 1;
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

int64_t round16(int64_t x) { return (x + 15) / 16 * 16; }

bool tc_path(int fmt, int T) { return fmt == ELQ_Q8_0 && T >= kTcMinT; }

struct ProjWs {
    int* err;
    int* counters;
    float* partial;
    uint8_t* bq;            // tensor-core path: packed activations
    float* bd;
    int64_t bstride;
    bool tc;
    WPlan plan;
    size_t total;
};

// allow_tc: whether the tensor-core path may be chosen (the allocation-free
// entry point always runs the GEMV its scratch bound is stated for).
ProjWs proj_layout(const elq_qmat* w, int T, void* base, bool allow_tc = true) {
    ProjWs ws;
    ws.tc = allow_tc && tc_path(w->fmt, T);
    ws.plan = plan_w(w->fmt, X_Q81_TOKEN, w->n_rows, w->k, dense_groups(T), T, std::min(T, kDenseTg));
    if (ws.tc) {
        ws.plan.partial_bytes = 0;
        ws.plan.counter_ints = 0;
    }
    Carve c;
    ws.err = c.take<int>(base, (64 + ws.plan.counter_ints) * sizeof(int));
    ws.counters = ws.err ? ws.err + 64 : nullptr;
    ws.partial = c.take<float>(base, ws.plan.partial_bytes);
    ws.bstride = round16(T);
    const int nb = w->k / 32;
    ws.bq = ws.tc ? c.take<uint8_t>(base, (size_t)nb * ws.bstride * 32) : nullptr;
    ws.bd = ws.tc ? c.take<float>(base, (size_t)nb * ws.bstride * 4) : nullptr;
    ws.total = c.off;
    return ws;
}

bool g_optin_tc[kMaxDevices];

cudaError_t launch_pack(const PackArgs& a, cudaStream_t s, bool pdl) {
    const int64_t n = a.bstride * a.nb;   // one thread per (block, slot)
    return launch(k_pack_b, dim3((unsigned)((n + 255) / 256)), dim3(256), 0, s, pdl, a);
}

// One kernel per output mode: each launch carries only its own epilogue.
template <int OM, bool F16>
cudaError_t launch_tc_t(const TcArgs& g, cudaStream_t s, bool pdl) {
    static bool optin[kMaxDevices];
    cudaError_t e = smem_optin(k_tcgemm<OM, F16>, tc_smem(F16), optin);
    if (e != cudaSuccess) return e;
    return launch(k_tcgemm<OM, F16>, dim3(sm_count()), dim3(kTcThreads), (size_t)tc_smem(F16), s, pdl, g);
}

// The driver's tensor-map encoder, looked up once through the runtime.
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, []() {
        void* f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
    });
    return fn;
}

bool encode_map(CUtensorMap* m, CUtensorMapDataType dt, cuuint32_t rank, const void* base, const cuuint64_t* dims,
                const cuuint64_t* strides, const cuuint32_t* box) {
    PFN_cuTensorMapEncodeTiled_v12000 fn = tensor_map_encoder();
    if (!fn) return false;
    const cuuint32_t es[5] = {1, 1, 1, 1, 1};
    return fn(m, dt, rank, const_cast<void*>(base), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
              CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// The four tensor maps of a k_tcgemm launch (layouts in TcArgs).  n_groups:
// the matrices of the arena (the experts, or 1).
bool tc_maps(TcArgs& g, int n_groups) {
    const cuuint64_t nb = (cuuint64_t)g.nb, tiles = (cuuint64_t)n_groups * g.rtiles;
    const cuuint64_t slots = (cuuint64_t)g.bstride;
    const cuuint64_t da[4] = {256, 4, nb, tiles}, sa[3] = {nb * 1024, 1024, nb * 4096};
    const cuuint32_t ba[4] = {256, 4, kTcKS, 1};
    const cuuint64_t dd[4] = {32, 4, nb, tiles}, sd[3] = {nb * 64, 64, nb * 256};
    const cuuint32_t bdd[4] = {32, 4, kTcKS, 1};
    const cuuint64_t db[3] = {64, slots / 8, nb}, sb[2] = {256, slots * 32};
    const cuuint32_t bb[3] = {64, kTcN / 8, kTcKS};
    // fp16 codes: [nb][2 halves][slots/8][64 words]
    const cuuint64_t db16[4] = {64, slots / 8, 2, nb}, sb16[3] = {256, slots * 32, slots * 64};
    const cuuint32_t bb16[4] = {64, kTcN / 8, 2, kTcKS};
    const cuuint64_t dbd[2] = {slots, nb}, sbd[1] = {slots * 4};
    const cuuint32_t bbd[2] = {kTcN, kTcKS};
    const bool bmap = g.q16 ? encode_map(&g.tm_b, CU_TENSOR_MAP_DATA_TYPE_UINT32, 4, g.bq, db16, sb16, bb16)
                            : encode_map(&g.tm_b, CU_TENSOR_MAP_DATA_TYPE_UINT32, 3, g.bq, db, sb, bb);
    return encode_map(&g.tm_a, CU_TENSOR_MAP_DATA_TYPE_UINT32, 4, g.q, da, sa, ba) &&
           encode_map(&g.tm_d, CU_TENSOR_MAP_DATA_TYPE_UINT16, 4, g.d, dd, sd, bdd) && bmap &&
           encode_map(&g.tm_bd, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, g.bd, dbd, sbd, bbd);
}

cudaError_t launch_tc(TcArgs g, cudaStream_t s, bool pdl) {
    g.budget_ns = kWaitBudgetNs;
    if (!tc_maps(g, g.n_groups)) return cudaErrorInvalidValue;
    // fp16 operands (kind::f16) when the matrix carries its fp16 codes; int8 (kind::i8) otherwise
    if (g.q16) {
        switch (g.out_mode) {
        case TC_OUT_F32: return launch_tc_t<TC_OUT_F32, true>(g, s, pdl);
        case TC_OUT_F32_Q81: return launch_tc_t<TC_OUT_F32_Q81, true>(g, s, pdl);
        case TC_OUT_SWIGLU: return launch_tc_t<TC_OUT_SWIGLU, true>(g, s, pdl);
        case TC_OUT_F32_ADD: return launch_tc_t<TC_OUT_F32_ADD, true>(g, s, pdl);
        default: return cudaErrorInvalidValue;
        }
    }
    switch (g.out_mode) {
    case TC_OUT_F32: return launch_tc_t<TC_OUT_F32, false>(g, s, pdl);
    case TC_OUT_F32_Q81: return launch_tc_t<TC_OUT_F32_Q81, false>(g, s, pdl);
    case TC_OUT_SWIGLU: return launch_tc_t<TC_OUT_SWIGLU, false>(g, s, pdl);
    case TC_OUT_F32_COMBINE: return launch_tc_t<TC_OUT_F32_COMBINE, false>(g, s, pdl);
    case TC_OUT_F32_ADD: return launch_tc_t<TC_OUT_F32_ADD, false>(g, s, pdl);
    default: return cudaErrorInvalidValue;
    }
}

TcArgs dense_tc(const elq_qmat* w, int T, const uint8_t* bq, const float* bd, int64_t bstride, int out_mode,
                float* y, uint8_t* yq, int* err) {
    TcArgs g;
    std::memset(&g, 0, sizeof(g));
    g.q = static_cast<const uint8_t*>(w->q);
    g.d = static_cast<const uint16_t*>(w->d);
    g.nb = w->k / 32;
    g.rtiles = w->n_rows / kTileRows;
    g.n_groups = 1;
    g.T = T;
    g.bq = bq;
    g.bd = bd;
    g.bstride = bstride;
    g.out_mode = out_mode;
    g.y = y;
    g.y_ld = w->n_rows;
    g.yq = yq;
    g.yq_ld = w->n_rows / 32;
    g.err = err;
    return g;
}

// The fused small-T kernel's shared-memory plan.
constexpr int kDecSmemMax = 227 * 1024;

struct DecPlanH {
    bool ok;
    int stages, stage_bytes, xq_chunks, header, smem;
};

// Chunks of x the largest CTA share of the D units (numbered chunk-major)
// spans, on a grid of `grid` CTAs.
int dec_xq_chunks(int tiles, int nchunks, int grid) {
    const int per_chunk = tiles * 4;
    const int n = per_chunk * nchunks;
    int most = 0;
    for (int b = 0; b < grid; ++b) {
        const int u0 = (int)((int64_t)n * b / grid), u1 = (int)((int64_t)n * (b + 1) / grid);
        if (u1 > u0) most = std::max(most, (u1 - 1) / per_chunk - u0 / per_chunk + 1);
    }
    return most;
}

DecPlanH plan_dec(const elq_layer* ly, int T) {
    DecPlanH d;
    std::memset(&d, 0, sizeof(d));
    if (!(ly->flags & ELQ_LAYER_FUSED)) return d;
    if (T < 1 || T > kDecMaxT || (int64_t)T * ly->k > kDecMaxPairs) return d;
    if (ly->D.fmt != ly->U.fmt || ly->gate_up.fmt != ly->down.fmt) return d;
    if (ly->gate_up.fmt == ELQ_NVFP4 || ext_fmt(ly->gate_up.fmt)) return d;   // the cluster GEMV path only
    if (ly->L / kTileRows > 64) return d;            // latent tiles the shared-memory mirror follows
    auto codes = [](int fmt) { return kChunk * (fmt == ELQ_Q8_0 ? 1024 : 512); };
    const size_t acts = (size_t)T * kChunk * 36;
    size_t need = std::max((size_t)codes(ly->D.fmt), (size_t)codes(ly->gate_up.fmt)) + kChunk * 64 + acts;
    need = std::max(need, (size_t)ly->L * 4);       // a router row
    need = std::max(need, (size_t)4096 + 256);      // the top-k and bucketing scratch
    d.stage_bytes = (int)round_up(need, 128);
    d.xq_chunks = dec_xq_chunks(ly->L / kTileRows, (ly->H / 32 + kChunk - 1) / kChunk, sm_count());
    const size_t xq = round_up((size_t)d.xq_chunks * acts, 128);
    d.header = dec_header_bytes(ly->L, ly->I);
    for (int st = kDecMaxStages; st >= 2; --st) {
        const size_t sm = (size_t)d.header + xq + (size_t)kDecWarps * st * d.stage_bytes;
        if (sm <= (size_t)kDecSmemMax) {
            d.stages = st;
            d.smem = (int)sm;
            d.ok = true;
            break;
        }
    }
    return d;
}

struct LayerWs {
    int* err;               // error word, then counters
    int* cnt_router;        // ceil(T/8) + 1
    int* cnt_d;
    int* cnt_gu;
    int* cnt_dn;
    int* cnt_u;
    int* cnt_comb;          // [T][L/128]
    uint8_t* xq;            // only when T > kRawMaxT
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
    // fused small-T path (one persistent kernel)
    bool fused;
    DecPlanH dec;
    int* sync;
    int4* grp;
    float* part_d;          // D chunk partials (fused path)
    // tensor-core path (int8; nvtc: NVFP4 experts on the block-scaled MMA)
    bool tc, nvtc;
    bool f16;               // tensor-core GEMMs on fp16-widened codes (every such matrix carries q16)
    int64_t tstride, sstride;   // slots of the dense (tokens) and the expert (pairs, padded) B buffers
    uint8_t *bxq, *bzq, *bhq, *byq;
    float *bxd, *bzd, *bhd, *byd;
    int32_t *slot_off, *tt_off, *pair_slot;
    int* cnt_comb_tc;
    WPlan pd, pgu, pdn, pu;
    bool raw;
    // small-T path: cluster router (k_route_small) and cluster GEMV (k_sgemv)
    bool small;
    SPlan sd, sgu, sdn, su;
    int rs_C, rs_epc;
    int32_t* gtok;          // [groups][8] tokens of each routed group's pairs
    size_t total;
};

LayerWs layer_layout(const elq_layer* ly, int T, void* base, int x_type) {
    LayerWs w;
    const int H = ly->H, L = ly->L, E = ly->E, k = ly->k, I = ly->I;
    const int64_t P = (int64_t)T * k;
    const int gmax = (int)std::min<int64_t>(E, P);
    w.tc = tc_path(ly->D.fmt, T) && tc_path(ly->U.fmt, T) && tc_path(ly->gate_up.fmt, T) && tc_path(ly->down.fmt, T);
    w.raw = T <= kRawMaxT;
    const int dmode = w.raw ? (x_type == ELQ_BF16 ? X_RAW_BF16 : X_RAW_F32) : X_Q81_TOKEN;
    w.pd = plan_w(ly->D.fmt, dmode, L, H, dense_groups(T), T, std::min(T, kDenseTg));
    w.pgu = plan_w(ly->gate_up.fmt, X_Q81_PAIR_TOKEN, 2 * I, L, gmax, P, std::min(T, kGroupTok));
    w.pdn = plan_w(ly->down.fmt, X_Q81_POSITION, L, I, gmax, P, std::min(T, kGroupTok));
    w.pu = plan_w(ly->U.fmt, X_Q81_TOKEN, H, L, dense_groups(T), T, std::min(T, kDenseTg));
    const int rblocks = (T + kRouterTok - 1) / kRouterTok;
    w.dec = plan_dec(ly, T);
    w.fused = !w.tc && w.dec.ok;
    w.small = false;
    // the cluster router: up to 8 CTAs (the portable cluster size), as few
    // experts per CTA as that allows (at most 16, one per warp)
    w.rs_C = 1;
    while ((E + w.rs_C - 1) / w.rs_C > 4 && w.rs_C < kSMaxCluster) w.rs_C *= 2;
    w.rs_epc = (E + w.rs_C - 1) / w.rs_C;
    // (NVFP4 experts take this path or none)
    if (!w.tc && !w.fused && w.raw && P <= kSMaxPairs && w.rs_epc <= kSMaxWarps &&
        rs_smem_bytes(T, L, E) + 16 <= kSSmemMax) {
        w.sd = plan_s(ly->D.fmt, dmode, false, L, H, 1, T, false);
        w.sgu = plan_s(ly->gate_up.fmt, X_Q81_PAIR_TOKEN, true, 2 * I, L, gmax, T, true);
        w.sdn = plan_s(ly->down.fmt, X_Q81_POSITION, false, L, I, gmax, T, true);
        w.su = plan_s(ly->U.fmt, X_Q81_TOKEN, false, H, L, 1, T, false);
        w.small = w.sd.ok && w.sgu.ok && w.sdn.ok && w.su.ok;
    }
    // NVFP4 experts beyond the cluster GEMV's sizes: D and U on the int8
    // tensor cores, the experts on the block-scaled ones
    w.nvtc = ly->gate_up.fmt == ELQ_NVFP4 && !w.small && ly->D.fmt == ELQ_Q8_0 && ly->U.fmt == ELQ_Q8_0;
    const bool tcbuf = w.tc || w.nvtc;
    // fp16-operand GEMMs when every int8 tensor-core matrix of the path carries its fp16 codes
    w.f16 = (w.tc && ly->D.q16 && ly->U.q16 && ly->gate_up.q16 && ly->down.q16) ||
            (w.nvtc && ly->D.q16 && ly->U.q16);
    const size_t cx = w.f16 ? 64 : 32;                     // bytes of a block's codes in the B buffers
    const size_t ce = (w.f16 && w.tc) ? 64 : 32;           // ... of the expert B buffers (NVFP4: packed codes)
    const size_t n_sync = w.fused ? (size_t)dec_sync_ints(T, L, I) : 0;
    const size_t n_cnt = 64 + (rblocks + 1) + w.pd.counter_ints + w.pgu.counter_ints + w.pdn.counter_ints +
                         w.pu.counter_ints + (size_t)T * (L / 32) + n_sync;
    Carve c;
    w.err = c.take<int>(base, n_cnt * sizeof(int));
    int* cur = w.err ? w.err + 64 : nullptr;
    auto adv = [&](size_t n) { int* r = cur; if (cur) cur += n; return r; };
    w.cnt_router = adv(rblocks + 1);
    w.cnt_d = adv(w.pd.counter_ints);
    w.cnt_gu = adv(w.pgu.counter_ints);
    w.cnt_dn = adv(w.pdn.counter_ints);
    w.cnt_u = adv(w.pu.counter_ints);
    w.cnt_comb = adv((size_t)T * (L / 32));     // per (token, 32-row block): covers the per-tile use too
    w.sync = w.fused ? adv(n_sync) : nullptr;
    w.xq = (w.raw && !w.nvtc) ? nullptr : c.take<uint8_t>(base, (size_t)T * (H / 32) * 36);
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
    w.tstride = round16(T);
    // NVFP4: token tiles of 128 slots start on whole scale atoms
    w.sstride = w.nvtc ? (int64_t)round_up((size_t)(P + kNvN * (int64_t)std::min<int64_t>(E, P)), 128)
                       : round16(P + 16 * (int64_t)std::min<int64_t>(E, P));
    w.grp = nullptr;
    w.gtok = nullptr;
    w.part_d = nullptr;
    if (w.small) {
        w.grp = c.take<int4>(base, (size_t)gmax * sizeof(int4));
        w.gtok = c.take<int32_t>(base, (size_t)gmax * kSMaxT * 4);
    }
    if (w.fused) {
        w.grp = c.take<int4>(base, (size_t)E * sizeof(int4));
        // D's chunk partials; the region also serves the separate-kernel
        // entry points that share this layout
        const size_t part = std::max(std::max(w.pd.partial_bytes, w.pgu.partial_bytes),
                                     std::max(w.pdn.partial_bytes, w.pu.partial_bytes));
        w.partial = c.take<float>(base, part);
        w.part_d = w.partial;
        w.bxq = w.bzq = w.bhq = w.byq = nullptr;
        w.bxd = w.bzd = w.bhd = w.byd = nullptr;
        w.slot_off = w.tt_off = w.pair_slot = nullptr;
        w.cnt_comb_tc = nullptr;
    } else if (!tcbuf) {
        const size_t part = std::max(std::max(w.pd.partial_bytes, w.pgu.partial_bytes),
                                     std::max(w.pdn.partial_bytes, w.pu.partial_bytes));
        w.partial = c.take<float>(base, part);
        w.bxq = w.bzq = w.bhq = w.byq = nullptr;
        w.bxd = w.bzd = w.bhd = w.byd = nullptr;
        w.slot_off = w.tt_off = w.pair_slot = nullptr;
        w.cnt_comb_tc = nullptr;
    } else {
        w.partial = nullptr;
        const int nbH = H / 32, nbL = L / 32, nbI = I / 32;
        w.bxq = c.take<uint8_t>(base, (size_t)nbH * w.tstride * cx);
        w.bxd = c.take<float>(base, (size_t)nbH * w.tstride * 4);
        w.bzq = c.take<uint8_t>(base, (size_t)nbL * w.sstride * ce);
        w.bzd = c.take<float>(base, (size_t)nbL * w.sstride * 4);
        w.bhq = c.take<uint8_t>(base, (size_t)nbI * w.sstride * ce);
        w.bhd = c.take<float>(base, (size_t)nbI * w.sstride * 4);
        w.byq = c.take<uint8_t>(base, (size_t)nbL * w.tstride * cx);
        w.byd = c.take<float>(base, (size_t)nbL * w.tstride * 4);
        w.slot_off = c.take<int32_t>(base, (size_t)(E + 1) * 4);
        w.tt_off = c.take<int32_t>(base, (size_t)(E + 1) * 4);
        w.pair_slot = c.take<int32_t>(base, (size_t)P * 4);
        w.cnt_comb_tc = c.take<int>(base, (size_t)T * (L / 32) * 4);
        // o is stored by slot on this path
        w.o = c.take<float>(base, (size_t)w.sstride * L * 4);
    }
    w.total = c.off;
    return w;
}

elq_status check_layer(const elq_layer* ly, int32_t T) {
    if (!ly) return ELQ_ERR_INVALID_ARG;
    if (T < 0) return ELQ_ERR_INVALID_ARG;
    const int H = ly->H, L = ly->L, E = ly->E, k = ly->k, I = ly->I;
    if (H <= 0 || L <= 0 || E <= 0 || k <= 0 || I <= 0) return ELQ_ERR_INVALID_ARG;
    if (k > E) return ELQ_ERR_INVALID_ARG;
    if (k > 32 || E > 1024 || L > kRouterMaxL) return ELQ_ERR_UNSUPPORTED;
    if (ly->flags & ~ELQ_LAYER_FUSED) return ELQ_ERR_INVALID_ARG;
    if (H % kTileRows || L % kTileRows || I % kTileRows) return ELQ_ERR_UNSUPPORTED;
    if ((int64_t)T * k > (int64_t)1 << 30) return ELQ_ERR_UNSUPPORTED;
    elq_status s;
    if ((s = check_qmat(&ly->D, L, H)) != ELQ_OK) return s;
    if ((s = check_qmat(&ly->U, H, L)) != ELQ_OK) return s;
    if ((int64_t)E * 2 * I > INT32_MAX || (int64_t)E * L > INT32_MAX) return ELQ_ERR_UNSUPPORTED;
    if ((s = check_qmat(&ly->gate_up, E * 2 * I, L, true)) != ELQ_OK) return s;
    if ((s = check_qmat(&ly->down, E * L, I, true)) != ELQ_OK) return s;
    if ((ly->gate_up.fmt == ELQ_NVFP4) != (ly->down.fmt == ELQ_NVFP4)) return ELQ_ERR_UNSUPPORTED;
    if ((ext_fmt(ly->gate_up.fmt) || ext_fmt(ly->down.fmt)) && ly->gate_up.fmt != ly->down.fmt)
        return ELQ_ERR_UNSUPPORTED;
    // Q5_1 / K-quant experts: the cluster GEMV's token and pair bounds only
    if (ext_fmt(ly->gate_up.fmt) && (T > kSMaxT || (int64_t)T * k > kSMaxPairs)) return ELQ_ERR_UNSUPPORTED;
    if (ly->gate_up.fmt == ELQ_NVFP4) {
        // one global scale per expert matrix; static activation scales
        if (ly->gate_up.gs_rows != 2 * I || ly->down.gs_rows != L) return ELQ_ERR_INVALID_ARG;
        if (!(ly->act_gz > 0.0f) || !(ly->act_gh > 0.0f) || !std::isfinite(ly->act_gz) ||
            !std::isfinite(ly->act_gh))
            return ELQ_ERR_INVALID_ARG;
        // beyond the cluster GEMV's token and pair bounds: the tensor-core
        // path, which takes D and U in Q8_0 only
        if ((T > kSMaxT || (int64_t)T * k > kSMaxPairs) && (ly->D.fmt != ELQ_Q8_0 || ly->U.fmt != ELQ_Q8_0))
            return ELQ_ERR_UNSUPPORTED;
    }
    if (!ly->router_w) return ELQ_ERR_INVALID_ARG;
    if (!aligned(ly->router_w, 16) || (ly->router_bias && !aligned(ly->router_bias, 4))) return ELQ_ERR_ALIGNMENT;
    return ELQ_OK;
}

// Router launch shape: 4 experts per CTA (one per warp) and one token block
// each while that grid stays within two CTAs per SM; beyond, 16 experts per
// CTA (8 warps of two) and about one CTA per SM, each streaming several token
// blocks.
struct RouterShape {
    int nw, epw, gx, gy, stages;
};

RouterShape router_shape(int T, int E) {
    RouterShape r;
    const int rblocks = (T + kRouterTok - 1) / kRouterTok;
    const int sms = sm_count();
    const bool small = (int64_t)rblocks * ((E + 3) / 4) <= 2 * (int64_t)sms;
    r.nw = small ? 4 : kRouterMaxWarps / 2;
    r.epw = small ? 1 : 2;
    r.gx = (E + r.nw * r.epw - 1) / (r.nw * r.epw);
    r.gy = r.nw == 4 ? rblocks : std::min(rblocks, std::max(1, sms / r.gx));
    r.stages = r.gy < rblocks ? 2 : 1;
    return r;
}

size_t router_smem(int T, int L, int E) {
    const RouterShape r = router_shape(T, E);
    const int Lp = (L + 255) & ~255;   // the kernel's padded row stride
    return (size_t)r.stages * std::min(T, kRouterTok) * Lp * 4 + (size_t)r.nw * E * 4;
}

bool router_shape_ok(int T, int L, int E) {
    return L <= kRouterMaxL && router_smem(T, L, E) <= (size_t)kRouterSmemMax;
}

cudaError_t launch_router(const float* z, const float* w, const float* bias, int T, int L, int E, int k,
                          int32_t* idx, float* wts, float* logits, int* cnt, bool do_bucket, int32_t* counts,
                          int32_t* offsets, int32_t* perm, int32_t* pos, int32_t* act, int32_t* n_act,
                          cudaStream_t s, bool pdl) {
    RouterArgs a;
    std::memset(&a, 0, sizeof(a));
    a.z = z; a.w = w; a.bias = bias; a.T = T; a.L = L; a.E = E; a.k = k;
    a.idx = idx; a.wts = wts; a.logits = logits;
    const int rblocks = (T + kRouterTok - 1) / kRouterTok;
    a.cnt_tok = cnt;
    a.cnt_all = cnt ? cnt + rblocks : nullptr;
    a.do_bucket = do_bucket ? 1 : 0;
    a.counts = counts; a.offsets = offsets; a.perm = perm; a.pos = pos; a.act = act; a.n_act = n_act;
    const RouterShape r = router_shape(T, E);
    if (r.epw == 2) {
        cudaError_t e = smem_optin(k_router<2>, kRouterSmemMax, g_optin_router2);
        if (e != cudaSuccess) return e;
        return launch(k_router<2>, dim3(r.gx, r.gy), dim3(r.nw * 32), router_smem(T, L, E), s, pdl, a);
    }
    cudaError_t e = smem_optin(k_router<1>, kRouterSmemMax, g_optin_router);
    if (e != cudaSuccess) return e;
    return launch(k_router<1>, dim3(r.gx, r.gy), dim3(r.nw * 32), router_smem(T, L, E), s, pdl, a);
}

// Grouped gate/up over the routed pairs: SwiGLU epilogue into hq.
WArgs gate_up_args(const elq_layer* ly, const LayerWs& w, int T, const uint8_t* zq, float* partial) {
    const int L = ly->L, k = ly->k, I = ly->I;
    WArgs g;
    std::memset(&g, 0, sizeof(g));
    g.q = static_cast<const uint8_t*>(ly->gate_up.q);
    g.d = static_cast<const uint16_t*>(ly->gate_up.d);
    g.nb = L / 32;
    g.q_gstride = (int64_t)(2 * I / kTileRows) * g.nb * slab_bytes(ly->gate_up.fmt);
    g.d_gstride = (int64_t)(2 * I / kTileRows) * g.nb * kTileRows;
    g.act = w.act; g.n_act = w.n_act; g.offsets = w.offsets; g.perm = w.perm; g.kslots = k; g.T = T;
    g.x = zq; g.x_mode = X_Q81_PAIR_TOKEN;
    g.out_mode = OUT_SWIGLU;
    g.yq = w.hq; g.yq_ld = I / 32;
    g.partial = partial; g.part_tok = (int64_t)T * k; g.counters = w.cnt_gu; g.err = w.err;
    return g;
}

// Grouped down over the routed pairs: o by pair position, weighted combine
// into y_lat and its Q8_1 rows.
WArgs down_args(const elq_layer* ly, const LayerWs& w, int T, const float* wts, float* y_lat, float* partial) {
    const int L = ly->L, k = ly->k, I = ly->I;
    WArgs h;
    std::memset(&h, 0, sizeof(h));
    h.q = static_cast<const uint8_t*>(ly->down.q);
    h.d = static_cast<const uint16_t*>(ly->down.d);
    h.nb = I / 32;
    h.q_gstride = (int64_t)(L / kTileRows) * h.nb * slab_bytes(ly->down.fmt);
    h.d_gstride = (int64_t)(L / kTileRows) * h.nb * kTileRows;
    h.act = w.act; h.n_act = w.n_act; h.offsets = w.offsets; h.perm = w.perm; h.kslots = k; h.T = T;
    h.x = w.hq; h.x_mode = X_Q81_POSITION;
    h.out_mode = OUT_F32_COMBINE;
    h.y = w.o; h.y_ld = L;
    h.wts = wts; h.pos = w.pos; h.cnt_comb = w.cnt_comb; h.ylat = y_lat; h.ylq = w.ylq;
    h.partial = partial; h.part_tok = (int64_t)T * k; h.counters = w.cnt_dn; h.err = w.err;
    return h;
}

// The expert projections on k_sgemv.  route: ROUTE_GROUPS (the layer call:
// the group table k_route_small wrote) or ROUTE_ARRAYS (the bucketed arrays
// in the workspace; wts the caller's).
SArgs gate_up_s(const elq_layer* ly, const LayerWs& w, int T, int route, const uint8_t* zq) {
    const int L = ly->L, E = ly->E, k = ly->k, I = ly->I;
    SArgs g;
    std::memset(&g, 0, sizeof(g));
    g.q = static_cast<const uint8_t*>(ly->gate_up.q);
    g.d = static_cast<const uint16_t*>(ly->gate_up.d);
    g.nb = L / 32;
    g.q_gstride = (int64_t)(2 * I / kTileRows) * g.nb * slab_bytes(ly->gate_up.fmt);
    g.d_gstride = (int64_t)(2 * I / kTileRows) * d_tile_elems(ly->gate_up.fmt, g.nb);
    g.groups_max = (int)std::min<int64_t>(E, (int64_t)T * k);
    g.route = route;
    g.T = T; g.E = E; g.k = k;
    g.act = w.act; g.n_act = w.n_act; g.offsets = w.offsets; g.perm = w.perm; g.pos = w.pos;
    g.grp = w.grp; g.gtok = w.gtok;
    g.x = zq;
    g.yq = w.hq; g.yq_ld = I / 32;
    g.wgs = ly->gate_up.gs; g.ags = ly->act_gz; g.ogs = ly->act_gh;
    g.L = L;
    g.err = w.err;
    g.early = 0;
    return g;
}

SArgs down_s(const elq_layer* ly, const LayerWs& w, int T, int route, const float* wts, float* y_lat) {
    const int L = ly->L, E = ly->E, k = ly->k, I = ly->I;
    SArgs h;
    std::memset(&h, 0, sizeof(h));
    h.q = static_cast<const uint8_t*>(ly->down.q);
    h.d = static_cast<const uint16_t*>(ly->down.d);
    h.nb = I / 32;
    h.q_gstride = (int64_t)(L / kTileRows) * h.nb * slab_bytes(ly->down.fmt);
    h.d_gstride = (int64_t)(L / kTileRows) * d_tile_elems(ly->down.fmt, h.nb);
    h.groups_max = (int)std::min<int64_t>(E, (int64_t)T * k);
    h.route = route;
    h.T = T; h.E = E; h.k = k;
    h.act = w.act; h.n_act = w.n_act; h.offsets = w.offsets; h.perm = w.perm; h.pos = w.pos;
    h.grp = w.grp; h.gtok = w.gtok;
    h.wts = wts;
    h.x = w.hq;
    h.y = w.o; h.y_ld = L;
    h.cnt_comb = w.cnt_comb; h.ylat = y_lat; h.ylq = w.ylq; h.L = L;
    h.wgs = ly->down.gs; h.ags = ly->act_gh;
    h.err = w.err;
    // the routing is complete before this kernel's upstream (gate/up) starts
    h.early = 1;
    return h;
}

// The small-T cluster router: one cluster of rs_C CTAs of rs_epc warps.
cudaError_t launch_route_small(const elq_layer* ly, const LayerWs& w, int T, cudaStream_t s, bool pdl) {
    static bool optin[kMaxDevices];
    cudaError_t e = smem_optin(k_route_small, kSSmemMax, optin);
    if (e != cudaSuccess) return e;
    RSArgs r;
    std::memset(&r, 0, sizeof(r));
    r.z = w.z; r.w = ly->router_w; r.bias = ly->router_bias;
    r.T = T; r.L = ly->L; r.E = ly->E; r.k = ly->k; r.C = w.rs_C; r.epc = w.rs_epc;
    r.logits = w.logits; r.idx = w.idx; r.wts = w.wts;
    r.counts = w.counts; r.offsets = w.offsets; r.perm = w.perm; r.pos = w.pos; r.act = w.act; r.n_act = w.n_act;
    r.grp = w.grp; r.gtok = w.gtok;
    cudaLaunchConfig_t cfg;
    std::memset(&cfg, 0, sizeof(cfg));
    cfg.gridDim = dim3((unsigned)w.rs_C);
    cfg.blockDim = dim3((unsigned)(32 * w.rs_epc));
    cfg.dynamicSmemBytes = (size_t)rs_smem_bytes(T, ly->L, ly->E) + 16;
    cfg.stream = s;
    cudaLaunchAttribute attr[2];
    int na = 0;
    if (w.rs_C > 1) {
        attr[na].id = cudaLaunchAttributeClusterDimension;
        attr[na].val.clusterDim.x = (unsigned)w.rs_C;
        attr[na].val.clusterDim.y = 1;
        attr[na].val.clusterDim.z = 1;
        ++na;
    }
    if (pdl) {
        attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[na].val.programmaticStreamSerializationAllowed = 1;
        ++na;
    }
    cfg.attrs = na ? attr : nullptr;
    cfg.numAttrs = na;
    return cudaLaunchKernelEx(&cfg, k_route_small, r);
}

// Kernel sequence of the grouped experts (gate/up, then down with the combine)
// routing_early_down: the routing was produced two kernels before the down
// projection (by the router, not by a bucketing kernel right before gate/up
// whose completion the down kernel could not otherwise rely on).
elq_status run_experts(const elq_layer* ly, const LayerWs& w, int T, const uint8_t* zq, const float* wts,
                       float* y_lat, cudaStream_t s, bool pdl, const std::function<bool()>& mark,
                       bool routing_early_down) {
    WArgs g = gate_up_args(ly, w, T, zq, w.partial);
    if (launch_w(g, ly->gate_up.fmt, w.pgu, s, pdl) != cudaSuccess || !mark()) return ELQ_ERR_CUDA;
    WArgs h = down_args(ly, w, T, wts, y_lat, w.partial);
    h.routing_early = routing_early_down ? 1 : 0;
    if (launch_w(h, ly->down.fmt, w.pdn, s, pdl) != cudaSuccess || !mark()) return ELQ_ERR_CUDA;
    return ELQ_OK;
}

// The fused small-T layer: one cooperative launch of k_decode_layer.
template <int FDU, int FEX>
cudaError_t launch_fused_t(const DecArgs& a, const DecPlanH& p, cudaStream_t s) {
    const int slot = (FDU == 8 ? 2 : 0) + (FEX == 8 ? 1 : 0);
    cudaError_t e = smem_optin(k_decode_layer<FDU, FEX>, kDecSmemMax, g_optin_dec[slot]);
    if (e != cudaSuccess) return e;
    return launch_coop(k_decode_layer<FDU, FEX>, dim3(sm_count()), dim3(kDecWarps * 32), (size_t)p.smem, s, a);
}

elq_status run_fused(const elq_layer* ly, const LayerWs& w, const void* x, int32_t x_type, int T, float* y,
                     cudaStream_t s, uint64_t budget_ns = kWaitBudgetNs, bool withhold_routing = false) {
    const int H = ly->H, L = ly->L, E = ly->E, k = ly->k, I = ly->I;
    const DecPlanH& p = w.dec;
    if (!p.ok) return ELQ_ERR_UNSUPPORTED;
    DecArgs a;
    std::memset(&a, 0, sizeof(a));
    // D reads the Q8_1 of x each CTA makes in shared memory
    a.dproj = dense_w(&ly->D, T, nullptr, X_Q81_TOKEN, 0, OUT_F32_Q81, w.z, w.zq, w.part_d, w.cnt_d, w.err);
    a.dproj.tiles = w.pd.tiles;
    a.dproj.nchunks = w.pd.nchunks;
    a.dproj.act_off = kChunk * (ly->D.fmt == ELQ_Q8_0 ? 1024 : 512) + kChunk * 64;
    a.dproj.act_bytes = kChunk * 36;
    a.dproj.stage_bytes = p.stage_bytes;
    a.dproj.stages = p.stages;
    a.dproj.tokcap = T;
    a.dproj.budget_ns = budget_ns;
    a.gu_q = static_cast<const uint8_t*>(ly->gate_up.q);
    a.gu_d = static_cast<const uint16_t*>(ly->gate_up.d);
    a.gu_qs = (int64_t)(2 * I / kTileRows) * (L / 32) * slab_bytes(ly->gate_up.fmt);
    a.gu_ds = (int64_t)(2 * I / kTileRows) * (L / 32) * kTileRows;
    a.dn_q = static_cast<const uint8_t*>(ly->down.q);
    a.dn_d = static_cast<const uint16_t*>(ly->down.d);
    a.dn_qs = (int64_t)(L / kTileRows) * (I / 32) * slab_bytes(ly->down.fmt);
    a.dn_ds = (int64_t)(L / kTileRows) * (I / 32) * kTileRows;
    a.u_q = static_cast<const uint8_t*>(ly->U.q);
    a.u_d = static_cast<const uint16_t*>(ly->U.d);
    a.T = T; a.H = H; a.L = L; a.E = E; a.k = k; a.I = I;
    a.rw = ly->router_w; a.rb = ly->router_bias;
    a.z = w.z; a.logits = w.logits; a.idx = w.idx; a.wts = w.wts;
    a.counts = w.counts; a.offsets = w.offsets; a.perm = w.perm; a.pos = w.pos; a.act = w.act; a.n_act = w.n_act;
    a.grp = w.grp;
    a.zq = w.zq; a.hq = w.hq; a.o = w.o; a.ylat = w.ylat; a.ylq = w.ylq; a.y = y;
    a.sync = w.sync;
    a.err = w.err;
    a.budget_ns = budget_ns;
    a.withhold_routing = withhold_routing ? 1 : 0;
    a.x = x;
    a.x_bf16 = (x_type == ELQ_BF16) ? 1 : 0;
    a.stages = p.stages; a.stage_bytes = p.stage_bytes; a.xq_chunks = p.xq_chunks; a.header = p.header;
    cudaError_t e;
    const bool du8 = ly->D.fmt == ELQ_Q8_0, ex8 = ly->gate_up.fmt == ELQ_Q8_0;
    if (du8 && ex8) e = launch_fused_t<8, 8>(a, p, s);
    else if (du8) e = launch_fused_t<8, 2>(a, p, s);
    else if (ex8) e = launch_fused_t<2, 8>(a, p, s);
    else e = launch_fused_t<2, 2>(a, p, s);
    return cuda_status(e);
}

elq_status run_layer(const elq_layer* layer, const void* x, int32_t x_type, int32_t T, float* y, void* ws,
                     size_t ws_bytes, void* stream, void* const* events, int32_t n_events, bool residual = false);

// Tensor-core experts: slots from the routing, gathered z codes, gate/up (+SwiGLU
// into the packed hq buffer), down (+combine into y_lat, Q8_1 rows and the
// packed buffer the U projection reads).
elq_status run_experts_tc(const elq_layer* ly, const LayerWs& w, int T, const uint8_t* zq, const float* wts,
                          float* y_lat, cudaStream_t s, bool pdl, const std::function<bool()>& mark) {
    const int L = ly->L, E = ly->E, k = ly->k, I = ly->I;
    const int P = T * k;
    if (launch(k_tc_route, dim3(1), dim3(1024), 0, s, pdl, (const int32_t*)w.offsets, (const int32_t*)w.act,
               (const int32_t*)w.n_act, (const int32_t*)w.idx, (const int32_t*)w.pos, P, E, w.slot_off, w.tt_off,
               w.pair_slot, 16, kTcN) != cudaSuccess ||
        !mark())
        return ELQ_ERR_CUDA;
    PackArgs pa;
    std::memset(&pa, 0, sizeof(pa));
    pa.x = zq;
    pa.nb = L / 32;
    pa.mode = PACK_SLOTS;
    pa.slot_off = w.slot_off;
    pa.offsets = w.offsets;
    pa.perm = w.perm;
    pa.E = E;
    pa.kslots = k;
    pa.bq = w.bzq;
    pa.bd = w.bzd;
    pa.bstride = w.sstride;
    pa.f16 = w.f16 ? 1 : 0;
    if (launch_pack(pa, s, pdl) != cudaSuccess || !mark()) return ELQ_ERR_CUDA;
    TcArgs g;
    std::memset(&g, 0, sizeof(g));
    g.q = static_cast<const uint8_t*>(ly->gate_up.q);
    g.d = static_cast<const uint16_t*>(ly->gate_up.d);
    g.nb = L / 32;
    g.rtiles = 2 * I / kTileRows;
    g.n_groups = E;
    g.q_gstride = (int64_t)g.rtiles * g.nb * kQ80Slab;
    g.d_gstride = (int64_t)g.rtiles * g.nb * kTileRows;
    g.q16 = w.f16 ? static_cast<const uint8_t*>(ly->gate_up.q16) : nullptr;
    g.q16_gstride = 2 * g.q_gstride;
    g.act = w.act; g.n_act = w.n_act; g.slot_off = w.slot_off; g.offsets = w.offsets; g.tt_off = w.tt_off;
    g.T = T;
    g.bq = w.bzq; g.bd = w.bzd; g.bstride = w.sstride;
    g.out_mode = TC_OUT_SWIGLU;
    g.cq = w.bhq; g.cd = w.bhd; g.cstride = w.sstride;
    g.err = w.err;
    if (launch_tc(g, s, pdl) != cudaSuccess || !mark()) return ELQ_ERR_CUDA;
    TcArgs h;
    std::memset(&h, 0, sizeof(h));
    h.q = static_cast<const uint8_t*>(ly->down.q);
    h.d = static_cast<const uint16_t*>(ly->down.d);
    h.nb = I / 32;
    h.rtiles = L / kTileRows;
    h.n_groups = E;
    h.q_gstride = (int64_t)h.rtiles * h.nb * kQ80Slab;
    h.d_gstride = (int64_t)h.rtiles * h.nb * kTileRows;
    h.q16 = w.f16 ? static_cast<const uint8_t*>(ly->down.q16) : nullptr;
    h.q16_gstride = 2 * h.q_gstride;
    h.act = w.act; h.n_act = w.n_act; h.slot_off = w.slot_off; h.offsets = w.offsets; h.tt_off = w.tt_off;
    h.T = T;
    h.bq = w.bhq; h.bd = w.bhd; h.bstride = w.sstride;
    h.out_mode = TC_OUT_F32;           // o by slot; the combine follows
    h.y = w.o; h.y_ld = L;
    h.err = w.err;
    if (launch_tc(h, s, pdl) != cudaSuccess || !mark()) return ELQ_ERR_CUDA;
    CombArgs c;
    std::memset(&c, 0, sizeof(c));
    c.o = w.o; c.wts = wts; c.pair_slot = w.pair_slot; c.T = T; c.L = L; c.k = k;
    c.ylat = y_lat; c.ylq = w.ylq; c.cq = w.byq; c.cd = w.byd; c.cstride = w.tstride;
    c.f16 = w.f16 ? 1 : 0;
    const int64_t threads = (int64_t)T * ((L / 32 + 3) / 4) * 32;   // one warp per (token, 4 blocks)
    if (launch(k_tc_combine, dim3((unsigned)((threads + 255) / 256)), dim3(256), 0, s, pdl, c) != cudaSuccess ||
        !mark())
        return ELQ_ERR_CUDA;
    return ELQ_OK;
}

// ---- NVFP4 experts on the block-scaled tensor cores --------------------------

template <int OM>
cudaError_t launch_nv_t(const NvArgs& g, cudaStream_t s, bool pdl) {
    static bool optin[kMaxDevices];
    cudaError_t e = smem_optin(k_nvgemm<OM>, kNvSmem, optin);
    if (e != cudaSuccess) return e;
    return launch(k_nvgemm<OM>, dim3(sm_count()), dim3(kTcThreads), (size_t)kNvSmem, s, pdl, g);
}

// An expert projection: weights m (n_rows = E * rows per expert, k), the
// activations packed in bq / sfb (K steps of 64 values, sstride slots).
NvArgs nv_args(const elq_qmat* m, int E, const LayerWs& w, int T, const uint8_t* bq, const uint8_t* sfb, float ags,
               bool& ok) {
    NvArgs g;
    std::memset(&g, 0, sizeof(g));
    const int nb = m->k / 32;
    g.d = static_cast<const uint8_t*>(m->d);
    g.d_tile_bytes = d_tile_elems(ELQ_NVFP4, nb) * 2;
    g.nb = nb;
    g.nks = m->k / 64;
    g.rtiles = m->n_rows / E / kTileRows;
    g.act = w.act; g.n_act = w.n_act; g.slot_off = w.slot_off; g.offsets = w.offsets; g.tt_off = w.tt_off;
    g.T = T;
    g.sfb = sfb;
    g.wgs = m->gs;
    g.ags = ags;
    g.sstride = w.sstride;
    g.err = w.err;
    g.budget_ns = kWaitBudgetNs;
    const cuuint64_t tiles = (cuuint64_t)m->n_rows / kTileRows, nbu = (cuuint64_t)nb;
    const cuuint64_t da[4] = {128, 4, nbu, tiles}, sa[3] = {nbu * 512, 512, nbu * 2048};
    const cuuint32_t ba[4] = {128, 4, 2 * kNvKS, 1};
    const cuuint64_t slots = (cuuint64_t)w.sstride;
    const cuuint64_t db[3] = {64, slots / 8, (cuuint64_t)g.nks}, sb[2] = {256, slots * 32};
    const cuuint32_t bb[3] = {64, kNvN / 8, kNvKS};
    ok = encode_map(&g.tm_a, CU_TENSOR_MAP_DATA_TYPE_UINT32, 4, m->q, da, sa, ba) &&
         encode_map(&g.tm_b, CU_TENSOR_MAP_DATA_TYPE_UINT32, 3, bq, db, sb, bb);
    return g;
}

// Slots from the routing, z packed, gate/up (+SwiGLU into the packed h),
// down (o by slot), the weighted combine (y_lat, its Q8_1 rows, and the
// packed buffer the U projection reads).  zq: NVFP4 rows under act_gz.
elq_status run_experts_nvtc(const elq_layer* ly, const LayerWs& w, int T, const uint8_t* zq, const float* wts,
                            float* y_lat, cudaStream_t s, bool pdl, const std::function<bool()>& mark) {
    const int L = ly->L, E = ly->E, k = ly->k, I = ly->I;
    const int P = T * k;
    if (launch(k_tc_route, dim3(1), dim3(1024), 0, s, pdl, (const int32_t*)w.offsets, (const int32_t*)w.act,
               (const int32_t*)w.n_act, (const int32_t*)w.idx, (const int32_t*)w.pos, P, E, w.slot_off, w.tt_off,
               w.pair_slot, kNvN, kNvN) != cudaSuccess ||
        !mark())
        return ELQ_ERR_CUDA;
    NvPackArgs pk;
    std::memset(&pk, 0, sizeof(pk));
    pk.x = zq;
    pk.nb = L / 32;
    pk.nks = L / 64;
    pk.slot_off = w.slot_off;
    pk.offsets = w.offsets;
    pk.perm = w.perm;
    pk.E = E;
    pk.kslots = k;
    pk.bq = w.bzq;
    pk.bsf = reinterpret_cast<uint8_t*>(w.bzd);
    pk.sstride = w.sstride;
    const int64_t n = w.sstride * pk.nks;   // one thread per (K-step, slot)
    if (launch(k_pack_nv, dim3((unsigned)((n + 255) / 256)), dim3(256), 0, s, pdl, pk) != cudaSuccess || !mark())
        return ELQ_ERR_CUDA;
    bool ok = false;
    NvArgs g = nv_args(&ly->gate_up, E, w, T, w.bzq, reinterpret_cast<const uint8_t*>(w.bzd), ly->act_gz, ok);
    if (!ok) return ELQ_ERR_CUDA;
    g.hq = w.bhq;
    g.hsf = reinterpret_cast<uint8_t*>(w.bhd);
    g.h_nks = I / 64;
    g.ogs = ly->act_gh;
    if (launch_nv_t<NV_OUT_SWIGLU>(g, s, pdl) != cudaSuccess || !mark()) return ELQ_ERR_CUDA;
    NvArgs h = nv_args(&ly->down, E, w, T, w.bhq, reinterpret_cast<const uint8_t*>(w.bhd), ly->act_gh, ok);
    if (!ok) return ELQ_ERR_CUDA;
    h.y = w.o;
    h.y_ld = L;
    if (launch_nv_t<NV_OUT_F32>(h, s, pdl) != cudaSuccess || !mark()) return ELQ_ERR_CUDA;
    CombArgs c;
    std::memset(&c, 0, sizeof(c));
    c.o = w.o; c.wts = wts; c.pair_slot = w.pair_slot; c.T = T; c.L = L; c.k = k;
    c.ylat = y_lat; c.ylq = w.ylq; c.cq = w.byq; c.cd = w.byd; c.cstride = w.tstride;
    c.f16 = w.f16 ? 1 : 0;
    const int64_t threads = (int64_t)T * ((L / 32 + 3) / 4) * 32;   // one warp per (token, 4 blocks)
    if (launch(k_tc_combine, dim3((unsigned)((threads + 255) / 256)), dim3(256), 0, s, pdl, c) != cudaSuccess ||
        !mark())
        return ELQ_ERR_CUDA;
    return ELQ_OK;
}

bool layer_tc(const elq_layer* ly, int T) {
    return tc_path(ly->D.fmt, T) && tc_path(ly->U.fmt, T) && tc_path(ly->gate_up.fmt, T) && tc_path(ly->down.fmt, T);
}

bool layer_fused(const elq_layer* ly, int T) { return !layer_tc(ly, T) && plan_dec(ly, T).ok; }

int layer_kernels(const elq_layer* ly, int T) {
    if (ly->gate_up.fmt == ELQ_NVFP4 || ext_fmt(ly->gate_up.fmt)) {
        const LayerWs w = layer_layout(ly, T, nullptr, ELQ_F32);
        return w.small ? 5 : w.nvtc ? 11 : 0;
    }
    if (layer_tc(ly, T)) return 10;
    if (layer_fused(ly, T)) return 1;
    return T <= kRawMaxT ? 5 : 6;
}

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

int32_t elq_version(void) { return 3; }

size_t elq_f16_bytes(const elq_qmat* w) {
    if (!w || w->fmt != ELQ_Q8_0 || w->n_rows <= 0 || w->k <= 0) return 0;
    return (size_t)w->n_rows * (size_t)w->k * 2;
}

elq_status elq_pack_f16(const elq_qmat* w, void* q16, void* stream) {
    if (!w || !q16 || !w->q) return ELQ_ERR_INVALID_ARG;
    if (w->fmt != ELQ_Q8_0) return ELQ_ERR_UNSUPPORTED;
    if (w->n_rows <= 0 || w->k <= 0 || w->n_rows % kTileRows || w->k % 32) return ELQ_ERR_INVALID_ARG;
    if (!aligned(w->q, 256) || !aligned(q16, 256)) return ELQ_ERR_ALIGNMENT;
    const int64_t pieces = (int64_t)w->n_rows * w->k / 16;   // 16-byte pieces of the int8 codes
    return cuda_status(launch(k_arena_f16, dim3((unsigned)((pieces + 255) / 256)), dim3(256), 0,
                              static_cast<cudaStream_t>(stream), false, static_cast<const uint8_t*>(w->q), pieces,
                              (int)(w->k / 32), static_cast<uint8_t*>(q16)));
}

size_t elq_arena_bytes(int32_t fmt, int32_t n_rows, int32_t k, size_t* q_bytes, size_t* d_bytes) {
    if (!arena_fmt_ok(fmt) || n_rows <= 0 || k <= 0 || n_rows % kTileRows || k % arena_k_unit(fmt)) {
        if (q_bytes) *q_bytes = 0;
        if (d_bytes) *d_bytes = 0;
        return 0;
    }
    const size_t slabs = (size_t)(n_rows / kTileRows) * (k / 32);
    // NVFP4: each tile's scales twice (per row, and as the tensor cores' atoms)
    const size_t q = slabs * slab_bytes(fmt), d = slabs * kScaleSlab * (fmt == ELQ_NVFP4 ? 2 : scale_units(fmt));
    if (q_bytes) *q_bytes = q;
    if (d_bytes) *d_bytes = d;
    return q + d;
}

elq_status elq_arena_pack(int32_t fmt, const void* aos, int32_t n_rows, int32_t k, void* q_out, void* d_out,
                          void* stream) {
    if (!arena_fmt_ok(fmt)) return ELQ_ERR_UNSUPPORTED;
    if (!aos || !q_out || !d_out || n_rows <= 0 || k <= 0) return ELQ_ERR_INVALID_ARG;
    if (n_rows % kTileRows || k % arena_k_unit(fmt)) return ELQ_ERR_UNSUPPORTED;
    if (!aligned(q_out, 256) || !aligned(d_out, 256)) return ELQ_ERR_ALIGNMENT;
    const int64_t n = (int64_t)n_rows * (k / 32);
    const dim3 grid((unsigned)((n + 255) / 256));
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    uint32_t* d32 = static_cast<uint32_t*>(d_out);
    const uint8_t* src = static_cast<const uint8_t*>(aos);
    uint8_t* q8 = static_cast<uint8_t*>(q_out);
    if (fmt == ELQ_Q5_1)
        k_arena_pack_ext<kQ51><<<grid, 256, 0, s>>>(src, n_rows, k, q8, d32);
    else if (fmt == ELQ_Q3_K)
        k_arena_pack_ext<kQ3K><<<grid, 256, 0, s>>>(src, n_rows, k, q8, d32);
    else if (fmt == ELQ_Q4_K)
        k_arena_pack_ext<kQ4K><<<grid, 256, 0, s>>>(src, n_rows, k, q8, d32);
    else if (fmt == ELQ_Q5_K)
        k_arena_pack_ext<kQ5K><<<grid, 256, 0, s>>>(src, n_rows, k, q8, d32);
    else if (fmt == ELQ_Q8_0)
        k_arena_pack<8><<<grid, 256, 0, s>>>(static_cast<const uint8_t*>(aos), n_rows, k,
                                             static_cast<uint8_t*>(q_out), static_cast<uint16_t*>(d_out));
    else if (fmt == ELQ_NVFP4)
        k_arena_pack<kNV><<<grid, 256, 0, s>>>(static_cast<const uint8_t*>(aos), n_rows, k,
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
    const dim3 grid((unsigned)((4 * nblk + 255) / 256));   // four threads per block
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (x_type == ELQ_BF16)
        return cuda_status(launch(k_quant_q8_1<true>, grid, dim3(256), 0, s, false, x, nblk,
                                  static_cast<uint8_t*>(out_q8_1)));
    return cuda_status(launch(k_quant_q8_1<false>, grid, dim3(256), 0, s, false, x, nblk,
                              static_cast<uint8_t*>(out_q8_1)));
}

elq_status elq_quantize_nvfp4(const void* x, int32_t x_type, int64_t rows, int64_t cols, float g, void* out,
                              void* stream) {
    if (x_type != ELQ_F32 && x_type != ELQ_BF16) return ELQ_ERR_UNSUPPORTED;
    if (rows < 0 || cols <= 0 || !(g > 0.0f) || !std::isfinite(g)) return ELQ_ERR_INVALID_ARG;
    if (cols % 32) return ELQ_ERR_UNSUPPORTED;
    if (rows == 0) return ELQ_OK;
    if (!x || !out) return ELQ_ERR_INVALID_ARG;
    if (!aligned(x, 4) || !aligned(out, 2)) return ELQ_ERR_ALIGNMENT;
    const int64_t nblk = rows * (cols / 32);
    const dim3 grid((unsigned)((nblk * 4 + 255) / 256));   // four threads per block
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (x_type == ELQ_BF16)
        return cuda_status(launch(k_quant_nvfp4<true>, grid, dim3(256), 0, s, false, x, nblk, g,
                                  static_cast<uint8_t*>(out)));
    return cuda_status(launch(k_quant_nvfp4<false>, grid, dim3(256), 0, s, false, x, nblk, g,
                              static_cast<uint8_t*>(out)));
}

elq_status elq_router_topk(const float* z, const float* w_router, const float* bias, int32_t T, int32_t L,
                           int32_t E, int32_t k, int32_t* idx, float* weights, float* logits, void* stream) {
    if (T < 0 || L <= 0 || E <= 0 || k <= 0 || k > E) return ELQ_ERR_INVALID_ARG;
    if (k > 32 || E > 1024 || L % 32 || L > kRouterMaxL) return ELQ_ERR_UNSUPPORTED;
    if (T == 0) return ELQ_OK;
    if (!z || !w_router || !idx || !weights || !logits) return ELQ_ERR_INVALID_ARG;
    if (!aligned(z, 16) || !aligned(w_router, 16) || (bias && !aligned(bias, 4)) || !aligned(idx, 4) ||
        !aligned(weights, 4) || !aligned(logits, 4))
        return ELQ_ERR_ALIGNMENT;
    if (!router_shape_ok(T, L, E)) return ELQ_ERR_UNSUPPORTED;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaError_t e = launch_router(z, w_router, bias, T, L, E, k, idx, weights, logits, nullptr, false, nullptr,
                                  nullptr, nullptr, nullptr, nullptr, nullptr, s, false);
    if (e != cudaSuccess) return ELQ_ERR_CUDA;
    e = smem_optin(k_topk, kRouterSmemMax, g_optin_topk);
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
    cudaError_t e = smem_optin(k_bucket, kRouterSmemMax, g_optin_bucket);
    if (e != cudaSuccess) return ELQ_ERR_CUDA;
    e = launch(k_bucket, dim3(1), dim3(nw * 32), (size_t)nw * E * 4, static_cast<cudaStream_t>(stream), false, idx,
               (int)(T * k), (int)E, counts, offsets, perm, pos, (int32_t*)nullptr, (int32_t*)nullptr);
    return cuda_status(e);
}

size_t elq_latent_proj_workspace_bytes(const elq_qmat* w, int32_t T) {
    if (!w || T <= 0) return 0;
    if (!fmt_ok(w->fmt) || w->n_rows <= 0 || w->k <= 0 || w->n_rows % kTileRows || w->k % 128) return 0;
    return proj_layout(w, T, nullptr).total;
}

elq_status elq_latent_proj(const elq_qmat* w, const void* x_q8_1, int32_t T, float* y, void* ws, size_t ws_bytes,
                           void* stream) {
    if (!w) return ELQ_ERR_INVALID_ARG;
    elq_status st = check_qmat(w, w->n_rows, w->k);
    if (st != ELQ_OK) return st;
    if (T < 0) return ELQ_ERR_INVALID_ARG;
    if (T == 0) return ELQ_OK;
    if (!x_q8_1 || !y) return ELQ_ERR_INVALID_ARG;
    if (!aligned(x_q8_1, 16) || !aligned(y, 16)) return ELQ_ERR_ALIGNMENT;
    ProjWs lay = proj_layout(w, T, ws);
    if (!ws || ws_bytes < lay.total) return ELQ_ERR_WORKSPACE;
    if (!aligned(ws, 256)) return ELQ_ERR_ALIGNMENT;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (lay.tc) {
        PackArgs pa;
        std::memset(&pa, 0, sizeof(pa));
        pa.x = static_cast<const uint8_t*>(x_q8_1);
        pa.nb = w->k / 32;
        pa.mode = PACK_DENSE;
        pa.T = T;
        pa.bq = lay.bq;
        pa.bd = lay.bd;
        pa.bstride = lay.bstride;
        if (launch_pack(pa, s, false) != cudaSuccess) return ELQ_ERR_CUDA;
        TcArgs g = dense_tc(w, T, lay.bq, lay.bd, lay.bstride, TC_OUT_F32, y, nullptr, lay.err);
        return cuda_status(launch_tc(g, s, true));
    }
    if (T <= kSMaxT) {
        const SPlan sp = plan_s(w->fmt, X_Q81_TOKEN, false, w->n_rows, w->k, 1, T, false);
        if (sp.ok)
            return cuda_status(launch_s(dense_s(w, T, x_q8_1, 0, y, nullptr, lay.err), w->fmt, X_Q81_TOKEN, OUT_F32,
                                        sp, s, false));
    }
    WArgs g = dense_w(w, T, x_q8_1, X_Q81_TOKEN, 0, OUT_F32, y, nullptr, lay.partial, lay.counters, lay.err);
    return cuda_status(launch_w(g, w->fmt, lay.plan, s, false));
}

size_t elq_workspace_bytes(const elq_layer* layer, int32_t T) {
    if (check_layer(layer, T) != ELQ_OK || T <= 0) return 0;
    // the larger of the two input types' layouts
    return std::max(layer_layout(layer, T, nullptr, ELQ_F32).total, layer_layout(layer, T, nullptr, ELQ_BF16).total);
}

elq_status elq_moe_experts_grouped(const elq_layer* layer, const void* z_q8_1, const int32_t* idx,
                                   const float* weights, int32_t T, float* y_lat, void* ws, size_t ws_bytes,
                                   void* stream) {
    elq_status st = check_layer(layer, T);
    if (st != ELQ_OK) return st;
    if (T == 0) return ELQ_OK;
    if (!z_q8_1 || !idx || !weights || !y_lat) return ELQ_ERR_INVALID_ARG;
    if (!aligned(z_q8_1, 16) || !aligned(idx, 4) || !aligned(weights, 4) || !aligned(y_lat, 16))
        return ELQ_ERR_ALIGNMENT;
    LayerWs w = layer_layout(layer, T, ws, ELQ_F32);
    if (!ws || ws_bytes < w.total) return ELQ_ERR_WORKSPACE;
    if (!aligned(ws, 256)) return ELQ_ERR_ALIGNMENT;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const int E = layer->E, k = layer->k;
    const int64_t P = (int64_t)T * k;
    const int nw = 32;
    const bool nv = layer->gate_up.fmt == ELQ_NVFP4 || ext_fmt(layer->gate_up.fmt);
    if (nv && !w.nvtc) {
        const int gmax = (int)std::min<int64_t>(E, P);
        if (!plan_s(layer->gate_up.fmt, X_Q81_PAIR_TOKEN, true, 2 * layer->I, layer->L, gmax, T, true).ok ||
            !plan_s(layer->down.fmt, X_Q81_POSITION, false, layer->L, layer->I, gmax, T, true).ok)
            return ELQ_ERR_UNSUPPORTED;
    }
    cudaError_t e = smem_optin(k_bucket, kRouterSmemMax, g_optin_bucket);
    if (e != cudaSuccess) return ELQ_ERR_CUDA;
    e = launch(k_bucket, dim3(1), dim3(nw * 32), (size_t)nw * E * 4, s, false, idx, (int)P, E, w.counts, w.offsets,
               w.perm, w.pos, w.act, w.n_act);
    if (e != cudaSuccess) return ELQ_ERR_CUDA;
    if (!w.tc && T <= kSMaxT && P <= kSMaxPairs) {
        const int gmax = (int)std::min<int64_t>(E, P);
        const SPlan pgu = plan_s(layer->gate_up.fmt, X_Q81_PAIR_TOKEN, true, 2 * layer->I, layer->L, gmax, T, true);
        const SPlan pdn = plan_s(layer->down.fmt, X_Q81_POSITION, false, layer->L, layer->I, gmax, T, true);
        if (pgu.ok && pdn.ok) {
            if (launch_s(gate_up_s(layer, w, T, ROUTE_ARRAYS, static_cast<const uint8_t*>(z_q8_1)),
                         layer->gate_up.fmt, X_Q81_PAIR_TOKEN, OUT_SWIGLU, pgu, s, true) != cudaSuccess)
                return ELQ_ERR_CUDA;
            return cuda_status(launch_s(down_s(layer, w, T, ROUTE_ARRAYS, weights, y_lat), layer->down.fmt,
                                        X_Q81_POSITION, OUT_F32_COMBINE, pdn, s, true));
        }
    }
    if (w.nvtc) {
        if (cudaMemcpyAsync(w.idx, idx, (size_t)P * 4, cudaMemcpyDeviceToDevice, s) != cudaSuccess) return ELQ_ERR_CUDA;
        return run_experts_nvtc(layer, w, T, static_cast<const uint8_t*>(z_q8_1), weights, y_lat, s, true,
                                []() { return true; });
    }
    if (w.tc) {
        // the slot map reads idx from the workspace copy the layer call would have
        if (cudaMemcpyAsync(w.idx, idx, (size_t)P * 4, cudaMemcpyDeviceToDevice, s) != cudaSuccess) return ELQ_ERR_CUDA;
        return run_experts_tc(layer, w, T, static_cast<const uint8_t*>(z_q8_1), weights, y_lat, s, true,
                              []() { return true; });
    }
    return run_experts(layer, w, T, static_cast<const uint8_t*>(z_q8_1), weights, y_lat, s, true,
                       []() { return true; }, true);
}

elq_status elq_moe_layer(const elq_layer* layer, const void* x, int32_t x_type, int32_t T, float* y, void* ws,
                         size_t ws_bytes, void* stream) {
    return run_layer(layer, x, x_type, T, y, ws, ws_bytes, stream, nullptr, 0);
}

elq_status elq_moe_stack(const elq_layer* layers, int32_t n_layers, const void* x, int32_t x_type, int32_t T,
                         float* h, void* ws, size_t ws_bytes, void* stream) {
    if (!layers || n_layers <= 0) return ELQ_ERR_INVALID_ARG;
    if (x_type != ELQ_F32 && x_type != ELQ_BF16) return ELQ_ERR_UNSUPPORTED;
    for (int l = 0; l < n_layers; ++l) {
        const elq_status st = check_layer(&layers[l], T);
        if (st != ELQ_OK) return st;
        const elq_layer& a = layers[l];
        const elq_layer& b = layers[0];
        if (a.H != b.H || a.L != b.L || a.E != b.E || a.k != b.k || a.I != b.I || a.D.fmt != b.D.fmt ||
            a.U.fmt != b.U.fmt || a.gate_up.fmt != b.gate_up.fmt || a.down.fmt != b.down.fmt ||
            (a.router_bias == nullptr) != (b.router_bias == nullptr))
            return ELQ_ERR_INVALID_ARG;
    }
    if (T == 0) return ELQ_OK;
    if (!x || !h) return ELQ_ERR_INVALID_ARG;
    if (!aligned(x, 16) || !aligned(h, 16)) return ELQ_ERR_ALIGNMENT;
    if (!router_shape_ok(T, layers[0].L, layers[0].E)) return ELQ_ERR_UNSUPPORTED;
    const size_t lay = layer_layout(&layers[0], T, nullptr, ELQ_F32).total;
    const size_t need = lay + round_up((size_t)T * layers[0].H * 4, 256);
    if (!ws || ws_bytes < need) return ELQ_ERR_WORKSPACE;
    if (!aligned(ws, 256)) return ELQ_ERR_ALIGNMENT;
    float* xn = reinterpret_cast<float*>(static_cast<char*>(ws) + lay);   // the normalised layer input
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const int H = layers[0].H;
    const int64_t n = (int64_t)T * H;
    const dim3 grid((unsigned)((n + 255) / 256));
    cudaError_t e = (x_type == ELQ_BF16) ? launch(k_to_f32<true>, grid, dim3(256), 0, s, false, x, n, h)
                                         : launch(k_to_f32<false>, grid, dim3(256), 0, s, false, x, n, h);
    if (e != cudaSuccess) return ELQ_ERR_CUDA;
    for (int l = 0; l < n_layers; ++l) {
        e = launch(k_rmsnorm, dim3((unsigned)((T + 7) / 8)), dim3(256), 0, s, false, (const float*)h, T, H, xn);
        if (e != cudaSuccess) return ELQ_ERR_CUDA;
        const elq_status st = run_layer(&layers[l], xn, ELQ_F32, T, h, ws, lay, stream, nullptr, 0, true);
        if (st != ELQ_OK) return st;
    }
    return ELQ_OK;
}

size_t elq_stack_workspace_bytes(const elq_layer* layer, int32_t T) {
    if (check_layer(layer, T) != ELQ_OK || T <= 0) return 0;
    return layer_layout(layer, T, nullptr, ELQ_F32).total + round_up((size_t)T * layer->H * 4, 256);
}

int32_t elq_layer_kernel_count(const elq_layer* layer, int32_t T) {
    if (check_layer(layer, T) != ELQ_OK || T <= 0) return 0;
    return layer_kernels(layer, T);
}

elq_status elq_moe_layer_profiled(const elq_layer* layer, const void* x, int32_t x_type, int32_t T, float* y,
                                  void* ws, size_t ws_bytes, void* const* events, int32_t n_events, void* stream) {
    if (!events || T <= 0 || check_layer(layer, T) != ELQ_OK) return ELQ_ERR_INVALID_ARG;
    const int nk = layer_kernels(layer, T);
    if (n_events < nk + 1) return ELQ_ERR_INVALID_ARG;
    for (int i = 0; i < nk + 1; ++i)
        if (!events[i]) return ELQ_ERR_INVALID_ARG;
    return run_layer(layer, x, x_type, T, y, ws, ws_bytes, stream, events, n_events);
}

elq_status elq_workspace_view(const elq_layer* layer, int32_t T, int32_t which, size_t* offset, size_t* bytes) {
    if (check_layer(layer, T) != ELQ_OK || T <= 0 || !offset || !bytes) return ELQ_ERR_INVALID_ARG;
    char* const base = reinterpret_cast<char*>((uintptr_t)1 << 40);   // only offsets are taken
    LayerWs w = layer_layout(layer, T, base, ELQ_F32);
    const size_t Tz = (size_t)T, P = (size_t)T * layer->k, L = layer->L, H = layer->H, E = layer->E,
                 I = layer->I;
    const void* p = nullptr;
    size_t n = 0;
    const size_t ablk = layer->gate_up.fmt == ELQ_NVFP4 ? 18 : 36;   // the experts' activation blocks
    switch (which) {
    case 0: p = w.xq; n = Tz * (H / 32) * 36; break;
    case 1: p = w.z; n = Tz * L * 4; break;
    case 2: p = w.zq; n = Tz * (L / 32) * ablk; break;
    case 3: p = w.logits; n = Tz * E * 4; break;
    case 4: p = w.idx; n = P * 4; break;
    case 5: p = w.wts; n = P * 4; break;
    case 6: p = w.counts; n = E * 4; break;
    case 7: p = w.offsets; n = (E + 1) * 4; break;
    case 8: p = w.perm; n = P * 4; break;
    case 9: p = w.pos; n = P * 4; break;
    case 10: p = (w.tc || w.nvtc) ? nullptr : w.hq; n = P * (I / 32) * ablk; break;
    case 11: p = (w.tc || w.nvtc) ? nullptr : w.o; n = P * L * 4; break;
    case 12: p = w.ylat; n = Tz * L * 4; break;
    case 13: p = w.ylq; n = Tz * (L / 32) * 36; break;
    case 14: p = w.n_act; n = 4; break;
    default: return ELQ_ERR_INVALID_ARG;
    }
    if (!p) return ELQ_ERR_INVALID_ARG;   // not materialised at this T
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

elq_status elq_test_fused_timeout(const elq_layer* layer, const void* x, int32_t x_type, int32_t T, float* y,
                                  void* ws, size_t ws_bytes, uint64_t budget_ns, void* stream) {
    elq_status st = check_layer(layer, T);
    if (st != ELQ_OK) return st;
    if (x_type != ELQ_F32 && x_type != ELQ_BF16) return ELQ_ERR_UNSUPPORTED;
    if (T <= 0 || !x || !y) return ELQ_ERR_INVALID_ARG;
    if (!aligned(x, 16) || !aligned(y, 16)) return ELQ_ERR_ALIGNMENT;
    if (budget_ns < 1000000ull || budget_ns > kWaitBudgetNs) return ELQ_ERR_INVALID_ARG;
    LayerWs w = layer_layout(layer, T, ws, x_type);
    if (!w.fused) return ELQ_ERR_UNSUPPORTED;
    if (!ws || ws_bytes < w.total) return ELQ_ERR_WORKSPACE;
    if (!aligned(ws, 256)) return ELQ_ERR_ALIGNMENT;
    return run_fused(layer, w, x, x_type, T, y, static_cast<cudaStream_t>(stream), budget_ns, true);
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

elq_status elq_test_mma_i8_rate(int32_t n_mma, int32_t* sink, int32_t* err, void* stream) {
    if (n_mma < 2 || !sink || !err) return ELQ_ERR_INVALID_ARG;
    static bool optin[kMaxDevices];
    cudaError_t e = smem_optin(k_test_mma_i8_rate, kRateSmem, optin);
    if (e != cudaSuccess) return ELQ_ERR_CUDA;
    return cuda_status(launch(k_test_mma_i8_rate, dim3(sm_count()), dim3(128), (size_t)kRateSmem,
                              static_cast<cudaStream_t>(stream), false, (int)n_mma, (int*)sink, (int*)err,
                              kWaitBudgetNs));
}

elq_status elq_test_mma_f16_rate(int32_t n_mma, int32_t* sink, int32_t* err, void* stream) {
    if (n_mma < 2 || !sink || !err) return ELQ_ERR_INVALID_ARG;
    static bool optin[kMaxDevices];
    cudaError_t e = smem_optin(k_test_mma_f16_rate, kRateSmem, optin);
    if (e != cudaSuccess) return ELQ_ERR_CUDA;
    return cuda_status(launch(k_test_mma_f16_rate, dim3(sm_count()), dim3(128), (size_t)kRateSmem,
                              static_cast<cudaStream_t>(stream), false, (int)n_mma, (int*)sink, (int*)err,
                              kWaitBudgetNs));
}

elq_status elq_test_mma_nvf4_rate(int32_t n_mma, int32_t n_cols, int32_t cp_each, int32_t* sink, int32_t* err,
                                  void* stream) {
    if (n_mma < 1 || !sink || !err) return ELQ_ERR_INVALID_ARG;
    if (n_cols < 16 || n_cols > 256 || n_cols % 16) return ELQ_ERR_INVALID_ARG;
    static bool optin[kMaxDevices];
    // the int8 rate kernel's shared-memory request: one CTA (and one TMEM allocation) per SM
    cudaError_t e = smem_optin(k_test_mma_nvf4_rate, kRateSmem, optin);
    if (e != cudaSuccess) return ELQ_ERR_CUDA;
    return cuda_status(launch(k_test_mma_nvf4_rate, dim3(sm_count()), dim3(128), (size_t)kRateSmem,
                              static_cast<cudaStream_t>(stream), false, (int)n_mma, (int)n_cols, (int)(cp_each != 0),
                              (int*)sink, (int*)err, kWaitBudgetNs));
}

elq_status elq_test_f32x2_rate(int32_t n, float* sink, void* stream) {
    if (n < 1 || !sink) return ELQ_ERR_INVALID_ARG;
    return cuda_status(launch(k_test_f32x2_rate, dim3(2 * sm_count()), dim3(1024), 0,
                              static_cast<cudaStream_t>(stream), false, (int)n, sink));
}

int32_t elq_sm_count(void) { return sm_count(); }

elq_status elq_test_expf(const float* in, float* out, int64_t n, void* stream) {
    if (n < 0) return ELQ_ERR_INVALID_ARG;
    if (n == 0) return ELQ_OK;
    if (!in || !out) return ELQ_ERR_INVALID_ARG;
    k_test_expf<<<(unsigned)((n + 255) / 256), 256, 0, static_cast<cudaStream_t>(stream)>>>(in, out, n);
    return cuda_status(cudaGetLastError());
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Allocation-free latent projection.  Its scratch (error word, tile counters,
// chunk partial sums) lives in one file-scope device array instead of a
// caller-provided workspace.  In host code the array's name only stands for
// the symbol: its device address is looked up with cudaGetSymbolAddress, once
// per device, with that device current.

namespace {
constexpr size_t kStaticScratchBytes = (size_t)4 << 20;   // 4 MiB, held by every GPU that loads the library
}

static __device__ __align__(256) unsigned char g_elq_static_scratch[kStaticScratchBytes];

namespace {
std::mutex g_static_mu;
void* g_static_addr[kMaxDevices];

elq_status static_scratch_address(void** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return ELQ_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return ELQ_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_static_mu);
    if (!g_static_addr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_elq_static_scratch) != cudaSuccess || !p) return ELQ_ERR_CUDA;
        g_static_addr[dev] = p;
    }
    *out = g_static_addr[dev];
    return ELQ_OK;
}
}  // namespace

extern "C" elq_status elq_latent_proj_noalloc(const elq_qmat* w, const void* x_q8_1, int32_t T, float* y,
                                              void* stream) {
    if (!w) return ELQ_ERR_INVALID_ARG;
    elq_status st = check_qmat(w, w->n_rows, w->k);
    if (st != ELQ_OK) return st;
    if (T < 0) return ELQ_ERR_INVALID_ARG;
    if (T == 0) return ELQ_OK;
    if (!x_q8_1 || !y) return ELQ_ERR_INVALID_ARG;
    if (!aligned(x_q8_1, 16) || !aligned(y, 16)) return ELQ_ERR_ALIGNMENT;
    if (proj_layout(w, T, nullptr, false).total > kStaticScratchBytes) return ELQ_ERR_WORKSPACE;
    void* base = nullptr;
    if ((st = static_scratch_address(&base)) != ELQ_OK) return st;
    ProjWs lay = proj_layout(w, T, base, false);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    // the array keeps the previous call's contents: the error word and the
    // tile counters must start at zero
    if (cudaMemsetAsync(lay.err, 0, (64 + lay.plan.counter_ints) * sizeof(int), s) != cudaSuccess)
        return ELQ_ERR_CUDA;
    WArgs g = dense_w(w, T, x_q8_1, X_Q81_TOKEN, 0, OUT_F32, y, nullptr, lay.partial, lay.counters, lay.err);
    return cuda_status(launch_w(g, w->fmt, lay.plan, s, false));
}

extern "C" elq_status elq_latent_proj_noalloc_status(void* stream) {
    void* base = nullptr;
    elq_status st = static_scratch_address(&base);
    if (st != ELQ_OK) return st;
    // the error word is the first int of the array (proj_layout's first carve)
    int v = 0;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (cudaMemcpyAsync(&v, base, sizeof(int), cudaMemcpyDeviceToHost, s) != cudaSuccess) return ELQ_ERR_CUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess) return ELQ_ERR_CUDA;
    return v == 0 ? ELQ_OK : ELQ_ERR_TIMEOUT;
}

namespace {

// residual: y = y + layer(x) (the stack; the separate-kernel GEMV path only)
elq_status run_layer(const elq_layer* layer, const void* x, int32_t x_type, int32_t T, float* y, void* ws,
                     size_t ws_bytes, void* stream, void* const* events, int32_t n_events, bool residual) {
    elq_status st = check_layer(layer, T);
    if (st != ELQ_OK) return st;
    if (x_type != ELQ_F32 && x_type != ELQ_BF16) return ELQ_ERR_UNSUPPORTED;
    if (T == 0) return ELQ_OK;
    if (!x || !y) return ELQ_ERR_INVALID_ARG;
    if (!aligned(x, 16) || !aligned(y, 16)) return ELQ_ERR_ALIGNMENT;
    if (events && n_events < layer_kernels(layer, T) + 1) return ELQ_ERR_INVALID_ARG;
    if (!router_shape_ok(T, layer->L, layer->E)) return ELQ_ERR_UNSUPPORTED;
    LayerWs w = layer_layout(layer, T, ws, x_type);
    const bool nv = layer->gate_up.fmt == ELQ_NVFP4;
    if ((nv || ext_fmt(layer->gate_up.fmt)) && !w.small && !w.nvtc) return ELQ_ERR_UNSUPPORTED;
    if (!ws || ws_bytes < w.total) return ELQ_ERR_WORKSPACE;
    if (!aligned(ws, 256)) return ELQ_ERR_ALIGNMENT;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const int H = layer->H, L = layer->L, E = layer->E, k = layer->k;
    int ev = 0;
    std::function<bool()> mark = [&]() -> bool {
        if (!events) return true;
        return cudaEventRecord(static_cast<cudaEvent_t>(events[ev++]), s) == cudaSuccess;
    };
    const bool pdl = (events == nullptr);
    cudaError_t e;
    if (!mark()) return ELQ_ERR_CUDA;
    if (w.fused && !residual) {
        st = run_fused(layer, w, x, x_type, T, y, s);
        if (st != ELQ_OK) return st;
        return mark() ? ELQ_OK : ELQ_ERR_CUDA;
    }
    if (w.nvtc) {
        // NVFP4 experts, many tokens: a1 quantiser, packed x, D on the int8
        // tensor cores (z), z's NVFP4 rows, router, the block-scaled experts, U
        const int64_t nblk = (int64_t)T * (H / 32);
        if (x_type == ELQ_BF16)
            e = launch(k_quant_q8_1<true>, dim3((unsigned)((4 * nblk + 255) / 256)), dim3(256), 0, s, false, x,
                       nblk, w.xq);
        else
            e = launch(k_quant_q8_1<false>, dim3((unsigned)((4 * nblk + 255) / 256)), dim3(256), 0, s, false, x,
                       nblk, w.xq);
        if (e != cudaSuccess || !mark()) return ELQ_ERR_CUDA;
        PackArgs pa;
        std::memset(&pa, 0, sizeof(pa));
        pa.x = w.xq;
        pa.nb = H / 32;
        pa.mode = PACK_DENSE;
        pa.T = T;
        pa.bq = w.bxq;
        pa.bd = w.bxd;
        pa.bstride = w.tstride;
        pa.f16 = w.f16 ? 1 : 0;
        if (launch_pack(pa, s, pdl) != cudaSuccess || !mark()) return ELQ_ERR_CUDA;
        TcArgs gd = dense_tc(&layer->D, T, w.bxq, w.bxd, w.tstride, TC_OUT_F32, w.z, nullptr, w.err);
        gd.q16 = w.f16 ? static_cast<const uint8_t*>(layer->D.q16) : nullptr;
        if (launch_tc(gd, s, pdl) != cudaSuccess || !mark()) return ELQ_ERR_CUDA;
        const int64_t zblk = (int64_t)T * (L / 32);
        e = launch(k_quant_nvfp4<false>, dim3((unsigned)((zblk * 4 + 255) / 256)), dim3(256), 0, s, pdl,
                   (const void*)w.z, zblk, layer->act_gz, w.zq);
        if (e != cudaSuccess || !mark()) return ELQ_ERR_CUDA;
        e = launch_router(w.z, layer->router_w, layer->router_bias, T, L, E, k, w.idx, w.wts, w.logits,
                          w.cnt_router, true, w.counts, w.offsets, w.perm, w.pos, w.act, w.n_act, s, pdl);
        if (e != cudaSuccess || !mark()) return ELQ_ERR_CUDA;
        st = run_experts_nvtc(layer, w, T, w.zq, w.wts, w.ylat, s, pdl, mark);
        if (st != ELQ_OK) return st;
        TcArgs gu = dense_tc(&layer->U, T, w.byq, w.byd, w.tstride, residual ? TC_OUT_F32_ADD : TC_OUT_F32, y,
                             nullptr, w.err);
        gu.q16 = w.f16 ? static_cast<const uint8_t*>(layer->U.q16) : nullptr;
        if (launch_tc(gu, s, pdl) != cudaSuccess || !mark()) return ELQ_ERR_CUDA;
        return ELQ_OK;
    }
    if (w.tc) {
        // prefill: a1 quantiser, packed x, D on the tensor cores (z, zq), router,
        // then the tensor-core experts and U
        const int64_t nblk = (int64_t)T * (H / 32);
        if (x_type == ELQ_BF16)
            e = launch(k_quant_q8_1<true>, dim3((unsigned)((4 * nblk + 255) / 256)), dim3(256), 0, s, false, x,
                       nblk, w.xq);
        else
            e = launch(k_quant_q8_1<false>, dim3((unsigned)((4 * nblk + 255) / 256)), dim3(256), 0, s, false, x,
                       nblk, w.xq);
        if (e != cudaSuccess || !mark()) return ELQ_ERR_CUDA;
        PackArgs pa;
        std::memset(&pa, 0, sizeof(pa));
        pa.x = w.xq;
        pa.nb = H / 32;
        pa.mode = PACK_DENSE;
        pa.T = T;
        pa.bq = w.bxq;
        pa.bd = w.bxd;
        pa.bstride = w.tstride;
        pa.f16 = w.f16 ? 1 : 0;
        if (launch_pack(pa, s, pdl) != cudaSuccess || !mark()) return ELQ_ERR_CUDA;
        TcArgs gd = dense_tc(&layer->D, T, w.bxq, w.bxd, w.tstride, TC_OUT_F32_Q81, w.z, w.zq, w.err);
        gd.q16 = w.f16 ? static_cast<const uint8_t*>(layer->D.q16) : nullptr;
        if (launch_tc(gd, s, pdl) != cudaSuccess || !mark()) return ELQ_ERR_CUDA;
        e = launch_router(w.z, layer->router_w, layer->router_bias, T, L, E, k, w.idx, w.wts, w.logits,
                          w.cnt_router, true, w.counts, w.offsets, w.perm, w.pos, w.act, w.n_act, s, pdl);
        if (e != cudaSuccess || !mark()) return ELQ_ERR_CUDA;
        st = run_experts_tc(layer, w, T, w.zq, w.wts, w.ylat, s, pdl, mark);
        if (st != ELQ_OK) return st;
        TcArgs gu = dense_tc(&layer->U, T, w.byq, w.byd, w.tstride, residual ? TC_OUT_F32_ADD : TC_OUT_F32, y,
                             nullptr, w.err);
        gu.q16 = w.f16 ? static_cast<const uint8_t*>(layer->U.q16) : nullptr;
        if (launch_tc(gu, s, pdl) != cudaSuccess || !mark()) return ELQ_ERR_CUDA;
        return ELQ_OK;
    }
    if (w.small) {
        // a1 + a2 + a4: D (x quantised in the kernel; z, zq), asking L2 for
        // the router rows and U, which later kernels of the layer read
        const int dmode = x_type == ELQ_BF16 ? X_RAW_BF16 : X_RAW_F32;
        SArgs gd = dense_s(&layer->D, T, x, H, w.z, w.zq, w.err);
        gd.ogs = layer->act_gz;                 // NVFP4 experts: z's blocks under act_gz
        gd.pf[0] = reinterpret_cast<const uint8_t*>(layer->router_w);
        gd.pf_bytes[0] = (int64_t)E * L * 4;
        gd.pf[1] = static_cast<const uint8_t*>(layer->U.q);
        gd.pf_bytes[1] = (int64_t)(H / kTileRows) * (L / 32) * slab_bytes(layer->U.fmt);
        gd.pf[2] = static_cast<const uint8_t*>(layer->U.d);
        gd.pf_bytes[2] = (int64_t)(H / kTileRows) * (L / 32) * kScaleSlab;
        if (launch_s(gd, layer->D.fmt, dmode, nv ? OUT_F32_NV : OUT_F32_Q81, w.sd, s, pdl) != cudaSuccess || !mark())
            return ELQ_ERR_CUDA;
        // a3 + a5: the cluster router (logits, top-k, softmax, bucketing, group table)
        if (launch_route_small(layer, w, T, s, pdl) != cudaSuccess || !mark()) return ELQ_ERR_CUDA;
        // a6 + a7, then a8 + a9
        if (launch_s(gate_up_s(layer, w, T, ROUTE_GROUPS, w.zq), layer->gate_up.fmt, X_Q81_PAIR_TOKEN, OUT_SWIGLU,
                     w.sgu, s, pdl) != cudaSuccess ||
            !mark())
            return ELQ_ERR_CUDA;
        if (launch_s(down_s(layer, w, T, ROUTE_GROUPS, w.wts, w.ylat), layer->down.fmt, X_Q81_POSITION,
                     OUT_F32_COMBINE, w.sdn, s, pdl) != cudaSuccess ||
            !mark())
            return ELQ_ERR_CUDA;
        // a10
        SArgs gu = dense_s(&layer->U, T, w.ylq, 0, y, nullptr, w.err);
        if (launch_s(gu, layer->U.fmt, X_Q81_TOKEN, residual ? OUT_F32_ADD : OUT_F32, w.su, s, pdl) != cudaSuccess ||
            !mark())
            return ELQ_ERR_CUDA;
        return ELQ_OK;
    }
    // a1 + a2 + a4: D projection of x (quantised by the GEMV itself at small T)
    WArgs gd;
    if (w.raw) {
        gd = dense_w(&layer->D, T, x, x_type == ELQ_BF16 ? X_RAW_BF16 : X_RAW_F32, H, OUT_F32_Q81, w.z, w.zq,
                     w.partial, w.cnt_d, w.err);
    } else {
        const int64_t nblk = (int64_t)T * (H / 32);
        if (x_type == ELQ_BF16)
            e = launch(k_quant_q8_1<true>, dim3((unsigned)((4 * nblk + 255) / 256)), dim3(256), 0, s, false, x,
                       nblk, w.xq);
        else
            e = launch(k_quant_q8_1<false>, dim3((unsigned)((4 * nblk + 255) / 256)), dim3(256), 0, s, false, x,
                       nblk, w.xq);
        if (e != cudaSuccess || !mark()) return ELQ_ERR_CUDA;
        gd = dense_w(&layer->D, T, w.xq, X_Q81_TOKEN, 0, OUT_F32_Q81, w.z, w.zq, w.partial, w.cnt_d, w.err);
    }
    if (launch_w(gd, layer->D.fmt, w.pd, s, pdl) != cudaSuccess || !mark()) return ELQ_ERR_CUDA;
    // a3 + a5
    e = launch_router(w.z, layer->router_w, layer->router_bias, T, L, E, k, w.idx, w.wts, w.logits, w.cnt_router,
                      true, w.counts, w.offsets, w.perm, w.pos, w.act, w.n_act, s, pdl);
    if (e != cudaSuccess || !mark()) return ELQ_ERR_CUDA;
    // a6 - a9
    st = run_experts(layer, w, T, w.zq, w.wts, w.ylat, s, pdl, mark, pdl);
    if (st != ELQ_OK) return st;
    // a10
    WArgs gu = dense_w(&layer->U, T, w.ylq, X_Q81_TOKEN, 0, residual ? OUT_F32_ADD : OUT_F32, y, nullptr, w.partial,
                       w.cnt_u, w.err);
    if (launch_w(gu, layer->U.fmt, w.pu, s, pdl) != cudaSuccess || !mark()) return ELQ_ERR_CUDA;
    return ELQ_OK;
}

}  // namespace
