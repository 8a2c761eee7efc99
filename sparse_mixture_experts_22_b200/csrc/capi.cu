// capi.cu -- the C ABI (include/moe.h): argument checks, the per-config plan,
// TMA descriptors and the launch sequence of the layer.
//
// Every entry point validates on the host before launching anything and
// returns a moe_status; it never throws, allocates device memory or
// synchronises (moe_read_device_status and moe_trace_end excepted, as the
// header says).
#include <stdarg.h>
#include <stdio.h>
#include <string.h>

#include <atomic>
#include <mutex>
#include <string>
#include <vector>

#include "../../include/moe.h"
#include "common.cuh"
#include "kernels.h"
#include "plan.h"

namespace moe {

// ---------------------------------------------------------------- errors

static thread_local std::string g_err;

static int fail(int code, const char* fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof buf, fmt, ap);
    va_end(ap);
    g_err = buf;
    return code;
}

static int ok() {
    g_err.clear();
    return MOE_OK;
}

// Records `text` as this thread's last error (cleared for MOE_OK); returns code.
int report_error(int code, const char* text) {
    if (code == MOE_OK) g_err.clear();
    else g_err = text;
    return code;
}

#define MOE_TRY(expr)                   \
    do {                                \
        int _s = (expr);                \
        if (_s != MOE_OK) return _s;    \
    } while (0)

cudaError_t& last_launch_error() {
    static thread_local cudaError_t e = cudaSuccess;
    return e;
}

static int launched(int rc, const char* what) {
    if (rc == 0) return MOE_OK;
    cudaError_t e = last_launch_error();
    last_launch_error() = cudaSuccess;
    if (e == cudaSuccess) e = cudaGetLastError();
    return fail(MOE_ERR_CUDA, "%s: launch failed: %s (%d)", what, cudaGetErrorString(e), (int)e);
}

// ---------------------------------------------------------------- plan

static size_t align256(size_t v) { return (v + 255) & ~(size_t)255; }

int make_plan(const moe_config* cfg, Plan* p, const char** why) {
    if (!cfg) { *why = "cfg is NULL"; return MOE_ERR_ARG; }
    const moe_config& c = *cfg;
    if (c.T < 0 || c.T > (1LL << 30)) { *why = "T must be in [0, 2^30]"; return MOE_ERR_SHAPE; }
    if (c.d < 128 || c.d % 128 || c.d > 65536) { *why = "d must be a multiple of 128 in [128, 65536]"; return MOE_ERR_SHAPE; }
    if (c.h < 128 || c.h % 128 || c.h > 262144) { *why = "h must be a multiple of 128 in [128, 262144]"; return MOE_ERR_SHAPE; }
    if (c.E < 1 || c.E > MAX_E) { *why = "E must be in [1, 1024]"; return MOE_ERR_SHAPE; }
    if (c.k < 1 || c.k > MAX_K || c.k > c.E) { *why = "k must be in [1, min(E, 8)]"; return MOE_ERR_SHAPE; }
    if (c.n_shared < 0 || c.n_shared > 64) { *why = "n_shared must be in [0, 64]"; return MOE_ERR_SHAPE; }
    if (c.n_shared > 0 && (c.h_shared < 128 || c.h_shared % 128)) { *why = "h_shared must be a multiple of 128"; return MOE_ERR_SHAPE; }
    if (c.cf_den < 0 || (c.cf_den > 0 && (c.cf_num <= 0 || c.cf_num > (1 << 20) || c.cf_den > (1 << 20)))) {
        *why = "capacity factor must be cf_num/cf_den with 0 < cf_num, cf_den <= 2^20 (cf_den = 0: no limit)";
        return MOE_ERR_ARG;
    }
    if (c.act_dtype != MOE_F32 && c.act_dtype != MOE_BF16) { *why = "act_dtype must be MOE_F32 or MOE_BF16"; return MOE_ERR_DTYPE; }
    if (c.has_bias != 0 && c.has_bias != 1) { *why = "has_bias must be 0 or 1"; return MOE_ERR_ARG; }
    if (c.overflow != MOE_OVERFLOW_DROP && c.overflow != MOE_OVERFLOW_REROUTE) {
        *why = "overflow must be MOE_OVERFLOW_DROP or MOE_OVERFLOW_REROUTE";
        return MOE_ERR_ARG;
    }
    if (c.train != 0 && c.train != 1) { *why = "train must be 0 or 1"; return MOE_ERR_ARG; }
    if (c.train && c.act_dtype != MOE_BF16) {
        *why = "train = 1 (backward pass) needs act_dtype MOE_BF16";
        return MOE_ERR_UNSUPPORTED;
    }
    if (c.hidden_mode != MOE_HIDDEN_AUTO && c.hidden_mode != MOE_HIDDEN_SPLIT &&
        c.hidden_mode != MOE_HIDDEN_BF16) {
        *why = "hidden_mode must be MOE_HIDDEN_AUTO, MOE_HIDDEN_SPLIT or MOE_HIDDEN_BF16";
        return MOE_ERR_ARG;
    }

    Plan& P = *p;
    P.T = c.T; P.d = c.d; P.h = c.h; P.E = c.E; P.k = c.k; P.S = c.n_shared;
    P.hs = c.n_shared ? c.h_shared : 0;
    P.hsum = P.S * P.hs;
    P.capped = c.cf_den > 0;
    P.reroute = P.capped && c.overflow == MOE_OVERFLOW_REROUTE;
    if (P.capped) {
        const int64_t num = c.T * (int64_t)c.k * c.cf_num;
        const int64_t den = (int64_t)c.E * c.cf_den;
        P.C = (num + den - 1) / den;
    } else {
        P.C = c.T;
    }
    const int64_t nmax = P.C < P.T ? P.C : P.T;  // most rows one expert can keep
    P.bf16 = c.act_dtype == MOE_BF16;
    P.act_bytes = P.bf16 ? 2 : 4;
    // H as two bf16 parts: asked for, or (auto) when no expert can keep more
    // than DOWN_SWAP_MAX_TOKENS rows -- the down projection then streams its
    // weights through swapped tiles, and the second MMA per K step runs on
    // tensor cores that wait for HBM anyway
    P.split = P.bf16 && (c.hidden_mode == MOE_HIDDEN_SPLIT ||
                         (c.hidden_mode == MOE_HIDDEN_AUTO && nmax <= DOWN_SWAP_MAX_TOKENS));
    if (!P.bf16) {
        P.path = PATH_F32;
        P.shared_path = PATH_F32;
        P.pad = 16;
    } else {
        P.path = nmax <= SWAP_MAX_TOKENS ? PATH_SWAP : PATH_TOKEN_MAJOR;
        P.shared_path = P.T <= SWAP_MAX_TOKENS ? PATH_SWAP : PATH_TOKEN_MAJOR;
        // the backward pass contracts whole 64-row blocks of each segment
        P.pad = P.path == PATH_TOKEN_MAJOR ? 128 : (c.train ? 64 : 16);
    }
    P.nt_max = (int)(((nmax > 0 ? nmax : 1) + 15) / 16 * 16);
    // split-K of the swapped down projection: enough units for ~6.5 waves of 148 SMs
    P.splits = 1;
    // split-K partials only for the swapped down projection, which serves groups
    // of at most 128 tokens (larger ones take the token-major down tiles)
    if (P.path == PATH_SWAP && P.nt_max <= DOWN_SWAP_MAX_TOKENS) {
        const int64_t units = (int64_t)P.E * (P.d / 128);
        const int kblocks = P.h / 64;
        while (P.splits < 8 && units * P.splits < 960 && kblocks % (P.splits * 2) == 0)
            P.splits *= 2;
    }
    // router: one CTA per token for small batches; tensor cores (three bf16 parts
    // of W_r) for larger bf16 batches; fp32 dot products for larger fp32 batches
    P.router_npad = P.E;
    P.router_ld = P.E;
    P.router_bn = 0;
    P.router_splits = 1;
    if (P.T <= SWAP_MAX_TOKENS) {
        P.router_kind = ROUTER_ROWS;
    } else if (P.bf16) {
        P.router_kind = ROUTER_TC;
        P.router_bn = 3 * P.E <= 128 ? 128 : 256;
        P.router_npad = (3 * P.E + P.router_bn - 1) / P.router_bn * P.router_bn;
        // split K four ways at least (each fp32 accumulation chain in TMEM
        // covers at most a quarter of d; the partial sums are added in fp32
        // afterwards) and further until the tiles cover most SMs
        const int64_t units = ((P.T + 127) / 128) * (P.router_npad / P.router_bn);
        const int kblocks = P.d / 64;
        while (P.router_splits < 8 && kblocks % (P.router_splits * 2) == 0 &&
               (P.router_splits < 4 || units * P.router_splits < 120))
            P.router_splits *= 2;
        P.router_ld = (3 * P.E + 3) / 4 * 4;
    } else {
        P.router_kind = ROUTER_SIMT;
    }
    const int64_t assign = c.T * (int64_t)c.k;
    const int64_t cap_all = (int64_t)c.E * nmax;
    const int64_t kept_max = assign < cap_all ? assign : cap_all;
    P.perm_rows = c.T > 0 ? kept_max + (int64_t)c.E * (P.pad - 1) : 0;
    P.nblk = (int)((c.T + ROUTE_BLOCK - 1) / ROUTE_BLOCK);
    // wide routing over more than one block: TOPK_SUB CTAs per block
    P.nsub = (c.E > TOPK_WARP_E && c.T > ROUTE_BLOCK) ? TOPK_SUB : 1;

    size_t o = 0;
    auto take = [&](size_t bytes) { size_t at = o; o = align256(o + bytes); return at; };
    P.off_status = take(256);
    P.off_logits = take((size_t)c.T * c.E * 4);
    P.off_wsplit = take(P.router_kind == ROUTER_TC ? (size_t)3 * c.E * c.d * 2 : 0);
    P.off_z3 = take(P.router_kind == ROUTER_TC ? (size_t)P.router_splits * c.T * P.router_ld * 4
                                               : 0);
    P.off_ppart = take((size_t)P.nblk * P.nsub * c.E * 4);
    P.off_hpart = take((size_t)P.nblk * P.nsub * 4);
    P.off_cnt = take((size_t)P.nblk * P.nsub * c.E * 4);
    P.off_tot = take((size_t)c.E * 4);
    P.off_expert = take(P.reroute ? (size_t)c.T * c.k * 4 : 0);
    P.off_rank = take(P.reroute ? (size_t)c.T * c.k * 4 : 0);
    P.off_offsets = take((size_t)(c.E + 1) * 4);
    P.off_perm = take((size_t)P.perm_rows * 4);
    P.off_xperm = take((size_t)P.perm_rows * c.d * P.act_bytes);
    // H [perm_rows][h]; split: the low parts in the next perm_rows rows
    P.off_H = take((size_t)(P.split ? 2 : 1) * P.perm_rows * c.h * P.act_bytes);
    P.off_y = take((size_t)P.splits * P.perm_rows * c.d * 4);
    P.off_Hs = take(P.S ? (size_t)(P.split ? 2 : 1) * c.T * P.hsum * P.act_bytes : 0);
    P.off_ys = take(P.S ? (size_t)c.T * c.d * 4 : 0);
    P.off_sums = take((size_t)(2 + 3 * c.E) * 8);
    P.train = c.train != 0;
    P.off_AB = take(P.train ? (size_t)P.perm_rows * 2 * c.h * 2 : 0);
    P.off_ABs = take(P.train && P.S ? (size_t)c.T * 2 * P.hsum * 2 : 0);
    P.total = o;

    // backward workspace
    P.wr_chunks = P.train ? wr_grad_chunks(c.T, c.d, c.E) : 1;
    o = 0;
    const bool tr = P.train;
    P.b_dY = take(tr ? (size_t)P.perm_rows * c.d * 2 : 0);
    P.b_dg = take(tr ? (size_t)c.T * c.k * 4 : 0);
    P.b_dz = take(tr ? (size_t)c.T * c.E * 4 : 0);
    P.b_dAB = take(tr ? (size_t)P.perm_rows * 2 * c.h * 2 : 0);
    P.b_dXp = take(tr ? (size_t)P.perm_rows * c.d * 4 : 0);
    const bool ts = tr && P.S > 0;
    P.b_dABs = take(ts ? (size_t)c.T * 2 * P.hsum * 2 : 0);
    P.b_dXs = take(ts ? (size_t)c.T * c.d * 4 : 0);
    P.b_wrpart = take(tr ? (size_t)P.wr_chunks * (c.d + 1) * c.E * 4 : 0);
    P.b_dxr = take(tr && c.E > 16 ? (size_t)c.T * c.d * 4 : 0);
    P.b_total = o;
    return MOE_OK;
}

static int plan_or_fail(const moe_config* cfg, Plan* p) {
    const char* why = "";
    int s = make_plan(cfg, p, &why);
    if (s != MOE_OK) return fail(s, "invalid config: %s", why);
    return MOE_OK;
}

// ---------------------------------------------------------------- device facts

struct Device {
    int sms = 0;
    int smem_optin = 0;
    bool sm100 = false;
};

static int device_facts(Device* dv) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return fail(MOE_ERR_CUDA, "cudaGetDevice failed");
    static std::mutex mu;
    static std::vector<Device> cache;
    std::lock_guard<std::mutex> lk(mu);
    if ((int)cache.size() <= dev) cache.resize(dev + 1);
    Device& c = cache[dev];
    if (c.sms == 0) {
        int major = 0, minor = 0;
        cudaDeviceGetAttribute(&c.sms, cudaDevAttrMultiProcessorCount, dev);
        cudaDeviceGetAttribute(&c.smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
        cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
        c.sm100 = (major == 10 && minor == 0);
        if (c.sms == 0) return fail(MOE_ERR_CUDA, "could not query the device");
    }
    *dv = c;
    if (!c.sm100) return fail(MOE_ERR_UNSUPPORTED, "this library is built for sm_100a (B200) only");
    return MOE_OK;
}

// ---------------------------------------------------------------- TMA descriptors

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

// bf16 row-major [rows][cols], box of 64 columns (128 B, 128-byte swizzle) x box_rows.
static int tmap_bf16(CUtensorMap* m, const void* ptr, int64_t rows, int64_t cols, int box_rows) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return fail(MOE_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable");
    cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)cols * 2};
    cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides,
                    box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS)
        return fail(MOE_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d) for a %lldx%lld tensor", (int)r,
                    (long long)rows, (long long)cols);
    return MOE_OK;
}

// ---------------------------------------------------------------- dependent launch

static int g_pdl_enabled = 1;
static thread_local bool g_pdl_in_forward = false;
// CTA-pair GEMM tiles: 0 none, 1 token-major tiles of groups that may hold
// >= PAIR_TOK_MIN_TOKENS rows, 2 also swapped tiles of groups of 129..256 rows
static int g_pair_enabled = 1;

bool pdl_active() { return g_pdl_enabled && g_pdl_in_forward; }

struct PdlScope {
    PdlScope() { g_pdl_in_forward = true; }
    ~PdlScope() { g_pdl_in_forward = false; }
};

// ---------------------------------------------------------------- launch count

static std::atomic<uint64_t> g_launches{0};

void note_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }

// ---------------------------------------------------------------- limits and tracing

static uint64_t g_wait_limit_ns = 2000000000ull;
static int g_test_stall = 0;

struct TraceMark {
    cudaEvent_t ev;
    const char* name;
    int call;
    bool pre;
};

// Per-kernel timing.  Without a filter every kernel of a moe_forward call is
// timed from the end of the previous one (one event after each launch).  With
// a filter only the named kernel is bracketed (one event before and one after
// its launch), which perturbs the rest of the step least.
struct Tracer {
    bool on = false;
    int max_calls = 0;
    int calls = 0;
    std::string only;
    std::vector<cudaEvent_t> pool;
    std::vector<TraceMark> marks;
};

static Tracer g_trace;

static void trace_record(cudaStream_t st, const char* name, bool pre) {
    if (!g_trace.on || g_trace.calls > g_trace.max_calls || g_trace.calls == 0) return;
    if (g_trace.marks.size() >= g_trace.pool.size()) return;
    cudaEvent_t ev = g_trace.pool[g_trace.marks.size()];
    cudaEventRecord(ev, st);
    g_trace.marks.push_back({ev, name, g_trace.calls, pre});
}

static void trace_pre(cudaStream_t st, const char* name) {
    if (g_trace.on && !g_trace.only.empty() && g_trace.only == name) trace_record(st, name, true);
}

static void trace_mark(cudaStream_t st, const char* name) {
    if (!g_trace.on) return;
    if (g_trace.only.empty() || g_trace.only == name) trace_record(st, name, false);
}

static void trace_call_begin(cudaStream_t st) {
    if (!g_trace.on) return;
    ++g_trace.calls;
    if (g_trace.only.empty()) trace_record(st, "begin", true);
}

// ---------------------------------------------------------------- checks

static int need_ws(const void* ws, size_t ws_bytes, const Plan& P) {
    if (!ws) return fail(MOE_ERR_ARG, "ws is NULL");
    if (reinterpret_cast<uintptr_t>(ws) & 255)
        return fail(MOE_ERR_ALIGN, "ws is not 256-byte aligned");
    if (ws_bytes < P.total)
        return fail(MOE_ERR_WORKSPACE, "workspace has %zu bytes; this config needs %zu", ws_bytes,
                    P.total);
    return MOE_OK;
}

static bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

static int need(const void* p, const char* name) {
    if (!p) return fail(MOE_ERR_ARG, "%s is NULL", name);
    if (!aligned16(p)) return fail(MOE_ERR_ALIGN, "%s is not 16-byte aligned", name);
    return MOE_OK;
}

static int maybe(const void* p, const char* name) {
    if (p && !aligned16(p)) return fail(MOE_ERR_ALIGN, "%s is not 16-byte aligned", name);
    return MOE_OK;
}

template <typename T>
static T* at(void* ws, size_t off) {
    return reinterpret_cast<T*>(reinterpret_cast<uint8_t*>(ws) + off);
}

template <typename T>
static const T* at(const void* ws, size_t off) {
    return reinterpret_cast<const T*>(reinterpret_cast<const uint8_t*>(ws) + off);
}

// ---------------------------------------------------------------- steps

static int run_tc_router(const Plan& P, const Device& dv, const void* x, const void* Ws,
                         float* z3, int32_t* status, cudaStream_t st) {
    CUtensorMap m_act, m_w;
    TcArgs a;
    memset(&a, 0, sizeof a);
    a.num_groups = 1;
    a.dense_rows = (int)P.T;
    a.K = P.d;
    a.n_feat = P.router_npad;
    a.w_rows_per_group = P.router_npad;
    a.status = status;
    a.wait_limit_ns = g_wait_limit_ns;
    a.out = z3;
    a.out_ld = P.router_ld;       // compact rows: only the 3E logit parts are stored
    a.out_cols = P.router_ld;
    a.splits = P.router_splits;
    a.split_stride = P.T * (int64_t)P.router_ld;
    // rows past 3E of the split weights lie outside the tensor map: TMA reads zeros there
    MOE_TRY(tmap_bf16(&m_act, x, P.T, P.d, 128));
    MOE_TRY(tmap_bf16(&m_w, Ws, 3LL * P.E, P.d, P.router_bn));
    a.stages = tc_max_stages(TC_DOWN_TOK, P.router_bn, 16, 1, false, dv.smem_optin);
    if (a.stages < 2) return fail(MOE_ERR_UNSUPPORTED, "shared memory too small for the GEMM tiles");
    trace_pre(st, "router_gemm");
    MOE_TRY(launched(launch_tc_gemm(TC_DOWN_TOK, P.router_bn, m_act, m_w, a, dv.sms, st),
                     "router_gemm"));
    trace_mark(st, "router_gemm");
    return MOE_OK;
}

// Router logits (partials), ready for top-k: fills r.src / nsplit / nparts / strides / bias.
static int step_logits(const Plan& P, const Device& dv, const void* x, const float* Wr,
                       const float* bias, void* ws, RouteParams& r, cudaStream_t st) {
    float* z = at<float>(ws, P.off_logits);
    float* z3 = at<float>(ws, P.off_z3);
    r.src = z;
    r.bias = bias;
    if (P.router_kind == ROUTER_ROWS) {
        trace_pre(st, "router_rows");
        MOE_TRY(launched(launch_router_rows(x, P.bf16, Wr, z, (int)P.T, P.d, P.E, st),
                         "router_rows"));
        trace_mark(st, "router_rows");
    } else if (P.router_kind == ROUTER_TC) {
        void* Ws = at<void>(ws, P.off_wsplit);
        trace_pre(st, "router_split");
        MOE_TRY(launched(launch_router_split(Wr, Ws, P.d, P.E, st), "router_split"));
        trace_mark(st, "router_split");
        MOE_TRY(run_tc_router(P, dv, x, Ws, z3, r.status, st));
        trace_pre(st, "router_reduce");
        MOE_TRY(launched(launch_router_reduce(z3, P.router_splits, P.T * (int64_t)P.router_ld,
                                              P.router_ld, 3, bias, z, P.T, P.E, st),
                         "router_reduce"));
        trace_mark(st, "router_reduce");
        r.bias = nullptr;  // already added
    } else {
        trace_pre(st, "router_logits");
        MOE_TRY(launched(launch_router_logits(x, P.bf16, Wr, z, P.T, P.d, P.E, dv.sms, st),
                         "router_logits"));
        trace_mark(st, "router_logits");
    }
    return MOE_OK;
}

static RouteParams route_params(const Plan& P, void* ws, int32_t* topk_idx, float* topk_gate,
                                float* logits) {
    RouteParams r;
    memset(&r, 0, sizeof r);
    r.zbuf = at<float>(ws, P.off_logits);
    r.logits = logits;
    r.T = P.T;
    r.E = P.E;
    r.k = P.k;
    r.topk_idx = topk_idx;
    r.topk_gate = topk_gate;
    r.ppart = at<float>(ws, P.off_ppart);
    r.hpart = at<float>(ws, P.off_hpart);
    r.cnt = at<int32_t>(ws, P.off_cnt);
    r.nsub = P.nsub;
    r.status = at<int32_t>(ws, P.off_status);
    return r;
}

static DispatchParams dispatch_params(const Plan& P, const void* x, int32_t* routed,
                                      int32_t* kept, int32_t* offsets, int32_t* perm_token,
                                      int32_t* slot_of, void* x_perm) {
    DispatchParams d;
    d.T = P.T;
    d.E = P.E;
    d.k = P.k;
    d.C = P.C;
    d.pad = P.pad;
    d.perm_rows = P.perm_rows;
    d.x = x;
    d.row_bytes = P.d * P.act_bytes;
    d.routed = routed;
    d.kept = kept;
    d.offsets = offsets;
    d.perm_token = perm_token;
    d.slot_of = slot_of;
    d.x_perm = x_perm;
    d.cap = nullptr;
    d.nsub = P.nsub;
    d.peer_rows = nullptr;  // one destination: x_perm
    d.npeer = 0;
    d.peer_start = nullptr;
    d.e_loc = P.E;
    return d;
}

static int empty_batch(const Plan& P, void* ws, int32_t* routed, int32_t* kept,
                       int32_t* offsets, cudaStream_t st) {
    // status reset; zero counts and offsets so later steps see no work
    if (cudaMemsetAsync(ws, 0, 256, st) != cudaSuccess ||
        (routed && cudaMemsetAsync(routed, 0, P.E * 4, st) != cudaSuccess) ||
        (kept && cudaMemsetAsync(kept, 0, P.E * 4, st) != cudaSuccess) ||
        (offsets && cudaMemsetAsync(offsets, 0, (P.E + 1) * 4, st) != cudaSuccess))
        return fail(MOE_ERR_CUDA, "memset failed");
    return MOE_OK;
}

static int step_route(const Plan& P, const Device& dv, const void* x, const float* Wr,
                      const float* bias, int32_t* topk_idx, float* topk_gate, float* logits,
                      void* ws, cudaStream_t st) {
    if (P.T == 0) return empty_batch(P, ws, nullptr, nullptr, nullptr, st);
    RouteParams r = route_params(P, ws, topk_idx, topk_gate, logits);
    MOE_TRY(step_logits(P, dv, x, Wr, bias, ws, r, st));
    // the reroute policy ranks spare experts by logit: keep logits + bias in ws
    if (P.reroute) r.logits = at<float>(ws, P.off_logits);
    trace_pre(st, "topk");
    MOE_TRY(launched(launch_topk(r, st), "topk"));
    trace_mark(st, "topk");
    if (P.reroute && logits &&
        cudaMemcpyAsync(logits, r.logits, (size_t)P.T * P.E * 4, cudaMemcpyDeviceToDevice, st) !=
            cudaSuccess)
        return fail(MOE_ERR_CUDA, "logits copy failed");
    return MOE_OK;
}

static int step_dispatch(const Plan& P, const Device& dv, const int32_t* topk_idx, const void* x,
                         int32_t* routed, int32_t* kept, int32_t* offsets, int32_t* perm_token,
                         int32_t* slot_of, void* x_perm, void* ws, cudaStream_t st) {
    if (P.T == 0) return empty_batch(P, ws, routed, kept, offsets, st);
    DispatchParams d = dispatch_params(P, x, routed, kept, offsets, perm_token, slot_of, x_perm);
    trace_pre(st, "dispatch");
    if (P.reroute)
        MOE_TRY(launched(launch_reroute_dispatch(d, topk_idx, at<int32_t>(ws, P.off_cnt),
                                                 at<int32_t>(ws, P.off_tot),
                                                 at<float>(ws, P.off_logits),
                                                 at<int32_t>(ws, P.off_expert),
                                                 at<int32_t>(ws, P.off_rank), dv.sms, st),
                         "dispatch"));
    else
        MOE_TRY(launched(launch_dispatch(d, topk_idx, at<int32_t>(ws, P.off_cnt),
                                         at<int32_t>(ws, P.off_tot), dv.sms, st),
                         "dispatch"));
    trace_mark(st, "dispatch");
    return MOE_OK;
}

// Router, top-k and dispatch of moe_forward: one fused launch for top-k and
// dispatch when the batch fits one routing block.
static int step_route_dispatch(const Plan& P, const Device& dv, const void* x, const float* Wr,
                               const float* bias, int32_t* topk_idx, float* topk_gate,
                               int32_t* routed, int32_t* kept, int32_t* offsets,
                               int32_t* perm_token, int32_t* slot_of, void* x_perm, void* ws,
                               cudaStream_t st) {
    if (P.T == 0) return empty_batch(P, ws, routed, kept, offsets, st);
    if (P.T > ROUTE_BLOCK || P.reroute) {
        MOE_TRY(step_route(P, dv, x, Wr, bias, topk_idx, topk_gate, nullptr, ws, st));
        return step_dispatch(P, dv, topk_idx, x, routed, kept, offsets, perm_token, slot_of,
                             x_perm, ws, st);
    }
    RouteParams r = route_params(P, ws, topk_idx, topk_gate, nullptr);
    MOE_TRY(step_logits(P, dv, x, Wr, bias, ws, r, st));
    DispatchParams d = dispatch_params(P, x, routed, kept, offsets, perm_token, slot_of, x_perm);
    trace_pre(st, "route_dispatch");
    MOE_TRY(launched(launch_route_dispatch(r, d, dv.sms, st), "route_dispatch"));
    trace_mark(st, "route_dispatch");
    return MOE_OK;
}

// One grouped GEMM pair (gate/up then down) on the tensor cores.
static int run_tc_ffn(const Plan& P, const Device& dv, int path, int groups,
                      const int32_t* rows, const int32_t* offs, const int32_t* group_w,
                      int dense_rows, const void* act,
                      int64_t act_rows, const void* W13, const void* W2p, int hid, void* H,
                      void* AB, float* y, int splits, int nt_max, int32_t* status,
                      cudaStream_t st, const char* tag1, const char* tag2, int ctr_slot = 0) {
    const bool tok = path == PATH_TOKEN_MAJOR;
    CUtensorMap m_act, m_w;
    TcArgs a;
    memset(&a, 0, sizeof a);
    a.num_groups = groups;
    a.group_rows = rows;
    a.group_off = offs;
    a.group_w = group_w;
    a.dense_rows = dense_rows;
    a.status = status;
    a.wait_limit_ns = g_wait_limit_ns;
    a.test_stall = g_test_stall;
    a.nt_max = nt_max;
    const int smem_limit = dv.smem_optin;

    // split H: its low bf16 parts follow the high ones, act_rows rows further
    a.lo_rows = P.split ? act_rows : 0;
    // the CTA-pair kernels take their units from a counter in the status area
    // (one per stream that may run them at once), zeroed before each launch
    a.unit_ctr = status + UNIT_CTR_WORD + ctr_slot;
    auto zero_ctr = [&]() -> int {
        if (cudaMemsetAsync(a.unit_ctr, 0, sizeof(int32_t), st) != cudaSuccess)
            return fail(MOE_ERR_CUDA, "memset failed");
        return MOE_OK;
    };

    // gate/up: act [act_rows][d] x W13 [groups * 2hid][d] -> H [act_rows][hid]
    const int mode1 = tok ? TC_GATEUP_TOK : TC_GATEUP_SWAP;
    MOE_TRY(tmap_bf16(&m_act, act, act_rows, P.d, tok ? 128 : swap_gateup_tok_box(nt_max)));
    MOE_TRY(tmap_bf16(&m_w, W13, (int64_t)groups * 2 * hid, P.d, tok ? 256 : 128));
    a.K = P.d;
    a.n_feat = hid;
    a.w_rows_per_group = 2 * hid;
    a.splits = 1;
    a.out = H;
    a.out_ld = hid;
    a.split_stride = 0;
    a.aux = AB;  // pre-activations for the backward pass (null: not kept)
    a.aux_ld = 2 * (int64_t)hid;
    // groups of more than 128 (and at most 256) tokens: swapped tiles on CTA
    // pairs, each SM staging half of the token rows
    const bool pair = !tok && g_pair_enabled >= 2 && nt_max > DOWN_SWAP_MAX_TOKENS;
    // groups that may hold thousands of tokens: token-major tiles of 256 tokens on
    // CTA pairs (a third less shared-memory fill per flop; the 256-row tiles pad
    // an expert's rows more than 128-row tiles, which pays off for large groups)
    const bool pair_tok = tok && g_pair_enabled >= 1 && nt_max >= PAIR_TOK_MIN_TOKENS &&
                          hid % 128 == 0 && P.d % 256 == 0;
    if (pair_tok) {
        MOE_TRY(tmap_bf16(&m_act, act, act_rows, P.d, 128));
        MOE_TRY(tmap_bf16(&m_w, W13, (int64_t)groups * 2 * hid, P.d, 128));
        a.stages = tc_pair_max_stages(TC_PAIR_GATEUP_TOK, nt_max, groups, false, smem_limit);
        if (a.stages < 2) return fail(MOE_ERR_UNSUPPORTED, "shared memory too small for the GEMM tiles");
        MOE_TRY(zero_ctr());
        trace_pre(st, tag1);
        MOE_TRY(launched(launch_tc_pair(TC_PAIR_GATEUP_TOK, m_act, m_w, a, dv.sms / 2, st), tag1));
        trace_mark(st, tag1);
        MOE_TRY(tmap_bf16(&m_act, H, (P.split ? 2 : 1) * act_rows, hid, 128));
        MOE_TRY(tmap_bf16(&m_w, W2p, (int64_t)groups * P.d, hid, 128));
        a.K = hid;
        a.n_feat = P.d;
        a.w_rows_per_group = P.d;
        a.splits = 1;
        a.out = y;
        a.out_ld = P.d;
        a.split_stride = act_rows * (int64_t)P.d;
        a.aux = nullptr;
        a.prefetch_kb = 0;
        a.stages = tc_pair_max_stages(TC_PAIR_DOWN_TOK, nt_max, groups, P.split, smem_limit);
        if (a.stages < 2) return fail(MOE_ERR_UNSUPPORTED, "shared memory too small for the GEMM tiles");
        MOE_TRY(zero_ctr());
        trace_pre(st, tag2);
        MOE_TRY(launched(launch_tc_pair(TC_PAIR_DOWN_TOK, m_act, m_w, a, dv.sms / 2, st), tag2));
        trace_mark(st, tag2);
        return MOE_OK;
    }
    if (pair) {
        MOE_TRY(tmap_bf16(&m_act, act, act_rows, P.d, pair_swap_tok_box(nt_max)));
        MOE_TRY(tmap_bf16(&m_w, W13, (int64_t)groups * 2 * hid, P.d, 64));
        a.stages = tc_pair_max_stages(TC_PAIR_GATEUP, nt_max, groups, false, smem_limit);
        if (a.stages < 2) return fail(MOE_ERR_UNSUPPORTED, "shared memory too small for the GEMM tiles");
        MOE_TRY(zero_ctr());
        trace_pre(st, tag1);
        MOE_TRY(launched(launch_tc_pair(TC_PAIR_GATEUP, m_act, m_w, a, dv.sms / 2, st), tag1));
        trace_mark(st, tag1);
    } else {
        a.stages = tc_max_stages(mode1, 256, nt_max, groups, false, smem_limit);
        // while the routing finishes, prefetch the start of each CTA's first weight
        // tile (the unit it gets when every expert has tokens) into L2
        a.prefetch_kb = (!tok && !group_w && pdl_active()) ? 16 : 0;
        if (a.stages < 2) return fail(MOE_ERR_UNSUPPORTED, "shared memory too small for the GEMM tiles");
        trace_pre(st, tag1);
        MOE_TRY(launched(launch_tc_gemm(mode1, 256, m_act, m_w, a, dv.sms, st), tag1));
        trace_mark(st, tag1);
    }

    // down: H [act_rows][hid] x W2p [groups * d][hid] -> y [splits][act_rows][d]
    // The down projection streams its weights through the wide B operand of the
    // token-major tiles whenever a group may hold more than 128 tokens: a 256-row
    // weight tile per stage keeps twice the weight bytes in flight of a swapped
    // tile next to a token tile that large, and the accumulator stays
    // double-buffered; the second token tile of a group is partly idle.
    const bool pair_down = pair && P.d % 256 == 0;
    if (pair_down) {
        MOE_TRY(tmap_bf16(&m_act, H, (P.split ? 2 : 1) * act_rows, hid, pair_swap_tok_box(nt_max)));
        MOE_TRY(tmap_bf16(&m_w, W2p, (int64_t)groups * P.d, hid, 128));
        a.K = hid;
        a.n_feat = P.d;
        a.w_rows_per_group = P.d;
        a.splits = 1;
        a.out = y;
        a.out_ld = P.d;
        a.split_stride = act_rows * (int64_t)P.d;
        a.aux = nullptr;
        a.prefetch_kb = 0;
        a.stages = tc_pair_max_stages(TC_PAIR_DOWN, nt_max, groups, P.split, smem_limit);
        if (a.stages < 2) return fail(MOE_ERR_UNSUPPORTED, "shared memory too small for the GEMM tiles");
        MOE_TRY(zero_ctr());
        trace_pre(st, tag2);
        MOE_TRY(launched(launch_tc_pair(TC_PAIR_DOWN, m_act, m_w, a, dv.sms / 2, st), tag2));
        trace_mark(st, tag2);
        return MOE_OK;
    }
    const bool dtok = tok || nt_max > DOWN_SWAP_MAX_TOKENS;
    // groups of 129..256 tokens (swapped gate/up): the down projection on the
    // token-major CTA-pair tile, one pair unit per expert and 256 output features,
    // each SM streaming its own 128 weight rows (6 stages of 16 KB) rather than
    // two one-SM m tiles sharing a 256-row weight tile through L2
    if (!tok && dtok && g_pair_enabled >= 1 && P.d % 256 == 0 && hid % 128 == 0) {
        MOE_TRY(tmap_bf16(&m_act, H, (P.split ? 2 : 1) * act_rows, hid, 128));
        MOE_TRY(tmap_bf16(&m_w, W2p, (int64_t)groups * P.d, hid, 128));
        a.K = hid;
        a.n_feat = P.d;
        a.w_rows_per_group = P.d;
        a.splits = 1;
        a.out = y;
        a.out_ld = P.d;
        a.split_stride = act_rows * (int64_t)P.d;
        a.aux = nullptr;
        a.prefetch_kb = 0;
        a.stages = tc_pair_max_stages(TC_PAIR_DOWN_TOK, nt_max, groups, P.split, smem_limit);
        if (a.stages < 2) return fail(MOE_ERR_UNSUPPORTED, "shared memory too small for the GEMM tiles");
        MOE_TRY(zero_ctr());
        trace_pre(st, tag2);
        MOE_TRY(launched(launch_tc_pair(TC_PAIR_DOWN_TOK, m_act, m_w, a, dv.sms / 2, st), tag2));
        trace_mark(st, tag2);
        return MOE_OK;
    }
    const int mode2 = dtok ? TC_DOWN_TOK : TC_DOWN_SWAP;
    const int bn = (P.d % 256 == 0) ? 256 : 128;
    MOE_TRY(tmap_bf16(&m_act, H, (P.split ? 2 : 1) * act_rows, hid, dtok ? 128 : 16));
    MOE_TRY(tmap_bf16(&m_w, W2p, (int64_t)groups * P.d, hid, dtok ? bn : 128));
    a.K = hid;
    a.n_feat = P.d;
    a.w_rows_per_group = P.d;
    a.splits = dtok ? 1 : splits;
    a.out = y;
    a.out_ld = P.d;
    a.split_stride = act_rows * (int64_t)P.d;
    a.aux = nullptr;
    a.prefetch_kb = 0;
    a.stages = tc_max_stages(mode2, bn, nt_max, groups, P.split, smem_limit);
    if (a.stages < 2) return fail(MOE_ERR_UNSUPPORTED, "shared memory too small for the GEMM tiles");
    trace_pre(st, tag2);
    MOE_TRY(launched(launch_tc_gemm(mode2, bn, m_act, m_w, a, dv.sms, st), tag2));
    trace_mark(st, tag2);
    return MOE_OK;
}

// The shared experts' FFN over every token (fused into one expert of width
// S * hs): gate 1, no capacity, reads x directly.
static int step_shared_ffn(const Plan& P, const Device& dv, const void* x, const void* W13s,
                           const void* W2s, float* y_shared, void* ws, cudaStream_t st) {
    if (P.T == 0 || P.S == 0) return MOE_OK;
    int32_t* status = at<int32_t>(ws, P.off_status);
    void* Hs = at<void>(ws, P.off_Hs);
    if (P.shared_path == PATH_F32) {
        MOE_TRY(launched(launch_f32_gateup(reinterpret_cast<const float*>(x),
                                           reinterpret_cast<const float*>(W13s),
                                           reinterpret_cast<float*>(Hs), 1, nullptr, nullptr,
                                           (int)P.T, P.T, P.d, P.hsum, st),
                         "f32_shared_gateup"));
        trace_mark(st, "f32_shared_gateup");
        MOE_TRY(launched(launch_f32_down(reinterpret_cast<const float*>(Hs),
                                         reinterpret_cast<const float*>(W2s), y_shared, 1,
                                         nullptr, nullptr, (int)P.T, P.T, P.d, P.hsum, st),
                         "f32_shared_down"));
        trace_mark(st, "f32_shared_down");
        return MOE_OK;
    }
    const int nt = (int)((P.T + 15) / 16 * 16);
    void* ABs = P.train ? at<void>(ws, P.off_ABs) : nullptr;
    return run_tc_ffn(P, dv, P.shared_path, 1, nullptr, nullptr, nullptr, (int)P.T, x, P.T, W13s,
                      W2s, P.hsum, Hs, ABs, y_shared, 1, nt, status, st, "gemm_shared_gateup",
                      "gemm_shared_down", 1);
}

// The routed experts' FFN over the dispatched rows; with `shared`, then the
// shared experts' on the same stream.
static int step_ffn(const Plan& P, const Device& dv, const void* x_perm, const int32_t* offsets,
                    const int32_t* kept, const void* W13, const void* W2p, const void* x,
                    const void* W13s, const void* W2s, float* y_perm, float* y_shared, void* ws,
                    cudaStream_t st, bool shared = true) {
    if (P.T == 0) return MOE_OK;
    void* H = at<void>(ws, P.off_H);
    int32_t* status = at<int32_t>(ws, P.off_status);
    if (P.path == PATH_F32) {
        MOE_TRY(launched(launch_f32_gateup(reinterpret_cast<const float*>(x_perm),
                                           reinterpret_cast<const float*>(W13),
                                           reinterpret_cast<float*>(H), P.E, kept, offsets, 0,
                                           P.perm_rows, P.d, P.h, st),
                         "f32_gateup"));
        trace_mark(st, "f32_gateup");
        MOE_TRY(launched(launch_f32_down(reinterpret_cast<const float*>(H),
                                         reinterpret_cast<const float*>(W2p), y_perm, P.E, kept,
                                         offsets, 0, P.perm_rows, P.d, P.h, st),
                         "f32_down"));
        trace_mark(st, "f32_down");
    } else {
        void* AB = P.train ? at<void>(ws, P.off_AB) : nullptr;
        MOE_TRY(run_tc_ffn(P, dv, P.path, P.E, kept, offsets, nullptr, 0, x_perm, P.perm_rows,
                           W13, W2p,
                           P.h, H, AB, y_perm, P.splits, P.nt_max, status, st, "gemm_gateup",
                           "gemm_down"));
    }
    if (shared) MOE_TRY(step_shared_ffn(P, dv, x, W13s, W2s, y_shared, ws, st));
    return MOE_OK;
}

// ---------------------------------------------------------------- shared experts beside the routed

// A second stream per device for the shared experts of moe_forward, and the
// events that fork it from and join it back into the caller's stream.
struct SideStream {
    cudaStream_t st = nullptr;
    cudaEvent_t fork = nullptr, join = nullptr;
};

static int side_stream(SideStream* out) {
    constexpr int kMaxDevices = 64;
    static std::mutex mu;
    static SideStream cache[kMaxDevices];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices)
        return fail(MOE_ERR_CUDA, "cudaGetDevice failed");
    std::lock_guard<std::mutex> lk(mu);
    SideStream& c = cache[dev];
    if (!c.st) {
        if (cudaStreamCreateWithFlags(&c.st, cudaStreamNonBlocking) != cudaSuccess ||
            cudaEventCreateWithFlags(&c.fork, cudaEventDisableTiming) != cudaSuccess ||
            cudaEventCreateWithFlags(&c.join, cudaEventDisableTiming) != cudaSuccess) {
            c = SideStream();
            return fail(MOE_ERR_CUDA, "could not create the shared-expert stream");
        }
    }
    *out = c;
    return MOE_OK;
}

static int g_shared_overlap = 1;
static int g_shared_sms = 0;  // SMs set aside for the shared experts (0: none)

static StatsParams stats_params(const Plan& P, const int32_t* routed, const int32_t* kept,
                                const void* ws, double* sums, moe_stats* stats) {
    StatsParams a;
    a.ppart = at<float>(ws, P.off_ppart);
    a.hpart = at<float>(ws, P.off_hpart);
    a.nblk = P.nblk * P.nsub;
    a.routed = routed;
    a.kept = kept;
    a.T = P.T;
    a.E = P.E;
    a.k = P.k;
    a.sums = sums;
    a.stats = stats;
    return a;
}

static int step_combine(const Plan& P, const float* y_perm, const int32_t* slot_of,
                        const float* gate, const float* y_shared, void* out,
                        const StatsParams* sp, cudaStream_t st) {
    const int splits = P.path == PATH_SWAP ? P.splits : 1;
    trace_pre(st, "combine");
    MOE_TRY(launched(launch_combine(y_perm, splits, P.perm_rows * (int64_t)P.d, slot_of, gate,
                                    P.S > 0 ? y_shared : nullptr, out, P.bf16, P.T, P.d, P.k, sp,
                                    st),
                     "combine"));
    trace_mark(st, "combine");
    return MOE_OK;
}

static int step_stats(const Plan& P, const int32_t* routed, const int32_t* kept, const void* ws,
                      double* sums, moe_stats* stats, cudaStream_t st) {
    trace_pre(st, "stats");
    MOE_TRY(launched(launch_stats(stats_params(P, routed, kept, ws, sums, stats), st), "stats"));
    trace_mark(st, "stats");
    return MOE_OK;
}

// ---------------------------------------------------------------- backward steps

// Backward GEMMs of one set of groups: dAB = SiLU*mul backward of dY W2t^T
// (bf16, interleaved like AB), then dX = dAB W13t^T (fp32).  nt_max bounds a
// group's rows: groups that may hold 1024+ rows take both on CTA-pair tiles, as
// the forward's GEMMs do.
static int run_tc_backward(const Plan& P, const Device& dv, int groups, const int32_t* rows,
                           const int32_t* offs, int dense_rows, int64_t act_rows, const void* dY,
                           const void* W2t, const void* AB, void* dAB, const void* W13t,
                           float* dX, int hid, int64_t nt_max, int32_t* status, cudaStream_t st,
                           const char* tag1, const char* tag2, int ctr_slot) {
    CUtensorMap m_act, m_w;
    TcArgs a;
    memset(&a, 0, sizeof a);
    a.num_groups = groups;
    a.group_rows = rows;
    a.group_off = offs;
    a.dense_rows = dense_rows;
    a.status = status;
    a.wait_limit_ns = g_wait_limit_ns;
    a.test_stall = g_test_stall;
    a.nt_max = 16;
    a.splits = 1;

    const int bn1 = hid % 256 == 0 ? 256 : 128;
    a.K = P.d;
    a.n_feat = hid;
    a.w_rows_per_group = hid;
    a.out = dAB;
    a.out_ld = 2 * (int64_t)hid;
    a.aux = const_cast<void*>(AB);
    a.aux_ld = 2 * (int64_t)hid;
    // groups that may hold 1024+ rows: dgate on CTA-pair tiles too
    const bool pair = g_pair_enabled >= 1 && nt_max >= PAIR_TOK_MIN_TOKENS && hid % 256 == 0;
    if (pair) {
        MOE_TRY(tmap_bf16(&m_act, dY, act_rows, P.d, 128));
        MOE_TRY(tmap_bf16(&m_w, W2t, (int64_t)groups * hid, P.d, 128));
        a.unit_ctr = status + UNIT_CTR_WORD + ctr_slot;
        a.stages = tc_pair_max_stages(TC_PAIR_DGATE_TOK, 256, groups, false, dv.smem_optin);
        if (a.stages < 2) return fail(MOE_ERR_UNSUPPORTED, "shared memory too small for the GEMM tiles");
        if (cudaMemsetAsync(a.unit_ctr, 0, sizeof(int32_t), st) != cudaSuccess)
            return fail(MOE_ERR_CUDA, "memset failed");
        trace_pre(st, tag1);
        MOE_TRY(launched(launch_tc_pair(TC_PAIR_DGATE_TOK, m_act, m_w, a, dv.sms / 2, st), tag1));
        trace_mark(st, tag1);
        a.unit_ctr = nullptr;
    } else {
        MOE_TRY(tmap_bf16(&m_act, dY, act_rows, P.d, 128));
        MOE_TRY(tmap_bf16(&m_w, W2t, (int64_t)groups * hid, P.d, bn1));
        a.stages = tc_max_stages(TC_DGATE_TOK, bn1, 16, groups, false, dv.smem_optin);
        if (a.stages < 2) return fail(MOE_ERR_UNSUPPORTED, "shared memory too small for the GEMM tiles");
        trace_pre(st, tag1);
        MOE_TRY(launched(launch_tc_gemm(TC_DGATE_TOK, bn1, m_act, m_w, a, dv.sms, st), tag1));
        trace_mark(st, tag1);
    }

    const int bn2 = P.d % 256 == 0 ? 256 : 128;
    a.K = 2 * hid;
    a.n_feat = P.d;
    a.w_rows_per_group = P.d;
    a.out = dX;
    a.out_ld = P.d;
    a.aux = nullptr;
    if (g_pair_enabled >= 1 && nt_max >= PAIR_TOK_MIN_TOKENS && P.d % 256 == 0) {
        MOE_TRY(tmap_bf16(&m_act, dAB, act_rows, 2 * hid, 128));
        MOE_TRY(tmap_bf16(&m_w, W13t, (int64_t)groups * P.d, 2 * hid, 128));
        a.unit_ctr = status + UNIT_CTR_WORD + ctr_slot;
        a.stages = tc_pair_max_stages(TC_PAIR_DOWN_TOK, 256, groups, false, dv.smem_optin);
        if (a.stages < 2) return fail(MOE_ERR_UNSUPPORTED, "shared memory too small for the GEMM tiles");
        if (cudaMemsetAsync(a.unit_ctr, 0, sizeof(int32_t), st) != cudaSuccess)
            return fail(MOE_ERR_CUDA, "memset failed");
        trace_pre(st, tag2);
        MOE_TRY(launched(launch_tc_pair(TC_PAIR_DOWN_TOK, m_act, m_w, a, dv.sms / 2, st), tag2));
        trace_mark(st, tag2);
        return MOE_OK;
    }
    MOE_TRY(tmap_bf16(&m_act, dAB, act_rows, 2 * hid, 128));
    MOE_TRY(tmap_bf16(&m_w, W13t, (int64_t)groups * P.d, 2 * hid, bn2));
    a.stages = tc_max_stages(TC_DOWN_TOK, bn2, 16, groups, false, dv.smem_optin);
    if (a.stages < 2) return fail(MOE_ERR_UNSUPPORTED, "shared memory too small for the GEMM tiles");
    trace_pre(st, tag2);
    MOE_TRY(launched(launch_tc_gemm(TC_DOWN_TOK, bn2, m_act, m_w, a, dv.sms, st), tag2));
    trace_mark(st, tag2);
    return MOE_OK;
}

// Weight gradient C[g] [m_rows][n_rows] = sum over the token rows r of group g
// of A[r][:]^T B[r][:]: A [act_rows][m_rows] and B [act_rows][n_rows] are the
// row-major activations, read as MN-major operands; group g covers the rows
// offs[g] .. offs[g] + rows[g] rounded up to 64 (offs a multiple of 64, the
// rows past rows[g] zero); dense: one group of dense_rows rows from row 0.
static int run_tc_wgrad(const Plan& P, const Device& dv, int groups, const int32_t* rows,
                        const int32_t* offs, int dense_rows, int64_t act_rows, const void* A,
                        int m_rows, const void* Bm, int n_rows, float* out, int32_t* status,
                        cudaStream_t st, const char* tag) {
    (void)P;
    CUtensorMap m_a, m_b;
    TcArgs a;
    memset(&a, 0, sizeof a);
    const int bn = n_rows % 256 == 0 ? 256 : 128;
    MOE_TRY(tmap_bf16(&m_a, A, act_rows, m_rows, 64));
    MOE_TRY(tmap_bf16(&m_b, Bm, act_rows, n_rows, 64));
    a.num_groups = groups;
    a.group_rows = rows;
    a.group_off = offs;
    a.dense_rows = dense_rows;
    a.status = status;
    a.wait_limit_ns = g_wait_limit_ns;
    a.test_stall = g_test_stall;
    a.nt_max = 16;
    a.splits = 1;
    a.n_feat = n_rows;
    a.m_rows = m_rows;
    a.out = out;
    a.out_ld = n_rows;
    a.group_stride = (int64_t)m_rows * n_rows;
    a.n_fastest = n_rows < m_rows ? 1 : 0;
    a.stages = tc_max_stages(TC_WGRAD, bn, 16, groups, false, dv.smem_optin);
    if (a.stages < 2) return fail(MOE_ERR_UNSUPPORTED, "shared memory too small for the GEMM tiles");
    trace_pre(st, tag);
    MOE_TRY(launched(launch_tc_gemm(TC_WGRAD, bn, m_a, m_b, a, dv.sms, st), tag));
    trace_mark(st, tag);
    return MOE_OK;
}

}  // namespace moe

using namespace moe;

// ================================================================ C ABI

extern "C" {

const char* moe_last_error(void) { return g_err.c_str(); }

int moe_capacity(const moe_config* cfg, int64_t* C) {
    if (!C) return fail(MOE_ERR_ARG, "C is NULL");
    Plan P;
    MOE_TRY(plan_or_fail(cfg, &P));
    if (cfg->cf_den == 0) {
        *C = cfg->T;
    } else {
        const int64_t num = cfg->T * (int64_t)cfg->k * cfg->cf_num;
        const int64_t den = (int64_t)cfg->E * cfg->cf_den;
        *C = (num + den - 1) / den;
    }
    return ok();
}

int moe_workspace_size(const moe_config* cfg, size_t* bytes) {
    if (!bytes) return fail(MOE_ERR_ARG, "bytes is NULL");
    Plan P;
    MOE_TRY(plan_or_fail(cfg, &P));
    *bytes = P.total;
    return ok();
}

int moe_perm_rows(const moe_config* cfg, int64_t* rows) {
    if (!rows) return fail(MOE_ERR_ARG, "rows is NULL");
    Plan P;
    MOE_TRY(plan_or_fail(cfg, &P));
    *rows = P.perm_rows;
    return ok();
}

int moe_ffn_splits(const moe_config* cfg, int32_t* splits) {
    if (!splits) return fail(MOE_ERR_ARG, "splits is NULL");
    Plan P;
    MOE_TRY(plan_or_fail(cfg, &P));
    *splits = P.path == PATH_SWAP ? P.splits : 1;
    return ok();
}

int moe_hidden_split(const moe_config* cfg, int32_t* split) {
    if (!split) return fail(MOE_ERR_ARG, "split is NULL");
    Plan P;
    MOE_TRY(plan_or_fail(cfg, &P));
    *split = P.split ? 1 : 0;
    return ok();
}

int moe_pack_weights(const moe_config* cfg, int which, const void* w1, const void* w3,
                     const void* w2, void* W13, void* W2p, void* stream) {
    Plan P;
    MOE_TRY(plan_or_fail(cfg, &P));
    if (which < 0 || which > 3)
        return fail(MOE_ERR_ARG, "which must be 0/1 (routed/shared) or 2/3 (backward layouts)");
    if ((which == 1 || which == 3) && P.S == 0) return fail(MOE_ERR_ARG, "config has no shared experts");
    if (which >= 2 && !P.bf16) return fail(MOE_ERR_DTYPE, "backward layouts are bf16 only");
    MOE_TRY(need(w1, "w1"));
    MOE_TRY(need(w3, "w3"));
    MOE_TRY(need(w2, "w2"));
    MOE_TRY(need(W13, "W13"));
    MOE_TRY(need(W2p, "W2p"));
    Device dv;
    MOE_TRY(device_facts(&dv));
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const int eb = P.act_bytes;
    const bool routed_set = which == 0 || which == 2;
    const int n = routed_set ? P.E : P.S;
    const int hid = routed_set ? P.h : P.hs;
    const int64_t d = P.d;
    const int64_t m13 = d * hid;  // elements of one w1 / w3 / w2 matrix
    if (which >= 2) {
        // W13t [n][d][2 hid] (routed) or [d][2 S hs] (shared): rows of w1 / w3
        // with the gate/up interleave along the hidden axis; W2t = w2 itself
        const bool routed = which == 2;
        const int64_t ld = routed ? 2 * (int64_t)hid : 2 * (int64_t)P.hsum;
        const int64_t dstride = routed ? d * 2 * hid : 0;
        const int step = routed ? 0 : hid;
        MOE_TRY(launched(launch_pack_cols(w1, W13, (int)d, hid, ld, 0, 0, n, m13, dstride, step, st),
                         "pack"));
        MOE_TRY(launched(launch_pack_cols(w3, W13, (int)d, hid, ld, 0, 1, n, m13, dstride, step, st),
                         "pack"));
        if (cudaMemcpyAsync(W2p, w2, (size_t)n * m13 * eb, cudaMemcpyDeviceToDevice, st) !=
            cudaSuccess)
            return fail(MOE_ERR_CUDA, "pack: copy of w2 failed");
        return ok();
    }
    if (which == 0) {
        // expert e: W13[e] [2h][d] and W2p[e] [d][h]
        MOE_TRY(launched(launch_pack(w1, W13, eb, (int)d, hid, d, 0, 0, n, m13, 2 * m13, 0, st),
                         "pack"));
        MOE_TRY(launched(launch_pack(w3, W13, eb, (int)d, hid, d, 0, 1, n, m13, 2 * m13, 0, st),
                         "pack"));
        MOE_TRY(launched(launch_pack(w2, W2p, eb, hid, (int)d, hid, 0, -1, n, m13, m13, 0, st),
                         "pack"));
    } else {
        // shared experts fused into one of width S*hs: hidden index e*hs + j
        MOE_TRY(launched(launch_pack(w1, W13, eb, (int)d, hid, d, 0, 0, n, m13, 0, hid, st),
                         "pack"));
        MOE_TRY(launched(launch_pack(w3, W13, eb, (int)d, hid, d, 0, 1, n, m13, 0, hid, st),
                         "pack"));
        MOE_TRY(launched(launch_pack(w2, W2p, eb, hid, (int)d, P.hsum, 0, -1, n, m13, hid, 0, st),
                         "pack"));
    }
    return ok();
}

int moe_route(const moe_config* cfg, const void* x, const float* Wr, const float* bias,
              int32_t* topk_idx, float* topk_gate, float* logits, void* ws, size_t ws_bytes,
              void* stream) {
    Plan P;
    MOE_TRY(plan_or_fail(cfg, &P));
    MOE_TRY(need_ws(ws, ws_bytes, P));
    if (P.T > 0) {
        MOE_TRY(need(x, "x"));
        MOE_TRY(need(Wr, "Wr"));
        MOE_TRY(need(topk_idx, "topk_idx"));
        MOE_TRY(need(topk_gate, "topk_gate"));
        if (cfg->has_bias) MOE_TRY(need(bias, "bias"));
        MOE_TRY(maybe(logits, "logits"));
    }
    Device dv;
    MOE_TRY(device_facts(&dv));
    MOE_TRY(step_route(P, dv, x, Wr, cfg->has_bias ? bias : nullptr, topk_idx, topk_gate, logits,
                       ws, reinterpret_cast<cudaStream_t>(stream)));
    return ok();
}

int moe_dispatch(const moe_config* cfg, const int32_t* topk_idx, const void* x, int32_t* routed,
                 int32_t* kept, int32_t* offsets, int32_t* perm_token, int32_t* slot_of,
                 void* x_perm, void* ws, size_t ws_bytes, void* stream) {
    Plan P;
    MOE_TRY(plan_or_fail(cfg, &P));
    MOE_TRY(need_ws(ws, ws_bytes, P));
    MOE_TRY(need(routed, "routed"));
    MOE_TRY(need(kept, "kept"));
    MOE_TRY(need(offsets, "offsets"));
    if (P.T > 0) {
        MOE_TRY(need(topk_idx, "topk_idx"));
        MOE_TRY(need(x, "x"));
        MOE_TRY(need(slot_of, "slot_of"));
        MOE_TRY(need(x_perm, "x_perm"));
        MOE_TRY(maybe(perm_token, "perm_token"));
    }
    Device dv;
    MOE_TRY(device_facts(&dv));
    MOE_TRY(step_dispatch(P, dv, topk_idx, x, routed, kept, offsets, perm_token, slot_of, x_perm,
                          ws, reinterpret_cast<cudaStream_t>(stream)));
    return ok();
}

int moe_expert_ffn(const moe_config* cfg, const void* x_perm, const int32_t* offsets,
                   const int32_t* kept, const void* W13, const void* W2p, const void* x,
                   const void* W13s, const void* W2s, float* y_perm, float* y_shared, void* ws,
                   size_t ws_bytes, void* stream) {
    Plan P;
    MOE_TRY(plan_or_fail(cfg, &P));
    MOE_TRY(need_ws(ws, ws_bytes, P));
    if (P.T > 0) {
        MOE_TRY(need(x_perm, "x_perm"));
        MOE_TRY(need(offsets, "offsets"));
        MOE_TRY(need(kept, "kept"));
        MOE_TRY(need(W13, "W13"));
        MOE_TRY(need(W2p, "W2p"));
        MOE_TRY(need(y_perm, "y_perm"));
        if (P.S > 0) {
            MOE_TRY(need(x, "x"));
            MOE_TRY(need(W13s, "W13s"));
            MOE_TRY(need(W2s, "W2s"));
            MOE_TRY(need(y_shared, "y_shared"));
        }
    }
    Device dv;
    MOE_TRY(device_facts(&dv));
    MOE_TRY(step_ffn(P, dv, x_perm, offsets, kept, W13, W2p, x, W13s, W2s, y_perm, y_shared, ws,
                     reinterpret_cast<cudaStream_t>(stream)));
    return ok();
}

int moe_combine(const moe_config* cfg, const float* y_perm, const int32_t* slot_of,
                const float* topk_gate, const float* y_shared, void* out, void* stream) {
    Plan P;
    MOE_TRY(plan_or_fail(cfg, &P));
    if (P.T > 0) {
        MOE_TRY(need(y_perm, "y_perm"));
        MOE_TRY(need(slot_of, "slot_of"));
        MOE_TRY(need(topk_gate, "topk_gate"));
        MOE_TRY(need(out, "out"));
        if (P.S > 0) MOE_TRY(need(y_shared, "y_shared"));
    }
    MOE_TRY(step_combine(P, y_perm, slot_of, topk_gate, y_shared, out, nullptr,
                         reinterpret_cast<cudaStream_t>(stream)));
    return ok();
}

int moe_stats_sums(const moe_config* cfg, const int32_t* routed, const int32_t* kept,
                   const void* ws, size_t ws_bytes, double* sums, void* stream) {
    Plan P;
    MOE_TRY(plan_or_fail(cfg, &P));
    MOE_TRY(need_ws(ws, ws_bytes, P));
    MOE_TRY(need(sums, "sums"));
    MOE_TRY(need(routed, "routed"));
    MOE_TRY(need(kept, "kept"));
    MOE_TRY(step_stats(P, routed, kept, ws, sums, nullptr, reinterpret_cast<cudaStream_t>(stream)));
    return ok();
}

int moe_stats_finalize(const moe_config* cfg, const double* sums, moe_stats* stats,
                       void* stream) {
    Plan P;
    MOE_TRY(plan_or_fail(cfg, &P));
    MOE_TRY(need(sums, "sums"));
    MOE_TRY(need(stats, "stats"));
    MOE_TRY(launched(launch_stats_finalize(sums, P.E, P.k, stats,
                                           reinterpret_cast<cudaStream_t>(stream)),
                     "stats_finalize"));
    return ok();
}

int moe_aux_stats(const moe_config* cfg, const int32_t* routed, const int32_t* kept,
                  const void* ws, size_t ws_bytes, moe_stats* stats, void* stream) {
    Plan P;
    MOE_TRY(plan_or_fail(cfg, &P));
    MOE_TRY(need_ws(ws, ws_bytes, P));
    MOE_TRY(need(stats, "stats"));
    MOE_TRY(need(routed, "routed"));
    MOE_TRY(need(kept, "kept"));
    double* sums = const_cast<double*>(at<double>(ws, P.off_sums));
    MOE_TRY(step_stats(P, routed, kept, ws, sums, stats, reinterpret_cast<cudaStream_t>(stream)));
    return ok();
}

int moe_forward(const moe_config* cfg, const void* x, const float* Wr, const float* bias,
                const void* W13, const void* W2p, const void* W13s, const void* W2s, void* out,
                int32_t* topk_idx, float* topk_gate, int32_t* routed, int32_t* kept,
                int32_t* slot_of, moe_stats* stats, void* ws, size_t ws_bytes, void* stream) {
    Plan P;
    MOE_TRY(plan_or_fail(cfg, &P));
    MOE_TRY(need_ws(ws, ws_bytes, P));
    MOE_TRY(need(routed, "routed"));
    MOE_TRY(need(kept, "kept"));
    MOE_TRY(maybe(stats, "stats"));
    if (P.T > 0) {
        MOE_TRY(need(x, "x"));
        MOE_TRY(need(Wr, "Wr"));
        MOE_TRY(need(W13, "W13"));
        MOE_TRY(need(W2p, "W2p"));
        MOE_TRY(need(out, "out"));
        MOE_TRY(need(topk_idx, "topk_idx"));
        MOE_TRY(need(topk_gate, "topk_gate"));
        MOE_TRY(need(slot_of, "slot_of"));
        if (cfg->has_bias) MOE_TRY(need(bias, "bias"));
        if (P.S > 0) {
            MOE_TRY(need(W13s, "W13s"));
            MOE_TRY(need(W2s, "W2s"));
        }
        if (out == x) return fail(MOE_ERR_ARG, "out must not alias x");
    }
    Device dv;
    MOE_TRY(device_facts(&dv));
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    trace_call_begin(st);
    PdlScope pdl;  // the forward chain's kernels may overlap their predecessors' tails
    int32_t* offsets = at<int32_t>(ws, P.off_offsets);
    int32_t* perm = at<int32_t>(ws, P.off_perm);
    void* x_perm = at<void>(ws, P.off_xperm);
    float* y = at<float>(ws, P.off_y);
    float* ys = P.S ? at<float>(ws, P.off_ys) : nullptr;
    // The shared experts need only x: with the overlap on they run on a second
    // stream from the start of the call, beside the routing and the routed
    // experts, and the combine waits for them.  (Off while every kernel is
    // being timed, whose events assume one stream.)
    const bool side = P.T > 0 && P.S > 0 && P.bf16 && g_shared_overlap &&
                      !(g_trace.on && g_trace.only.empty());
    // With SMs set aside for them, the shared experts' GEMMs take that many SMs
    // and the routed experts' the rest, so that the two run side by side (the
    // routed GEMMs stream weights from HBM; the shared ones are compute-bound)
    // rather than one in the tail of the other.
    Device dv_routed = dv, dv_shared = dv;
    if (side && g_shared_sms > 0 && g_shared_sms <= dv.sms - 32) {
        dv_shared.sms = g_shared_sms;
        dv_routed.sms = dv.sms - g_shared_sms;
    }
    SideStream ss;
    if (side) {
        MOE_TRY(side_stream(&ss));
        if (cudaEventRecord(ss.fork, st) != cudaSuccess ||
            cudaStreamWaitEvent(ss.st, ss.fork, 0) != cudaSuccess)
            return fail(MOE_ERR_CUDA, "could not fork the shared-expert stream");
        g_pdl_in_forward = false;  // the first launch on the side stream follows an event
        const int rc = step_shared_ffn(P, dv_shared, x, W13s, W2s, ys, ws, ss.st);
        g_pdl_in_forward = true;
        MOE_TRY(rc);
        if (cudaEventRecord(ss.join, ss.st) != cudaSuccess)
            return fail(MOE_ERR_CUDA, "could not join the shared-expert stream");
    }
    MOE_TRY(step_route_dispatch(P, dv, x, Wr, cfg->has_bias ? bias : nullptr, topk_idx, topk_gate,
                                routed, kept, offsets, perm, slot_of, x_perm, ws, st));
    MOE_TRY(step_ffn(P, dv_routed, x_perm, offsets, kept, W13, W2p, x, W13s, W2s, y, ys, ws, st,
                     !side));
    if (side && cudaStreamWaitEvent(st, ss.join, 0) != cudaSuccess)
        return fail(MOE_ERR_CUDA, "could not join the shared-expert stream");
    // combine, with the statistics computed by one extra block of the same launch
    StatsParams sp = stats_params(P, routed, kept, ws, at<double>(ws, P.off_sums), stats);
    if (P.T > 0)
        MOE_TRY(step_combine(P, y, slot_of, topk_gate, ys, out, stats ? &sp : nullptr, st));
    else if (stats)
        MOE_TRY(step_stats(P, routed, kept, ws, at<double>(ws, P.off_sums), stats, st));
    return ok();
}

// ---------------------------------------------------------------- expert parallelism

int moe_segment_pad(const moe_config* cfg, int32_t* pad) {
    if (!pad) return fail(MOE_ERR_ARG, "pad is NULL");
    Plan P;
    MOE_TRY(plan_or_fail(cfg, &P));
    *pad = P.pad;
    return ok();
}

int moe_route_counts(const moe_config* cfg, const void* ws, size_t ws_bytes, int32_t* counts,
                     void* stream) {
    Plan P;
    MOE_TRY(plan_or_fail(cfg, &P));
    MOE_TRY(need_ws(ws, ws_bytes, P));
    MOE_TRY(need(counts, "counts"));
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (P.T == 0) {
        if (cudaMemsetAsync(counts, 0, (size_t)P.E * 4, st) != cudaSuccess)
            return fail(MOE_ERR_CUDA, "memset failed");
        return ok();
    }
    MOE_TRY(launched(launch_route_counts(at<int32_t>(ws, P.off_cnt), P.nblk * P.nsub, P.E, counts, st),
                     "route_counts"));
    return ok();
}

int moe_ep_plan(const moe_config* cfg, int32_t world, int32_t rank, const int32_t* counts,
                int64_t C, int32_t* cap, int32_t* row_start, int32_t* group_rows,
                int32_t* group_off, int32_t* group_weight, int32_t* recv_rows, void* stream) {
    Plan P;
    MOE_TRY(plan_or_fail(cfg, &P));
    if (world < 1 || world > MAX_PEERS) return fail(MOE_ERR_ARG, "world must be 1..MOE_MAX_PEERS");
    if (P.E % world) return fail(MOE_ERR_SHAPE, "E must be a multiple of world");
    if (rank < 0 || rank >= world) return fail(MOE_ERR_ARG, "rank must be in [0, world)");
    if (C < 0) return fail(MOE_ERR_ARG, "C must be >= 0");
    MOE_TRY(need(counts, "counts"));
    MOE_TRY(need(cap, "cap"));
    MOE_TRY(need(row_start, "row_start"));
    MOE_TRY(need(group_rows, "group_rows"));
    MOE_TRY(need(group_off, "group_off"));
    MOE_TRY(need(group_weight, "group_weight"));
    MOE_TRY(need(recv_rows, "recv_rows"));
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    MOE_TRY(launched(launch_ep_plan(counts, world, P.E, rank, C, P.pad, cap, row_start,
                                    group_rows, group_off, group_weight, recv_rows, st),
                     "ep_plan"));
    return ok();
}

int moe_dispatch_capped(const moe_config* cfg, const int32_t* topk_idx, const void* x,
                        const int32_t* cap, int32_t* routed, int32_t* kept, int32_t* offsets,
                        int32_t* perm_token, int32_t* slot_of, void* x_perm, void* ws,
                        size_t ws_bytes, void* stream) {
    Plan P;
    MOE_TRY(plan_or_fail(cfg, &P));
    if (P.reroute) return fail(MOE_ERR_UNSUPPORTED, "moe_dispatch_capped: the drop policy only");
    MOE_TRY(need_ws(ws, ws_bytes, P));
    MOE_TRY(need(cap, "cap"));
    MOE_TRY(need(routed, "routed"));
    MOE_TRY(need(kept, "kept"));
    MOE_TRY(need(offsets, "offsets"));
    if (P.T > 0) {
        MOE_TRY(need(topk_idx, "topk_idx"));
        MOE_TRY(need(x, "x"));
        MOE_TRY(need(slot_of, "slot_of"));
        MOE_TRY(need(x_perm, "x_perm"));
        MOE_TRY(maybe(perm_token, "perm_token"));
    }
    Device dv;
    MOE_TRY(device_facts(&dv));
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (P.T == 0) return empty_batch(P, ws, routed, kept, offsets, st) == MOE_OK ? ok() : MOE_ERR_CUDA;
    DispatchParams d = dispatch_params(P, x, routed, kept, offsets, perm_token, slot_of, x_perm);
    d.cap = cap;
    MOE_TRY(launched(launch_dispatch(d, topk_idx, at<int32_t>(ws, P.off_cnt),
                                     at<int32_t>(ws, P.off_tot), dv.sms, st),
                     "dispatch"));
    return ok();
}

static_assert(MOE_MAX_PEERS == MAX_PEERS, "peer table sizes differ");

static int check_peers(const Plan& P, int32_t world, const void* const* ptrs, const char* what) {
    if (world < 1 || world > MAX_PEERS) return fail(MOE_ERR_ARG, "world must be 1..MOE_MAX_PEERS");
    if (P.E % world) return fail(MOE_ERR_SHAPE, "E must be a multiple of world");
    if (P.reroute) return fail(MOE_ERR_UNSUPPORTED, "expert parallelism: the drop policy only");
    if (!ptrs) return fail(MOE_ERR_ARG, what);
    for (int q = 0; q < world; ++q) {
        if (!ptrs[q]) return fail(MOE_ERR_ARG, what);
        if (reinterpret_cast<uintptr_t>(ptrs[q]) & 15)
            return fail(MOE_ERR_ALIGN, "peer row pointers must be 16-byte aligned");
    }
    return MOE_OK;
}

int moe_dispatch_peers(const moe_config* cfg, const int32_t* topk_idx, const void* x,
                       const int32_t* cap, int32_t world, void* const* dst_rows,
                       const int32_t* dst_row_start, int32_t* routed, int32_t* kept,
                       int32_t* offsets, int32_t* perm_token, int32_t* slot_of, void* ws,
                       size_t ws_bytes, void* stream) {
    Plan P;
    MOE_TRY(plan_or_fail(cfg, &P));
    if (!P.bf16) return fail(MOE_ERR_DTYPE, "moe_dispatch_peers: bf16 only");
    MOE_TRY(need_ws(ws, ws_bytes, P));
    MOE_TRY(need(cap, "cap"));
    MOE_TRY(need(routed, "routed"));
    MOE_TRY(need(kept, "kept"));
    MOE_TRY(need(offsets, "offsets"));
    if (P.T > 0) {
        MOE_TRY(check_peers(P, world, reinterpret_cast<const void* const*>(dst_rows),
                            "dst_rows is NULL or holds a NULL pointer"));
        MOE_TRY(need(topk_idx, "topk_idx"));
        MOE_TRY(need(x, "x"));
        MOE_TRY(need(slot_of, "slot_of"));
        MOE_TRY(maybe(perm_token, "perm_token"));
    }
    Device dv;
    MOE_TRY(device_facts(&dv));
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (P.T == 0) return empty_batch(P, ws, routed, kept, offsets, st) == MOE_OK ? ok() : MOE_ERR_CUDA;
    DispatchParams d = dispatch_params(P, x, routed, kept, offsets, perm_token, slot_of, nullptr);
    d.cap = cap;
    d.peer_rows = dst_rows;
    d.npeer = world;
    d.peer_start = dst_row_start;
    d.e_loc = P.E / world;
    MOE_TRY(launched(launch_dispatch(d, topk_idx, at<int32_t>(ws, P.off_cnt),
                                     at<int32_t>(ws, P.off_tot), dv.sms, st),
                     "dispatch"));
    return ok();
}

int moe_combine_peers(const moe_config* cfg, int32_t world, const float* const* y_rows,
                      const int32_t* y_row_start, const int32_t* topk_idx,
                      const int32_t* offsets, const int32_t* slot_of, const float* topk_gate,
                      const float* y_shared, void* out, void* stream) {
    Plan P;
    MOE_TRY(plan_or_fail(cfg, &P));
    if (P.T > 0) {
        MOE_TRY(check_peers(P, world, reinterpret_cast<const void* const*>(y_rows),
                            "y_rows is NULL or holds a NULL pointer"));
        MOE_TRY(need(topk_idx, "topk_idx"));
        MOE_TRY(need(offsets, "offsets"));
        MOE_TRY(need(slot_of, "slot_of"));
        MOE_TRY(need(topk_gate, "topk_gate"));
        MOE_TRY(need(out, "out"));
        if (P.S > 0) MOE_TRY(need(y_shared, "y_shared"));
    }
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    trace_pre(st, "combine");
    MOE_TRY(maybe(y_row_start, "y_row_start"));
    MOE_TRY(launched(launch_combine_peers(y_rows, y_row_start, world, P.E / world, topk_idx,
                                          offsets, slot_of, topk_gate,
                                          P.S > 0 ? y_shared : nullptr, out, P.bf16, P.T, P.d,
                                          P.k, st),
                     "combine"));
    trace_mark(st, "combine");
    return ok();
}

int moe_combine_rows(const moe_config* cfg, const float* y_rows, const int32_t* slot_of,
                     const float* topk_gate, const float* y_shared, void* out, void* stream) {
    Plan P;
    MOE_TRY(plan_or_fail(cfg, &P));
    if (P.T > 0) {
        MOE_TRY(need(y_rows, "y_rows"));
        MOE_TRY(need(slot_of, "slot_of"));
        MOE_TRY(need(topk_gate, "topk_gate"));
        MOE_TRY(need(out, "out"));
        if (P.S > 0) MOE_TRY(need(y_shared, "y_shared"));
    }
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    trace_pre(st, "combine");
    MOE_TRY(launched(launch_combine(y_rows, 1, 0, slot_of, topk_gate,
                                    P.S > 0 ? y_shared : nullptr, out, P.bf16, P.T, P.d, P.k,
                                    nullptr, st),
                     "combine"));
    trace_mark(st, "combine");
    return ok();
}

static size_t grouped_h_offset() { return 256; }

int moe_grouped_workspace_size(const moe_config* cfg, int64_t rows, int32_t max_group_rows,
                               size_t* bytes) {
    if (!bytes) return fail(MOE_ERR_ARG, "bytes is NULL");
    Plan P;
    MOE_TRY(plan_or_fail(cfg, &P));
    if (rows < 0 || max_group_rows < 0) return fail(MOE_ERR_ARG, "rows and max_group_rows must be >= 0");
    *bytes = grouped_h_offset() + align256((size_t)(P.split ? 2 : 1) * rows * P.h * P.act_bytes);
    return ok();
}

int moe_expert_ffn_grouped(const moe_config* cfg, const void* x_rows, int64_t rows,
                           int32_t n_groups, const int32_t* group_rows, const int32_t* group_off,
                           const int32_t* group_weight, int32_t max_group_rows, const void* W13,
                           const void* W2p, float* y_rows, void* ws, size_t ws_bytes,
                           void* stream) {
    Plan P;
    MOE_TRY(plan_or_fail(cfg, &P));
    if (!P.bf16) return fail(MOE_ERR_DTYPE, "moe_expert_ffn_grouped: bf16 only");
    if (rows < 0 || n_groups < 0 || n_groups > 65536 || max_group_rows < 0)
        return fail(MOE_ERR_ARG, "moe_expert_ffn_grouped: bad sizes");
    if (!ws) return fail(MOE_ERR_ARG, "ws is NULL");
    if (reinterpret_cast<uintptr_t>(ws) & 255) return fail(MOE_ERR_ALIGN, "ws is not 256-byte aligned");
    const size_t need_bytes =
        grouped_h_offset() + align256((size_t)(P.split ? 2 : 1) * rows * P.h * P.act_bytes);
    if (ws_bytes < need_bytes)
        return fail(MOE_ERR_WORKSPACE, "workspace has %zu bytes; this call needs %zu", ws_bytes,
                    need_bytes);
    if (rows == 0 || n_groups == 0) return ok();
    MOE_TRY(need(x_rows, "x_rows"));
    MOE_TRY(need(group_rows, "group_rows"));
    MOE_TRY(need(group_off, "group_off"));
    MOE_TRY(need(group_weight, "group_weight"));
    MOE_TRY(need(W13, "W13"));
    MOE_TRY(need(W2p, "W2p"));
    MOE_TRY(need(y_rows, "y_rows"));
    Device dv;
    MOE_TRY(device_facts(&dv));
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const int nmax = max_group_rows > 0 ? max_group_rows : 1;
    const int path = nmax <= SWAP_MAX_TOKENS ? PATH_SWAP : PATH_TOKEN_MAJOR;
    const int nt_max = (nmax + 15) / 16 * 16;
    int32_t* status = at<int32_t>(ws, 0);
    if (cudaMemsetAsync(status, 0, 4, st) != cudaSuccess) return fail(MOE_ERR_CUDA, "memset failed");
    void* H = at<void>(ws, grouped_h_offset());
    MOE_TRY(run_tc_ffn(P, dv, path, n_groups, group_rows, group_off, group_weight, 0, x_rows, rows,
                       W13, W2p, P.h, H, nullptr, y_rows, 1, nt_max, status, st,
                       "gemm_grouped_gateup", "gemm_grouped_down"));
    return ok();
}

int moe_backward_workspace_size(const moe_config* cfg, size_t* bytes) {
    if (!bytes) return fail(MOE_ERR_ARG, "bytes is NULL");
    Plan P;
    MOE_TRY(plan_or_fail(cfg, &P));
    if (!P.train) return fail(MOE_ERR_ARG, "the backward pass needs cfg->train = 1");
    *bytes = P.b_total;
    return ok();
}

int moe_backward(const moe_config* cfg, const void* grad_out, float aux_coef, const void* x,
                 const float* Wr, const float* bias, const void* W13t, const void* W2t,
                 const void* W13st, const void* W2st, const int32_t* topk_idx,
                 const float* topk_gate, const int32_t* routed, const int32_t* kept,
                 const int32_t* slot_of, void* ws, size_t ws_bytes, float* dx, float* dWr,
                 float* db, float* dW13, float* dW2p, float* dW13s, float* dW2s, float* dlogits,
                 void* bws, size_t bws_bytes, void* stream) {
    Plan P;
    MOE_TRY(plan_or_fail(cfg, &P));
    if (!P.train) return fail(MOE_ERR_ARG, "the backward pass needs cfg->train = 1");
    MOE_TRY(need_ws(ws, ws_bytes, P));
    if (!bws) return fail(MOE_ERR_ARG, "bws is NULL");
    if (reinterpret_cast<uintptr_t>(bws) & 255)
        return fail(MOE_ERR_ALIGN, "bws is not 256-byte aligned");
    if (bws_bytes < P.b_total)
        return fail(MOE_ERR_WORKSPACE, "backward workspace has %zu bytes; this config needs %zu",
                    bws_bytes, P.b_total);
    MOE_TRY(need(dWr, "dWr"));
    MOE_TRY(need(dW13, "dW13"));
    MOE_TRY(need(dW2p, "dW2p"));
    MOE_TRY(maybe(db, "db"));
    MOE_TRY(maybe(dlogits, "dlogits"));
    if (P.S > 0) {
        MOE_TRY(need(dW13s, "dW13s"));
        MOE_TRY(need(dW2s, "dW2s"));
    }
    if (P.T > 0) {
        MOE_TRY(need(grad_out, "grad_out"));
        MOE_TRY(need(x, "x"));
        MOE_TRY(need(Wr, "Wr"));
        MOE_TRY(need(W13t, "W13t"));
        MOE_TRY(need(W2t, "W2t"));
        MOE_TRY(need(topk_idx, "topk_idx"));
        MOE_TRY(need(topk_gate, "topk_gate"));
        MOE_TRY(need(routed, "routed"));
        MOE_TRY(need(kept, "kept"));
        MOE_TRY(need(slot_of, "slot_of"));
        MOE_TRY(need(dx, "dx"));
        if (cfg->has_bias) MOE_TRY(need(bias, "bias"));
        if (P.S > 0) {
            MOE_TRY(need(W13st, "W13st"));
            MOE_TRY(need(W2st, "W2st"));
        }
    }
    Device dv;
    MOE_TRY(device_facts(&dv));
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const int64_t T = P.T;
    const int d = P.d, h = P.h, E = P.E, k = P.k;
    if (T == 0) {
        // nothing was routed: every gradient is zero
        if (cudaMemsetAsync(dWr, 0, (size_t)d * E * 4, st) != cudaSuccess ||
            (db && cfg->has_bias && cudaMemsetAsync(db, 0, (size_t)E * 4, st) != cudaSuccess) ||
            cudaMemsetAsync(dW13, 0, (size_t)E * 2 * h * d * 4, st) != cudaSuccess ||
            cudaMemsetAsync(dW2p, 0, (size_t)E * d * h * 4, st) != cudaSuccess ||
            (P.S && cudaMemsetAsync(dW13s, 0, (size_t)2 * P.hsum * d * 4, st) != cudaSuccess) ||
            (P.S && cudaMemsetAsync(dW2s, 0, (size_t)d * P.hsum * 4, st) != cudaSuccess))
            return fail(MOE_ERR_CUDA, "memset failed");
        return ok();
    }
    trace_call_begin(st);
    int32_t* status = at<int32_t>(ws, P.off_status);
    const int32_t* offsets = at<int32_t>(ws, P.off_offsets);
    const void* x_perm = at<void>(ws, P.off_xperm);
    const void* H = at<void>(ws, P.off_H);
    const float* y = at<float>(ws, P.off_y);
    const void* AB = at<void>(ws, P.off_AB);
    const float* z = at<float>(ws, P.off_logits);
    void* dY = at<void>(bws, P.b_dY);
    float* dg = at<float>(bws, P.b_dg);
    float* dz = dlogits ? dlogits : at<float>(bws, P.b_dz);
    void* dAB = at<void>(bws, P.b_dAB);
    float* dXp = at<float>(bws, P.b_dXp);
    const int splits = P.path == PATH_SWAP ? P.splits : 1;

    // gate-scaled output gradients per kept slot, and the gate gradients
    trace_pre(st, "bwd_gather");
    MOE_TRY(launched(launch_bwd_gather(grad_out, y, splits, P.perm_rows * (int64_t)d, slot_of,
                                       topk_gate, dY, dg, T, d, k, dv.sms, st),
                     "bwd_gather"));
    trace_mark(st, "bwd_gather");
    // router logits: the forward left z with the bias added on these paths
    const bool z_has_bias = P.router_kind == ROUTER_TC || P.reroute;
    const float* b_add = (cfg->has_bias && !z_has_bias) ? bias : nullptr;
    trace_pre(st, "router_bwd");
    MOE_TRY(launched(launch_router_bwd(z, b_add, topk_idx, topk_gate, dg, routed, aux_coef, dz, T,
                                       E, k, dv.sms, st),
                     "router_bwd"));
    trace_mark(st, "router_bwd");
    trace_pre(st, "wr_grad");
    MOE_TRY(launched(launch_wr_grad(x, dz, at<float>(bws, P.b_wrpart), dWr,
                                    cfg->has_bias ? db : nullptr, T, d, E, st),
                     "wr_grad"));
    trace_mark(st, "wr_grad");

    // routed experts: dAB, dX, then the weight gradients over each expert's tokens
    MOE_TRY(run_tc_backward(P, dv, E, kept, offsets, 0, P.perm_rows, dY, W2t, AB, dAB, W13t, dXp, h,
                            P.nt_max, status, st, "gemm_dgate", "gemm_dx", 0));
    // the rows between each expert's tokens and the next multiple of 64 are
    // zeroed in the four activations the weight gradients contract
    PadJobs pj;
    pj.n = 4;
    pj.job[0] = {const_cast<void*>(x_perm), d};
    pj.job[1] = {const_cast<void*>(H), h};
    pj.job[2] = {dY, d};
    pj.job[3] = {dAB, 2 * h};
    pj.off = offsets;
    pj.rows = kept;
    pj.groups = E;
    trace_pre(st, "zero_pad");
    MOE_TRY(launched(launch_zero_pad(pj, st), "zero_pad"));
    trace_mark(st, "zero_pad");
    MOE_TRY(run_tc_wgrad(P, dv, E, kept, offsets, 0, P.perm_rows, dY, d, H, h, dW2p, status, st,
                         "gemm_dw2"));
    MOE_TRY(run_tc_wgrad(P, dv, E, kept, offsets, 0, P.perm_rows, dAB, 2 * h, x_perm, d, dW13,
                         status, st, "gemm_dw13"));

    // shared experts: gate 1, every token
    float* dXs = nullptr;
    if (P.S > 0) {
        const void* Hs = at<void>(ws, P.off_Hs);
        const void* ABs = at<void>(ws, P.off_ABs);
        void* dABs = at<void>(bws, P.b_dABs);
        dXs = at<float>(bws, P.b_dXs);
        MOE_TRY(run_tc_backward(P, dv, 1, nullptr, nullptr, (int)T, T, grad_out, W2st, ABs, dABs,
                                W13st, dXs, P.hsum, T, status, st, "gemm_shared_dgate",
                                "gemm_shared_dx", 1));
        MOE_TRY(run_tc_wgrad(P, dv, 1, nullptr, nullptr, (int)T, T, grad_out, d, Hs, P.hsum,
                             dW2s, status, st, "gemm_shared_dw2"));
        MOE_TRY(run_tc_wgrad(P, dv, 1, nullptr, nullptr, (int)T, T, dABs, 2 * P.hsum, x, d,
                             dW13s, status, st, "gemm_shared_dw13"));
    }

    trace_pre(st, "combine_bwd");
    MOE_TRY(launched(launch_combine_bwd(dXp, slot_of, dXs, dz, Wr, at<float>(bws, P.b_dxr), dx,
                                        T, d, k, E, st),
                     "combine_bwd"));
    trace_mark(st, "combine_bwd");
    return ok();
}

int moe_read_device_status(const void* ws, int32_t* status, void* stream) {
    MOE_TRY(need(ws, "ws"));
    if (!status) return fail(MOE_ERR_ARG, "status is NULL");
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    int32_t v = 0;
    if (cudaMemcpyAsync(&v, ws, sizeof v, cudaMemcpyDeviceToHost, st) != cudaSuccess ||
        cudaStreamSynchronize(st) != cudaSuccess)
        return fail(MOE_ERR_CUDA, "reading the device status failed: %s",
                    cudaGetErrorString(cudaGetLastError()));
    if (cudaMemsetAsync(const_cast<void*>(ws), 0, sizeof v, st) != cudaSuccess)
        return fail(MOE_ERR_CUDA, "clearing the device status failed");
    *status = v;
    return ok();
}

int moe_launch_count(uint64_t* n) {
    if (!n) return fail(MOE_ERR_ARG, "n is NULL");
    *n = g_launches.load(std::memory_order_relaxed);
    return ok();
}

int moe_set_pdl(int on) {
    g_pdl_enabled = on ? 1 : 0;
    return ok();
}

int moe_set_pair_tiles(int mode) {
    if (mode < 0 || mode > 2) return fail(MOE_ERR_ARG, "mode must be 0, 1 or 2");
    g_pair_enabled = mode;
    return ok();
}

int moe_set_shared_overlap(int on) {
    g_shared_overlap = on ? 1 : 0;
    return ok();
}

int moe_set_shared_sms(int sms) {
    if (sms < 0 || sms > 1024 || sms % 2)
        return fail(MOE_ERR_ARG, "sms must be an even count in [0, 1024]");
    g_shared_sms = sms;
    return ok();
}

int moe_set_wait_limit_ns(uint64_t ns) {
    g_wait_limit_ns = ns;
    return ok();
}

int moe_set_test_stall(int on) {
    g_test_stall = on ? 1 : 0;
    return ok();
}

int moe_trace_begin(int max_calls, const char* only) {
    if (max_calls < 1 || max_calls > 100000) return fail(MOE_ERR_ARG, "max_calls out of range");
    const size_t need_ev = (size_t)max_calls * 24;
    while (g_trace.pool.size() < need_ev) {
        cudaEvent_t ev;
        if (cudaEventCreate(&ev) != cudaSuccess) return fail(MOE_ERR_CUDA, "cudaEventCreate failed");
        g_trace.pool.push_back(ev);
    }
    g_trace.marks.clear();
    g_trace.calls = 0;
    g_trace.max_calls = max_calls;
    g_trace.only = only ? only : "";
    g_trace.on = true;
    return ok();
}

int moe_trace_end(char (*names)[32], int* launches, double* ms, int cap, int* n_out) {
    g_trace.on = false;
    if (!n_out) return fail(MOE_ERR_ARG, "n_out is NULL");
    std::vector<std::string> nm;
    std::vector<int> cnt;
    std::vector<double> tot;
    for (size_t i = 1; i < g_trace.marks.size(); ++i) {
        const TraceMark& a = g_trace.marks[i - 1];
        const TraceMark& b = g_trace.marks[i];
        if (a.call != b.call || b.pre) continue;
        if (cudaEventSynchronize(b.ev) != cudaSuccess)
            return fail(MOE_ERR_CUDA, "cudaEventSynchronize failed");
        float t = 0.f;
        if (cudaEventElapsedTime(&t, a.ev, b.ev) != cudaSuccess)
            return fail(MOE_ERR_CUDA, "cudaEventElapsedTime failed");
        size_t j = 0;
        while (j < nm.size() && nm[j] != b.name) ++j;
        if (j == nm.size()) {
            nm.push_back(b.name);
            cnt.push_back(0);
            tot.push_back(0.0);
        }
        cnt[j] += 1;
        tot[j] += t;
    }
    int n = 0;
    for (size_t j = 0; j < nm.size() && n < cap; ++j, ++n) {
        if (names) {
            strncpy(names[n], nm[j].c_str(), 31);
            names[n][31] = 0;
        }
        if (launches) launches[n] = cnt[j];
        if (ms) ms[n] = tot[j];
    }
    *n_out = n;
    g_trace.marks.clear();
    return ok();
}

}  // extern "C"
