// route_static.cu -- the router / top-k step without a caller workspace.
//
// Some callers cannot allocate device memory for a workspace: code running
// inside a framework whose allocator they do not control, a plugin given only
// input and output buffers, or a process that must not grow its device
// footprint after start-up.  moe_route_static serves them: it runs the same
// kernels as moe_route (one CTA per token for the logits, then top-k and the
// gates), but its scratch -- the logits and the per-block statistics
// partials -- lives in one fixed array of device memory owned by this
// library (MOE_ROUTE_STATIC_SCRATCH bytes), held by a GPU from the first call
// on it until the process exits.
//
// Host code cannot use the array's name as a device address (on the host it
// names a stand-in object), so the device address is looked up once per
// device with cudaGetSymbolAddress, with that device current, on the first
// call that runs on the device.  Under CUDA's lazy module loading (the
// default) that lookup is also when the array comes into being on the
// device, so a caller that must keep its device footprint fixed makes one
// warm-up call per device at start-up; that first call should also come
// before any stream capture.  The address is cached with the id of the
// context it belongs to and looked up again if the device's context changes
// (after a cudaDeviceReset, say).  All calls share the array and each call
// overwrites what the previous one left there; calls that overlap on the GPU
// (two streams, two threads) race on it and must be serialised by the caller.
#include <string.h>

#include <mutex>

#include "../../include/moe.h"
#include "common.cuh"
#include "kernels.h"
#include "plan.h"

namespace moe {

int report_error(int code, const char* text);  // capi.cu

namespace {

constexpr size_t kScratchBytes = MOE_ROUTE_STATIC_SCRATCH;
constexpr int kMaxDevices = 64;

__device__ __align__(256) uint8_t g_route_scratch[kScratchBytes];

std::mutex g_mu;
void* g_scratch_ptr[kMaxDevices] = {nullptr};
unsigned long long g_scratch_ctx[kMaxDevices] = {0};

// Unique id of the current thread's CUDA context (cuCtxGetId through the
// runtime's driver entry point; 0 when it cannot be had).
unsigned long long current_context_id() {
    typedef CUresult (*GetCurrent)(CUcontext*);
    typedef CUresult (*GetId)(CUcontext, unsigned long long*);
    static GetCurrent get_current = nullptr;
    static GetId get_id = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) ==
                cudaSuccess && q == cudaDriverEntryPointSuccess)
            get_current = reinterpret_cast<GetCurrent>(p);
        p = nullptr;
        if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_id = reinterpret_cast<GetId>(p);
    });
    CUcontext ctx = nullptr;
    unsigned long long id = 0;
    if (get_current && get_id && get_current(&ctx) == CUDA_SUCCESS && ctx &&
        get_id(ctx, &id) == CUDA_SUCCESS)
        return id;
    return 0;
}

// Device address of the scratch array for the current device, looked up on
// the first call on the device (and again when its context has changed).
int scratch_for_current_device(uint8_t** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices)
        return report_error(MOE_ERR_CUDA, "moe_route_static: cudaGetDevice failed");
    // 0 when no context is current yet: the lookup below then makes the
    // device's primary context current
    const unsigned long long ctx = current_context_id();
    std::lock_guard<std::mutex> lk(g_mu);
    if (!g_scratch_ptr[dev] || ctx == 0 || ctx != g_scratch_ctx[dev]) {
        void* p = nullptr;
        const cudaError_t e = cudaGetSymbolAddress(&p, g_route_scratch);
        if (e != cudaSuccess || !p)
            return report_error(MOE_ERR_CUDA,
                                "moe_route_static: cudaGetSymbolAddress of the scratch failed");
        g_scratch_ptr[dev] = p;
        g_scratch_ctx[dev] = ctx != 0 ? ctx : current_context_id();
    }
    *out = static_cast<uint8_t*>(g_scratch_ptr[dev]);
    return MOE_OK;
}

size_t up256(size_t v) { return (v + 255) & ~(size_t)255; }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

}  // namespace

}  // namespace moe

using namespace moe;

extern "C" MOE_API int moe_route_static(const moe_config* cfg, const void* x, const float* Wr,
                                        const float* bias, int32_t* topk_idx, float* topk_gate,
                                        void* stream) {
    Plan P;
    const char* why = "";
    int s = make_plan(cfg, &P, &why);
    if (s != MOE_OK) return report_error(s, why);
    if (P.T > MOE_ROUTE_STATIC_MAX_T)
        return report_error(MOE_ERR_SHAPE, "moe_route_static: T is above MOE_ROUTE_STATIC_MAX_T");
    if (P.T * (int64_t)P.E > MOE_ROUTE_STATIC_MAX_TE)
        return report_error(MOE_ERR_SHAPE,
                            "moe_route_static: T * E is above MOE_ROUTE_STATIC_MAX_TE");
    // layout of the scratch: status words | logits [T][E] | P partials | entropy
    // partials | histograms (sized by the limits above, well inside the array)
    const size_t o_z = 256;
    const size_t o_pp = o_z + up256((size_t)P.T * P.E * 4);
    const size_t nrows = (size_t)P.nblk * P.nsub;  // partial rows (top-k CTAs)
    const size_t o_hp = o_pp + up256(nrows * P.E * 4);
    const size_t o_cnt = o_hp + up256(nrows * 4);
    const size_t total = o_cnt + up256(nrows * P.E * 4);
    if (total > kScratchBytes)
        return report_error(MOE_ERR_SHAPE, "moe_route_static: scratch array too small");
    if (P.T == 0) return report_error(MOE_OK, "");
    if (!x || !Wr || !topk_idx || !topk_gate || (cfg->has_bias && !bias))
        return report_error(MOE_ERR_ARG, "moe_route_static: a required pointer is NULL");
    if (!aligned16(x) || !aligned16(Wr) || !aligned16(topk_idx) || !aligned16(topk_gate) ||
        (cfg->has_bias && !aligned16(bias)))
        return report_error(MOE_ERR_ALIGN, "moe_route_static: a pointer is not 16-byte aligned");

    uint8_t* scratch = nullptr;
    s = scratch_for_current_device(&scratch);
    if (s != MOE_OK) return s;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    float* z = reinterpret_cast<float*>(scratch + o_z);

    if (launch_router_rows(x, P.bf16, Wr, z, (int)P.T, P.d, P.E, st) != 0)
        return report_error(MOE_ERR_CUDA, "moe_route_static: router launch failed");
    RouteParams r;
    memset(&r, 0, sizeof r);
    r.src = z;
    r.bias = cfg->has_bias ? bias : nullptr;
    r.zbuf = z;
    r.logits = nullptr;
    r.T = P.T;
    r.E = P.E;
    r.k = P.k;
    r.topk_idx = topk_idx;
    r.topk_gate = topk_gate;
    r.ppart = reinterpret_cast<float*>(scratch + o_pp);
    r.hpart = reinterpret_cast<float*>(scratch + o_hp);
    r.cnt = reinterpret_cast<int32_t*>(scratch + o_cnt);
    r.status = reinterpret_cast<int32_t*>(scratch);  // cleared by the top-k kernel
    r.nsub = P.nsub;
    if (launch_topk(r, st) != 0)
        return report_error(MOE_ERR_CUDA, "moe_route_static: top-k launch failed");
    return report_error(MOE_OK, "");
}
