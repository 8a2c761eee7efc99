// router.cu -- the linear router, top-k selection and gates.
//
// [Mixtral 8x7B and MoE explained, "Easy explanation" ¶3]: the router scores
// every expert like a classifier, keeps the top k and softmaxes over those k
// to weight the experts' outputs.  [MoE routing fully explained, "Easy
// explanation" ¶2]: the router's full distribution over all experts, used
// here only for the load-balancing statistics.
//
// Kernel 1 (router_logits): z = x W_r + b in fp32.  A CTA owns 8 experts and
// a run of tokens; the 8 columns of W_r sit transposed in shared memory and
// every warp streams its tokens' rows of x once, each lane covering 8 of
// every 256 elements with 16-byte (fp32) or 8-byte (bf16) loads.  The work is
// HBM-bound for E = 8 (x is read once) and FP32-pipe bound for E = 160.
//
// Small batches (<= 256 tokens) use one CTA per token instead, and
// bf16 batches above that a tensor-core GEMM against W_r split into three
// bf16 parts; the partial sums are added in a fixed order (router_reduce, or
// inside the top-k kernel).  Top-k and gates live in routing.cu.
#include <math.h>

#include "common.cuh"
#include "kernels.h"
#include "plan.h"

namespace moe {

namespace {

constexpr int RT_WARPS = 8;
constexpr int RT_EXP = 8;         // experts per CTA
constexpr int RT_DCH = 4096;      // max d elements per shared-memory chunk

template <typename XT>
__device__ __forceinline__ void load4(const XT* p, float* v);

template <>
__device__ __forceinline__ void load4<float>(const float* p, float* v) {
    float4 f = *reinterpret_cast<const float4*>(p);
    v[0] = f.x; v[1] = f.y; v[2] = f.z; v[3] = f.w;
}

template <>
__device__ __forceinline__ void load4<__nv_bfloat16>(const __nv_bfloat16* p, float* v) {
    uint2 u = *reinterpret_cast<const uint2*>(p);
    v[0] = __uint_as_float(u.x << 16);
    v[1] = __uint_as_float(u.x & 0xFFFF0000u);
    v[2] = __uint_as_float(u.y << 16);
    v[3] = __uint_as_float(u.y & 0xFFFF0000u);
}

template <typename XT, int TPW>
__global__ void __launch_bounds__(RT_WARPS * 32)
    router_logits_kernel(const XT* __restrict__ x, const float* __restrict__ Wr,
                         float* __restrict__ z, int64_t T, int d, int E, int dch) {
    // W_r columns e0..e0+7, transposed: [RT_EXP][dch + 4] (the +4 staggers banks)
    extern __shared__ float ws[];
    const int pitch = dch + 4;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int e0 = blockIdx.y * RT_EXP;
    const int ne = min(RT_EXP, E - e0);
    const int64_t t0 = ((int64_t)blockIdx.x * RT_WARPS + warp) * TPW;

    float acc[TPW][RT_EXP];
#pragma unroll
    for (int i = 0; i < TPW; ++i)
#pragma unroll
        for (int e = 0; e < RT_EXP; ++e) acc[i][e] = 0.f;

    for (int c0 = 0; c0 < d; c0 += dch) {
        const int len = min(dch, d - c0);
        __syncthreads();
        for (int i = threadIdx.x; i < len * RT_EXP; i += blockDim.x) {
            const int c = i / RT_EXP, e = i % RT_EXP;
            ws[e * pitch + c] = (e < ne) ? Wr[(int64_t)(c0 + c) * E + e0 + e] : 0.f;
        }
        __syncthreads();
        for (int s = 0; s < len; s += 256) {
            float xv[TPW][8];
            bool have[2];
#pragma unroll
            for (int v = 0; v < 2; ++v) have[v] = (s + 4 * (lane + 32 * v)) < len;
#pragma unroll
            for (int i = 0; i < TPW; ++i) {
                const int64_t t = t0 + i;
#pragma unroll
                for (int v = 0; v < 2; ++v) {
                    if (t < T && have[v])
                        load4<XT>(x + t * d + c0 + s + 4 * (lane + 32 * v), &xv[i][4 * v]);
                    else
                        xv[i][4 * v] = xv[i][4 * v + 1] = xv[i][4 * v + 2] = xv[i][4 * v + 3] = 0.f;
                }
            }
#pragma unroll
            for (int e = 0; e < RT_EXP; ++e) {
                float w[8];
#pragma unroll
                for (int v = 0; v < 2; ++v) {
                    if (have[v]) {
                        float4 f = *reinterpret_cast<const float4*>(
                            &ws[e * pitch + s + 4 * (lane + 32 * v)]);
                        w[4 * v] = f.x; w[4 * v + 1] = f.y; w[4 * v + 2] = f.z; w[4 * v + 3] = f.w;
                    } else {
                        w[4 * v] = w[4 * v + 1] = w[4 * v + 2] = w[4 * v + 3] = 0.f;
                    }
                }
#pragma unroll
                for (int i = 0; i < TPW; ++i)
#pragma unroll
                    for (int j = 0; j < 8; ++j) acc[i][e] = fmaf(xv[i][j], w[j], acc[i][e]);
            }
        }
    }
#pragma unroll
    for (int i = 0; i < TPW; ++i)
#pragma unroll
        for (int e = 0; e < RT_EXP; ++e) {
            float v = acc[i][e];
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
            acc[i][e] = v;
        }
    if (lane < RT_EXP && lane < ne) {
#pragma unroll
        for (int i = 0; i < TPW; ++i) {
            const int64_t t = t0 + i;
            float v = 0.f;
#pragma unroll
            for (int e = 0; e < RT_EXP; ++e)
                if (e == lane) v = acc[i][e];
            if (t < T) z[t * E + e0 + lane] = v;
        }
    }
}

template <typename XT, int TPW>
int launch_logits_t(const XT* x, const float* Wr, float* z, int64_t T, int d, int E,
                    cudaStream_t st) {
    const int tok_per_cta = RT_WARPS * TPW;
    dim3 grid((unsigned)((T + tok_per_cta - 1) / tok_per_cta), (E + RT_EXP - 1) / RT_EXP);
    const int dch = d < RT_DCH ? d : RT_DCH;
    const size_t smem = (size_t)RT_EXP * (dch + 4) * sizeof(float);
    auto kern = router_logits_kernel<XT, TPW>;
    // the opt-in is per device: set it on every launch that needs it
    if (smem > 48 * 1024 &&
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
            cudaSuccess)
        return -1;
    kern<<<grid, RT_WARPS * 32, smem, st>>>(x, Wr, z, T, d, E, dch);
    note_launch();
    return launch_result();
}

template <typename XT>
int launch_logits_dispatch(const XT* x, const float* Wr, float* z, int64_t T, int d, int E,
                           int num_sms, cudaStream_t st) {
    // tokens per warp: as many as keep at least ~2 CTAs per SM busy
    const int64_t ctas_e = (E + RT_EXP - 1) / RT_EXP;
    const int64_t want = 2LL * num_sms;
    if ((T + 63) / 64 * ctas_e >= want) return launch_logits_t<XT, 8>(x, Wr, z, T, d, E, st);
    if ((T + 31) / 32 * ctas_e >= want) return launch_logits_t<XT, 4>(x, Wr, z, T, d, E, st);
    if ((T + 15) / 16 * ctas_e >= want) return launch_logits_t<XT, 2>(x, Wr, z, T, d, E, st);
    return launch_logits_t<XT, 1>(x, Wr, z, T, d, E, st);
}

// ---------------------------------------------------------------- small batches
//
// With at most 256 tokens the router is a latency problem, not a bandwidth
// one.  One CTA per (token, group of 8 experts): its 256 threads split the d
// dimension (8 contiguous elements per thread per 2048-wide slab), multiply
// by the matching rows of W_r, and a fixed-order block reduction (warp
// shuffles, then the 8 warp sums in order) gives the token's 8 logits.  Every
// CTA issues all of its loads at once, so the whole router takes about two
// memory latencies.
constexpr int RR_THREADS = 256;
constexpr int RR_SLAB = RR_THREADS * 8;

template <typename XT>
__device__ __forceinline__ void load8(const XT* p, float* v);

template <>
__device__ __forceinline__ void load8<float>(const float* p, float* v) {
    const float4 a = *reinterpret_cast<const float4*>(p);
    const float4 b = *reinterpret_cast<const float4*>(p + 4);
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}

template <>
__device__ __forceinline__ void load8<__nv_bfloat16>(const __nv_bfloat16* p, float* v) {
    const uint4 u = *reinterpret_cast<const uint4*>(p);
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        v[2 * i] = __uint_as_float(w[i] << 16);
        v[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
}

template <typename XT>
__global__ void __launch_bounds__(RR_THREADS)
    router_rows_kernel(const XT* __restrict__ x, const float* __restrict__ Wr,
                       float* __restrict__ z, int d, int E) {
    __shared__ float red[RR_THREADS / 32][RT_EXP];
    pdl_wait();
    pdl_trigger();
    const int t = blockIdx.x;
    const int e0 = blockIdx.y * RT_EXP;
    const int ne = min(RT_EXP, E - e0);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    float acc[RT_EXP];
#pragma unroll
    for (int e = 0; e < RT_EXP; ++e) acc[e] = 0.f;
    const bool full8 = ne == RT_EXP && (E % 4) == 0;
    for (int c0 = 8 * tid; c0 < d; c0 += RR_SLAB) {
        float xv[8];
        load8<XT>(x + (int64_t)t * d + c0, xv);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const float* wrow = Wr + (int64_t)(c0 + j) * E + e0;
            float w[RT_EXP];
            if (full8) {
                const float4 a = *reinterpret_cast<const float4*>(wrow);
                const float4 b = *reinterpret_cast<const float4*>(wrow + 4);
                w[0] = a.x; w[1] = a.y; w[2] = a.z; w[3] = a.w;
                w[4] = b.x; w[5] = b.y; w[6] = b.z; w[7] = b.w;
            } else {
#pragma unroll
                for (int e = 0; e < RT_EXP; ++e) w[e] = e < ne ? wrow[e] : 0.f;
            }
#pragma unroll
            for (int e = 0; e < RT_EXP; ++e) acc[e] = fmaf(xv[j], w[e], acc[e]);
        }
    }
#pragma unroll
    for (int e = 0; e < RT_EXP; ++e) {
        float v = acc[e];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
        if (lane == 0) red[warp][e] = v;
    }
    __syncthreads();
    if (tid < ne) {
        float v = 0.f;
#pragma unroll
        for (int w = 0; w < RR_THREADS / 32; ++w) v += red[w][tid];
        z[(int64_t)t * E + e0 + tid] = v;
    }
}

// ---------------------------------------------------------------- router on the tensor cores
//
// For bf16 tokens the logits run as a tensor-core GEMM (gemm_tc.cu) against
// W_r split into three bf16 parts, W = W_hi + W_mid + W_lo (each part the
// bf16 rounding of what the earlier parts leave), stored transposed
// (K-major): Ws[p*E + e][c].  Every product of a bf16 token element with a
// bf16 part is exact in fp32 and the three partial sums together carry W to
// 24 bits, so the logits keep fp32 accuracy.  topk sums the parts.
__global__ void router_split_kernel(const float* __restrict__ Wr, __nv_bfloat16* __restrict__ Ws,
                                    int d, int E) {
    // 32 x 32 tile of W_r (rows c, columns e) transposed through shared memory
    __shared__ float tile[32][33];
    const int c0 = blockIdx.x * 32, e0 = blockIdx.y * 32;
    for (int i = threadIdx.y; i < 32; i += blockDim.y) {
        const int c = c0 + i, e = e0 + threadIdx.x;
        tile[i][threadIdx.x] = (c < d && e < E) ? Wr[(int64_t)c * E + e] : 0.f;
    }
    __syncthreads();
    for (int i = threadIdx.y; i < 32; i += blockDim.y) {
        const int e = e0 + i, c = c0 + threadIdx.x;
        if (e >= E || c >= d) continue;
        const float w = tile[threadIdx.x][i];
        const __nv_bfloat16 hi = __float2bfloat16_rn(w);
        const float r1 = w - __bfloat162float(hi);
        const __nv_bfloat16 mid = __float2bfloat16_rn(r1);
        const float r2 = r1 - __bfloat162float(mid);
        const __nv_bfloat16 lo = __float2bfloat16_rn(r2);
        Ws[(int64_t)e * d + c] = hi;
        Ws[(int64_t)(E + e) * d + c] = mid;
        Ws[(int64_t)(2 * E + e) * d + c] = lo;
    }
}

// ---------------------------------------------------------------- partial-sum reduction
//
// z[t][e] = bias[e] + sum over splits s and parts p of src[s][t][p*E + e], in
// that fixed order; one thread per logit, coalesced along e.
__global__ void __launch_bounds__(256)
    router_reduce_kernel(const float* __restrict__ src, int nsplit, int64_t split_stride,
                         int row_stride, int nparts, const float* __restrict__ bias,
                         float* __restrict__ z, int64_t T, int E) {
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= T * E) return;
    const int64_t t = i / E;
    const int e = (int)(i % E);
    float v = bias ? bias[e] : 0.f;
    const float* base = src + t * row_stride + e;
    if (nparts == 3) {
        // all loads first (independent), then the adds in fixed order
        float part[8][3];
#pragma unroll
        for (int q = 0; q < 8; ++q)
            if (q < nsplit)
#pragma unroll
                for (int p = 0; p < 3; ++p) part[q][p] = base[q * split_stride + p * E];
#pragma unroll
        for (int q = 0; q < 8; ++q)
            if (q < nsplit)
#pragma unroll
                for (int p = 0; p < 3; ++p) v += part[q][p];
        for (int q = 8; q < nsplit; ++q)
            for (int p = 0; p < 3; ++p) v += base[q * split_stride + p * E];
    } else {
        for (int q = 0; q < nsplit; ++q) {
            const float* r = base + q * split_stride;
            for (int p = 0; p < nparts; ++p) v += r[p * E];
        }
    }
    z[i] = v;
}

}  // namespace

int launch_router_logits(const void* x, bool x_bf16, const float* Wr, float* z, int64_t T, int d,
                         int E, int num_sms, cudaStream_t st) {
    if (T == 0) return 0;
    if (x_bf16)
        return launch_logits_dispatch(reinterpret_cast<const __nv_bfloat16*>(x), Wr, z, T, d, E,
                                      num_sms, st);
    return launch_logits_dispatch(reinterpret_cast<const float*>(x), Wr, z, T, d, E, num_sms, st);
}

int launch_router_rows(const void* x, bool x_bf16, const float* Wr, float* z, int T, int d,
                       int E, cudaStream_t st) {
    if (T == 0) return 0;
    dim3 grid(T, (E + RT_EXP - 1) / RT_EXP);
    if (x_bf16)
        launch_ex(pdl_active(), router_rows_kernel<__nv_bfloat16>, grid, dim3(RR_THREADS), 0, st,
                  reinterpret_cast<const __nv_bfloat16*>(x), Wr, z, d, E);
    else
        launch_ex(pdl_active(), router_rows_kernel<float>, grid, dim3(RR_THREADS), 0, st,
                  reinterpret_cast<const float*>(x), Wr, z, d, E);
    note_launch();
    return launch_result();
}

int launch_router_reduce(const float* src, int nsplit, int64_t split_stride, int row_stride,
                         int nparts, const float* bias, float* z, int64_t T, int E,
                         cudaStream_t st) {
    if (T == 0) return 0;
    const int64_t n = T * E;
    router_reduce_kernel<<<(unsigned)((n + 255) / 256), 256, 0, st>>>(
        src, nsplit, split_stride, row_stride, nparts, bias, z, T, E);
    note_launch();
    return launch_result();
}

int launch_router_split(const float* Wr, void* Ws, int d, int E, cudaStream_t st) {
    dim3 grid((d + 31) / 32, (E + 31) / 32), block(32, 8);
    router_split_kernel<<<grid, block, 0, st>>>(Wr, reinterpret_cast<__nv_bfloat16*>(Ws), d, E);
    note_launch();
    return launch_result();
}

}  // namespace moe
