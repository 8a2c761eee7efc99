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
// Kernel 2 (topk): one thread per token.  Keeps the k largest logits in
// registers (strictly greater wins, so the lower index keeps a tie), gates
// = softmax over the kept k, then the full softmax for the block partial sums
// of P_e, the per-token entropy and the per-block expert histogram that
// dispatch scans.  All block sums run in a fixed order (deterministic).
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
                         const float* __restrict__ bias, float* __restrict__ z, int64_t T, int d,
                         int E, int dch) {
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
        const float b = bias ? bias[e0 + lane] : 0.f;
#pragma unroll
        for (int i = 0; i < TPW; ++i) {
            const int64_t t = t0 + i;
            float v = 0.f;
#pragma unroll
            for (int e = 0; e < RT_EXP; ++e)
                if (e == lane) v = acc[i][e];
            if (t < T) z[t * E + e0 + lane] = v + b;
        }
    }
}

template <typename XT, int TPW>
int launch_logits_t(const XT* x, const float* Wr, const float* bias, float* z, int64_t T, int d,
                    int E, cudaStream_t st) {
    const int tok_per_cta = RT_WARPS * TPW;
    dim3 grid((unsigned)((T + tok_per_cta - 1) / tok_per_cta), (E + RT_EXP - 1) / RT_EXP);
    const int dch = d < RT_DCH ? d : RT_DCH;
    const size_t smem = (size_t)RT_EXP * (dch + 4) * sizeof(float);
    auto kern = router_logits_kernel<XT, TPW>;
    static size_t configured = 0;
    if (smem > 48 * 1024 && smem > configured) {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
            cudaSuccess)
            return -1;
        configured = smem;
    }
    kern<<<grid, RT_WARPS * 32, smem, st>>>(x, Wr, bias, z, T, d, E, dch);
    return cudaGetLastError() == cudaSuccess ? 0 : -1;
}

template <typename XT>
int launch_logits_dispatch(const XT* x, const float* Wr, const float* bias, float* z, int64_t T,
                           int d, int E, int num_sms, cudaStream_t st) {
    // tokens per warp: as many as keep at least ~2 CTAs per SM busy
    const int64_t ctas_e = (E + RT_EXP - 1) / RT_EXP;
    const int64_t want = 2LL * num_sms;
    if ((T + 63) / 64 * ctas_e >= want) return launch_logits_t<XT, 8>(x, Wr, bias, z, T, d, E, st);
    if ((T + 31) / 32 * ctas_e >= want) return launch_logits_t<XT, 4>(x, Wr, bias, z, T, d, E, st);
    if ((T + 15) / 16 * ctas_e >= want) return launch_logits_t<XT, 2>(x, Wr, bias, z, T, d, E, st);
    return launch_logits_t<XT, 1>(x, Wr, bias, z, T, d, E, st);
}

// ---------------------------------------------------------------- top-k

constexpr int TK_CHUNK = 32;  // experts per shared-memory pass of the P partial sums

__global__ void __launch_bounds__(ROUTE_BLOCK)
    topk_kernel(const float* __restrict__ z, int64_t T, int E, int k, int32_t* __restrict__ idx,
                float* __restrict__ gate, float* __restrict__ ppart, float* __restrict__ hpart,
                int32_t* __restrict__ cnt, int32_t* __restrict__ status) {
    __shared__ float ps[ROUTE_BLOCK][TK_CHUNK + 1];
    __shared__ float hs[ROUTE_BLOCK];
    extern __shared__ int32_t hist[];  // [E]
    const int tid = threadIdx.x;
    const int64_t t = (int64_t)blockIdx.x * ROUTE_BLOCK + tid;
    const bool valid = t < T;
    const float* zt = z + (valid ? t : 0) * E;

    for (int e = tid; e < E; e += ROUTE_BLOCK) hist[e] = 0;
    // a new layer call starts here: clear the device status word
    if (blockIdx.x == 0 && tid == 0 && status) *status = DEV_OK;

    float val[MAX_K];
    int id[MAX_K];
#pragma unroll
    for (int j = 0; j < MAX_K; ++j) {
        val[j] = -INFINITY;
        id[j] = -1;
    }
    if (valid) {
        for (int e = 0; e < E; ++e) {
            float v = zt[e];
            if (v != v) v = -INFINITY;  // a NaN logit ranks last
            // insert if larger than the current k-th (or a slot is still empty):
            // walk the sorted list; from the insertion point on, every entry
            // shifts down one place and the old k-th falls off
            if (id[k - 1] < 0 || v > val[k - 1]) {
                float cv = v;
                int ci = e;
                bool ins = false;
#pragma unroll
                for (int q = 0; q < MAX_K; ++q) {
                    if (q < k && (ins || id[q] < 0 || cv > val[q])) {
                        const float tv = val[q];
                        const int ti = id[q];
                        val[q] = cv;
                        id[q] = ci;
                        cv = tv;
                        ci = ti;
                        ins = true;
                    }
                }
            }
        }
    }
    __syncthreads();  // hist cleared
    float m = val[0];
    if (valid) {
        float s = 0.f;
#pragma unroll
        for (int j = 0; j < MAX_K; ++j)
            if (j < k) s += __expf(val[j] - m);
        const float inv = 1.f / s;
#pragma unroll
        for (int j = 0; j < MAX_K; ++j)
            if (j < k) {
                idx[t * k + j] = id[j];
                gate[t * k + j] = __expf(val[j] - m) * inv;
                atomicAdd(&hist[id[j]], 1);
            }
    }
    // full softmax over E: S = sum exp(z - m); p = exp(z - m) / S;
    // entropy = ln S - sum p (z - m)
    float S = 0.f;
    if (valid)
        for (int e = 0; e < E; ++e) {
            float v = zt[e];
            S += __expf((v != v ? -INFINITY : v) - m);
        }
    const float invS = valid ? 1.f / S : 0.f;
    float pz = 0.f;
    for (int c0 = 0; c0 < E; c0 += TK_CHUNK) {
        const int n = min(TK_CHUNK, E - c0);
        for (int i = 0; i < n; ++i) {
            float p = 0.f;
            if (valid) {
                float v = zt[c0 + i];
                v = (v != v) ? -INFINITY : v;
                p = __expf(v - m) * invS;
                if (p > 0.f) pz += p * (v - m);
            }
            ps[tid][i] = p;
        }
        __syncthreads();
        if (tid < n) {
            float acc = 0.f;
            for (int r = 0; r < ROUTE_BLOCK; ++r) acc += ps[r][tid];
            ppart[(int64_t)blockIdx.x * E + c0 + tid] = acc;
        }
        __syncthreads();
    }
    hs[tid] = valid ? (__logf(S) - pz) : 0.f;
    __syncthreads();
    if (tid == 0) {
        float acc = 0.f;
        for (int r = 0; r < ROUTE_BLOCK; ++r) acc += hs[r];
        hpart[blockIdx.x] = acc;
    }
    for (int e = tid; e < E; e += ROUTE_BLOCK) cnt[(int64_t)blockIdx.x * E + e] = hist[e];
}

}  // namespace

int launch_router_logits(const void* x, bool x_bf16, const float* Wr, const float* bias,
                         float* z, int64_t T, int d, int E, int num_sms, cudaStream_t st) {
    if (T == 0) return 0;
    if (x_bf16)
        return launch_logits_dispatch(reinterpret_cast<const __nv_bfloat16*>(x), Wr, bias, z, T, d,
                                      E, num_sms, st);
    return launch_logits_dispatch(reinterpret_cast<const float*>(x), Wr, bias, z, T, d, E,
                                  num_sms, st);
}

int launch_topk(const float* z, int64_t T, int E, int k, int32_t* topk_idx, float* topk_gate,
                float* ppart, float* hpart, int32_t* cnt, int32_t* status, cudaStream_t st) {
    if (T == 0) return 0;
    const unsigned blocks = (unsigned)((T + ROUTE_BLOCK - 1) / ROUTE_BLOCK);
    topk_kernel<<<blocks, ROUTE_BLOCK, E * sizeof(int32_t), st>>>(z, T, E, k, topk_idx, topk_gate,
                                                                  ppart, hpart, cnt, status);
    return cudaGetLastError() == cudaSuccess ? 0 : -1;
}

}  // namespace moe
