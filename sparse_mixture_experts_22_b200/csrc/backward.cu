// backward.cu -- the layer's backward pass outside the tensor-core GEMMs.
//
// Loss L = sum_t <G_t, out_t> + aux_coef * aux.  The pages motivate the
// gradients (the router's softmax weighting and the load-balancing loss are
// what training acts on: MoE routing fully explained, "Easy explanation" ¶2
// and ¶4); the readings are those of the header: routing decisions and the
// routed counts f_e carry no gradient, gates are not renormalised after a
// drop, and under reroute the gate gradient goes to the router's choice.
//
//   gather     dY[r] = g G_t (bf16) for every kept slot r of token t, and
//              dg = <G_t, y_r> (y summed over its split-K partials)
//   router     dz_t = softmax-over-k backward of dg + aux term
//              aux_coef (E / T) p_te (f_e - sum_i f_i p_ti)
//   wr_grad    dWr = x^T dz and db = column sums of dz, split over token
//              chunks into partials reduced in a fixed order
//   dxr        the router's share of dx: dz Wr^T
//   kofs       each expert's 64-aligned offset along the token axis of the
//              transposed activations the weight-gradient GEMMs contract
//   transpose  [rows][features] -> [features][tokens] per expert segment,
//              zero-filled up to the next multiple of 64 tokens
//   combine    dx_t = sum over kept slots of dXp + shared dX + router dX
// Every sum runs in a fixed order: the results are identical run to run.
#include "common.cuh"
#include "kernels.h"

namespace moe {

namespace {

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

// ---------------------------------------------------------------- gather

constexpr int GATHER_THREADS = 256;

__global__ void __launch_bounds__(GATHER_THREADS)
    bwd_gather_kernel(const __nv_bfloat16* __restrict__ G, const float* __restrict__ y,
                      int splits, int64_t split_stride, const int32_t* __restrict__ slot_of,
                      const float* __restrict__ gate, __nv_bfloat16* __restrict__ dY,
                      float* __restrict__ dg, int64_t T, int d, int k) {
    __shared__ float red[GATHER_THREADS / 32];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    for (int64_t t = blockIdx.x; t < T; t += gridDim.x) {
        const __nv_bfloat16* g = G + t * d;
        for (int j = 0; j < k; ++j) {
            const int32_t r = slot_of[t * k + j];
            if (r < 0) {
                if (tid == 0) dg[t * k + j] = 0.0f;
                continue;
            }
            const float gj = gate[t * k + j];
            float part = 0.0f;
            for (int c = tid * 16; c < d; c += GATHER_THREADS * 16) {
                float gv[16], yv[16], o[16];
                load_bf16x16(g + c, gv);
#pragma unroll
                for (int i = 0; i < 16; ++i) yv[i] = 0.0f;
                for (int s = 0; s < splits; ++s) {
                    const float4* yp =
                        reinterpret_cast<const float4*>(y + s * split_stride + (int64_t)r * d + c);
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const float4 w = yp[q];
                        yv[4 * q] += w.x;
                        yv[4 * q + 1] += w.y;
                        yv[4 * q + 2] += w.z;
                        yv[4 * q + 3] += w.w;
                    }
                }
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    part += gv[i] * yv[i];
                    o[i] = gj * gv[i];
                }
                store_bf16x16(dY + (int64_t)r * d + c, o);
            }
            part = warp_sum(part);
            if (lane == 0) red[warp] = part;
            __syncthreads();
            if (tid == 0) {
                float s = 0.0f;
                for (int w = 0; w < GATHER_THREADS / 32; ++w) s += red[w];
                dg[t * k + j] = s;
            }
            __syncthreads();
        }
    }
}

// ---------------------------------------------------------------- router logits

// One warp per token; lane l handles experts l, l + 32, ...
__global__ void __launch_bounds__(256)
    router_bwd_kernel(const float* __restrict__ z, const float* __restrict__ bias,
                      const int32_t* __restrict__ idx, const float* __restrict__ gate,
                      const float* __restrict__ dg, const int32_t* __restrict__ routed,
                      float aux_coef, float* __restrict__ dz, int64_t T, int E, int k) {
    const int lane = threadIdx.x & 31;
    const int64_t warps = (int64_t)gridDim.x * (blockDim.x >> 5);
    const float inv_assign = 1.0f / (float)(T * k);
    const float scale = aux_coef * (float)E / (float)T;
    for (int64_t t = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); t < T;
         t += warps) {
        const float* zt = z + t * E;
        float m = -INFINITY;
        for (int e = lane; e < E; e += 32) m = fmaxf(m, zt[e] + (bias ? bias[e] : 0.0f));
        m = warp_max(m);
        float den = 0.0f, fq = 0.0f;
        for (int e = lane; e < E; e += 32) {
            const float p = expf(zt[e] + (bias ? bias[e] : 0.0f) - m);
            den += p;
            fq += (float)routed[e] * inv_assign * p;
        }
        den = warp_sum(den);
        fq = warp_sum(fq);
        const float inv_den = 1.0f / den;
        const float q = fq * inv_den;  // sum_i f_i p_i
        float mg = 0.0f;               // sum_j g_j dg_j
        for (int j = 0; j < k; ++j) mg += gate[t * k + j] * dg[t * k + j];
        for (int e = lane; e < E; e += 32) {
            const float p = expf(zt[e] + (bias ? bias[e] : 0.0f) - m) * inv_den;
            float v = scale * p * ((float)routed[e] * inv_assign - q);
            for (int j = 0; j < k; ++j)
                if (idx[t * k + j] == e) v += gate[t * k + j] * (dg[t * k + j] - mg);
            dz[t * E + e] = v;
        }
    }
}

// ---------------------------------------------------------------- router weights

constexpr int WR_THREADS = 128;
constexpr int WR_ET = 32;   // experts per block
constexpr int WR_TT = 32;   // tokens staged per step

// part[ch][c][e] = sum over the chunk's tokens of x[t][c] dz[t][e]; row c == d
// holds the column sums of dz (the bias gradient).
template <typename XT>
__global__ void __launch_bounds__(WR_THREADS)
    wr_grad_kernel(const XT* __restrict__ x, const float* __restrict__ dz, float* __restrict__ part,
                   int64_t T, int d, int E, int64_t chunk) {
    __shared__ float dzs[WR_TT][WR_ET];
    const int c = blockIdx.x * WR_THREADS + threadIdx.x;
    const int e0 = blockIdx.z * WR_ET;
    const int ne = min(WR_ET, E - e0);
    const int64_t t0 = (int64_t)blockIdx.y * chunk;
    const int64_t t1 = min(T, t0 + chunk);
    float acc[WR_ET];
#pragma unroll
    for (int i = 0; i < WR_ET; ++i) acc[i] = 0.0f;
    for (int64_t tb = t0; tb < t1; tb += WR_TT) {
        __syncthreads();
        for (int i = threadIdx.x; i < WR_TT * WR_ET; i += WR_THREADS) {
            const int tt = i / WR_ET, ee = i % WR_ET;
            dzs[tt][ee] = (tb + tt < t1 && ee < ne) ? dz[(tb + tt) * E + e0 + ee] : 0.0f;
        }
        __syncthreads();
        if (c <= d) {
            const int nt = (int)min((int64_t)WR_TT, t1 - tb);
            for (int tt = 0; tt < nt; ++tt) {
                const float xv = c < d ? (float)x[(tb + tt) * d + c] : 1.0f;
#pragma unroll
                for (int i = 0; i < WR_ET; ++i) acc[i] += xv * dzs[tt][i];
            }
        }
    }
    if (c <= d) {
        float* dst = part + ((int64_t)blockIdx.y * (d + 1) + c) * E + e0;
#pragma unroll
        for (int i = 0; i < WR_ET; ++i)
            if (i < ne) dst[i] = acc[i];
    }
}

// out[i] = sum over chunks (in order) of part[ch][i]; i < d*E -> dWr, the
// last E entries -> db (when given)
__global__ void wr_reduce_kernel(const float* __restrict__ part, int nch, int64_t n_main, int E,
                                 float* __restrict__ dWr, float* __restrict__ db) {
    const int64_t n = n_main + E;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
         i += (int64_t)gridDim.x * blockDim.x) {
        float s = 0.0f;
        for (int ch = 0; ch < nch; ++ch) s += part[(int64_t)ch * n + i];
        if (i < n_main) dWr[i] = s;
        else if (db) db[i - n_main] = s;
    }
}

// ---------------------------------------------------------------- router share of dx

constexpr int DXR_TT = 32;   // tokens per block
constexpr int DXR_CT = 128;  // model columns per block (one per thread)
constexpr int DXR_EK = 32;   // experts staged per step

// dxr[t][c] = sum_e dz[t][e] Wr[c][e]
__global__ void __launch_bounds__(DXR_CT)
    dxr_kernel(const float* __restrict__ dz, const float* __restrict__ Wr, float* __restrict__ dxr,
               int64_t T, int d, int E) {
    __shared__ float zs[DXR_TT][DXR_EK + 1];
    __shared__ float ws[DXR_CT][DXR_EK + 1];
    const int64_t t0 = (int64_t)blockIdx.y * DXR_TT;
    const int c0 = blockIdx.x * DXR_CT;
    const int tid = threadIdx.x;
    float acc[DXR_TT];
#pragma unroll
    for (int i = 0; i < DXR_TT; ++i) acc[i] = 0.0f;
    for (int e0 = 0; e0 < E; e0 += DXR_EK) {
        __syncthreads();
        for (int i = tid; i < DXR_TT * DXR_EK; i += DXR_CT) {
            const int tt = i / DXR_EK, ee = i % DXR_EK;
            zs[tt][ee] = (t0 + tt < T && e0 + ee < E) ? dz[(t0 + tt) * E + e0 + ee] : 0.0f;
        }
        for (int i = tid; i < DXR_CT * DXR_EK; i += DXR_CT) {
            const int cc = i / DXR_EK, ee = i % DXR_EK;
            ws[cc][ee] = (e0 + ee < E) ? Wr[(int64_t)(c0 + cc) * E + e0 + ee] : 0.0f;
        }
        __syncthreads();
#pragma unroll 4
        for (int ee = 0; ee < DXR_EK; ++ee) {
            const float w = ws[tid][ee];
#pragma unroll
            for (int tt = 0; tt < DXR_TT; ++tt) acc[tt] += zs[tt][ee] * w;
        }
    }
    for (int tt = 0; tt < DXR_TT; ++tt)
        if (t0 + tt < T) dxr[(t0 + tt) * d + c0 + tid] = acc[tt];
}

// ---------------------------------------------------------------- token offsets

// kofs[g] = sum over g' < g of rows[g'] rounded up to 64; kofs[G] = total
__global__ void kofs_kernel(const int32_t* __restrict__ rows, int G, int32_t* __restrict__ kofs) {
    if (threadIdx.x != 0 || blockIdx.x != 0) return;
    int32_t acc = 0;
    for (int g = 0; g < G; ++g) {
        kofs[g] = acc;
        acc += (rows[g] + 63) / 64 * 64;
    }
    kofs[G] = acc;
}

// ---------------------------------------------------------------- transpose

constexpr int TP = 64;  // tile: 64 tokens x 64 features

// dst[f][kofs[g] + i] = src[off[g] + i][f] for i < rows[g]; zero for
// rows[g] <= i < the next multiple of 64.  Dense jobs use one group of
// `dense_rows` rows at offset 0 (rows == null).
__global__ void __launch_bounds__(256)
    transpose_kernel(TransposeJobs jobs) {
    __shared__ uint16_t tile[TP][TP + 2];
    const TransposeJob& jb = jobs.job[blockIdx.z];
    const int f0 = blockIdx.y * TP;
    if (f0 >= jb.features) return;
    const int G = jb.groups;
    const int32_t* kofs = jb.kofs;
    const int kt = blockIdx.x * TP;
    const int total = kofs ? kofs[G] : (jb.dense_rows + TP - 1) / TP * TP;
    if (kt >= total) return;
    int g = 0, local = kt, n = jb.dense_rows, r0 = 0;
    if (kofs) {
        int lo = 0, hi = G - 1;
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (kofs[mid] <= kt) lo = mid; else hi = mid - 1;
        }
        g = lo;
        local = kt - kofs[g];
        n = jb.rows[g];
        r0 = jb.off[g];
    }
    const int valid = min(TP, n - local);
    const uint16_t* src = reinterpret_cast<const uint16_t*>(jb.src);
    // load: 64 rows x 64 features, 8 features (16 bytes) per access
    for (int i = threadIdx.x; i < TP * (TP / 8); i += blockDim.x) {
        const int rr = i / (TP / 8), cc = (i % (TP / 8)) * 8;
        uint4 v = make_uint4(0, 0, 0, 0);
        if (rr < valid)
            v = *reinterpret_cast<const uint4*>(src + (int64_t)(r0 + local + rr) * jb.src_ld +
                                                f0 + cc);
        const uint16_t* pv = reinterpret_cast<const uint16_t*>(&v);
#pragma unroll
        for (int q = 0; q < 8; ++q) tile[rr][cc + q] = pv[q];
    }
    __syncthreads();
    uint16_t* dst = reinterpret_cast<uint16_t*>(jb.dst);
    for (int i = threadIdx.x; i < TP * (TP / 8); i += blockDim.x) {
        const int ff = i / (TP / 8), tt = (i % (TP / 8)) * 8;
        uint16_t pv[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) pv[q] = tile[tt + q][ff];
        *reinterpret_cast<uint4*>(dst + (int64_t)(f0 + ff) * jb.dst_ld + kt + tt) =
            *reinterpret_cast<const uint4*>(pv);
    }
}

// ---------------------------------------------------------------- dx

// dx[t] = sum_j dXp[slot_of[t][j]] (kept slots, in j order) + dXs[t] + dXr[t]
__global__ void combine_bwd_kernel(const float* __restrict__ dXp, const int32_t* __restrict__ slot_of,
                                   const float* __restrict__ dXs, const float* __restrict__ dXr,
                                   float* __restrict__ dx, int64_t T, int d, int k) {
    const int q = d / 4;
    const int64_t n = T * q;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
         i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t t = i / q;
        const int c = (int)(i % q) * 4;
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int j = 0; j < k; ++j) {
            const int32_t r = slot_of[t * k + j];
            if (r < 0) continue;
            const float4 v = *reinterpret_cast<const float4*>(dXp + (int64_t)r * d + c);
            acc.x += v.x; acc.y += v.y; acc.z += v.z; acc.w += v.w;
        }
        if (dXs) {
            const float4 v = *reinterpret_cast<const float4*>(dXs + t * d + c);
            acc.x += v.x; acc.y += v.y; acc.z += v.z; acc.w += v.w;
        }
        const float4 v = *reinterpret_cast<const float4*>(dXr + t * d + c);
        acc.x += v.x; acc.y += v.y; acc.z += v.z; acc.w += v.w;
        *reinterpret_cast<float4*>(dx + t * d + c) = acc;
    }
}

// ---------------------------------------------------------------- backward weight layout

// dst[r][col(c)] = src[r][c] (bf16, 8 columns per access) for n matrices
// [R][Cc]; col(c) = c + col_off, or with interleave >= 0 the gate/up
// interleave of 128-wide hidden blocks: j = c + col_off ->
// 256 * (j / 128) + 128 * interleave + j % 128.
__global__ void pack_cols_kernel(const uint16_t* __restrict__ src, uint16_t* __restrict__ dst,
                                 int R, int Cc, int64_t ld_dst, int col_off, int interleave,
                                 int64_t src_stride, int64_t dst_stride, int col_step) {
    src += blockIdx.y * src_stride;
    dst += blockIdx.y * dst_stride;
    col_off += blockIdx.y * col_step;
    const int q = Cc / 8;
    const int64_t n = (int64_t)R * q;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
         i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t r = i / q;
        const int c = (int)(i % q) * 8;
        const int j = c + col_off;
        const int64_t col =
            interleave < 0 ? j : (int64_t)256 * (j / 128) + 128 * interleave + (j % 128);
        *reinterpret_cast<uint4*>(dst + r * ld_dst + col) =
            *reinterpret_cast<const uint4*>(src + r * Cc + c);
    }
}

int grid_for(int64_t n, int threads, int cap) {
    int64_t b = (n + threads - 1) / threads;
    if (b < 1) b = 1;
    return (int)(b < cap ? b : cap);
}

}  // namespace

int launch_bwd_gather(const void* G, const float* y, int splits, int64_t split_stride,
                      const int32_t* slot_of, const float* gate, void* dY, float* dg, int64_t T,
                      int d, int k, int num_sms, cudaStream_t st) {
    const int grid = (int)(T < (int64_t)num_sms * 16 ? T : (int64_t)num_sms * 16);
    bwd_gather_kernel<<<grid, GATHER_THREADS, 0, st>>>(
        reinterpret_cast<const __nv_bfloat16*>(G), y, splits, split_stride, slot_of, gate,
        reinterpret_cast<__nv_bfloat16*>(dY), dg, T, d, k);
    note_launch();
    return launch_result();
}

int launch_router_bwd(const float* z, const float* bias, const int32_t* idx, const float* gate,
                      const float* dg, const int32_t* routed, float aux_coef, float* dz, int64_t T,
                      int E, int k, int num_sms, cudaStream_t st) {
    const int64_t blocks = (T + 7) / 8;
    const int grid = (int)(blocks < (int64_t)num_sms * 8 ? blocks : (int64_t)num_sms * 8);
    router_bwd_kernel<<<grid, 256, 0, st>>>(z, bias, idx, gate, dg, routed, aux_coef, dz, T, E, k);
    note_launch();
    return launch_result();
}

int wr_grad_chunks(int64_t T, int d, int E) {
    int64_t nch = (T + 255) / 256;
    if (nch > 64) nch = 64;
    const int64_t cap = (int64_t)(256u << 20) / ((int64_t)(d + 1) * E * 4);
    if (nch > cap) nch = cap;
    return (int)(nch < 1 ? 1 : nch);
}

int launch_wr_grad(const void* x, const float* dz, float* part, float* dWr, float* db, int64_t T,
                   int d, int E, cudaStream_t st) {
    const int nch = wr_grad_chunks(T, d, E);
    const int64_t chunk = ((T + nch - 1) / nch + WR_TT - 1) / WR_TT * WR_TT;
    dim3 grid((d + 1 + WR_THREADS - 1) / WR_THREADS, nch, (E + WR_ET - 1) / WR_ET);
    wr_grad_kernel<__nv_bfloat16><<<grid, WR_THREADS, 0, st>>>(
        reinterpret_cast<const __nv_bfloat16*>(x), dz, part, T, d, E, chunk);
    note_launch();
    if (launch_result() != 0) return -1;
    const int64_t n = (int64_t)(d + 1) * E;
    wr_reduce_kernel<<<grid_for(n, 256, 4096), 256, 0, st>>>(part, nch, (int64_t)d * E, E, dWr, db);
    note_launch();
    return launch_result();
}

int launch_dxr(const float* dz, const float* Wr, float* dxr, int64_t T, int d, int E,
               cudaStream_t st) {
    dim3 grid(d / DXR_CT, (unsigned)((T + DXR_TT - 1) / DXR_TT));
    dxr_kernel<<<grid, DXR_CT, 0, st>>>(dz, Wr, dxr, T, d, E);
    note_launch();
    return launch_result();
}

int launch_kofs(const int32_t* rows, int G, int32_t* kofs, cudaStream_t st) {
    kofs_kernel<<<1, 32, 0, st>>>(rows, G, kofs);
    note_launch();
    return launch_result();
}

int launch_transpose(const TransposeJobs& jobs, int64_t k_bound, cudaStream_t st) {
    int fmax = 0;
    for (int i = 0; i < jobs.n; ++i) fmax = jobs.job[i].features > fmax ? jobs.job[i].features : fmax;
    if (jobs.n == 0 || k_bound <= 0) return 0;
    dim3 grid((unsigned)((k_bound + TP - 1) / TP), (fmax + TP - 1) / TP, jobs.n);
    transpose_kernel<<<grid, 256, 0, st>>>(jobs);
    note_launch();
    return launch_result();
}

int launch_combine_bwd(const float* dXp, const int32_t* slot_of, const float* dXs,
                       const float* dXr, float* dx, int64_t T, int d, int k, int num_sms,
                       cudaStream_t st) {
    combine_bwd_kernel<<<grid_for(T * (d / 4), 256, num_sms * 16), 256, 0, st>>>(
        dXp, slot_of, dXs, dXr, dx, T, d, k);
    note_launch();
    return launch_result();
}

int launch_pack_cols(const void* src, void* dst, int R, int Cc, int64_t ld_dst, int col_off,
                     int interleave, int n, int64_t src_stride, int64_t dst_stride, int col_step,
                     cudaStream_t st) {
    dim3 grid(grid_for((int64_t)R * (Cc / 8), 256, 2048), n);
    pack_cols_kernel<<<grid, 256, 0, st>>>(reinterpret_cast<const uint16_t*>(src),
                                           reinterpret_cast<uint16_t*>(dst), R, Cc, ld_dst,
                                           col_off, interleave, src_stride, dst_stride, col_step);
    note_launch();
    return launch_result();
}

}  // namespace moe
