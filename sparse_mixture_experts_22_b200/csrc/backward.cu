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
//   zero_pad   zeros in the rows between an expert's last token and the next
//              multiple of 64 (the weight-gradient GEMMs read whole 64-row
//              blocks of the row-major activations as MN-major operands)
//   combine    dx_t = sum over kept slots of dXp + shared dX + dz_t Wr^T
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
constexpr int WR_TT = 32;   // tokens staged per step

// part[ch][c][e] = sum over the chunk's tokens of x[t][c] dz[t][e]; row c == d
// holds the column sums of dz (the bias gradient).  A thread owns CV
// consecutive columns (one vector load of x per token) and ET experts.
template <int CV, int ET>
__global__ void __launch_bounds__(WR_THREADS)
    wr_grad_kernel(const __nv_bfloat16* __restrict__ x, const float* __restrict__ dz,
                   float* __restrict__ part, int64_t T, int d, int E, int64_t chunk) {
    __shared__ float dzs[WR_TT][ET];
    const int c0 = (blockIdx.x * WR_THREADS + threadIdx.x) * CV;
    const int e0 = blockIdx.z * ET;
    const int ne = min(ET, E - e0);
    const int64_t t0 = (int64_t)blockIdx.y * chunk;
    const int64_t t1 = min(T, t0 + chunk);
    const bool ones = c0 == d;  // the bias row
    float acc[CV][ET];
#pragma unroll
    for (int i = 0; i < CV; ++i)
#pragma unroll
        for (int j = 0; j < ET; ++j) acc[i][j] = 0.0f;
    for (int64_t tb = t0; tb < t1; tb += WR_TT) {
        __syncthreads();
        for (int i = threadIdx.x; i < WR_TT * ET; i += WR_THREADS) {
            const int tt = i / ET, ee = i % ET;
            dzs[tt][ee] = (tb + tt < t1 && ee < ne) ? dz[(tb + tt) * E + e0 + ee] : 0.0f;
        }
        __syncthreads();
        if (c0 <= d) {
            const int nt = (int)min((int64_t)WR_TT, t1 - tb);
            for (int tt = 0; tt < nt; ++tt) {
                float xv[CV];
                if (!ones) {
                    const __nv_bfloat16* px = x + (tb + tt) * d + c0;
                    if (CV == 8) {
                        load_bf16x8(px, xv);
                    } else {
#pragma unroll
                        for (int i = 0; i < CV; ++i) xv[i] = __bfloat162float(px[i]);
                    }
                } else {
#pragma unroll
                    for (int i = 0; i < CV; ++i) xv[i] = i == 0 ? 1.0f : 0.0f;
                }
#pragma unroll
                for (int j = 0; j < ET; ++j) {
                    const float z = dzs[tt][j];
#pragma unroll
                    for (int i = 0; i < CV; ++i) acc[i][j] += xv[i] * z;
                }
            }
        }
    }
    if (c0 <= d) {
        const int nrow = ones ? 1 : CV;
#pragma unroll
        for (int i = 0; i < CV; ++i) {
            if (i >= nrow) break;
            float* dst = part + ((int64_t)blockIdx.y * (d + 1) + c0 + i) * E + e0;
#pragma unroll
            for (int j = 0; j < ET; ++j)
                if (j < ne) dst[j] = acc[i][j];
        }
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

// ---------------------------------------------------------------- padding rows

// Zeroes rows [off[g] + rows[g], off[g] + rows[g] rounded up to 64) of each
// bf16 buffer: the weight-gradient GEMMs contract whole 64-row blocks of every
// expert segment, so the rows past an expert's tokens must hold zeros.
__global__ void __launch_bounds__(256) zero_pad_kernel(PadJobs p) {
    const int g = blockIdx.x;
    const PadJob& jb = p.job[blockIdx.y];
    const int32_t n = p.rows[g];
    const int64_t r0 = (int64_t)p.off[g] + n;
    const int64_t r1 = (int64_t)p.off[g] + (n + 63) / 64 * 64;
    const int w8 = jb.width / 8;
    const int64_t total = (r1 - r0) * w8;
    uint4* base = reinterpret_cast<uint4*>(jb.buf);
    for (int64_t i = (int64_t)blockIdx.z * blockDim.x + threadIdx.x; i < total;
         i += (int64_t)gridDim.z * blockDim.x) {
        const int64_t row = r0 + i / w8;
        base[row * w8 + i % w8] = make_uint4(0, 0, 0, 0);
    }
}

// ---------------------------------------------------------------- dx

// The router's share of dx is dz_t Wr^T, a product with K = E.  Up to
// E = 16 a thread keeps Wr's rows for its four columns in registers and the
// share is formed inside the combine; for more experts it is a tiled product
// of its own (dxr), which the combine then adds.

constexpr int CB_TOK = 64;   // tokens per block of the combine

// dx[t][c..c+3] = sum_j dXp[slot_of[t][j]][c..] (kept slots, j order)
//               + dXs[t][c..] + (EREG ? sum_e dz[t][e] Wr[c..][e] : dxr[t][c..])
template <int EREG>
__global__ void __launch_bounds__(256)
    combine_bwd_kernel(const float* __restrict__ dXp, const int32_t* __restrict__ slot_of,
                       const float* __restrict__ dXs, const float* __restrict__ dz,
                       const float* __restrict__ Wr, const float* __restrict__ dxr,
                       float* __restrict__ dx, int64_t T, int d, int k, int E) {
    constexpr int ER = EREG > 0 ? EREG : 1;
    __shared__ float zs[CB_TOK][ER];
    __shared__ int32_t slots[CB_TOK][8];
    const int64_t t0 = (int64_t)blockIdx.y * CB_TOK;
    const int c = (blockIdx.x * 256 + threadIdx.x) * 4;
    for (int i = threadIdx.x; i < CB_TOK * 8; i += 256) {
        const int tt = i / 8, j = i % 8;
        slots[tt][j] = (t0 + tt < T && j < k) ? slot_of[(t0 + tt) * k + j] : -1;
    }
    float w[4][EREG > 0 ? EREG : 1];
    if (EREG > 0) {
        for (int i = threadIdx.x; i < CB_TOK * ER; i += 256) {
            const int tt = i / ER, e = i % ER;
            zs[tt][e] = (t0 + tt < T && e < E) ? dz[(t0 + tt) * E + e] : 0.0f;
        }
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int e = 0; e < (EREG > 0 ? EREG : 1); ++e)
                w[i][e] = (c < d && e < E) ? Wr[(int64_t)(c + i) * E + e] : 0.0f;
    }
    __syncthreads();
    if (c >= d) return;
    const int nt = (int)min((int64_t)CB_TOK, T - t0);
    for (int tt = 0; tt < nt; ++tt) {
        const int64_t t = t0 + tt;
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int j = 0; j < k; ++j) {
            const int32_t r = slots[tt][j];
            if (r < 0) continue;
            const float4 v = *reinterpret_cast<const float4*>(dXp + (int64_t)r * d + c);
            acc.x += v.x; acc.y += v.y; acc.z += v.z; acc.w += v.w;
        }
        if (dXs) {
            const float4 v = *reinterpret_cast<const float4*>(dXs + t * d + c);
            acc.x += v.x; acc.y += v.y; acc.z += v.z; acc.w += v.w;
        }
        if (EREG > 0) {
            float r[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int e = 0; e < (EREG > 0 ? EREG : 1); ++e) {
                const float z = zs[tt][e];
#pragma unroll
                for (int i = 0; i < 4; ++i) r[i] += z * w[i][e];
            }
            acc.x += r[0]; acc.y += r[1]; acc.z += r[2]; acc.w += r[3];
        } else {
            const float4 v = *reinterpret_cast<const float4*>(dxr + t * d + c);
            acc.x += v.x; acc.y += v.y; acc.z += v.z; acc.w += v.w;
        }
        *reinterpret_cast<float4*>(dx + t * d + c) = acc;
    }
}

constexpr int DXR_TT = 32;   // tokens per block
constexpr int DXR_CT = 128;  // model columns per block (one per thread)
constexpr int DXR_EK = 32;   // experts staged per step

// dxr[t][c] = sum_e dz[t][e] Wr[c][e], tiled over e through shared memory
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
            const float wv = ws[tid][ee];
#pragma unroll
            for (int tt = 0; tt < DXR_TT; ++tt) acc[tt] += zs[tt][ee] * wv;
        }
    }
#pragma unroll
    for (int tt = 0; tt < DXR_TT; ++tt)
        if (t0 + tt < T) dxr[(t0 + tt) * d + c0 + tid] = acc[tt];
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
    const __nv_bfloat16* xb = reinterpret_cast<const __nv_bfloat16*>(x);
    if (E <= 8) {
        // one extra thread (column d) computes the bias row
        dim3 grid((d + 8 + WR_THREADS * 8 - 1) / (WR_THREADS * 8), nch, 1);
        wr_grad_kernel<8, 8><<<grid, WR_THREADS, 0, st>>>(xb, dz, part, T, d, E, chunk);
    } else {
        dim3 grid((d + 4 + WR_THREADS * 4 - 1) / (WR_THREADS * 4), nch, (E + 15) / 16);
        wr_grad_kernel<4, 16><<<grid, WR_THREADS, 0, st>>>(xb, dz, part, T, d, E, chunk);
    }
    note_launch();
    if (launch_result() != 0) return -1;
    const int64_t n = (int64_t)(d + 1) * E;
    wr_reduce_kernel<<<grid_for(n, 256, 4096), 256, 0, st>>>(part, nch, (int64_t)d * E, E, dWr, db);
    note_launch();
    return launch_result();
}

int launch_zero_pad(const PadJobs& p, cudaStream_t st) {
    if (p.n == 0 || p.groups == 0) return 0;
    // blocks per (segment, buffer): enough for the widest buffer's 63 padding
    // rows, but about 1200 blocks over the whole launch
    int wmax = 0;
    for (int i = 0; i < p.n; ++i) wmax = p.job[i].width > wmax ? p.job[i].width : wmax;
    const int per = (int)(((int64_t)63 * (wmax / 8) + 255) / 256);
    const int share = 1200 / (p.groups * p.n);
    int z = per < share ? per : share;
    z = z < 1 ? 1 : (z > 64 ? 64 : z);
    zero_pad_kernel<<<dim3(p.groups, p.n, z), 256, 0, st>>>(p);
    note_launch();
    return launch_result();
}

int launch_combine_bwd(const float* dXp, const int32_t* slot_of, const float* dXs,
                       const float* dz, const float* Wr, float* dxr, float* dx, int64_t T, int d,
                       int k, int E, cudaStream_t st) {
    dim3 grid((d / 4 + 255) / 256, (unsigned)((T + CB_TOK - 1) / CB_TOK));
    if (E <= 8) {
        combine_bwd_kernel<8><<<grid, 256, 0, st>>>(dXp, slot_of, dXs, dz, Wr, nullptr, dx, T, d,
                                                    k, E);
        note_launch();
        return launch_result();
    }
    if (E <= 16) {
        combine_bwd_kernel<16><<<grid, 256, 0, st>>>(dXp, slot_of, dXs, dz, Wr, nullptr, dx, T,
                                                     d, k, E);
        note_launch();
        return launch_result();
    }
    dim3 gr(d / DXR_CT, (unsigned)((T + DXR_TT - 1) / DXR_TT));
    dxr_kernel<<<gr, DXR_CT, 0, st>>>(dz, Wr, dxr, T, d, E);
    note_launch();
    if (launch_result() != 0) return -1;
    combine_bwd_kernel<0><<<grid, 256, 0, st>>>(dXp, slot_of, dXs, dz, Wr, dxr, dx, T, d, k, E);
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
