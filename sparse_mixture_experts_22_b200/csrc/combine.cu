// combine.cu -- gate-weighted combine, routing statistics and weight packing.
//
// Combine [Mixtral 8x7B and MoE explained, "Easy explanation" ¶3: the chosen
// experts' outputs are summed with the gate weights; "Mixture of experts"
// wiki, "How it works": weighted by the router's confidence; MoE routing
// fully explained, "Easy explanation" ¶4: shared experts see every token]:
//   out[t] = sum_j g[t,j] * (sum_s y[s][slot(t,j)]) + y_shared[t]
// with j and s in fixed order, fp32, one thread per 8 output columns (two
// 16-byte loads per row read, one 16-byte bf16x8 store).  A dropped
// assignment contributes nothing and the other gates are not renormalised.
//
// Statistics [MoE routing fully explained, "Easy explanation" ¶4, "Main
// insights" ¶3]: the load-balancing loss E * sum_e f_e P_e, the overflow
// rate and the mean router entropy, reduced from the per-block partials in a
// fixed order in fp64.
#include <string.h>

#include "common.cuh"
#include "kernels.h"
#include "plan.h"

namespace moe {

namespace {

__device__ void finalize_stats(const double* sums, int E, int k, moe_stats* st) {
    const double T = sums[0];
    moe_stats r{0.0, 0.0, 0.0, T, 0.0};
    if (T > 0.0) {
        const double tk = T * k;
        double aux = 0.0, dropped = 0.0;
        for (int e = 0; e < E; ++e) {
            const double f = sums[2 + E + e] / tk;  // share of assignments (before the limit)
            const double P = sums[2 + e] / T;       // mean router probability
            aux += f * P;
            dropped += sums[2 + E + e] - sums[2 + 2 * E + e];
        }
        r.aux_loss = (double)E * aux;
        r.overflow_rate = dropped / tk;
        r.mean_entropy = sums[1] / T;
        r.dropped = dropped;
    }
    *st = r;
}

// sums = [T, entropy sum, P sums (E), routed (E), kept (E)], each a fixed-order
// fp64 reduction of the router's per-block partials; then the statistics.
// Run by one block of any size.
__device__ __noinline__ void stats_block(const StatsParams& a) {
    const float* ppart = a.ppart;
    const float* hpart = a.hpart;
    const int nblk = a.nblk, E = a.E, k = a.k;
    const int32_t* routed = a.routed;
    const int32_t* kept = a.kept;
    const int64_t T = a.T;
    double* sums = a.sums;
    moe_stats* st = reinterpret_cast<moe_stats*>(a.stats);
    const int tid = threadIdx.x;
    if (tid == 0) {
        double h = 0.0;
        for (int b = 0; b < nblk; ++b) h += (double)hpart[b];
        sums[0] = (double)T;
        sums[1] = h;
    }
    for (int e = tid; e < E; e += blockDim.x) {
        double p = 0.0;
        for (int b = 0; b < nblk; ++b) p += (double)ppart[(int64_t)b * E + e];
        sums[2 + e] = p;
        sums[2 + E + e] = T > 0 ? (double)routed[e] : 0.0;
        sums[2 + 2 * E + e] = T > 0 ? (double)kept[e] : 0.0;
    }
    if (!st) return;
    __syncthreads();
    if (tid == 0) finalize_stats(sums, E, k, st);
}

__global__ void stats_kernel(StatsParams a) { stats_block(a); }

// The last block of the grid computes the statistics instead when
// sp.sums is set (they need only the router partials and the counts).
// KMAX >= k bounds the per-thread arrays: sized for the config's k, the
// kernel keeps few registers and many threads (so many row loads) in flight.
template <bool OUT_BF16, int KMAX>
__global__ void __launch_bounds__(256)
    combine_kernel(const float* __restrict__ y, int splits, int64_t split_stride,
                   const int32_t* __restrict__ slot_of, const float* __restrict__ gate,
                   const float* __restrict__ ys, void* __restrict__ out, int64_t T, int d, int k,
                   StatsParams sp) {
    pdl_wait();
    if (sp.sums && blockIdx.x == gridDim.x - 1) {
        stats_block(sp);
        return;
    }
    const int vecs = d / 8;
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= T * vecs) return;
    const int64_t t = i / vecs;
    const int c = (int)(i % vecs) * 8;
    // all slots and gates first, so that every row load below is independent
    int32_t slot[KMAX];
    float g[KMAX];
#pragma unroll
    for (int j = 0; j < KMAX; ++j) {
        slot[j] = j < k ? slot_of[t * k + j] : -1;
        g[j] = j < k ? gate[t * k + j] : 0.f;
    }
    float acc[8];
#pragma unroll
    for (int q = 0; q < 8; ++q) acc[q] = 0.f;
    // the shared experts' row is requested together with the routed rows
    float4 sa = make_float4(0.f, 0.f, 0.f, 0.f), sb = sa;
    if (ys) {
        const float* p = ys + t * d + c;
        sa = __ldg(reinterpret_cast<const float4*>(p));
        sb = __ldg(reinterpret_cast<const float4*>(p + 4));
    }
    if (splits == 1) {
        // every kept row's 32 bytes are requested before any is used, so the
        // k loads of a thread are in flight together
        float4 ra[KMAX], rb[KMAX];
#pragma unroll
        for (int j = 0; j < KMAX; ++j) {
            ra[j] = make_float4(0.f, 0.f, 0.f, 0.f);
            rb[j] = ra[j];
            if (slot[j] >= 0) {
                const float* p = y + (int64_t)slot[j] * d + c;
                ra[j] = __ldg(reinterpret_cast<const float4*>(p));
                rb[j] = __ldg(reinterpret_cast<const float4*>(p + 4));
            }
        }
#pragma unroll
        for (int j = 0; j < KMAX; ++j) {
            if (slot[j] < 0) continue;
            acc[0] = fmaf(g[j], ra[j].x, acc[0]);
            acc[1] = fmaf(g[j], ra[j].y, acc[1]);
            acc[2] = fmaf(g[j], ra[j].z, acc[2]);
            acc[3] = fmaf(g[j], ra[j].w, acc[3]);
            acc[4] = fmaf(g[j], rb[j].x, acc[4]);
            acc[5] = fmaf(g[j], rb[j].y, acc[5]);
            acc[6] = fmaf(g[j], rb[j].z, acc[6]);
            acc[7] = fmaf(g[j], rb[j].w, acc[7]);
        }
    }
#pragma unroll
    for (int j = 0; j < KMAX; ++j) {
        if (splits == 1 || slot[j] < 0) continue;
        float v[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) v[q] = 0.f;
        for (int s = 0; s < splits; ++s) {
            const float* p = y + s * split_stride + (int64_t)slot[j] * d + c;
            const float4 a = __ldg(reinterpret_cast<const float4*>(p));
            const float4 b = __ldg(reinterpret_cast<const float4*>(p + 4));
            v[0] += a.x; v[1] += a.y; v[2] += a.z; v[3] += a.w;
            v[4] += b.x; v[5] += b.y; v[6] += b.z; v[7] += b.w;
        }
#pragma unroll
        for (int q = 0; q < 8; ++q) acc[q] = fmaf(g[j], v[q], acc[q]);
    }
    if (ys) {
        acc[0] += sa.x; acc[1] += sa.y; acc[2] += sa.z; acc[3] += sa.w;
        acc[4] += sb.x; acc[5] += sb.y; acc[6] += sb.z; acc[7] += sb.w;
    }
    if (OUT_BF16) {
        uint4 o;
        o.x = pack_bf16x2(acc[0], acc[1]);
        o.y = pack_bf16x2(acc[2], acc[3]);
        o.z = pack_bf16x2(acc[4], acc[5]);
        o.w = pack_bf16x2(acc[6], acc[7]);
        *reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(out) + t * d + c) = o;
    } else {
        float* p = reinterpret_cast<float*>(out) + t * d + c;
        *reinterpret_cast<float4*>(p) = make_float4(acc[0], acc[1], acc[2], acc[3]);
        *reinterpret_cast<float4*>(p + 4) = make_float4(acc[4], acc[5], acc[6], acc[7]);
    }
}

// k <= 2, one partial per row, d % 16 == 0: 16 columns per thread, so that each
// thread keeps twice the row bytes in flight (same arithmetic order as
// combine_kernel; the large layer's combine: 168 -> 144 us).
template <bool OUT_BF16>
__global__ void __launch_bounds__(256)
    combine16_kernel(const float* __restrict__ y, const int32_t* __restrict__ slot_of,
                     const float* __restrict__ gate, const float* __restrict__ ys,
                     void* __restrict__ out, int64_t T, int d, int k, StatsParams sp) {
    pdl_wait();
    if (sp.sums && blockIdx.x == gridDim.x - 1) {
        stats_block(sp);
        return;
    }
    const int vecs = d / 16;
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= T * vecs) return;
    const int64_t t = i / vecs;
    const int c = (int)(i % vecs) * 16;
    int32_t slot[2];
    float g[2];
#pragma unroll
    for (int j = 0; j < 2; ++j) {
        slot[j] = j < k ? slot_of[t * k + j] : -1;
        g[j] = j < k ? gate[t * k + j] : 0.f;
    }
    float4 sv[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) sv[q] = make_float4(0.f, 0.f, 0.f, 0.f);
    if (ys) {
        const float4* p = reinterpret_cast<const float4*>(ys + t * d + c);
#pragma unroll
        for (int q = 0; q < 4; ++q) sv[q] = __ldg(p + q);
    }
    float4 r[2][4];
#pragma unroll
    for (int j = 0; j < 2; ++j) {
#pragma unroll
        for (int q = 0; q < 4; ++q) r[j][q] = make_float4(0.f, 0.f, 0.f, 0.f);
        if (slot[j] >= 0) {
            const float4* p = reinterpret_cast<const float4*>(y + (int64_t)slot[j] * d + c);
#pragma unroll
            for (int q = 0; q < 4; ++q) r[j][q] = __ldg(p + q);
        }
    }
    float acc[16];
#pragma unroll
    for (int q = 0; q < 16; ++q) acc[q] = 0.f;
#pragma unroll
    for (int j = 0; j < 2; ++j) {
        if (slot[j] < 0) continue;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            acc[4 * q + 0] = fmaf(g[j], r[j][q].x, acc[4 * q + 0]);
            acc[4 * q + 1] = fmaf(g[j], r[j][q].y, acc[4 * q + 1]);
            acc[4 * q + 2] = fmaf(g[j], r[j][q].z, acc[4 * q + 2]);
            acc[4 * q + 3] = fmaf(g[j], r[j][q].w, acc[4 * q + 3]);
        }
    }
    if (ys) {
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            acc[4 * q + 0] += sv[q].x;
            acc[4 * q + 1] += sv[q].y;
            acc[4 * q + 2] += sv[q].z;
            acc[4 * q + 3] += sv[q].w;
        }
    }
    if (OUT_BF16) {
        uint4 o0, o1;
        o0.x = pack_bf16x2(acc[0], acc[1]);
        o0.y = pack_bf16x2(acc[2], acc[3]);
        o0.z = pack_bf16x2(acc[4], acc[5]);
        o0.w = pack_bf16x2(acc[6], acc[7]);
        o1.x = pack_bf16x2(acc[8], acc[9]);
        o1.y = pack_bf16x2(acc[10], acc[11]);
        o1.z = pack_bf16x2(acc[12], acc[13]);
        o1.w = pack_bf16x2(acc[14], acc[15]);
        uint4* o = reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(out) + t * d + c);
        o[0] = o0;
        o[1] = o1;
    } else {
        float4* o = reinterpret_cast<float4*>(reinterpret_cast<float*>(out) + t * d + c);
#pragma unroll
        for (int q = 0; q < 4; ++q)
            o[q] = make_float4(acc[4 * q], acc[4 * q + 1], acc[4 * q + 2], acc[4 * q + 3]);
    }
}

// Destinations of the expert-parallel combine: y row bases of the owners.
struct PeerY {
    const float* base[MAX_PEERS];
    const int32_t* start;  // device [npeer] rows to skip at each owner, or null
    int npeer, e_loc;
};

// The combine with the expert outputs at their owners (expert parallelism):
// the row of (t, j) is read from the owner of expert topk_idx[t][j], in this
// GPU's memory or a peer's (NVLink loads), at its position in the segments
// this rank sent there.  Same arithmetic and order as combine_kernel.
template <bool OUT_BF16>
__global__ void __launch_bounds__(256)
    combine_peers_kernel(PeerY py, const int32_t* __restrict__ topk_idx,
                         const int32_t* __restrict__ offsets,
                         const int32_t* __restrict__ slot_of, const float* __restrict__ gate,
                         const float* __restrict__ ys, void* __restrict__ out, int64_t T, int d,
                         int k) {
    __shared__ const float* sbase[MAX_PEERS];
    __shared__ int32_t sfirst[MAX_PEERS];  // first slot of each owner's segments
    if (threadIdx.x == 0) {
#pragma unroll
        for (int i = 0; i < MAX_PEERS; ++i)
            if (i < py.npeer) sbase[i] = py.base[i];
    }
    // row of slot s at owner o: s - offsets[o * e_loc] + start[o]
    if (threadIdx.x < py.npeer)
        sfirst[threadIdx.x] = offsets[threadIdx.x * py.e_loc] -
                              (py.start ? py.start[threadIdx.x] : 0);
    __syncthreads();
    const int vecs = d / 8;
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= T * vecs) return;
    const int64_t t = i / vecs;
    const int c = (int)(i % vecs) * 8;
    float acc[8];
#pragma unroll
    for (int q = 0; q < 8; ++q) acc[q] = 0.f;
    // every kept row is requested before any is used
    float4 ra[MAX_K], rb[MAX_K];
    float g[MAX_K];
    bool kept[MAX_K];
#pragma unroll
    for (int j = 0; j < MAX_K; ++j) {
        ra[j] = make_float4(0.f, 0.f, 0.f, 0.f);
        rb[j] = ra[j];
        g[j] = 0.f;
        const int32_t slot = j < k ? slot_of[t * k + j] : -1;
        kept[j] = slot >= 0;
        if (kept[j]) {
            const int o = topk_idx[t * k + j] / py.e_loc;
            const float* p = sbase[o] + (int64_t)(slot - sfirst[o]) * d + c;
            ra[j] = *reinterpret_cast<const float4*>(p);
            rb[j] = *reinterpret_cast<const float4*>(p + 4);
            g[j] = gate[t * k + j];
        }
    }
#pragma unroll
    for (int j = 0; j < MAX_K; ++j) {
        if (!kept[j]) continue;
        acc[0] = fmaf(g[j], ra[j].x, acc[0]);
        acc[1] = fmaf(g[j], ra[j].y, acc[1]);
        acc[2] = fmaf(g[j], ra[j].z, acc[2]);
        acc[3] = fmaf(g[j], ra[j].w, acc[3]);
        acc[4] = fmaf(g[j], rb[j].x, acc[4]);
        acc[5] = fmaf(g[j], rb[j].y, acc[5]);
        acc[6] = fmaf(g[j], rb[j].z, acc[6]);
        acc[7] = fmaf(g[j], rb[j].w, acc[7]);
    }
    if (ys) {
        const float* p = ys + t * d + c;
        const float4 a = *reinterpret_cast<const float4*>(p);
        const float4 b = *reinterpret_cast<const float4*>(p + 4);
        acc[0] += a.x; acc[1] += a.y; acc[2] += a.z; acc[3] += a.w;
        acc[4] += b.x; acc[5] += b.y; acc[6] += b.z; acc[7] += b.w;
    }
    if (OUT_BF16) {
        uint4 o;
        o.x = pack_bf16x2(acc[0], acc[1]);
        o.y = pack_bf16x2(acc[2], acc[3]);
        o.z = pack_bf16x2(acc[4], acc[5]);
        o.w = pack_bf16x2(acc[6], acc[7]);
        *reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(out) + t * d + c) = o;
    } else {
        float* p = reinterpret_cast<float*>(out) + t * d + c;
        *reinterpret_cast<float4*>(p) = make_float4(acc[0], acc[1], acc[2], acc[3]);
        *reinterpret_cast<float4*>(p + 4) = make_float4(acc[4], acc[5], acc[6], acc[7]);
    }
}

__global__ void stats_finalize_kernel(const double* __restrict__ sums, int E, int k,
                                      moe_stats* __restrict__ st) {
    if (threadIdx.x == 0) finalize_stats(sums, E, k, st);
}

// Tiled transpose with a row remap for the packed weight layouts.
// src [R][Cc]; dst[row(c)][r + 0] with row(c) = c + col_off, or, when
// interleave >= 0, the gate/up interleave of 128-wide hidden blocks:
// hidden index j = c + col_off -> row 256 * (j / 128) + 128 * interleave + j % 128.
template <typename Tv>
__global__ void pack_kernel(const Tv* __restrict__ src, Tv* __restrict__ dst, int R, int Cc,
                            int64_t ld_dst, int col_off, int interleave, int64_t src_stride,
                            int64_t dst_stride, int col_step) {
    __shared__ Tv tile[32][33];
    src += blockIdx.z * src_stride;
    dst += blockIdx.z * dst_stride;
    col_off += blockIdx.z * col_step;
    const int r0 = blockIdx.y * 32, c0 = blockIdx.x * 32;
    for (int i = threadIdx.y; i < 32; i += blockDim.y) {
        const int r = r0 + i, c = c0 + threadIdx.x;
        if (r < R && c < Cc) tile[i][threadIdx.x] = src[(int64_t)r * Cc + c];
    }
    __syncthreads();
    for (int i = threadIdx.y; i < 32; i += blockDim.y) {
        const int c = c0 + i, r = r0 + threadIdx.x;
        if (r < R && c < Cc) {
            const int j = c + col_off;
            const int64_t row =
                interleave < 0 ? j : (int64_t)256 * (j / 128) + 128 * interleave + (j % 128);
            dst[row * ld_dst + r] = tile[threadIdx.x][i];
        }
    }
}

}  // namespace

int launch_combine(const float* y, int splits, int64_t split_stride, const int32_t* slot_of,
                   const float* gate, const float* y_shared, void* out, bool out_bf16, int64_t T,
                   int d, int k, const StatsParams* sp, cudaStream_t st) {
    if (T == 0) return sp ? launch_stats(*sp, st) : 0;
    const int64_t n = T * (d / 8);
    StatsParams none;
    memset(&none, 0, sizeof none);
    const StatsParams& s = sp ? *sp : none;
    const unsigned blocks = (unsigned)((n + 255) / 256) + (sp ? 1 : 0);
    auto go = [&](auto kern) {
        launch_ex(pdl_active(), kern, dim3(blocks), dim3(256), 0, st, y, splits, split_stride,
                  slot_of, gate, y_shared, out, T, d, k, s);
    };
    if (k <= 2 && splits == 1 && d % 16 == 0) {
        const int64_t n16 = T * (d / 16);
        const unsigned b16 = (unsigned)((n16 + 255) / 256) + (sp ? 1 : 0);
        auto kern = out_bf16 ? combine16_kernel<true> : combine16_kernel<false>;
        launch_ex(pdl_active(), kern, dim3(b16), dim3(256), 0, st, y, slot_of, gate, y_shared,
                  out, T, d, k, s);
    } else if (k <= 2) {
        out_bf16 ? go(combine_kernel<true, 2>) : go(combine_kernel<false, 2>);
    }
    else if (k <= 4)
        out_bf16 ? go(combine_kernel<true, 4>) : go(combine_kernel<false, 4>);
    else
        out_bf16 ? go(combine_kernel<true, MAX_K>) : go(combine_kernel<false, MAX_K>);
    note_launch();
    return launch_result();
}

int launch_combine_peers(const float* const* y_rows, const int32_t* y_start, int npeer,
                         int e_loc, const int32_t* topk_idx, const int32_t* offsets,
                         const int32_t* slot_of, const float* gate, const float* y_shared,
                         void* out, bool out_bf16, int64_t T, int d, int k, cudaStream_t st) {
    if (T == 0) return 0;
    if (npeer < 1 || npeer > MAX_PEERS || e_loc < 1) return -1;
    PeerY py;
    for (int i = 0; i < MAX_PEERS; ++i) py.base[i] = i < npeer ? y_rows[i] : nullptr;
    py.npeer = npeer;
    py.e_loc = e_loc;
    py.start = y_start;
    const int64_t n = T * (d / 8);
    const unsigned blocks = (unsigned)((n + 255) / 256);
    if (out_bf16)
        combine_peers_kernel<true><<<blocks, 256, 0, st>>>(py, topk_idx, offsets, slot_of, gate,
                                                          y_shared, out, T, d, k);
    else
        combine_peers_kernel<false><<<blocks, 256, 0, st>>>(py, topk_idx, offsets, slot_of, gate,
                                                           y_shared, out, T, d, k);
    note_launch();
    return launch_result();
}

int launch_stats(const StatsParams& a, cudaStream_t st) {
    stats_kernel<<<1, 256, 0, st>>>(a);
    note_launch();
    return launch_result();
}

int launch_stats_finalize(const double* sums, int E, int k, void* stats, cudaStream_t st) {
    stats_finalize_kernel<<<1, 32, 0, st>>>(sums, E, k, reinterpret_cast<moe_stats*>(stats));
    note_launch();
    return launch_result();
}

int launch_pack(const void* src, void* dst, int elem_bytes, int R, int Cc, int64_t ld_dst,
                int col_off, int interleave, int n, int64_t src_stride, int64_t dst_stride,
                int col_step, cudaStream_t st) {
    dim3 grid((Cc + 31) / 32, (R + 31) / 32, n), block(32, 8);
    if (elem_bytes == 2)
        pack_kernel<uint16_t><<<grid, block, 0, st>>>(
            reinterpret_cast<const uint16_t*>(src), reinterpret_cast<uint16_t*>(dst), R, Cc,
            ld_dst, col_off, interleave, src_stride, dst_stride, col_step);
    else
        pack_kernel<float><<<grid, block, 0, st>>>(
            reinterpret_cast<const float*>(src), reinterpret_cast<float*>(dst), R, Cc, ld_dst,
            col_off, interleave, src_stride, dst_stride, col_step);
    note_launch();
    return launch_result();
}

}  // namespace moe
