// gemm_f32.cu -- expert FFN in fp32 on the CUDA cores, for fp32 layers.
//
// The tensor cores have no fp32 multiply without TF32 rounding, which would
// not meet the fp32 tolerance, so fp32 configurations run the same grouped
// gate/up and down products (see gemm_tc.cu for the bf16 path) as plain
// fp32 dot products with 16x16 shared-memory tiles.  Same packed weight
// layout, same expert segments, fp32 H.
#include <math.h>

#include "common.cuh"
#include "kernels.h"

namespace moe {

namespace {

constexpr int TILE = 16;

__device__ __forceinline__ int group_of_row(int64_t r, int groups, const int32_t* rows,
                                            const int32_t* off, int dense_rows, int64_t* first) {
    if (!rows) {
        *first = 0;
        return r < dense_rows ? 0 : -1;
    }
    int lo = 0, hi = groups - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (off[mid] <= r) lo = mid; else hi = mid - 1;
    }
    if (r < off[lo] || r >= (int64_t)off[lo] + rows[lo]) return -1;
    *first = off[lo];
    return lo;
}

// One thread per output (r, f).  A 16 x 16 tile of activation rows is staged
// in shared memory per K step; the rows of one tile may belong to different
// groups, so each thread reads its own group's weight row from global memory
// (L1-cached: the 16 threads of a tile column share it).
template <bool GATEUP>
__global__ void __launch_bounds__(TILE * TILE)
    f32_ffn_kernel(const float* __restrict__ A, const float* __restrict__ W, float* __restrict__ O,
                   int groups, const int32_t* __restrict__ rows, const int32_t* __restrict__ off,
                   int dense_rows, int64_t rows_bound, int K, int nout, int64_t w_rows_per_group) {
    __shared__ float As[TILE][TILE + 1];
    const int tx = threadIdx.x, ty = threadIdx.y;
    const int64_t r = (int64_t)blockIdx.y * TILE + ty;
    const int f = blockIdx.x * TILE + tx;
    int64_t first = 0;
    const int g = r < rows_bound ? group_of_row(r, groups, rows, off, dense_rows, &first) : -1;
    const bool live = g >= 0 && f < nout;
    int64_t wg = 0, wu = 0;
    if (live) {
        if (GATEUP) {
            wg = (int64_t)g * w_rows_per_group + 256 * (f / 128) + (f % 128);  // gate row
            wu = wg + 128;                                                       // up row
        } else {
            wg = (int64_t)g * w_rows_per_group + f;
        }
    }
    float a = 0.f, b = 0.f;
    for (int k0 = 0; k0 < K; k0 += TILE) {
        As[ty][tx] = (g >= 0 && k0 + tx < K) ? A[r * K + k0 + tx] : 0.f;
        __syncthreads();
        if (live) {
            const int kend = min(TILE, K - k0);
            for (int kk = 0; kk < kend; ++kk) {
                const float xv = As[ty][kk];
                a = fmaf(xv, W[wg * K + k0 + kk], a);
                if (GATEUP) b = fmaf(xv, W[wu * K + k0 + kk], b);
            }
        }
        __syncthreads();
    }
    if (live) O[r * nout + f] = GATEUP ? a / (1.0f + expf(-a)) * b : a;
}

}  // namespace

int launch_f32_gateup(const float* A, const float* W13, float* H, int num_groups,
                      const int32_t* group_rows, const int32_t* group_off, int dense_rows,
                      int64_t rows_bound, int d, int h, cudaStream_t st) {
    if (rows_bound == 0) return 0;
    dim3 grid((h + TILE - 1) / TILE, (unsigned)((rows_bound + TILE - 1) / TILE));
    f32_ffn_kernel<true><<<grid, dim3(TILE, TILE), 0, st>>>(
        A, W13, H, num_groups, group_rows, group_off, dense_rows, rows_bound, d, h, 2LL * h);
    note_launch();
    return launch_result();
}

int launch_f32_down(const float* H, const float* W2p, float* Y, int num_groups,
                    const int32_t* group_rows, const int32_t* group_off, int dense_rows,
                    int64_t rows_bound, int d, int h, cudaStream_t st) {
    if (rows_bound == 0) return 0;
    dim3 grid((d + TILE - 1) / TILE, (unsigned)((rows_bound + TILE - 1) / TILE));
    f32_ffn_kernel<false><<<grid, dim3(TILE, TILE), 0, st>>>(
        H, W2p, Y, num_groups, group_rows, group_off, dense_rows, rows_bound, h, d, (int64_t)d);
    note_launch();
    return launch_result();
}

}  // namespace moe
