// dispatch.cu -- capacity-limited dispatch of token rows to experts.
//
// [MoE routing fully explained, "Easy explanation" ¶3 and ¶5]: every expert
// takes at most C = ceil(T k cf / E) tokens per batch; the overflow is
// dropped.  The drop order is arrival order by token index: an expert's
// queue fills with its tokens in increasing t.  So the rank of assignment
// (t, j) in expert e is the number of earlier tokens that chose e, and it is
// kept if rank < C.  The rank is computed without atomics on the order:
//
//   1. topk_kernel left a histogram cnt[block][e] per 128-token block;
//   2. each CTA scans the histograms of the blocks before it (base[e]) and of
//      all blocks (routed[e]), then kept[e] = min(routed[e], C) and the
//      padded segment offsets of every expert;
//   3. inside the block, a warp ballot per expert gives each lane the number
//      of earlier lanes that chose the same expert, and per-warp counts give
//      the offset of each warp.
//
// The result is identical on every run.  Several CTAs may share one token
// block (grid.y); they repeat the cheap ranking and split the row copies
// into x_perm, so even a 32-token decode batch spreads its gather over many
// SMs.
#include "common.cuh"
#include "kernels.h"
#include "plan.h"

namespace moe {

namespace {

constexpr int DWARPS = ROUTE_BLOCK / 32;

__global__ void __launch_bounds__(ROUTE_BLOCK)
    dispatch_kernel(const int32_t* __restrict__ topk_idx, const int32_t* __restrict__ cnt,
                    int64_t T, int E, int k, int64_t C, int pad, int64_t perm_rows,
                    const uint4* __restrict__ x, int row_vecs, int32_t* __restrict__ routed_out,
                    int32_t* __restrict__ kept_out, int32_t* __restrict__ offsets_out,
                    int32_t* __restrict__ perm_token, int32_t* __restrict__ slot_of,
                    uint4* __restrict__ x_perm) {
    extern __shared__ int32_t sm[];
    int32_t* base = sm;                 // [E]  assignments to e in earlier blocks
    int32_t* tot = base + E;            // [E]  all assignments to e
    int32_t* off = tot + E;             // [E+1] padded segment starts
    int32_t* wcnt = off + E + 1;        // [DWARPS][E]
    int32_t* slots = wcnt + DWARPS * E; // [ROUTE_BLOCK * k]

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int blk = blockIdx.x;
    const int nblk = gridDim.x;

    for (int e = tid; e < E; e += ROUTE_BLOCK) {
        int32_t b = 0, a = 0;
        for (int q = 0; q < nblk; ++q) {
            const int32_t c = cnt[(int64_t)q * E + e];
            if (q < blk) b += c;
            a += c;
        }
        base[e] = b;
        tot[e] = a;
    }
    __syncthreads();
    if (tid == 0) {
        int32_t o = 0;
        for (int e = 0; e < E; ++e) {
            off[e] = o;
            const int32_t kept = (int64_t)tot[e] < C ? tot[e] : (int32_t)C;
            o += (kept + pad - 1) / pad * pad;
        }
        off[E] = o;
    }
    __syncthreads();
    const bool writer = blockIdx.y == 0;
    if (writer) {
        if (blk == 0) {
            for (int e = tid; e < E; e += ROUTE_BLOCK) {
                routed_out[e] = tot[e];
                kept_out[e] = (int64_t)tot[e] < C ? tot[e] : (int32_t)C;
            }
            for (int e = tid; e <= E; e += ROUTE_BLOCK) offsets_out[e] = off[e];
        }
        if (perm_token) {
            // padding rows of each expert segment, and the unused tail, hold -1
            for (int e = blk; e < E; e += nblk) {
                const int32_t kept = (int64_t)tot[e] < C ? tot[e] : (int32_t)C;
                for (int r = off[e] + kept + tid; r < off[e + 1]; r += ROUTE_BLOCK) perm_token[r] = -1;
            }
            for (int64_t r = off[E] + (int64_t)blk * ROUTE_BLOCK + tid; r < perm_rows;
                 r += (int64_t)nblk * ROUTE_BLOCK)
                perm_token[r] = -1;
        }
    }

    // ranks inside the block
    const int64_t t = (int64_t)blk * ROUTE_BLOCK + tid;
    const bool valid = t < T;
    int32_t my[MAX_K];
    int32_t rank_w[MAX_K];
#pragma unroll
    for (int j = 0; j < MAX_K; ++j) {
        my[j] = (valid && j < k) ? topk_idx[t * k + j] : -1;
        rank_w[j] = 0;
    }
    const unsigned lt = (1u << lane) - 1u;
    for (int e = 0; e < E; ++e) {
        bool chose = false;
#pragma unroll
        for (int j = 0; j < MAX_K; ++j) chose |= (my[j] == e);
        const unsigned m = __ballot_sync(0xffffffffu, chose);
        if (lane == 0) wcnt[warp * E + e] = __popc(m);
        if (chose) {
            const int r = __popc(m & lt);
#pragma unroll
            for (int j = 0; j < MAX_K; ++j)
                if (my[j] == e) rank_w[j] = r;
        }
    }
    __syncthreads();
#pragma unroll
    for (int j = 0; j < MAX_K; ++j) {
        if (j >= k) break;
        int32_t slot = -1;
        if (valid) {
            const int e = my[j];
            int32_t r = base[e] + rank_w[j];
            for (int w = 0; w < warp; ++w) r += wcnt[w * E + e];
            if ((int64_t)r < C) slot = off[e] + r;
            if (writer) {
                slot_of[t * k + j] = slot;
                if (slot >= 0 && perm_token) perm_token[slot] = (int32_t)t;
            }
        }
        slots[tid * k + j] = slot;
    }
    __syncthreads();

    // gather: this CTA copies every gridDim.y-th (t, j) row of its block
    const int nrow = ROUTE_BLOCK * k;
    for (int r = blockIdx.y; r < nrow; r += gridDim.y) {
        const int32_t slot = slots[r];
        if (slot < 0) continue;
        const int64_t tok = (int64_t)blk * ROUTE_BLOCK + r / k;
        const uint4* src = x + tok * row_vecs;
        uint4* dst = x_perm + (int64_t)slot * row_vecs;
#pragma unroll 4
        for (int c = tid; c < row_vecs; c += ROUTE_BLOCK) dst[c] = src[c];
    }
}

}  // namespace

int launch_dispatch(const int32_t* topk_idx, const int32_t* cnt, int64_t T, int E, int k,
                    int64_t C, int pad, int64_t perm_rows, const void* x, int row_bytes,
                    int32_t* routed, int32_t* kept, int32_t* offsets, int32_t* perm_token,
                    int32_t* slot_of, void* x_perm, int num_sms, cudaStream_t st) {
    if (T == 0) return 0;
    const int nblk = (int)((T + ROUTE_BLOCK - 1) / ROUTE_BLOCK);
    // CTAs per token block: enough to keep about two per SM copying rows
    int ny = (2 * num_sms + nblk - 1) / nblk;
    if (ny > ROUTE_BLOCK * k) ny = ROUTE_BLOCK * k;
    if (ny < 1) ny = 1;
    const size_t smem = sizeof(int32_t) * ((size_t)3 * E + 1 + (size_t)DWARPS * E + ROUTE_BLOCK * k);
    if (smem > 48 * 1024) {
        if (cudaFuncSetAttribute(dispatch_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)smem) != cudaSuccess)
            return -1;
    }
    dim3 grid(nblk, ny);
    dispatch_kernel<<<grid, ROUTE_BLOCK, smem, st>>>(
        topk_idx, cnt, T, E, k, C, pad, perm_rows, reinterpret_cast<const uint4*>(x),
        row_bytes / 16, routed, kept, offsets, perm_token, slot_of, reinterpret_cast<uint4*>(x_perm));
    return cudaGetLastError() == cudaSuccess ? 0 : -1;
}

}  // namespace moe
