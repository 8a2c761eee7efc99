// ep_plan.cu -- the expert-parallel plan of one rank, on the device.
//
// Expert parallelism [Mixtral 8x7B and MoE explained, "Easy explanation" ¶4:
// the experts can be spread over GPUs; MoE routing fully explained, "Easy
// explanation" ¶3: tokens travel to the GPU of their expert] computes the
// single-GPU layer of the concatenated batches of G ranks, so the capacity
// C of the whole batch [same page, ¶5] is shared out in rank order: rank s
// may keep, of expert e, what the lower ranks left of C.  From the gathered
// routed counts [G][E] one block computes, for rank `rank`:
//   cap[e]        = max(C - base[rank][e], 0), base[s][e] = sum_{s' < s} counts[s'][e]
//   row_start[q]  = sum_{s < rank} sum_{e of q} seg[s][e]   (rows before this
//                   rank's at owner q), seg = kept rounded up to the padding,
//                   kept[s][e] = min(counts[s][e], max(C - base[s][e], 0))
//   the groups this rank receives, (source s, local expert el) in that
//   order: rows kept[s][e], first row the running sum of seg, expert el
//   recv[0]       = the total of those segments.
// All integer arithmetic; the host never reads the counts.
#include "common.cuh"
#include "kernels.h"
#include "plan.h"

namespace moe {

namespace {

constexpr int EP_THREADS = 1024;  // one thread per expert (E <= MAX_E)

__device__ __forceinline__ int64_t seg_of(int64_t kept, int pad) {
    return (kept + pad - 1) / pad * pad;
}

// Exclusive prefix sum of v over the block (int64); *total gets the sum.
__device__ int64_t block_exclusive_scan(int64_t v, int64_t* warp_sums, int64_t* total) {
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    int64_t incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int64_t t = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += t;
    }
    if (lane == 31) warp_sums[w] = incl;
    __syncthreads();
    if (w == 0) {
        int64_t s = lane < (int)(blockDim.x >> 5) ? warp_sums[lane] : 0;
        int64_t si = s;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int64_t t = __shfl_up_sync(0xffffffffu, si, o);
            if (lane >= o) si += t;
        }
        warp_sums[lane] = si - s;  // exclusive prefix of the warp sums
        if (lane == 31) warp_sums[32] = si;
    }
    __syncthreads();
    const int64_t r = warp_sums[w] + incl - v;
    *total = warp_sums[32];
    __syncthreads();
    return r;
}

__global__ void __launch_bounds__(EP_THREADS)
    ep_plan_kernel(const int32_t* __restrict__ counts, int G, int E, int rank, int64_t C,
                   int pad, int32_t* __restrict__ cap, int32_t* __restrict__ row_start,
                   int32_t* __restrict__ g_rows, int32_t* __restrict__ g_off,
                   int32_t* __restrict__ g_w, int32_t* __restrict__ recv) {
    __shared__ unsigned long long s_start[MAX_PEERS];
    __shared__ int64_t warp_sums[33];
    const int E_loc = E / G;
    const int tid = threadIdx.x;
    if (tid < G) s_start[tid] = 0;
    __syncthreads();
    // caps of this rank; the rows lower ranks send to each owner
    for (int e = tid; e < E; e += blockDim.x) {
        int64_t base = 0, below = 0;
        for (int s = 0; s < rank; ++s) {
            const int64_t c = counts[(int64_t)s * E + e];
            const int64_t room = C - base > 0 ? C - base : 0;
            below += seg_of(c < room ? c : room, pad);
            base += c;
        }
        const int64_t room = C - base > 0 ? C - base : 0;
        cap[e] = (int32_t)(room < 0x7fffffffLL ? room : 0x7fffffffLL);
        atomicAdd(&s_start[e / E_loc], (unsigned long long)below);
    }
    __syncthreads();
    if (tid < G) row_start[tid] = (int32_t)s_start[tid];
    // the groups this rank receives: thread el follows expert rank * E_loc + el
    // through the sources (its base grows source by source)
    const int el = tid;
    const bool mine = el < E_loc;
    const int e = rank * E_loc + el;
    int64_t base = 0, at = 0;
    for (int s = 0; s < G; ++s) {
        int64_t kept = 0;
        if (mine) {
            const int64_t c = counts[(int64_t)s * E + e];
            const int64_t room = C - base > 0 ? C - base : 0;
            kept = c < room ? c : room;
            base += c;
        }
        int64_t tot = 0;
        const int64_t off = block_exclusive_scan(mine ? seg_of(kept, pad) : 0, warp_sums, &tot);
        if (mine) {
            const int64_t gi = (int64_t)s * E_loc + el;
            g_rows[gi] = (int32_t)kept;
            g_off[gi] = (int32_t)(at + off);
            g_w[gi] = el;
        }
        at += tot;
    }
    if (tid == 0) recv[0] = (int32_t)at;
}

}  // namespace

int launch_ep_plan(const int32_t* counts, int G, int E, int rank, int64_t C, int pad,
                   int32_t* cap, int32_t* row_start, int32_t* g_rows, int32_t* g_off,
                   int32_t* g_w, int32_t* recv, cudaStream_t st) {
    if (G < 1 || G > MAX_PEERS || E < 1 || E > MAX_E || E % G || rank < 0 || rank >= G ||
        pad < 1)
        return -1;
    ep_plan_kernel<<<1, EP_THREADS, 0, st>>>(counts, G, E, rank, C, pad, cap, row_start, g_rows,
                                             g_off, g_w, recv);
    note_launch();
    return launch_result();
}

}  // namespace moe
