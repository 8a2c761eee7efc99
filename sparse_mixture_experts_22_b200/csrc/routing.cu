// routing.cu -- top-k selection, gates, router statistics partials, and the
// capacity-limited dispatch of token rows to experts.
//
// Top-k and gates [Mixtral 8x7B and MoE explained, "Easy explanation" ¶3]:
// keep the k highest-scoring experts and softmax over those k to weight their
// outputs.  One thread per token keeps the k largest logits in registers
// (strictly greater wins, so the lower expert index keeps a tie).  The full
// softmax over all E experts [MoE routing fully explained, "Easy explanation"
// ¶2] feeds the per-block partial sums of P_e and of the token entropy.
//
// Dispatch [MoE routing fully explained, "Easy explanation" ¶3 and ¶5]: every
// expert takes at most C = ceil(T k cf / E) tokens per batch and the overflow
// is dropped, in arrival order by token index: the rank of assignment (t, j)
// in expert e is the number of earlier tokens that chose e, kept if rank < C.
// The rank needs no atomics on the order: per-128-token block histograms, a
// scan over earlier blocks, then inside the block one warp ballot per expert
// and per-warp counts.  Results are identical on every run.
//
// Batches of at most 128 tokens run top-k and dispatch in one kernel
// (route_dispatch_kernel); several CTAs repeat the cheap routing and share the
// row copies into x_perm, so a decode batch spreads its gather over many SMs.
#include <math.h>

#include <map>
#include <mutex>
#include <utility>

#include "common.cuh"
#include "kernels.h"
#include "plan.h"

namespace moe {

namespace {

constexpr int TK_CHUNK = 32;     // experts per shared-memory pass of the P partial sums
constexpr int TK_SMEM_E = 256;   // up to this many experts a block's logits sit in shared memory
constexpr int DWARPS = ROUTE_BLOCK / 32;

struct TopkArgs {
    const float* src;      // router logits without bias [T][E]
    const float* bias;     // may be null
    float* zbuf;           // [T][E] logits + bias, for E > TK_SMEM_E (may equal src)
    float* logits;         // optional user copy of z [T][E]
    int64_t T;
    int E, k;
    int32_t* idx;          // [T][k]
    float* gate;           // [T][k]
    float* ppart;          // [blocks][E]
    float* hpart;          // [blocks]
    int32_t* status;       // device status word (cleared here: a layer call starts)
    int nsub;              // CTAs per block of ROUTE_BLOCK tokens (1, or TOPK_SUB for E > TK_WARP_E)
};

constexpr int TK_WARP_E = TOPK_WARP_E;  // above this many experts one warp routes one token
constexpr int TK_WIDE_THREADS = 512;  // threads of the standalone top-k kernel in that case

// Shared memory of topk_block for `nthreads` threads: hist [E] int32, then
// (E <= TK_SMEM_E) the block's logits [ROUTE_BLOCK][E + 1] fp32, then
// (E > TK_WARP_E) per-warp sums of the full softmax [nthreads/32][E] fp32.
__host__ __device__ inline size_t topk_smem_bytes(int E, int nthreads) {
    size_t b = (size_t)E * sizeof(int32_t);
    if (E <= TK_SMEM_E) b += (size_t)ROUTE_BLOCK * (E + 1) * sizeof(float);
    if (E > TK_WARP_E) b += (size_t)(nthreads / 32) * E * sizeof(float);
    return b;
}

__device__ __forceinline__ float finite_or_minus_inf(float v) { return v != v ? -INFINITY : v; }

// Inserts (v, e) into a descending list of at most k entries held in
// registers; a larger value goes first, an equal one after the entries
// already there (experts arrive in increasing index, so the lower index keeps
// a tie).  From the insertion point on every entry shifts down one place and
// the old k-th falls off.
__device__ __forceinline__ void topk_insert(float* val, int* id, int k, float v, int e) {
    if (!(id[k - 1] < 0 || v > val[k - 1])) return;
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

// Routes part `sub` of `nsub` of the ROUTE_BLOCK tokens of block `blk` with
// blockDim.x >= ROUTE_BLOCK threads (nsub > 1 only above TK_WARP_E experts:
// the tokens of a block are then shared by nsub CTAs so that a batch of few
// blocks still spreads over the SMs).  Leaves the per-expert histogram of its
// tokens in hist[] (shared) and, with nsub == 1, for threads below
// ROUTE_BLOCK, the kept experts of token `tid` in my[] (-1 past k or for
// padding).  Global outputs are written only when `write` is set; the
// partials go to row blk * nsub + sub.  Up to TK_WARP_E experts one thread
// routes one token; above that one warp routes one token: each lane keeps the
// top k of its experts, and k rounds of a warp-wide arg-max over the lanes'
// heads merge them.
__device__ void topk_block(const TopkArgs& a, int blk, int sub, int nsub, bool write,
                           int32_t* hist, float* zs, int32_t* my) {
    __shared__ float ps[ROUTE_BLOCK][TK_CHUNK + 1];
    __shared__ float hs[ROUTE_BLOCK];
    __shared__ int32_t sel[ROUTE_BLOCK][MAX_K];
    const int E = a.E, k = a.k;
    const bool in_smem = E <= TK_SMEM_E;
    const int tid = threadIdx.x, NT = blockDim.x;
    const int span = ROUTE_BLOCK / nsub;  // tokens of this CTA
    const int64_t pidx = (int64_t)blk * nsub + sub;  // its partials' row
    const int64_t tb = (int64_t)blk * ROUTE_BLOCK + (int64_t)sub * span;
    const int nvalid = (int)(a.T - tb < span ? (a.T - tb > 0 ? a.T - tb : 0) : span);
    const int64_t t = tb + tid;
    const bool valid = tid < nvalid;
    float* pw = reinterpret_cast<float*>(zs) + (in_smem ? ROUTE_BLOCK * (E + 1) : 0);

    for (int e = tid; e < E; e += NT) hist[e] = 0;
    if (tid < ROUTE_BLOCK) hs[tid] = 0.f;

    // logits of the block (+ bias), all threads, coalesced, eight loads in
    // flight per thread
    {
        const int n = nvalid * E;
        const float* zsrc = a.src + tb * E;
        for (int i0 = tid; i0 < n; i0 += 8 * NT) {
            float v[8];
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                const int i = i0 + q * NT;
                v[q] = i < n ? zsrc[i] : 0.f;
            }
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                const int i = i0 + q * NT;
                if (i >= n) break;
                const int tl = i / E, e = i - tl * E;
                const float z = a.bias ? v[q] + a.bias[e] : v[q];
                if (in_smem) zs[tl * (E + 1) + e] = z;
                else a.zbuf[(tb + tl) * E + e] = z;
                if (write && a.logits) a.logits[(tb + tl) * E + e] = z;
            }
        }
    }
    __syncthreads();

    if (E <= TK_WARP_E) {
        // ---------------------------------------------- one thread per token
        const bool mine = tid < ROUTE_BLOCK;
        const float* zt = in_smem ? zs + (mine ? tid : 0) * (E + 1) : a.zbuf + (valid ? t : 0) * E;
        float val[MAX_K];
        int id[MAX_K];
#pragma unroll
        for (int j = 0; j < MAX_K; ++j) {
            val[j] = -INFINITY;
            id[j] = -1;
        }
        if (valid)
            for (int e = 0; e < E; ++e) topk_insert(val, id, k, finite_or_minus_inf(zt[e]), e);
        const float m = val[0];
        if (valid) {
            float s = 0.f;
#pragma unroll
            for (int j = 0; j < MAX_K; ++j)
                if (j < k) s += __expf(val[j] - m);
            const float inv = 1.f / s;
#pragma unroll
            for (int j = 0; j < MAX_K; ++j)
                if (j < k) {
                    if (write) {
                        a.idx[t * k + j] = id[j];
                        a.gate[t * k + j] = __expf(val[j] - m) * inv;
                    }
                    atomicAdd(&hist[id[j]], 1);
                }
        }
#pragma unroll
        for (int j = 0; j < MAX_K; ++j) my[j] = (valid && j < k) ? id[j] : -1;

        // full softmax over E: S = sum exp(z - m); p = exp(z - m) / S;
        // entropy = ln S - sum p (z - m)
        float S = 0.f;
        if (valid)
            for (int e = 0; e < E; ++e) S += __expf(finite_or_minus_inf(zt[e]) - m);
        const float invS = valid ? 1.f / S : 0.f;
        float pz = 0.f;
        for (int c0 = 0; c0 < E; c0 += TK_CHUNK) {
            const int n = min(TK_CHUNK, E - c0);
            if (mine)
                for (int i = 0; i < n; ++i) {
                    float p = 0.f;
                    if (valid) {
                        const float v = finite_or_minus_inf(zt[c0 + i]);
                        p = __expf(v - m) * invS;
                        if (p > 0.f) pz += p * (v - m);
                    }
                    ps[tid][i] = p;
                }
            __syncthreads();
            if (write && tid < n) {
                float acc = 0.f;
                // rows past the block's tokens hold +0, which adds nothing
                for (int r = 0; r < nvalid; ++r) acc += ps[r][tid];
                a.ppart[pidx * E + c0 + tid] = acc;
            }
            __syncthreads();
        }
        if (mine) hs[tid] = valid ? (__logf(S) - pz) : 0.f;
    } else {
        // ---------------------------------------------- one warp per token
        const int lane = tid & 31, warp = tid >> 5, nw = NT >> 5;
        for (int e = lane; e < E; e += 32) pw[warp * E + e] = 0.f;
        for (int tl = warp; tl < nvalid; tl += nw) {
            const int64_t tt = tb + tl;
            const float* zr = in_smem ? zs + tl * (E + 1) : a.zbuf + tt * E;
            float lv[MAX_K];
            int li[MAX_K];
#pragma unroll
            for (int j = 0; j < MAX_K; ++j) {
                lv[j] = -INFINITY;
                li[j] = -1;
            }
            for (int e = lane; e < E; e += 32) topk_insert(lv, li, k, finite_or_minus_inf(zr[e]), e);
            float vsel[MAX_K];
            int isel[MAX_K];
#pragma unroll
            for (int j = 0; j < MAX_K; ++j) {
                vsel[j] = -INFINITY;
                isel[j] = -1;
                if (j >= k) continue;
                // arg-max of the lanes' heads: larger value, then lower index
                float bv = lv[0];
                int bi = li[0] < 0 ? 0x7fffffff : li[0];
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) {
                    const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
                    const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
                    if (ov > bv || (ov == bv && oi < bi)) {
                        bv = ov;
                        bi = oi;
                    }
                }
                vsel[j] = bv;
                isel[j] = bi;
                if (li[0] == bi) {  // the winning lane pops its head
#pragma unroll
                    for (int q = 0; q < MAX_K - 1; ++q) {
                        lv[q] = lv[q + 1];
                        li[q] = li[q + 1];
                    }
                    lv[MAX_K - 1] = -INFINITY;
                    li[MAX_K - 1] = -1;
                }
            }
            const float m = vsel[0];
            float s = 0.f;
#pragma unroll
            for (int j = 0; j < MAX_K; ++j)
                if (j < k) s += __expf(vsel[j] - m);
            const float inv = 1.f / s;
            if (lane == 0) {
#pragma unroll
                for (int j = 0; j < MAX_K; ++j)
                    if (j < k) {
                        if (write) {
                            a.idx[tt * k + j] = isel[j];
                            a.gate[tt * k + j] = __expf(vsel[j] - m) * inv;
                        }
                        atomicAdd(&hist[isel[j]], 1);
                        sel[tl][j] = isel[j];
                    }
            }
            // full softmax, each lane over its experts, then a fixed shuffle tree
            float Sl = 0.f;
            for (int e = lane; e < E; e += 32) Sl += __expf(finite_or_minus_inf(zr[e]) - m);
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) Sl += __shfl_xor_sync(0xffffffffu, Sl, o);
            const float invS = 1.f / Sl;
            float pz = 0.f;
            for (int e = lane; e < E; e += 32) {
                const float v = finite_or_minus_inf(zr[e]);
                const float p = __expf(v - m) * invS;
                pw[warp * E + e] += p;
                if (p > 0.f) pz += p * (v - m);
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) pz += __shfl_xor_sync(0xffffffffu, pz, o);
            if (lane == 0) hs[tl] = __logf(Sl) - pz;
        }
        __syncthreads();
        if (write)
            for (int e = tid; e < E; e += NT) {
                float acc = 0.f;
                for (int w = 0; w < nw; ++w) acc += pw[w * E + e];
                a.ppart[pidx * E + e] = acc;
            }
        if (tid < ROUTE_BLOCK) {
#pragma unroll
            for (int j = 0; j < MAX_K; ++j) my[j] = (valid && j < k) ? sel[tid][j] : -1;
        }
    }
    __syncthreads();
    if (write && tid == 0) {
        float acc = 0.f;
        for (int r = 0; r < nvalid; ++r) acc += hs[r];
        a.hpart[pidx] = acc;
    }
}

struct DispatchArgs {
    int64_t T;
    int E, k;
    int64_t C;
    int pad;
    int64_t perm_rows;
    const uint4* x;
    int row_vecs;          // 16-byte vectors per row of x
    int32_t* routed;       // [E]
    int32_t* kept;         // [E]
    int32_t* offsets;      // [E+1]
    int32_t* perm_token;   // [perm_rows] (may be null)
    int32_t* slot_of;      // [T][k]
    uint4* x_perm;         // [perm_rows][d]
    const int32_t* cap;    // [E] per-expert capacity (min with C), or null
    int nsub;              // histogram rows per block (the top-k CTAs of a block)
    int npeer, e_loc;      // row destinations: expert e -> peer[e / e_loc] (see place_rows)
    uint4* peer[MAX_PEERS];
    const int32_t* peer_start;  // device [npeer] first row at each destination, or null (0)
};

__device__ __forceinline__ int64_t expert_cap(const DispatchArgs& a, int e) {
    if (!a.cap) return a.C;
    const int64_t c = a.cap[e];
    return c < a.C ? (c < 0 ? 0 : c) : a.C;
}

// Shared memory of the dispatch kernels: base [E], tot [E], rows [E],
// off [E+1], wcnt [DWARPS][E], slots [ROUTE_BLOCK * k], owner [ROUTE_BLOCK * k],
// then (8-byte aligned) the destination table [MAX_PEERS] and its first rows
// [MAX_PEERS].
__host__ __device__ inline size_t dispatch_smem_bytes(int E, int k) {
    return sizeof(int32_t) *
               ((size_t)4 * E + 1 + (size_t)DWARPS * E + (size_t)2 * ROUTE_BLOCK * k) +
           8 + sizeof(uint4*) * MAX_PEERS + sizeof(int32_t) * MAX_PEERS;
}

struct DispatchSmem {
    int32_t* base;   // assignments to e in earlier blocks
    int32_t* tot;    // assignments to e in the batch (routed)
    int32_t* rows;   // rows e serves (kept)
    int32_t* off;    // padded segment starts [E+1]
    int32_t* wcnt;   // per-warp counts [DWARPS][E]
    int32_t* slots;  // [ROUTE_BLOCK * k] destination row of each (token, j), -1: dropped
    int32_t* owner;  // [ROUTE_BLOCK * k] destination of each (token, j)
    uint4** peer;    // [MAX_PEERS] destination bases
    int32_t* start;  // [MAX_PEERS] first row of this rank's rows at each destination
};

__device__ __forceinline__ DispatchSmem dispatch_smem(int32_t* sm, int E, int k) {
    DispatchSmem d;
    d.base = sm;
    d.tot = d.base + E;
    d.rows = d.tot + E;
    d.off = d.rows + E;
    d.wcnt = d.off + E + 1;
    d.slots = d.wcnt + DWARPS * E;
    d.owner = d.slots + ROUTE_BLOCK * k;
    const uintptr_t p = reinterpret_cast<uintptr_t>(d.owner + ROUTE_BLOCK * k);
    d.peer = reinterpret_cast<uint4**>((p + 7) & ~static_cast<uintptr_t>(7));
    d.start = reinterpret_cast<int32_t*>(d.peer + MAX_PEERS);
    return d;
}

__device__ __forceinline__ int32_t capped(int32_t n, int64_t C) {
    return (int64_t)n < C ? n : (int32_t)C;
}

// Thread 0: padded segment starts from the rows each expert serves.
__device__ void segment_offsets(const int32_t* rows, int E, int pad, int32_t* off) {
    if (threadIdx.x != 0) return;
    int32_t o = 0;
    for (int e = 0; e < E; ++e) {
        off[e] = o;
        o += (rows[e] + pad - 1) / pad * pad;
    }
    off[E] = o;
}

// Global rank of each of the thread's assignments in its expert's queue
// (token order): earlier blocks (base), earlier warps (per-warp ballot
// counts), earlier lanes (ballot).  Called by all ROUTE_BLOCK threads.
__device__ void block_ranks(int E, const int32_t* base, int32_t* wcnt, const int32_t* my,
                            int32_t* rank) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    int32_t rank_w[MAX_K];
#pragma unroll
    for (int j = 0; j < MAX_K; ++j) rank_w[j] = 0;
    const unsigned lt = (1u << lane) - 1u;
    for (int e = 0; e < E; ++e) {
        bool chose = false;
#pragma unroll
        for (int j = 0; j < MAX_K; ++j) chose |= (my[j] == e);
        const unsigned msk = __ballot_sync(0xffffffffu, chose);
        if (lane == 0) wcnt[warp * E + e] = __popc(msk);
        if (chose) {
            const int r = __popc(msk & lt);
#pragma unroll
            for (int j = 0; j < MAX_K; ++j)
                if (my[j] == e) rank_w[j] = r;
        }
    }
    __syncthreads();
#pragma unroll
    for (int j = 0; j < MAX_K; ++j) {
        rank[j] = -1;
        if (my[j] < 0) continue;
        const int e = my[j];
        int32_t r = base[e] + rank_w[j];
        for (int w = 0; w < warp; ++w) r += wcnt[w * E + e];
        rank[j] = r;
    }
}

// Slots and row copies of block `blk`: assignment j of this thread's token is
// served by expert[j] at position rank[j] of its queue, kept if rank < C.
// d.off and d.rows must be filled.  When `writer`, writes slot_of and
// perm_token (with -1 in padding rows and the unused tail).  `split`/`nsplit`:
// this CTA copies every nsplit-th row.  The row of slot s of expert e goes to
// destination o = e / e_loc at row s - off[o * e_loc]: with one destination
// (e_loc = E) that is x_perm at row s; with expert parallelism, the receive
// buffer of e's owner, in this GPU's memory or a peer's (NVLink stores).
__device__ void place_rows(const DispatchArgs& a, int blk, int nblk, bool writer, int split,
                           int nsplit, const DispatchSmem& d, const int32_t* expert,
                           const int32_t* rank) {
    const int E = a.E, k = a.k;
    const int tid = threadIdx.x;
    if (writer && a.perm_token) {
        for (int e = blk; e < E; e += nblk)
            for (int r = d.off[e] + d.rows[e] + tid; r < d.off[e + 1]; r += ROUTE_BLOCK)
                a.perm_token[r] = -1;
        for (int64_t r = d.off[E] + (int64_t)blk * ROUTE_BLOCK + tid; r < a.perm_rows;
             r += (int64_t)nblk * ROUTE_BLOCK)
            a.perm_token[r] = -1;
    }
    if (tid == 0) {
        // the destination table, indexed statically so it stays in the
        // parameter space
#pragma unroll
        for (int i = 0; i < MAX_PEERS; ++i)
            if (i < a.npeer) d.peer[i] = a.peer[i];
    }
    if (tid < a.npeer) d.start[tid] = a.peer_start ? a.peer_start[tid] : 0;
    const int64_t t = (int64_t)blk * ROUTE_BLOCK + tid;
    const bool valid = t < a.T;
#pragma unroll
    for (int j = 0; j < MAX_K; ++j) {
        if (j >= k) break;
        int32_t slot = -1, row = -1, own = 0;
        if (valid) {
            if (rank[j] >= 0 && (int64_t)rank[j] < expert_cap(a, expert[j]))
                slot = d.off[expert[j]] + rank[j];
            if (writer) {
                a.slot_of[t * k + j] = slot;
                if (slot >= 0 && a.perm_token) a.perm_token[slot] = (int32_t)t;
            }
            if (slot >= 0) {
                own = expert[j] / a.e_loc;
                row = slot - d.off[own * a.e_loc];
            }
        }
        d.slots[tid * k + j] = row;
        d.owner[tid * k + j] = own;
    }
    __syncthreads();

    // gather: every token's row is read once and stored to each slot it keeps.
    // Warp w of this CTA takes the block's tokens split + nsplit * (w + W i);
    // when the CTAs of a block outnumber its tokens' warps' work, the columns
    // of a row are split between the warps that share the token.
    constexpr int W = ROUTE_BLOCK / 32;
    constexpr int G = 8;
    const int warp = tid >> 5, lane = tid & 31;
    const int nv = a.row_vecs;
    const int64_t tok0 = (int64_t)blk * ROUTE_BLOCK;
    const int ntok = (int)((a.T - tok0) < ROUTE_BLOCK ? (a.T - tok0) : ROUTE_BLOCK);
    const int workers = nsplit * W;                       // warps over this block
    const int wid = split + nsplit * warp;                // this warp among them
    const int cparts = workers > ntok ? workers / ntok : 1;  // column parts per token
    const int cp = wid % cparts;                          // this warp's column part
    for (int tl = wid / cparts; tl < ntok; tl += workers / cparts) {
        uint4* dst[MAX_K];
        bool any = false;
#pragma unroll
        for (int j = 0; j < MAX_K; ++j) {
            const int32_t row = j < k ? d.slots[tl * k + j] : -1;
            dst[j] = row >= 0 ? d.peer[d.owner[tl * k + j]] +
                                    (int64_t)(row + d.start[d.owner[tl * k + j]]) * nv
                              : nullptr;
            any |= row >= 0;
        }
        if (!any) continue;
        const uint4* src = a.x + (tok0 + tl) * nv;
        // this warp's share of the row's 16-byte columns
        const int c_lo = (int)((int64_t)nv * cp / cparts);
        const int c_hi = (int)((int64_t)nv * (cp + 1) / cparts);
        for (int c0 = c_lo + lane; c0 < c_hi; c0 += 32 * G) {
            uint4 v[G];
#pragma unroll
            for (int q = 0; q < G; ++q)
                if (c0 + 32 * q < c_hi) v[q] = __ldg(src + c0 + 32 * q);
#pragma unroll
            for (int j = 0; j < MAX_K; ++j) {
                if (!dst[j]) continue;
#pragma unroll
                for (int q = 0; q < G; ++q)
                    if (c0 + 32 * q < c_hi) dst[j][c0 + 32 * q] = v[q];
            }
        }
    }
}

// The drop policy: ranks, capacity, slots and row copies of block `blk`.
// d.base and d.tot must be filled; my[] holds the thread's token choices.
__device__ void dispatch_block(const DispatchArgs& a, int blk, int nblk, bool writer, int split,
                               int nsplit, const DispatchSmem& d, const int32_t* my) {
    const int E = a.E;
    const int tid = threadIdx.x;
    for (int e = tid; e < E; e += ROUTE_BLOCK) d.rows[e] = capped(d.tot[e], expert_cap(a, e));
    __syncthreads();
    segment_offsets(d.rows, E, a.pad, d.off);
    __syncthreads();
    if (writer && blk == 0) {
        for (int e = tid; e < E; e += ROUTE_BLOCK) {
            a.routed[e] = d.tot[e];
            a.kept[e] = d.rows[e];
        }
        for (int e = tid; e <= E; e += ROUTE_BLOCK) a.offsets[e] = d.off[e];
    }
    int32_t rank[MAX_K];
    block_ranks(E, d.base, d.wcnt, my, rank);
    place_rows(a, blk, nblk, writer, split, nsplit, d, my, rank);
}

__global__ void __launch_bounds__(TK_WIDE_THREADS)
    topk_kernel(TopkArgs a, int32_t* __restrict__ cnt) {
    extern __shared__ int32_t dyn[];
    int32_t* hist = dyn;
    float* zs = reinterpret_cast<float*>(dyn + a.E);
    int32_t my[MAX_K];
    if (blockIdx.x == 0 && threadIdx.x == 0 && a.status) {
        a.status[0] = DEV_OK;  // a new layer call starts here
        a.status[1] = 0;       // combine's completion ticket
    }
    // CTA b routes part b % nsub of block b / nsub; its histogram is row b
    topk_block(a, blockIdx.x / a.nsub, blockIdx.x % a.nsub, a.nsub, true, hist, zs, my);
    __syncthreads();
    for (int e = threadIdx.x; e < a.E; e += blockDim.x)
        cnt[(int64_t)blockIdx.x * a.E + e] = hist[e];
}

// counts[e] = sum over routing blocks of the histograms (the batch's routed
// assignments per expert).  One warp per expert; integer sums.
__global__ void route_counts_kernel(const int32_t* __restrict__ cnt, int nblk, int E,
                                    int32_t* __restrict__ counts) {
    const int e = (int)((blockIdx.x * (int64_t)blockDim.x + threadIdx.x) >> 5);
    const int lane = threadIdx.x & 31;
    if (e >= E) return;
    int32_t s = 0;
    for (int b = lane; b < nblk; b += 32) s += cnt[(int64_t)b * E + e];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    if (lane == 0) counts[e] = s;
}

// Per expert e, the exclusive prefix over blocks of the histograms (in place:
// cnt[b][e] becomes the number of assignments to e in blocks before b) and
// the total tot[e].  One warp per expert; integer sums, any order is exact.
__global__ void dispatch_scan_kernel(int32_t* __restrict__ cnt, int32_t* __restrict__ tot,
                                     int nblk, int E) {
    const int e = (int)((blockIdx.x * (int64_t)blockDim.x + threadIdx.x) >> 5);
    const int lane = threadIdx.x & 31;
    if (e >= E) return;
    int32_t carry = 0;
    for (int q0 = 0; q0 < nblk; q0 += 32) {
        const int q = q0 + lane;
        const int32_t c = q < nblk ? cnt[(int64_t)q * E + e] : 0;
        int32_t incl = c;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int32_t v = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += v;
        }
        if (q < nblk) cnt[(int64_t)q * E + e] = carry + incl - c;
        carry += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (lane == 0) tot[e] = carry;
}

__global__ void __launch_bounds__(ROUTE_BLOCK)
    dispatch_kernel(DispatchArgs a, const int32_t* __restrict__ topk_idx,
                    const int32_t* __restrict__ base_in, const int32_t* __restrict__ tot_in) {
    extern __shared__ int32_t sm[];
    const DispatchSmem d = dispatch_smem(sm, a.E, a.k);
    const int blk = blockIdx.x, nblk = gridDim.x;
    for (int e = threadIdx.x; e < a.E; e += ROUTE_BLOCK) {
        d.base[e] = base_in[(int64_t)blk * a.nsub * a.E + e];
        d.tot[e] = tot_in[e];
    }
    const int64_t t = (int64_t)blk * ROUTE_BLOCK + threadIdx.x;
    int32_t my[MAX_K];
#pragma unroll
    for (int j = 0; j < MAX_K; ++j) my[j] = (t < a.T && j < a.k) ? topk_idx[t * a.k + j] : -1;
    __syncthreads();
    dispatch_block(a, blk, nblk, blockIdx.y == 0, blockIdx.y, gridDim.y, d, my);
}

// ---------------------------------------------------------------- reroute policy
//
// [MoE routing fully explained, "Easy explanation" ¶3: the second way to treat
// tokens beyond capacity, rerouting them to a spare expert].  Three steps:
// rank_kernel records every assignment's rank in its expert's queue;
// reroute_kernel visits the dropped ones in token order and moves each to the
// token's best-scoring unused expert that still has room (it keeps its gate);
// the rule is sequential, and the kernel reproduces it in a few parallel
// rounds (see reroute_kernel); place_kernel then writes slots and copies rows
// as for the drop policy.

__global__ void __launch_bounds__(ROUTE_BLOCK)
    rank_kernel(DispatchArgs a, const int32_t* __restrict__ topk_idx,
                const int32_t* __restrict__ base_in, int32_t* __restrict__ expert_of,
                int32_t* __restrict__ rank_of) {
    extern __shared__ int32_t sm[];
    const DispatchSmem d = dispatch_smem(sm, a.E, a.k);
    const int blk = blockIdx.x;
    for (int e = threadIdx.x; e < a.E; e += ROUTE_BLOCK)
        d.base[e] = base_in[(int64_t)blk * a.nsub * a.E + e];
    const int64_t t = (int64_t)blk * ROUTE_BLOCK + threadIdx.x;
    int32_t my[MAX_K], rank[MAX_K];
#pragma unroll
    for (int j = 0; j < MAX_K; ++j) my[j] = (t < a.T && j < a.k) ? topk_idx[t * a.k + j] : -1;
    __syncthreads();
    block_ranks(a.E, d.base, d.wcnt, my, rank);
    if (t < a.T)
#pragma unroll
        for (int j = 0; j < MAX_K; ++j)
            if (j < a.k) {
                expert_of[t * a.k + j] = my[j];
                rank_of[t * a.k + j] = rank[j];
            }
}

constexpr int RR_THREADS = 1024;  // one token per thread, chunks of 1024 tokens

__host__ __device__ inline size_t reroute_smem_bytes(int E, int k) {
    // fill [E] | warp sums [32] | control [4] | unresolved masks [1024] (int32)
    // | picks and serving experts [1024][k] (int16) | ordered pick list [1024 k] (uint16)
    return sizeof(int32_t) * ((size_t)E + 32 + 4 + RR_THREADS) +
           3 * sizeof(int16_t) * (size_t)RR_THREADS * k;
}

// The reroute pass in rounds.  Each thread owns one token of a 1024-token
// chunk.  In a round every thread picks, for each of its unresolved dropped
// assignments in j order, the best-scoring expert (ties: lower index) that
// still has room under the fill levels at the start of the round and that the
// token does not use.  The picks are listed in (token, j) order and warp 0
// commits them 32 at a time -- a pick's queue position is its expert's fill
// plus the earlier picks of the same expert in the list (__match_any_sync) --
// stopping at the first pick whose expert is full by then.  Up to that point
// the picks equal those of the one-at-a-time rule (room only shrinks, so an
// expert that was best with room stays best while it has room); the next
// round re-picks from there.  Every stop leaves one more expert full, so a
// chunk takes at most E + 1 rounds.
__global__ void __launch_bounds__(RR_THREADS)
    reroute_kernel(const int32_t* __restrict__ topk_idx, int32_t* __restrict__ expert_of,
                   int32_t* __restrict__ rank_of, const int32_t* __restrict__ tot,
                   const float* __restrict__ z, const float* __restrict__ bias, int64_t T, int E,
                   int k, int64_t C, int pad, int32_t* __restrict__ routed,
                   int32_t* __restrict__ kept, int32_t* __restrict__ offsets) {
    extern __shared__ int32_t sm[];
    int32_t* fill = sm;                                            // [E]
    int32_t* wsum = fill + E;                                      // [32] per-warp pick counts
    int32_t* ctl = wsum + 32;                                      // [0] done, [1] list length
    uint32_t* um = reinterpret_cast<uint32_t*>(ctl + 4);           // [1024] unresolved j bits
    int16_t* pick = reinterpret_cast<int16_t*>(um + RR_THREADS);   // [1024][k]
    int16_t* srv = pick + RR_THREADS * k;                          // [1024][k] serving experts
    uint16_t* plist = reinterpret_cast<uint16_t*>(srv + RR_THREADS * k);  // [1024 k] tl*8 + j
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    for (int e = tid; e < E; e += RR_THREADS) {
        fill[e] = capped(tot[e], C);
        routed[e] = tot[e];
    }
    for (int64_t t0 = 0; t0 < T; t0 += RR_THREADS) {
        const int64_t t = t0 + tid;
        const bool have = t < T;
        int32_t ch[MAX_K];
        uint32_t unres = 0;
#pragma unroll
        for (int j = 0; j < MAX_K; ++j) {
            ch[j] = (have && j < k) ? topk_idx[t * k + j] : -1;
            if (have && j < k) {
                srv[tid * k + j] = (int16_t)ch[j];
                if ((int64_t)rank_of[t * k + j] >= C) unres |= 1u << j;
            }
        }
        um[tid] = unres;
        if (!__syncthreads_or(unres != 0)) continue;
        for (int round = 0; round <= E + 1; ++round) {
            // ------------------------------------------------ picks (all threads)
            if (unres) {
                const float* zt = z + t * E;
                int32_t mine[MAX_K];  // experts this token picked earlier in the round
#pragma unroll
                for (int j = 0; j < MAX_K; ++j) mine[j] = -1;
                for (int j = 0; j < k; ++j) {
                    if (!((unres >> j) & 1u)) continue;
                    int best = -1;
                    float bv = -INFINITY;
                    for (int e = 0; e < E; ++e) {
                        if ((int64_t)fill[e] >= C) continue;
                        bool used = false;
                        for (int q = 0; q < k; ++q)
                            used |= ch[q] == e || srv[tid * k + q] == e || mine[q] == e;
                        if (used) continue;
                        const float v = finite_or_minus_inf(zt[e] + (bias ? bias[e] : 0.0f));
                        if (best < 0 || v > bv) {
                            best = e;
                            bv = v;
                        }
                    }
                    pick[tid * k + j] = (int16_t)best;
                    mine[j] = best;
                }
            }
            // ------------------------------------------------ ordered pick list (block scan)
            const int cnt = __popc(unres);
            int incl = cnt;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int v = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += v;
            }
            if (lane == 31) wsum[warp] = incl;
            __syncthreads();
            if (warp == 0) {
                int w = wsum[lane];
                int wi = w;
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const int v = __shfl_up_sync(0xffffffffu, wi, o);
                    if (lane >= o) wi += v;
                }
                wsum[lane] = wi - w;  // exclusive prefix of the warp totals
                if (lane == 31) ctl[1] = wi;
            }
            __syncthreads();
            {
                int pos = wsum[warp] + incl - cnt;
                uint32_t u = unres;
                while (u) {
                    const int j = __ffs(u) - 1;
                    u &= u - 1;
                    plist[pos++] = (uint16_t)(tid * 8 + j);
                }
            }
            __syncthreads();
            // ------------------------------------------------ commit walk (warp 0)
            if (warp == 0) {
                const int n = ctl[1];
                bool cut = false;
                for (int base = 0; base < n && !cut; base += 32) {
                    const int i = base + lane;
                    const bool act = i < n;
                    const int ent = act ? plist[i] : 0;
                    const int tl = ent >> 3, j = ent & 7;
                    const int p = act ? pick[tl * k + j] : -1;
                    // inactive lanes and picks without room get keys no one else has
                    const int key = (act && p >= 0) ? p : -1 - lane;
                    const uint32_t grp = __match_any_sync(0xffffffffu, key);
                    const int before = __popc(grp & ((1u << lane) - 1u));
                    const int f = (act && p >= 0) ? fill[p] : 0;
                    const bool full = act && p >= 0 && (int64_t)(f + before) >= C;
                    const uint32_t fullm = __ballot_sync(0xffffffffu, full);
                    const int lim = fullm ? __ffs(fullm) - 1 : 32;
                    const bool commit = act && lane < lim;
                    const uint32_t cm = __ballot_sync(0xffffffffu, commit);
                    if (commit) {
                        if (p >= 0) {
                            const int64_t g = (t0 + tl) * k + j;
                            srv[tl * k + j] = (int16_t)p;
                            expert_of[g] = p;
                            rank_of[g] = f + before;
                        }
                        // p < 0: no expert has room; the assignment stays dropped
                        atomicAnd(&um[tl], ~(1u << j));
                    }
                    // the last committing pick of each expert advances its fill
                    const uint32_t mine_c = grp & cm;
                    if (commit && p >= 0 && (31 - __clz(mine_c)) == lane) fill[p] = f + before + 1;
                    __syncwarp();
                    cut = fullm != 0;
                }
                if (lane == 0) ctl[0] = cut ? 0 : 1;
            }
            __syncthreads();
            unres = um[tid];
            const bool done = ctl[0] != 0;
            __syncthreads();
            if (done) break;
        }
        __syncthreads();
    }
    for (int e = tid; e < E; e += RR_THREADS) kept[e] = fill[e];
    __syncthreads();
    if (tid == 0) {
        int32_t o = 0;
        for (int e = 0; e < E; ++e) {
            offsets[e] = o;
            o += (fill[e] + pad - 1) / pad * pad;
        }
        offsets[E] = o;
    }
}

__global__ void __launch_bounds__(ROUTE_BLOCK)
    place_kernel(DispatchArgs a, const int32_t* __restrict__ expert_of,
                 const int32_t* __restrict__ rank_of) {
    extern __shared__ int32_t sm[];
    const DispatchSmem d = dispatch_smem(sm, a.E, a.k);
    const int blk = blockIdx.x, nblk = gridDim.x;
    for (int e = threadIdx.x; e < a.E; e += ROUTE_BLOCK) d.rows[e] = a.kept[e];
    for (int e = threadIdx.x; e <= a.E; e += ROUTE_BLOCK) d.off[e] = a.offsets[e];
    const int64_t t = (int64_t)blk * ROUTE_BLOCK + threadIdx.x;
    int32_t ex[MAX_K], rank[MAX_K];
#pragma unroll
    for (int j = 0; j < MAX_K; ++j) {
        const bool v = t < a.T && j < a.k;
        ex[j] = v ? expert_of[t * a.k + j] : -1;
        rank[j] = v ? rank_of[t * a.k + j] : -1;
    }
    __syncthreads();
    place_rows(a, blk, nblk, blockIdx.y == 0, blockIdx.y, gridDim.y, d, ex, rank);
}

// T <= ROUTE_BLOCK: top-k and dispatch in one launch.  Every CTA routes the
// whole batch (cheap) and copies its share of the rows; CTA 0 writes the
// routing outputs.
__global__ void __launch_bounds__(ROUTE_BLOCK)
    route_dispatch_kernel(TopkArgs ta, DispatchArgs da, int32_t* __restrict__ cnt) {
    extern __shared__ int32_t dyn[];
    pdl_wait();
    pdl_trigger();
    const int E = ta.E;
    int32_t* hist = dyn;
    float* zs = reinterpret_cast<float*>(dyn + E);
    int32_t* dsm =
        reinterpret_cast<int32_t*>(reinterpret_cast<uint8_t*>(dyn) + topk_smem_bytes(E, ROUTE_BLOCK));
    const DispatchSmem d = dispatch_smem(dsm, E, da.k);
    const bool leader = blockIdx.x == 0;
    if (leader && threadIdx.x == 0 && ta.status) {
        ta.status[0] = DEV_OK;
        ta.status[1] = 0;
    }
    int32_t my[MAX_K];
    topk_block(ta, 0, 0, 1, leader, hist, zs, my);
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += ROUTE_BLOCK) {
        d.base[e] = 0;
        d.tot[e] = hist[e];
        if (leader) cnt[e] = hist[e];
    }
    __syncthreads();
    dispatch_block(da, 0, 1, leader, blockIdx.x, gridDim.x, d, my);
}

// Opts the kernel in to `bytes` of dynamic shared memory when its static plus
// dynamic shared memory exceeds the 48 KB a launch gets without opting in
// (the top-k kernels hold ~21.5 KB of static arrays beside their dynamic
// buffer).  Per device and kernel the limit only ever grows, so callers with
// smaller needs on other threads are not cut short.
template <typename K>
int set_smem(K kern, size_t bytes) {
    struct Entry {
        size_t static_bytes;
        size_t optin;
    };
    static std::mutex mu;
    static std::map<std::pair<int, const void*>, Entry> cache;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return -1;
    std::lock_guard<std::mutex> lk(mu);
    const auto key = std::make_pair(dev, reinterpret_cast<const void*>(kern));
    auto it = cache.find(key);
    if (it == cache.end()) {
        cudaFuncAttributes fa;
        if (cudaFuncGetAttributes(&fa, kern) != cudaSuccess) return -1;
        it = cache.emplace(key, Entry{fa.sharedSizeBytes, 0}).first;
    }
    if (it->second.static_bytes + bytes <= 48 * 1024 || bytes <= it->second.optin) return 0;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes) !=
        cudaSuccess)
        return -1;
    it->second.optin = bytes;
    return 0;
}

TopkArgs topk_args(const RouteParams& r) {
    TopkArgs a;
    a.src = r.src;
    a.bias = r.bias;
    a.zbuf = r.zbuf;
    a.logits = r.logits;
    a.T = r.T;
    a.E = r.E;
    a.k = r.k;
    a.idx = r.topk_idx;
    a.gate = r.topk_gate;
    a.ppart = r.ppart;
    a.hpart = r.hpart;
    a.status = r.status;
    a.nsub = r.nsub > 0 ? r.nsub : 1;
    return a;
}

DispatchArgs dispatch_args(const DispatchParams& p) {
    DispatchArgs a;
    a.T = p.T;
    a.E = p.E;
    a.k = p.k;
    a.C = p.C;
    a.pad = p.pad;
    a.perm_rows = p.perm_rows;
    a.x = reinterpret_cast<const uint4*>(p.x);
    a.row_vecs = p.row_bytes / 16;
    a.routed = p.routed;
    a.kept = p.kept;
    a.offsets = p.offsets;
    a.perm_token = p.perm_token;
    a.slot_of = p.slot_of;
    a.x_perm = reinterpret_cast<uint4*>(p.x_perm);
    a.cap = p.cap;
    a.nsub = p.nsub > 0 ? p.nsub : 1;
    a.peer_start = p.peer_start;
    for (int i = 0; i < MAX_PEERS; ++i) a.peer[i] = nullptr;
    if (p.npeer > 0) {
        a.npeer = p.npeer;
        a.e_loc = p.e_loc;
        for (int i = 0; i < p.npeer; ++i) a.peer[i] = reinterpret_cast<uint4*>(p.peer_rows[i]);
    } else {
        a.npeer = 1;
        a.e_loc = p.E;
        a.peer[0] = a.x_perm;
    }
    return a;
}

// CTAs per token block for the row copies: about two per SM in total, and no
// more than the block has rows
int copy_splits(int nblk, int64_t T, int k, int num_sms) {
    int ny = (2 * num_sms + nblk - 1) / nblk;
    const int64_t rows = (T < ROUTE_BLOCK ? T : ROUTE_BLOCK) * (int64_t)k;
    if (ny > rows) ny = (int)rows;
    return ny < 1 ? 1 : ny;
}

}  // namespace

int launch_route_counts(const int32_t* cnt, int nblk, int E, int32_t* counts, cudaStream_t st) {
    const int64_t threads = (int64_t)E * 32;
    route_counts_kernel<<<(unsigned)((threads + 255) / 256), 256, 0, st>>>(cnt, nblk, E, counts);
    note_launch();
    return launch_result();
}

int launch_topk(const RouteParams& r, cudaStream_t st) {
    if (r.T == 0) return 0;
    const int nsub = r.nsub > 0 ? r.nsub : 1;
    if (nsub > 1 && (r.E <= TK_WARP_E || ROUTE_BLOCK % nsub != 0)) return -1;
    const unsigned blocks = (unsigned)((r.T + ROUTE_BLOCK - 1) / ROUTE_BLOCK) * nsub;
    const int nthreads = r.E > TK_WARP_E ? TK_WIDE_THREADS : ROUTE_BLOCK;
    const size_t smem = topk_smem_bytes(r.E, nthreads);
    if (set_smem(topk_kernel, smem)) return -1;
    topk_kernel<<<blocks, nthreads, smem, st>>>(topk_args(r), r.cnt);
    note_launch();
    return launch_result();
}

int launch_dispatch(const DispatchParams& p, const int32_t* topk_idx, int32_t* cnt, int32_t* tot,
                    int num_sms, cudaStream_t st) {
    if (p.T == 0) return 0;
    const int nblk = (int)((p.T + ROUTE_BLOCK - 1) / ROUTE_BLOCK);
    const int nrows = nblk * (p.nsub > 0 ? p.nsub : 1);  // histogram rows
    const int64_t scan_threads = (int64_t)p.E * 32;
    dispatch_scan_kernel<<<(unsigned)((scan_threads + 255) / 256), 256, 0, st>>>(cnt, tot, nrows,
                                                                                p.E);
    note_launch();
    if (launch_result() != 0) return -1;
    const size_t smem = dispatch_smem_bytes(p.E, p.k);
    if (set_smem(dispatch_kernel, smem)) return -1;
    dim3 grid(nblk, copy_splits(nblk, p.T, p.k, num_sms));
    dispatch_kernel<<<grid, ROUTE_BLOCK, smem, st>>>(dispatch_args(p), topk_idx, cnt, tot);
    note_launch();
    return launch_result();
}

int launch_reroute_dispatch(const DispatchParams& p, const int32_t* topk_idx, int32_t* cnt,
                            int32_t* tot, const float* z, int32_t* expert_of, int32_t* rank_of,
                            int num_sms, cudaStream_t st) {
    if (p.T == 0) return 0;
    const int nblk = (int)((p.T + ROUTE_BLOCK - 1) / ROUTE_BLOCK);
    const DispatchArgs a = dispatch_args(p);
    const int nrows = nblk * a.nsub;  // histogram rows
    const int64_t scan_threads = (int64_t)p.E * 32;
    dispatch_scan_kernel<<<(unsigned)((scan_threads + 255) / 256), 256, 0, st>>>(cnt, tot, nrows,
                                                                                p.E);
    note_launch();
    if (launch_result() != 0) return -1;
    const size_t smem = dispatch_smem_bytes(p.E, p.k);
    if (set_smem(rank_kernel, smem) || set_smem(place_kernel, smem)) return -1;
    rank_kernel<<<nblk, ROUTE_BLOCK, smem, st>>>(a, topk_idx, cnt, expert_of, rank_of);
    note_launch();
    if (launch_result() != 0) return -1;
    const size_t rsmem = reroute_smem_bytes(p.E, p.k);
    if (set_smem(reroute_kernel, rsmem)) return -1;
    reroute_kernel<<<1, RR_THREADS, rsmem, st>>>(topk_idx, expert_of, rank_of, tot, z, nullptr,
                                                 p.T, p.E, p.k, p.C, p.pad, p.routed, p.kept,
                                                 p.offsets);
    note_launch();
    if (launch_result() != 0) return -1;
    dim3 grid(nblk, copy_splits(nblk, p.T, p.k, num_sms));
    place_kernel<<<grid, ROUTE_BLOCK, smem, st>>>(a, expert_of, rank_of);
    note_launch();
    return launch_result();
}

int launch_route_dispatch(const RouteParams& r, const DispatchParams& p, int num_sms,
                          cudaStream_t st) {
    if (r.T == 0) return 0;
    if (r.T > ROUTE_BLOCK) return -1;
    const size_t smem = topk_smem_bytes(r.E, ROUTE_BLOCK) + dispatch_smem_bytes(p.E, p.k);
    if (set_smem(route_dispatch_kernel, smem)) return -1;
    launch_ex(pdl_active(), route_dispatch_kernel, dim3(copy_splits(1, p.T, p.k, num_sms)),
              dim3(ROUTE_BLOCK), smem, st, topk_args(r), dispatch_args(p), r.cnt);
    note_launch();
    return launch_result();
}

}  // namespace moe
