// kernels.h -- internal launchers of the MoE library's CUDA kernels.
// Each returns 0 on a successful launch, -1 otherwise.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace moe {

// Counts one kernel launch (every launch site calls it; moe_launch_count).
void note_launch();

// The calling thread's error of its last failed launch (cudaSuccess if none).
cudaError_t& last_launch_error();

// True while moe_forward launches its kernels on this thread: the kernels of
// its chain are then launched with programmatic stream serialization (they
// call pdl_wait() before touching memory their predecessor writes).
bool pdl_active();

// Launches `kern`, with programmatic stream serialization when `pdl` is set.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_ex(bool pdl, void (*kern)(KArgs...), dim3 grid, dim3 block,
                             size_t smem, cudaStream_t st, Args... args) {
    cudaLaunchConfig_t c = {};
    c.gridDim = grid;
    c.blockDim = block;
    c.dynamicSmemBytes = smem;
    c.stream = st;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[0].val.programmaticStreamSerializationAllowed = 1;
    c.attrs = pdl ? at : nullptr;
    c.numAttrs = pdl ? 1 : 0;
    return cudaLaunchKernelEx(&c, kern, args...);
}

// 0 if the launches so far succeeded; else records the error and returns -1.
inline int launch_result() {
    const cudaError_t e = cudaGetLastError();
    if (e == cudaSuccess) return 0;
    last_launch_error() = e;
    return -1;
}

// ---------------------------------------------------------------- router
// logits z[T][E] = x[T][d] Wr[d][E] on the CUDA cores (fp32 accumulate, no bias)
int launch_router_logits(const void* x, bool x_bf16, const float* Wr, float* z, int64_t T, int d,
                         int E, int num_sms, cudaStream_t st);
// small batches: z[T][E] = x W_r (no bias), one CTA per (token, 8 experts)
int launch_router_rows(const void* x, bool x_bf16, const float* Wr, float* z, int T, int d,
                       int E, cudaStream_t st);
// W_r [d][E] fp32 -> three bf16 parts, K-major: Ws[p*E + e][d]
int launch_router_split(const float* Wr, void* Ws, int d, int E, cudaStream_t st);
// z[t][e] = bias[e] + sum_s sum_p src[s*split_stride + t*row_stride + p*E + e]
int launch_router_reduce(const float* src, int nsplit, int64_t split_stride, int row_stride,
                         int nparts, const float* bias, float* z, int64_t T, int E,
                         cudaStream_t st);

// ---------------------------------------------------------------- top-k and dispatch
struct RouteParams {
    const float* src;       // router logits without bias [T][E]
    const float* bias;      // may be null
    float* zbuf;            // [T][E] scratch (may equal src)
    float* logits;          // optional copy of the logits for the caller
    int64_t T;
    int E, k;
    int32_t* topk_idx;      // [T][k]
    float* topk_gate;       // [T][k]
    float* ppart;           // [blocks * nsub][E] full-softmax partial sums
    float* hpart;           // [blocks * nsub] entropy partial sums
    int32_t* cnt;           // [blocks * nsub][E] histogram of kept-expert choices
    int32_t* status;        // device status word (+ combine ticket)
    int nsub;               // top-k CTAs per block of ROUTE_BLOCK tokens (E > TOPK_WARP_E)
};

struct DispatchParams {
    int64_t T;
    int E, k;
    int64_t C;
    int pad;
    int64_t perm_rows;
    const void* x;
    int row_bytes;
    int32_t* routed;
    int32_t* kept;
    int32_t* offsets;
    int32_t* perm_token;    // may be null
    int32_t* slot_of;
    void* x_perm;
    const int32_t* cap;     // device [E] per-expert capacity (min with C), or null
    int nsub;               // histogram rows per block of ROUTE_BLOCK tokens (see RouteParams)
    // Destinations of the row copies.  npeer == 0: x_perm, row = slot.  Else
    // expert e's rows go to rank o = e / e_loc: row (slot - offsets[o * e_loc])
    // of peer_rows[o] (a host array of npeer device pointers, read at launch).
    void* const* peer_rows;
    int npeer, e_loc;
    const int32_t* peer_start;  // device [npeer]: rows to skip at each destination, or null
};

int launch_topk(const RouteParams& r, cudaStream_t st);
// counts[e] = routed assignments of the batch to expert e, from the top-k
// histograms cnt [blocks][E] (before dispatch turns them into prefixes)
int launch_route_counts(const int32_t* cnt, int nblk, int E, int32_t* counts, cudaStream_t st);
// cnt [blocks][E] is turned in place into exclusive prefixes over blocks;
// tot [E] receives the totals
int launch_dispatch(const DispatchParams& p, const int32_t* topk_idx, int32_t* cnt, int32_t* tot,
                    int num_sms, cudaStream_t st);
// Reroute policy: ranks, then dropped assignments moved in token order to the
// token's best unused expert with room (z = logits with bias), then slots and
// row copies.  expert_of / rank_of [T][k] receive the serving expert and rank.
int launch_reroute_dispatch(const DispatchParams& p, const int32_t* topk_idx, int32_t* cnt,
                            int32_t* tot, const float* z, int32_t* expert_of, int32_t* rank_of,
                            int num_sms, cudaStream_t st);
// T <= 128: top-k and dispatch in one launch
int launch_route_dispatch(const RouteParams& r, const DispatchParams& p, int num_sms,
                          cudaStream_t st);

// ---------------------------------------------------------------- tensor-core GEMMs
// One persistent CTA per SM: a TMA producer warp, an MMA-issuing warp and the
// epilogue warps (four; sixteen for the swapped gate/up, whose accumulator is
// single-buffered for wide token tiles).  The down projection takes the
// swapped tiles only while every group fits 128 tokens.
enum TcMode : int {
    TC_GATEUP_TOK = 0,   // H = silu(A w1) * (A w3), token-major tiles
    TC_DOWN_TOK = 1,     // y = A W^T (fp32), token-major tiles, optional split-K
    TC_GATEUP_SWAP = 2,  // gate/up with weight rows as M (few tokens per group)
    TC_DOWN_SWAP = 3,    // down with weight rows as M, split-K
    TC_DGATE_TOK = 4,    // backward: dH = dY W2^T, SiLU*mul backward in the epilogue
    TC_WGRAD = 5,        // backward: C[g] = A[:, K_g] B[:, K_g]^T over each group's token range
    TC_PAIR_GATEUP = 6,  // gate/up on CTA pairs: 2 x (64 gate + 64 up weight rows) x the tokens
    TC_PAIR_DOWN = 7,    // down on CTA pairs: 2 x 128 weight rows x the tokens (fp32 out)
    TC_PAIR_GATEUP_TOK = 8,  // gate/up on CTA pairs, token-major: 2 x 128 tokens x 256
    TC_PAIR_DOWN_TOK = 9,    // down on CTA pairs, token-major: 2 x 128 tokens x 256 (fp32 out)
    TC_PAIR_DGATE_TOK = 10,  // backward dgate on CTA pairs, token-major: 2 x 128 tokens x 256
};

struct TcArgs {
    int num_groups;
    const int32_t* group_rows;  // device [num_groups] valid rows, or nullptr -> dense_rows
    const int32_t* group_off;   // device [num_groups] first row, or nullptr -> 0
    int dense_rows;
    int K;                      // reduction length
    int n_feat;                 // gate/up: hidden width; down: model width
    int w_rows_per_group;       // weight rows per group (gate/up: 2h; down: d)
    int splits;                 // split-K (down projection / router; 1 for gate/up)
    int nt_max;                 // swapped: max tokens per group, multiple of 16
    int stages;                 // shared-memory pipeline depth
    void* out;                  // H (bf16) or y (fp32)
    int64_t out_ld;             // elements per output row
    int out_cols;               // token-major down: columns written (0 = all)
    int64_t split_stride;       // elements between split-K partial outputs
    int32_t* status;            // device status word
    uint64_t wait_limit_ns;
    int test_stall;             // test hook: CTA 0 withholds its first accumulator-ready signal
    void* aux;                  // gate/up: pre-activation output AB (bf16, may be null);
                                // dgate: AB input
    int64_t aux_ld;             // elements per AB row (2 x hidden width)
    int m_rows;                 // wgrad: rows of A (output rows per group)
    int64_t group_stride;       // wgrad: elements between the groups' outputs
    int n_fastest;              // wgrad: consecutive units step through N tiles first
    const int32_t* group_w;     // device [num_groups] weight index of each group, or null -> g
    int prefetch_kb;            // swapped gate/up: k-blocks of the first weight tile to prefetch
                                // into L2 before waiting on the predecessor (0: none)
    int32_t* unit_ctr;          // CTA-pair kernels: device counter the pairs take their units
                                // from (zero at launch)
    int64_t lo_rows;            // H as bf16 high + low parts (0: bf16 H alone): gate/up writes
                                // row r's low parts to row r + lo_rows of `out`; down reads
                                // them there from the activation tensor and issues a second
                                // MMA per K step into the same accumulator
};

// Token rows per TMA box of the swapped gate/up (TC_GATEUP_SWAP): nt_max up to
// 64, else 64, so that a stage of up to 256 token rows takes at most four copies
// (a copy's fixed cost, not its bytes, bounds a stage of many 16-row boxes).
// The tensor map of the token rows must use this box height; a stage's token
// region holds nt_max rows rounded up to a whole box.  Rows of a group's last
// box past its tokens are the next group's (or the zero fill past the tensor)
// and lie outside the MMA's N columns.
__host__ __device__ inline int swap_gateup_tok_box(int nt_max) { return nt_max < 64 ? nt_max : 64; }

// The same for the swapped CTA-pair tiles (TC_PAIR_GATEUP, TC_PAIR_DOWN), where
// each CTA stages half of a unit's token rows: nt_max / 2 up to 64, else 64.
__host__ __device__ inline int pair_swap_tok_box(int nt_max) {
    return nt_max / 2 < 64 ? nt_max / 2 : 64;
}

// Deepest pipeline (2..8 stages) whose shared memory fits smem_limit; `split`
// sizes the down projection's stages for H's two parts.
int tc_max_stages(int mode, int bn, int nt_max, int groups, bool split, int smem_limit);
int launch_tc_gemm(int mode, int bn, const CUtensorMap& act, const CUtensorMap& w,
                   const TcArgs& a, int grid, cudaStream_t st);

// Tiles on CTA pairs (clusters of two; gemm_pair.cu).  Swapped, for groups of up
// to 256 tokens: TC_PAIR_GATEUP (act = x rows, pair_swap_tok_box rows; w = W13, 64-row
// boxes; n_feat = hidden width) and TC_PAIR_DOWN (act = H rows, pair_swap_tok_box rows;
// w = W2p, 128-row boxes; n_feat = model width, a multiple of 256); nt_max is a
// multiple of 16 in [16, 256].  Token-major, for groups of any size:
// TC_PAIR_GATEUP_TOK, TC_PAIR_DOWN_TOK and the backward TC_PAIR_DGATE_TOK (act =
// dY rows, w = W2t, aux = AB, out = dAB; n_feat a multiple of 256) with act and
// w both in 128-row boxes.  The
// grid is `pairs` clusters of two CTAs (one per two SMs); the pairs take their
// units from a counter, so pairs that are not resident at once only start
// later and find less work.
int tc_pair_max_stages(int mode, int nt_max, int groups, bool split, int smem_limit);
int launch_tc_pair(int mode, const CUtensorMap& act, const CUtensorMap& w, const TcArgs& a,
                   int pairs, cudaStream_t st);

// ---------------------------------------------------------------- fp32 SIMT FFN
// gate/up: H[r][f] = silu(A_r . W13[g][gate f]) * (A_r . W13[g][up f]);
// down: Y[r][o] = H_r . W2p[g][o].  Groups as in TcArgs.
int launch_f32_gateup(const float* A, const float* W13, float* H, int num_groups,
                      const int32_t* group_rows, const int32_t* group_off, int dense_rows,
                      int64_t rows_bound, int d, int h, cudaStream_t st);
int launch_f32_down(const float* H, const float* W2p, float* Y, int num_groups,
                    const int32_t* group_rows, const int32_t* group_off, int dense_rows,
                    int64_t rows_bound, int d, int h, cudaStream_t st);

// ---------------------------------------------------------------- combine / stats / pack
struct StatsParams {
    const float* ppart;     // [nblk][E]
    const float* hpart;     // [nblk]
    int nblk;
    const int32_t* routed;  // [E]
    const int32_t* kept;    // [E]
    int64_t T;
    int E, k;
    double* sums;           // [2 + 3E]: T, entropy sum, P sums, routed, kept
    void* stats;            // moe_stats, or null for the sums alone
};

// out[t] = sum_j gate * sum_s y[s][slot] + y_shared[t]; with sp, one more block
// computes the statistics in the same launch
// out[t] = sum over kept j of gate * y row of (t, j) (+ y_shared[t]), the y
// row found at the expert's owner: expert e = topk_idx[t][j] belongs to rank
// o = e / e_loc, and its row is slot - offsets[o * e_loc] of y_rows[o] (a host
// array of npeer device pointers, read at launch).
// y_start (device [npeer], or null) skips that many rows at each owner first.
int launch_combine_peers(const float* const* y_rows, const int32_t* y_start, int npeer,
                         int e_loc, const int32_t* topk_idx, const int32_t* offsets,
                         const int32_t* slot_of, const float* gate, const float* y_shared,
                         void* out, bool out_bf16, int64_t T, int d, int k, cudaStream_t st);

// Expert-parallel plan of rank `rank` of G from the gathered counts [G][E]
// (device), all on the device: cap [E], row_start [G] (rows of lower ranks
// at each owner), and the (source, local expert) groups this rank receives:
// g_rows, g_off, g_w [G * E/G], recv [1] their padded total.
int launch_ep_plan(const int32_t* counts, int G, int E, int rank, int64_t C, int pad,
                   int32_t* cap, int32_t* row_start, int32_t* g_rows, int32_t* g_off,
                   int32_t* g_w, int32_t* recv, cudaStream_t st);
int launch_combine(const float* y, int splits, int64_t split_stride, const int32_t* slot_of,
                   const float* gate, const float* y_shared, void* out, bool out_bf16,
                   int64_t T, int d, int k, const StatsParams* sp, cudaStream_t st);
int launch_stats(const StatsParams& a, cudaStream_t st);
int launch_stats_finalize(const double* sums, int E, int k, void* stats, cudaStream_t st);
// dst[remap(c)][r + row_off] = src[r][c] for a [R][Cc] source; remap interleaves
// 128-wide hidden blocks (gate/up) when `interleave` >= 0 (0 = gate, 1 = up).
// n independent matrices: src + i * src_stride -> dst + i * dst_stride, and the
// hidden column offset grows by col_step per matrix (fused shared experts)
int launch_pack(const void* src, void* dst, int elem_bytes, int R, int Cc, int64_t ld_dst,
                int col_off, int interleave, int n, int64_t src_stride, int64_t dst_stride,
                int col_step, cudaStream_t st);

// ---------------------------------------------------------------- backward pass
// dY[slot] = gate * G[t] (bf16) for every kept slot; dg[t][j] = <G[t], y[slot]>
// (y summed over its split-K partials), 0 for dropped assignments
int launch_bwd_gather(const void* G, const float* y, int splits, int64_t split_stride,
                      const int32_t* slot_of, const float* gate, void* dY, float* dg, int64_t T,
                      int d, int k, int num_sms, cudaStream_t st);
// dz[t][e] = softmax-over-k backward of dg + aux_coef (E/T) p (f - sum f p);
// z are the forward logits, bias added here when given
int launch_router_bwd(const float* z, const float* bias, const int32_t* idx, const float* gate,
                      const float* dg, const int32_t* routed, float aux_coef, float* dz, int64_t T,
                      int E, int k, int num_sms, cudaStream_t st);
// token chunks of the router-weight gradient (partials [chunks][d + 1][E])
int wr_grad_chunks(int64_t T, int d, int E);
// dWr = x^T dz, db = column sums of dz (db may be null)
int launch_wr_grad(const void* x, const float* dz, float* part, float* dWr, float* db, int64_t T,
                   int d, int E, cudaStream_t st);
struct PadJob {
    void* buf;              // bf16 [rows][width], width a multiple of 8
    int width;
};
struct PadJobs {
    PadJob job[4];
    int n;
    const int32_t* off;     // device [groups] segment starts
    const int32_t* rows;    // device [groups] rows in use
    int groups;
};
// zeroes rows [off[g] + rows[g], off[g] + rows[g] rounded up to 64) of each buffer
int launch_zero_pad(const PadJobs& p, cudaStream_t st);
// dx[t] = sum over kept slots of dXp[slot] + dXs[t] (may be null) + sum_e dz[t][e] Wr[:, e];
// dxr [T][d] is scratch for the router's share when E > 16
int launch_combine_bwd(const float* dXp, const int32_t* slot_of, const float* dXs,
                       const float* dz, const float* Wr, float* dxr, float* dx, int64_t T, int d,
                       int k, int E, cudaStream_t st);
// dst[r][col(c)] = src[r][c], bf16, no transpose (backward weight layout)
int launch_pack_cols(const void* src, void* dst, int R, int Cc, int64_t ld_dst, int col_off,
                     int interleave, int n, int64_t src_stride, int64_t dst_stride, int col_step,
                     cudaStream_t st);

}  // namespace moe
