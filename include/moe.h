/*
 * moe.h -- C ABI of the B200 (sm_100a) sparse top-k mixture-of-experts layer.
 *
 * The layer (pages: "Mixtral 8x7B and MoE explained: sparse mixture of
 * experts, only 2 experts active per token", section "Easy explanation";
 * "Mixture of experts" wiki entry, section "How it works"; "MoE routing fully
 * explained: the expert-mixture structure Mixtral and DeepSeek use, load
 * balancing, capacity factor", sections "Easy explanation" and "Main
 * insights") computes, for a batch x[T][d]:
 *
 *   z      = x W_r + b                      linear router, fp32 logits
 *   S_t    = the k largest z[t][.]          ties go to the lower expert index
 *   g[t,j] = softmax of z over S_t          gates over the kept k only
 *   C      = ceil(T k cf / E)               expert capacity (cf = inf: C = T)
 *   each expert keeps its first C assignments in token order; the rest drop
 *   out[t] = sum_{kept j} g[t,j] FFN_{S_t[j]}(x_t) + sum_s FFNshared_s(x_t)
 *   FFN(x) = (silu(x w1) * (x w3)) w2
 *   aux    = E sum_e f_e P_e,  f_e = routed_e / (T k),  P_e = mean_t softmax(z_t)_e
 *
 * Conventions for every call:
 *   - All pointers are DEVICE pointers unless stated; the caller owns every
 *     buffer.  The library never allocates device memory and never
 *     synchronises the stream (except moe_read_device_status, which says so).
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default).
 *   - Calls are asynchronous.  The return value reports host-side argument
 *     checks and launch errors only; nothing is launched when a check fails.
 *     A device-side error (a bounded wait that ran out) is recorded in the
 *     status word inside the workspace; read it with moe_read_device_status.
 *   - 16-byte alignment is required for every tensor pointer.
 *   - `ws`/`ws_bytes` is the caller's workspace of at least
 *     moe_workspace_size(cfg) bytes (else MOE_ERR_WORKSPACE).
 *   - Row-major layouts throughout.  "act" is the activation/weight dtype
 *     of the config (bf16 or fp32).
 *   - moe_last_error() returns a thread-local text for the last failing call.
 */
#ifndef MOE_B200_H
#define MOE_B200_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define MOE_API __attribute__((visibility("default")))
#else
#define MOE_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    MOE_OK = 0,
    MOE_ERR_ARG = 1,         /* null pointer or invalid scalar argument */
    MOE_ERR_SHAPE = 2,       /* unsupported sizes (see moe_config) */
    MOE_ERR_DTYPE = 3,       /* unsupported dtype */
    MOE_ERR_ALIGN = 4,       /* pointer not 16-byte aligned */
    MOE_ERR_WORKSPACE = 5,   /* workspace smaller than moe_workspace_size */
    MOE_ERR_CUDA = 6,        /* a CUDA runtime call or launch failed */
    MOE_ERR_TIMEOUT = 7,     /* a device-side bounded wait ran out (device status) */
    MOE_ERR_UNSUPPORTED = 8  /* no sm_100 device, or a feature not built */
} moe_status;

typedef enum { MOE_F32 = 0, MOE_BF16 = 1 } moe_dtype;

/* What happens to assignments beyond an expert's capacity [MoE routing fully
 * explained, "Easy explanation" ¶3 names three choices]:
 *   MOE_OVERFLOW_DROP     drop them (fast, loses their contribution)
 *   MOE_OVERFLOW_REROUTE  move each, in token order, to the token's
 *                         highest-scoring expert it does not already use that
 *                         still has room; it keeps its gate (else it drops)
 * The third choice, processing everything, is cf_den = 0 (no limit). */
typedef enum { MOE_OVERFLOW_DROP = 0, MOE_OVERFLOW_REROUTE = 1 } moe_overflow;

/* How the expert hidden activations H = silu(x w1) * (x w3) reach the down
 * projection in bf16 configs [the FFN's expand-then-contract, Mixtral 8x7B and
 * MoE explained, "Easy explanation" ¶2].  H is computed in fp32; rounding it
 * to bf16 alone costs about 2^-9 relative per element, which after the
 * h-long sum leaves the layer output about 0.8e-3 (relative L1) further from
 * the exact result than the bf16 store of the output does on its own.
 *   MOE_HIDDEN_AUTO   split (below) when no expert can keep more than 128
 *                     rows (min(C, T) <= 128): the down projection then
 *                     streams its weights through tiles of 128 weight rows x
 *                     the expert's tokens, and the extra MMAs run on tensor
 *                     cores that wait for HBM anyway; bf16 otherwise
 *   MOE_HIDDEN_SPLIT  H = H_hi + H_lo with H_hi = bf16(H), H_lo = bf16(H - H_hi)
 *                     (16 significant bits); the down projection issues two
 *                     MMAs per K step into one fp32 accumulator.  Costs 2 N d h
 *                     more tensor FLOPs (a third more per layer), N h 2 bytes
 *                     of workspace and their write and read.
 *   MOE_HIDDEN_BF16   H rounded to bf16: one MMA per K step, the fastest.
 * fp32 configs keep H in fp32 and ignore the field. */
typedef enum { MOE_HIDDEN_AUTO = 0, MOE_HIDDEN_SPLIT = 1, MOE_HIDDEN_BF16 = 2 } moe_hidden_mode;

/* Layer configuration.
 *   T         tokens in the batch (0 allowed: every call is a no-op that
 *             writes zero statistics)
 *   d         model width, multiple of 128
 *   h         routed-expert hidden width, multiple of 128
 *   E         routed experts, 1..1024
 *   k         experts kept per token, 1..min(E, 8)
 *   n_shared  shared experts applied to every token (0 = none); they are
 *             fused into one expert of width n_shared * h_shared
 *   h_shared  hidden width of each shared expert, multiple of 128
 *   cf_num / cf_den  capacity factor; cf_den == 0 means no capacity limit
 *   act_dtype MOE_BF16 (tensor-core path) or MOE_F32 (fp32 SIMT path; no TF32)
 *   has_bias  1 if the router has a bias vector b[E]
 *   overflow  moe_overflow (0 = drop)
 *   train     1: moe_forward also keeps in ws what moe_backward reads (the
 *             gate/up pre-activations, bf16); bf16 configs only.  The
 *             workspace grows accordingly (moe_workspace_size).
 *   hidden_mode  moe_hidden_mode (0 = auto)                               */
typedef struct {
    int64_t T;
    int32_t d, h, E, k, n_shared, h_shared;
    int64_t cf_num, cf_den;
    int32_t act_dtype;
    int32_t has_bias;
    int32_t overflow;
    int32_t train;
    int32_t hidden_mode;
} moe_config;

/* Routing statistics [MoE routing fully explained, "Easy explanation" ¶4 and
 * "Main insights" ¶3], written to DEVICE memory by moe_aux_stats.
 *   aux_loss       E * sum_e f_e P_e  (f from assignments before the capacity
 *                  limit; exactly 1 for perfectly even routing)
 *   overflow_rate  dropped assignments / (T k)
 *   mean_entropy   mean over tokens of -sum_e p ln p of the full softmax (nats)
 *   tokens, dropped  T and the dropped assignment count (as doubles)      */
typedef struct {
    double aux_loss;
    double overflow_rate;
    double mean_entropy;
    double tokens;
    double dropped;
} moe_stats;

/* ---- host-only helpers (no device work) -------------------------------- */

/* Expert capacity C = ceil(T k cf_num / (E cf_den)) in exact integer
 * arithmetic [MoE routing fully explained, "Easy explanation" ¶5: batch x
 * top-k x capacity factor / experts, e.g. 2048, 8, top-2, 1.25 -> 640].
 * cf_den == 0 gives C = T.  Writes *C; returns MOE_OK or MOE_ERR_ARG. */
MOE_API int moe_capacity(const moe_config* cfg, int64_t* C);

/* Bytes of device workspace every call below needs for this config (the same
 * buffer may be reused across calls with the same config).  Layout inside is
 * private; its first 256 bytes hold the device status word. */
MOE_API int moe_workspace_size(const moe_config* cfg, size_t* bytes);

/* Upper bound on the rows of the permuted (expert-sorted, padded) buffers
 * x_perm / y_perm that moe_dispatch and moe_expert_ffn use. */
MOE_API int moe_perm_rows(const moe_config* cfg, int64_t* rows);

/* Number of split-K partial buffers moe_expert_ffn writes into y_perm
 * (y_perm is [splits][moe_perm_rows][d] fp32). */
MOE_API int moe_ffn_splits(const moe_config* cfg, int32_t* splits);

/* *split = 1 if this config feeds the hidden activations to the down
 * projection as two bf16 parts (moe_hidden_mode: MOE_HIDDEN_SPLIT, or
 * MOE_HIDDEN_AUTO with min(C, T) <= 128; bf16 configs), else 0. */
MOE_API int moe_hidden_split(const moe_config* cfg, int32_t* split);

/* Text of the last failing call on this thread ("" if none). */
MOE_API const char* moe_last_error(void);

/* ---- layout transform -------------------------------------------------- */

/* Packs expert weights from the y = x W layout into the tensor-core layout.
 * which = 0 (routed): w1, w3 [E][d][h], w2 [E][h][d] ->
 *   W13 [E][2h][d]: for hidden block b (128 wide) rows 256b..256b+127 are
 *   columns 128b.. of w1 (gate) transposed, rows 256b+128.. the same columns
 *   of w3 (up); W2p [E][d][h] = w2 transposed (reduction dim contiguous).
 * which = 1 (shared): w1, w3 [S][d][hs], w2 [S][hs][d] are fused into one
 *   expert of width S*hs (hidden index s*hs + j) and packed the same way:
 *   W13 [2*S*hs][d], W2p [d][S*hs].
 * which = 2 (routed, backward layout; bf16): the transposes the backward
 *   GEMMs read, W13 <- W13t [E][d][2h] (row c holds w1[c][:] and w3[c][:] with
 *   the same 128-wide block interleave along 2h) and W2p <- W2t [E][h][d]
 *   (= w2, the model dim contiguous).
 * which = 3 (shared, backward layout; bf16): the fused shared expert the same
 *   way, W13t [d][2*S*hs] and W2t [S*hs][d].
 * All in act dtype.  Inputs are not modified.  Training re-packs after each
 * weight update (the packed tensors are the layer's parameters as stored). */
MOE_API int moe_pack_weights(const moe_config* cfg, int which, const void* w1, const void* w3,
                     const void* w2, void* W13, void* W2p, void* stream);

/* ---- the layer's steps ------------------------------------------------- */

/* Router [Mixtral explained, "Easy explanation" ¶3]: z = x W_r + b in fp32,
 * top-k per token (descending logit, ties to the lower index) and gates
 * softmax over the kept k.  Also writes the full-softmax partial sums used
 * by moe_aux_stats into ws.
 *   x [T][d] act; Wr [d][E] fp32; bias [E] fp32 (ignored unless has_bias)
 *   topk_idx [T][k] int32; topk_gate [T][k] fp32
 *   logits [T][E] fp32, optional (NULL = not written): the router logits z.
 * Precision: for bf16 batches of more than 256 tokens the logits run on the
 * tensor cores against W_r split into three bf16 parts (carrying W_r to 24
 * bits) with fp32 accumulation; otherwise as fp32 dot products.            */
MOE_API int moe_route(const moe_config* cfg, const void* x, const float* Wr, const float* bias,
              int32_t* topk_idx, float* topk_gate, float* logits, void* ws, size_t ws_bytes,
              void* stream);

/* Dispatch under capacity [MoE routing fully explained, "Easy explanation"
 * ¶3 and ¶5]: per-expert counts, stable rank of every assignment within its
 * expert by token index, truncation at C (overflow dropped), and the gather
 * of kept rows into expert-sorted order.  Needs ws from moe_route (block
 * histograms, which this call consumes: run moe_route before each dispatch).
 *   routed [E], kept [E] int32      assignments the router made / rows each
 *                                   expert serves (rerouted rows included)
 *   offsets [E+1] int32             first row of each expert in x_perm
 *                                   (segments padded for the tensor-core tiles)
 *   perm_token [moe_perm_rows] int32  token of each row (-1 in padding)
 *   slot_of [T][k] int32            row of x_perm holding (t, j), -1 if dropped
 *   x_perm [moe_perm_rows][d] act   gathered rows (padding rows undefined)   */
MOE_API int moe_dispatch(const moe_config* cfg, const int32_t* topk_idx, const void* x,
                 int32_t* routed, int32_t* kept, int32_t* offsets, int32_t* perm_token,
                 int32_t* slot_of, void* x_perm, void* ws, size_t ws_bytes,
                 void* stream);

/* Expert FFNs [Mixtral explained, "Easy explanation" ¶2 and ¶4]: for every
 * expert with kept tokens, H = silu(x_perm W1) * (x_perm W3) then y = H W2,
 * as grouped GEMMs on the tensor cores (bf16 in, fp32 accumulate, H stored
 * bf16); experts with no tokens are not read.  The shared experts (if any)
 * run on x directly.
 *   x_perm, offsets, kept  from moe_dispatch
 *   W13, W2p               packed routed weights; W13s, W2s packed shared
 *   y_perm [splits][moe_perm_rows][d] fp32  split-K partial outputs (ungated)
 *   y_shared [T][d] fp32   sum of the shared experts (may be NULL if none)  */
MOE_API int moe_expert_ffn(const moe_config* cfg, const void* x_perm, const int32_t* offsets,
                   const int32_t* kept, const void* W13, const void* W2p, const void* x,
                   const void* W13s, const void* W2s, float* y_perm, float* y_shared,
                   void* ws, size_t ws_bytes, void* stream);

/* Combine [Mixtral explained, "Easy explanation" ¶3; wiki, "How it works"]:
 * out[t] = sum_j gate[t][j] * (sum over splits of y_perm[.][slot_of[t][j]])
 * + y_shared[t], summed in fixed j order in fp32, stored in act dtype.
 *   out [T][d] act; must not alias x                                        */
MOE_API int moe_combine(const moe_config* cfg, const float* y_perm, const int32_t* slot_of,
                const float* topk_gate, const float* y_shared, void* out, void* stream);

/* Statistics [MoE routing fully explained, "Easy explanation" ¶4, "Main
 * insights" ¶3]: reduces the router partials in ws (fixed order, fp64) with
 * the counts into *stats (device).  Needs ws from moe_route. */
MOE_API int moe_aux_stats(const moe_config* cfg, const int32_t* routed, const int32_t* kept,
                  const void* ws, size_t ws_bytes, moe_stats* stats, void* stream);

/* Split form of moe_aux_stats for data-parallel use: moe_stats_sums writes
 * the additive sums [2 + 3E] doubles (T, entropy sum, P sums [E], routed [E],
 * kept [E]) to `sums` (device); after the caller has summed them across
 * ranks, moe_stats_finalize turns them into *stats. */
MOE_API int moe_stats_sums(const moe_config* cfg, const int32_t* routed, const int32_t* kept,
                   const void* ws, size_t ws_bytes, double* sums, void* stream);
MOE_API int moe_stats_finalize(const moe_config* cfg, const double* sums, moe_stats* stats,
                       void* stream);

/* The whole layer: moe_route, moe_dispatch, moe_expert_ffn, moe_combine and
 * moe_aux_stats in sequence on `stream`, with the intermediates in ws (the
 * shared experts may run on a second stream forked from and joined back into
 * `stream`, see moe_set_shared_overlap).  W13s/W2s may be NULL when
 * n_shared == 0; bias may be NULL when !has_bias; stats may be NULL to skip
 * the statistics.  The call reads nothing back to the host, so it can be
 * captured in a CUDA graph once one uncaptured call on the device has set the
 * kernels' attributes and created the second stream; every replay gives the
 * bits of an uncaptured call on the same inputs. */
MOE_API int moe_forward(const moe_config* cfg, const void* x, const float* Wr, const float* bias,
                const void* W13, const void* W2p, const void* W13s, const void* W2s,
                void* out, int32_t* topk_idx, float* topk_gate, int32_t* routed,
                int32_t* kept, int32_t* slot_of, moe_stats* stats, void* ws, size_t ws_bytes,
                void* stream);

/* ---- backward pass ------------------------------------------------------ */

/* Bytes of the second workspace moe_backward needs for this config. */
MOE_API int moe_backward_workspace_size(const moe_config* cfg, size_t* bytes);

/* Gradients of the layer [the softmax weighting and the load-balancing loss
 * the pages describe are what training acts on: MoE routing fully explained,
 * "Easy explanation" ¶2 and ¶4] for the loss
 *   L = sum_t <grad_out_t, out_t> + aux_coef * aux_loss,
 * after a moe_forward of the same batch with cfg->train = 1 (bf16 only).
 * Readings: the top-k choice, the capacity decision and the routed counts f_e
 * are piecewise constant and carry no gradient (aux reaches the router
 * through P_e); gates are not renormalised after a drop, so a dropped
 * assignment has gate gradient 0 but its logit still receives the
 * softmax-over-k terms; under reroute the gate gradient goes to the router's
 * chosen expert while the serving expert's FFN is differentiated.
 * Inputs:
 *   grad_out [T][d] act dtype; aux_coef the weight of the aux loss
 *   x, Wr, bias        the forward's inputs (bias ignored unless has_bias)
 *   W13t, W2t          routed weights in the backward layout (pack which = 2)
 *   W13st, W2st        shared expert, backward layout (pack which = 3), or NULL
 *   topk_idx, topk_gate, routed, kept, slot_of   the forward's outputs
 *   ws, ws_bytes       the forward's workspace, unchanged since that call
 * Outputs (device, fp32, overwritten):
 *   dx [T][d]; dWr [d][E]; db [E] (NULL allowed; written only with has_bias);
 *   dW13 [E][2h][d] and dW2p [E][d][h] in the forward packed layout (which = 0);
 *   dW13s [2*S*hs][d], dW2s [d][S*hs] (shared; NULL when n_shared == 0);
 *   dlogits [T][E] (optional, NULL = not written): dL/dz.
 * bws, bws_bytes: the backward workspace (moe_backward_workspace_size),
 * 256-byte aligned.  Asynchronous on `stream`; bounded waits record
 * MOE_ERR_TIMEOUT in ws's status word like the forward. */
MOE_API int moe_backward(const moe_config* cfg, const void* grad_out, float aux_coef,
                         const void* x, const float* Wr, const float* bias, const void* W13t,
                         const void* W2t, const void* W13st, const void* W2st,
                         const int32_t* topk_idx, const float* topk_gate,
                         const int32_t* routed, const int32_t* kept, const int32_t* slot_of,
                         void* ws, size_t ws_bytes, float* dx, float* dWr, float* db,
                         float* dW13, float* dW2p, float* dW13s, float* dW2s, float* dlogits,
                         void* bws, size_t bws_bytes, void* stream);

/* ---- expert parallelism --------------------------------------------------- */

/* Building blocks of the layer with its experts partitioned across G ranks
 * [Mixtral explained, "Easy explanation" ¶4 and MoE routing fully explained,
 * ¶3: experts spread over GPUs, tokens sent to the GPU that holds their
 * expert].  The reading the library implements: G ranks with their own
 * batches together compute exactly the single-GPU layer on the concatenated
 * batch (rank 0's tokens first): capacity C = ceil(T_all k cf / E) and the
 * arrival order run over the whole concatenation.  A rank calls moe_route on
 * its batch (with a local config whose cf_den = 0), exchanges the per-expert
 * counts (moe_route_counts), keeps for expert e at most
 * cap[e] = C - (assignments to e on lower ranks) with moe_dispatch_capped,
 * sends each expert's rows to its owner, which runs moe_expert_ffn_grouped on
 * the (source rank, expert) groups it received, and gets the output rows back
 * for moe_combine.  The exchanges live in the Python package (ep.py); the
 * plan (caps, where each rank's rows land, the groups an owner receives) is
 * either computed there on the host or on the device by moe_ep_plan. */

/* Row padding of each expert segment in x_perm for this config (the
 * receiver of a segment needs it to find the next one). */
MOE_API int moe_segment_pad(const moe_config* cfg, int32_t* pad);

/* counts[e] (device int32 [E]) = assignments of the batch to expert e,
 * before any capacity limit.  Call after moe_route and before any dispatch
 * on the same ws (dispatch consumes the router's histograms). */
MOE_API int moe_route_counts(const moe_config* cfg, const void* ws, size_t ws_bytes,
                             int32_t* counts, void* stream);

/* moe_dispatch with a per-expert capacity: expert e keeps the first
 * min(C, cap[e]) of the batch's assignments to it (token order); cap is
 * device int32 [E] (negative counts as 0).  Drop policy only. */
MOE_API int moe_dispatch_capped(const moe_config* cfg, const int32_t* topk_idx, const void* x,
                                const int32_t* cap, int32_t* routed, int32_t* kept,
                                int32_t* offsets, int32_t* perm_token, int32_t* slot_of,
                                void* x_perm, void* ws, size_t ws_bytes, void* stream);

/* The expert-parallel plan of rank `rank` of `world`, on the device, from
 * counts (device int32 [world][E]: every rank's moe_route_counts, gathered in
 * rank order) and the capacity C of the whole concatenated batch [MoE routing
 * fully explained, "Easy explanation" ¶5]; cfg is the rank's local config
 * (its segment padding is used).  With base[s][e] = sum of counts[s'][e] over
 * s' < s, rank s keeps kept[s][e] = min(counts[s][e], max(C - base[s][e], 0))
 * rows of expert e in a segment of seg[s][e] = kept rounded up to the padding:
 *   cap [E]            max(C - base[rank][e], 0): moe_dispatch_capped's cap
 *   row_start [world]  for owner q, the rows lower ranks send to q (the
 *                      segments of q's experts): where this rank's rows begin
 *                      in q's receive and output buffers
 *   group_rows / group_off / group_weight [world * E/world]  the (source,
 *                      local expert) groups this rank receives, sources in
 *                      order, then experts: kept rows, first row, expert
 *   recv_rows [1]      the rows this rank receives (padded)
 * all device int32.  Nothing is read back to the host, so a step of the
 * peer-memory form needs no host synchronisation.  Errors: world out of
 * range or not dividing E, rank out of range, C < 0, a NULL or misaligned
 * pointer; reported before any launch. */
MOE_API int moe_ep_plan(const moe_config* cfg, int32_t world, int32_t rank,
                        const int32_t* counts, int64_t C, int32_t* cap, int32_t* row_start,
                        int32_t* group_rows, int32_t* group_off, int32_t* group_weight,
                        int32_t* recv_rows, void* stream);

/* Workspace of moe_expert_ffn_grouped for `rows` input rows. */
MOE_API int moe_grouped_workspace_size(const moe_config* cfg, int64_t rows,
                                       int32_t max_group_rows, size_t* bytes);

/* The expert FFN (as moe_expert_ffn, bf16) over explicit groups of rows:
 * group g is rows group_off[g] .. + group_rows[g] of x_rows [rows][d] and uses
 * expert group_weight[g] of W13 / W2p (packed as moe_pack_weights which = 0,
 * holding however many experts the caller owns; every index must be below
 * that count).  All three arrays are device int32 [n_groups]; max_group_rows
 * (host) bounds every group_rows[g] -- a larger one is clamped and
 * MOE_ERR_SHAPE recorded in ws's status word.  y_rows [rows][d] fp32 receives
 * the outputs of the group rows (other rows are not written). */
MOE_API int moe_expert_ffn_grouped(const moe_config* cfg, const void* x_rows, int64_t rows,
                                   int32_t n_groups, const int32_t* group_rows,
                                   const int32_t* group_off, const int32_t* group_weight,
                                   int32_t max_group_rows, const void* W13, const void* W2p,
                                   float* y_rows, void* ws, size_t ws_bytes, void* stream);

/* moe_combine with the expert outputs in one fp32 buffer y_rows [rows][d]
 * (no split-K partials), e.g. as returned by the expert owners: out[t] =
 * sum over kept j of gate * y_rows[slot_of[t][j]] (+ y_shared[t]). */
MOE_API int moe_combine_rows(const moe_config* cfg, const float* y_rows, const int32_t* slot_of,
                             const float* topk_gate, const float* y_shared, void* out,
                             void* stream);

/* Expert parallelism over peer memory: the same step with the two
 * exchanges folded into the dispatch and the combine.  World ranks, rank q
 * owning experts q * E_loc .. (q + 1) * E_loc - 1 (E_loc = E / world).
 *
 * moe_dispatch_peers is moe_dispatch_capped whose row copies go straight to
 * the owners: the kept rows of expert e (owner q = e / E_loc) are written,
 * segment by segment as moe_dispatch_capped lays them out in x_perm, starting
 * at row dst_row_start[q] of dst_rows[q] -- rank q's receive buffer, where
 * this rank's rows begin after the rows that lower ranks send to q.
 * dst_rows is a host array of `world` device pointers (16-byte aligned,
 * [rows][d] of the activation type), each this GPU's memory or a peer's
 * mapped into this process (CUDA IPC, symmetric memory); the kernel stores
 * through them over NVLink.  dst_row_start is device int32 [world] (e.g.
 * moe_ep_plan's row_start), or NULL when dst_rows[q] already point at this
 * rank's first row.  offsets, slot_of and perm_token keep their local
 * (x_perm) meaning.  The caller orders the stores before the owners read
 * them (a stream-ordered barrier across the ranks).
 *
 * moe_combine_peers is moe_combine_rows with each output row read from its
 * owner: y_rows is a host array of `world` device pointers, y_rows[q] = rank
 * q's fp32 output rows [rows][d], this rank's rows from row y_row_start[q]
 * on (device int32 [world], or NULL = 0); topk_idx and offsets are this
 * rank's, from the dispatch.  1 <= world <= MOE_MAX_PEERS, E % world == 0;
 * drop policy; the dispatch takes bf16 activations (MOE_ERR_DTYPE
 * otherwise).  Errors: bad world, a NULL or misaligned pointer, or a reroute
 * config are reported before any launch. */
#define MOE_MAX_PEERS 64
MOE_API int moe_dispatch_peers(const moe_config* cfg, const int32_t* topk_idx, const void* x,
                               const int32_t* cap, int32_t world, void* const* dst_rows,
                               const int32_t* dst_row_start, int32_t* routed, int32_t* kept,
                               int32_t* offsets, int32_t* perm_token, int32_t* slot_of, void* ws,
                               size_t ws_bytes, void* stream);
MOE_API int moe_combine_peers(const moe_config* cfg, int32_t world, const float* const* y_rows,
                              const int32_t* y_row_start, const int32_t* topk_idx,
                              const int32_t* offsets, const int32_t* slot_of,
                              const float* topk_gate, const float* y_shared, void* out,
                              void* stream);

/* ---- routing without a workspace ----------------------------------------- */

/* The pages have no counterpart to this call; it exists for callers that
 * cannot allocate device memory: code running inside a framework whose
 * allocator they do not control, a plugin handed only its input and output
 * buffers, or a process that must not grow its device footprint after it
 * starts.  moe_route_static computes exactly what moe_route computes (same
 * kernels, same results: topk_idx [T][k] int32 and topk_gate [T][k] fp32) but
 * takes no workspace and allocates nothing.  Its scratch (the logits and the
 * statistics partials) is a file-scope device array of
 * MOE_ROUTE_STATIC_SCRATCH bytes inside the library, held by a GPU from the
 * first call on it until the process exits.  Limits: T <= MOE_ROUTE_STATIC_MAX_T
 * and T * E <= MOE_ROUTE_STATIC_MAX_TE, else MOE_ERR_SHAPE.  The first call on a
 * device looks up the array's device address (cudaGetSymbolAddress); under
 * CUDA's lazy module loading (the default) that is also when the array is
 * placed on the device, so a caller whose device footprint must not grow later
 * makes one warm-up call per device at start-up, and that first call should
 * come before any stream capture.  The address is looked up again when the
 * device's context changes (after cudaDeviceReset).  All calls share the
 * array and each call overwrites what the last one left; calls that overlap on
 * the GPU race, so the caller must serialise them (one stream, or events
 * between streams). */
#define MOE_ROUTE_STATIC_SCRATCH (512u * 1024u)
#define MOE_ROUTE_STATIC_MAX_T 256
#define MOE_ROUTE_STATIC_MAX_TE 65536
MOE_API int moe_route_static(const moe_config* cfg, const void* x, const float* Wr,
                             const float* bias, int32_t* topk_idx, float* topk_gate,
                             void* stream);

/* ---- status, tracing, limits ------------------------------------------- */

/* Copies the device status word from ws to *status (MOE_OK or
 * MOE_ERR_TIMEOUT) and clears it.  This call synchronises `stream`. */
MOE_API int moe_read_device_status(const void* ws, int32_t* status, void* stream);

/* Kernels this library has launched since it was loaded, over all threads
 * and devices (a running count; the difference of two reads counts the
 * launches in between). */
MOE_API int moe_launch_count(uint64_t* n);

/* Programmatic dependent launch inside moe_forward (default on): the
 * kernels of the layer's chain may start while their predecessor finishes,
 * each waiting on the device before it reads what the predecessor writes, and
 * the swapped gate/up GEMM prefetches its first weight tiles into L2 while the
 * routing runs.  Results are identical either way.  Process-wide. */
MOE_API int moe_set_pdl(int on);

/* Expert GEMM tiles on pairs of SMs (a cluster of two CTAs running one
 * tcgen05 MMA, M = 256, each SM staging half of A and half of B), process-wide:
 *   0  one SM per tile everywhere
 *   1  (default) token-major tiles of 256 tokens x 256 features on SM pairs
 *      for expert groups that may hold >= 1024 rows (the large prefill layer,
 *      a shared expert over a long batch): a third less shared-memory fill per
 *      flop than the one-SM 128 x 256 tile; and the down projection of groups
 *      of 129..256 tokens (one pair tile per 256 output features, each weight
 *      row read once)
 *   2  also the swapped gate/up and down tiles (weight rows x tokens) of
 *      experts that keep 129..256 tokens on SM pairs -- measured level with
 *      one SM per tile on the DeepSeek-V2-style layer (its gate/up within 2 %,
 *      the layer slightly slower), so off by default
 * Results are identical in every mode (the fp32 sums run in the same order).
 * MOE_ERR_ARG for another value. */
MOE_API int moe_set_pair_tiles(int mode);

/* Shared experts beside the routed ones in moe_forward (default on): they
 * need only x, so they run on a second stream (one per device, created by the
 * library on first use) from the start of the call, beside the routing and
 * the routed experts, and the combine waits for them; the call still returns
 * with all its work ordered on `stream`.  Calls from several threads on one
 * device share that second stream.  Off: one stream, shared experts after the
 * routed ones.  Results are identical either way.  Process-wide. */
MOE_API int moe_set_shared_overlap(int on);

/* SMs set aside for the shared experts while they overlap the routed ones
 * (default 0: none).  With sms > 0, moe_forward launches the shared experts'
 * GEMMs with grids of `sms` SMs and the routed experts' GEMMs with grids of
 * the rest, so that the HBM-bound routed GEMMs and the compute-bound shared
 * ones run side by side instead of the second starting in the tail of the
 * first.  Applies only when the overlap is on, the layer has shared experts
 * and at least 32 SMs remain for the routed ones; the block scheduler decides
 * where the CTAs land, so this shapes the grids, it does not pin SMs.  Results
 * are identical for every value.  MOE_ERR_ARG unless sms is even and in
 * [0, 1024].  Process-wide. */
MOE_API int moe_set_shared_sms(int sms);

/* Upper bound, in nanoseconds, on every device-side wait of the tensor-core
 * kernels (default 2e9).  A wait that runs out records MOE_ERR_TIMEOUT in
 * the device status word and its kernel returns early.  Process-wide. */
MOE_API int moe_set_wait_limit_ns(uint64_t ns);

/* Test hook for the time-out path (off by default).  When on, in every expert
 * FFN GEMM launch work unit 0 (whichever CTA or CTA pair takes it) withholds
 * its "accumulator ready" signal, so that its epilogue wait can only run out:
 * after the wait limit (set a short one with moe_set_wait_limit_ns) the
 * kernel records MOE_ERR_TIMEOUT, drains its in-flight copies and MMAs,
 * releases tensor memory and returns.  Results of such a call are garbage;
 * the device stays usable.  Process-wide. */
MOE_API int moe_set_test_stall(int on);

/* Per-kernel timing of moe_forward.  moe_trace_begin(n, only) records CUDA
 * events for up to n moe_forward calls: with only == NULL, one event after
 * every kernel launch (each kernel is timed from the end of the previous
 * one); with only naming a kernel (e.g. "gemm_gateup"), one event before and
 * one after that kernel alone.  moe_trace_end synchronises and writes, per
 * kernel, its name, launch count and summed milliseconds (up to cap entries;
 * *n_out = entries written).  Process-wide; not thread-safe. */
MOE_API int moe_trace_begin(int max_calls, const char* only);
MOE_API int moe_trace_end(char (*names)[32], int* launches, double* ms, int cap, int* n_out);

#ifdef __cplusplus
}
#endif
#endif /* MOE_B200_H */
