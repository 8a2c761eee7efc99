// plan.h -- host-side plan of one layer configuration: which kernels run,
// how expert segments are padded, and where each intermediate lives inside
// the caller's workspace.  A pure function of moe_config.
#pragma once

#include <stddef.h>
#include <stdint.h>

#include "../../include/moe.h"

namespace moe {

// How the expert FFN GEMMs are laid out.
enum FfnPath : int {
    PATH_TOKEN_MAJOR = 0,  // tensor cores, 128 tokens x 256 features per tile
    PATH_SWAP = 1,         // tensor cores, 128 weight rows x (tokens of one expert) per tile
    PATH_F32 = 2,          // fp32 SIMT (fp32 configs; no TF32)
};

// How the router logits are computed.
enum RouterKind : int {
    ROUTER_ROWS = 0,     // T <= 256: one CTA per token on the CUDA cores (fp32)
    ROUTER_TC = 1,       // bf16, T > 256: tensor-core GEMM against 3 bf16 parts of W_r
    ROUTER_SIMT = 2,     // fp32, T > 256: fp32 dot products on the CUDA cores
};

constexpr int ROUTE_BLOCK = 128;  // tokens per router / dispatch block
constexpr int TOPK_WARP_E = 32;   // above this many experts one warp routes one token
constexpr int TOPK_SUB = 4;       // ... and (batches above one block) a block's tokens are
                                  // routed by TOPK_SUB CTAs, each with its own partials
constexpr int MAX_E = 1024;
constexpr int MAX_K = 8;
constexpr int MAX_PEERS = 64;     // expert-parallel ranks one dispatch or combine addresses
constexpr int SWAP_MAX_TOKENS = 256;  // largest per-expert token count the swap path covers
constexpr int DOWN_SWAP_MAX_TOKENS = 128;  // above this the down projection takes token-major tiles
constexpr int PAIR_TOK_MIN_TOKENS = 1024;  // token-major tiles on CTA pairs from this group bound on
// int32 words of the workspace's 256-byte status area: [0] the status word,
// [1] the combine's ticket, [8..9] the CTA-pair kernels' unit counters (one per
// stream of a moe_forward: the routed experts', the shared experts')
constexpr int UNIT_CTR_WORD = 8;

struct Plan {
    int64_t T;
    int d, h, E, k, S, hs;
    int64_t C;          // capacity (T when unlimited)
    bool capped;
    bool reroute;       // overflow rerouted to a spare expert (else dropped)
    bool bf16;
    int act_bytes;
    int path;           // FfnPath for the routed experts
    int shared_path;    // FfnPath for the fused shared expert
    int pad;            // row padding of each expert segment in x_perm
    int nt_max;         // swap path: max tokens per expert, rounded up to 16
    int splits;         // split-K partials of the down projection
    int64_t perm_rows;  // rows of x_perm / each y_perm split
    int nblk;           // router blocks of ROUTE_BLOCK tokens
    int nsub;           // top-k CTAs per router block (1 or TOPK_SUB); the routing partials
                        // (histograms, P and entropy sums) are per CTA: nblk * nsub of them
    int hsum;           // S * hs (fused shared width)
    int router_kind;    // RouterKind
    int router_npad;    // tensor cores: padded GEMM width of the 3 bf16 parts of W_r
    int router_bn;      // tensor cores: tile width of the router GEMM
    int router_ld;      // tensor cores: row length of the partial logits (3E rounded to 4)
    int router_splits;  // tensor cores: split-K
    bool train;         // forward keeps the gate/up pre-activations for the backward pass
    bool split;         // H reaches the down projection as bf16 high + low parts
    int wr_chunks;      // backward: token chunks of the router-weight gradient

    // workspace byte offsets
    size_t off_status, off_logits, off_wsplit, off_z3, off_ppart, off_hpart, off_cnt, off_tot, off_expert, off_rank, off_offsets, off_perm,
        off_xperm, off_H, off_y, off_Hs, off_ys, off_sums, off_AB, off_ABs, total;
    // backward workspace byte offsets
    size_t b_dY, b_dg, b_dz, b_dAB, b_dXp, b_dABs, b_dXs, b_wrpart, b_dxr, b_total;
};

// Fills *p; returns MOE_OK or an error code with the message in *why.
int make_plan(const moe_config* cfg, Plan* p, const char** why);

}  // namespace moe
