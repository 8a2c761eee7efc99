// gemm_tc.cu -- grouped expert GEMMs on the sm_100a tensor cores.
//
// The expert FFN [Mixtral 8x7B and MoE explained, "Easy explanation" ¶2: each
// expert widens the ~4k embedding to a ~14k hidden size and narrows it back;
// ¶4: unselected experts are not computed at all] runs as two grouped GEMMs
// over the expert-sorted token rows that dispatch produced:
//
//   gate/up : H[r, f] = silu(x_r . w1[:, f]) * (x_r . w3[:, f])   (bf16 out)
//   down    : y[r, o] = H_r . w2[:, o]                              (fp32 out)
//
// One group per expert (or one dense group for the fused shared expert).
// Group sizes live on the device (kept counts from dispatch); the host never
// reads them, so the whole layer runs without a host synchronisation.
//
// Two tile layouts, chosen on the host from the largest possible group:
//   token-major  (groups may exceed 256 rows: prefill)
//     D[128 tokens x BN] = A(tokens, K-major) * B(weights, K-major)^T
//     gate/up tiles hold 128 gate + 128 up features of the same hidden block
//     (the packed W13 layout interleaves them), so the SiLU*mul epilogue
//     finds both operands in one thread's TMEM lane.
//   swapped      (every group has <= 256 rows: decode, many small experts)
//     D[128 weight rows x N tokens] = A(weights) * B(tokens)^T, N = the
//     group's token count rounded up to 16; each expert's weights are read
//     exactly once.  gate and up rows go to two accumulators; the down
//     projection may be split along K into partial outputs.
//
// Structure (one persistent CTA per SM, 6 warps):
//   warp 0      TMA producer: fills a ring of shared-memory stages
//   warp 1      MMA issuer (one thread) and TMEM owner
//   warps 2..5  epilogue: TMEM -> registers -> global
// Barriers: full/empty per stage (TMA <-> MMA), acc_full/acc_empty per TMEM
// accumulator buffer (MMA <-> epilogue).  Every wait is bounded; a wait that
// runs out records a timeout in the status word and the CTA winds down,
// letting its in-flight copies and MMAs finish before TMEM is released.
#include <stdio.h>

#include <mutex>

#include "common.cuh"
#include "kernels.h"

namespace moe {

namespace {

constexpr int BM = 128;      // MMA M (TMEM lanes)
constexpr int BK = 64;       // K elements per stage: one 128-byte swizzle row of bf16
constexpr int UK = 16;       // K per tcgen05.mma (bf16)
constexpr int THREADS = 192;

// Threads of a CTA: the producer warp, the MMA warp and four epilogue warps
// (one per TMEM lane quarter); the swapped gate/up has sixteen, four per
// quarter, splitting the token columns: its accumulator is single-buffered
// for wide token tiles, so the epilogue's length is time the MMAs wait
// (measured on deepseek: 4 -> 8 -> 12 -> 16 warps, 1133 -> 1036 -> 1010 -> 991 us).
template <int MODE>
constexpr int threads_of() {
    return MODE == TC_GATEUP_SWAP ? 64 + 16 * 32 : THREADS;
}
constexpr uint64_t TEARDOWN_NS = 200000000ull;  // 0.2 s bound on draining in-flight work

struct SharedLayout {
    uint32_t a_bytes, b_bytes, stage_bytes;
    uint32_t stg_off;  // fp32 epilogue staging (token-major down, weight gradient)
    uint32_t bar_off, grp_off, total;
};

// fp32 epilogues stage each warp's 32 x 32 block in shared memory so that a
// warp stores whole 128-byte row segments; rows padded to 36 floats.
constexpr int STG_LD = 36;
constexpr uint32_t STG_WARP_BYTES = 32 * STG_LD * 4;

__host__ __device__ inline bool staged_epilogue(int mode) {
    return mode == TC_DOWN_TOK || mode == TC_WGRAD;
}

__host__ __device__ inline uint32_t align_up(uint32_t v, uint32_t a) { return (v + a - 1) / a * a; }

// Whether a launch's down projection reads H as two bf16 parts (high, low):
// its activation tiles are then staged twice per K step.
__host__ __device__ inline bool down_split(int mode, int64_t lo_rows) {
    return (mode == TC_DOWN_TOK || mode == TC_DOWN_SWAP) && lo_rows != 0;
}

// Bytes of operand per stage for each mode.  With a split H the token-major
// down stages the high and the low 128-row tile one after the other (A); the
// swapped down stages a unit's ntok high-part rows and right after them its
// ntok low-part rows (B, room for 2 nt_max rows), read by one MMA of N = 2 ntok.
__host__ __device__ inline void stage_bytes(int mode, int bn, int nt_max, bool split, uint32_t* a,
                                            uint32_t* b) {
    const uint32_t parts = split ? 2 : 1;
    switch (mode) {
        case TC_GATEUP_TOK:
        case TC_DOWN_TOK:
        case TC_DGATE_TOK:
        case TC_WGRAD:
            *a = (mode == TC_DOWN_TOK ? parts : 1) * BM * BK * 2;
            *b = bn * BK * 2;
            break;
        case TC_GATEUP_SWAP: {
            const int tb = swap_gateup_tok_box(nt_max);
            *a = 2 * BM * BK * 2;
            *b = (nt_max + tb - 1) / tb * tb * BK * 2;
            break;
        }
        default:
            *a = BM * BK * 2;
            *b = parts * nt_max * BK * 2;
            break;
    }
}

__host__ __device__ inline SharedLayout shared_layout(int mode, int bn, int nt_max, int stages,
                                                      int groups, bool split) {
    SharedLayout L;
    stage_bytes(mode, bn, nt_max, split, &L.a_bytes, &L.b_bytes);
    L.a_bytes = align_up(L.a_bytes, 1024);
    L.b_bytes = align_up(L.b_bytes, 1024);
    L.stage_bytes = L.a_bytes + L.b_bytes;
    L.stg_off = L.stage_bytes * stages;
    L.bar_off = L.stg_off + (staged_epilogue(mode) ? 4 * STG_WARP_BYTES : 0);
    // full[S], empty[S], acc_full[2], acc_empty[2], drain, tmem slot
    L.grp_off = L.bar_off + align_up((2 * stages + 5) * 8 + 8, 16);
    L.total = L.grp_off + (4 * groups + 1) * 4 + 1024;  // + 1 KB for base alignment
    return L;
}

// Where one unit of work sits.
struct Unit {
    int g;        // group
    int w;        // weight index of the group
    int rows;     // valid rows of the group
    int row0;     // first row of the group in the activation/output tensors
    int mt, nb;   // token-major: m tile, n tile;  swapped: feature block
    int ks;       // split-K index (swapped down)
    int kb0, kb1; // k-block range
    int ntok;     // swapped: token columns (multiple of 16)
};

struct GroupTable {
    const int* start;  // [groups + 1] unit prefix
    const int* rows;   // [groups]
    const int* off;    // [groups]
    const int* wi;     // [groups] weight index
    int groups;
};

__device__ __forceinline__ int find_group(const GroupTable& t, int u) {
    int lo = 0, hi = t.groups - 1;
    while (lo < hi) {
        int mid = (lo + hi + 1) >> 1;
        if (t.start[mid] <= u) lo = mid; else hi = mid - 1;
    }
    return lo;
}

template <int MODE, int BN>
__device__ __forceinline__ Unit decode_unit(const GroupTable& t, int u, const TcArgs& a) {
    Unit x;
    x.g = find_group(t, u);
    x.w = t.wi[x.g];
    x.rows = t.rows[x.g];
    x.row0 = t.off[x.g];
    const int local = u - t.start[x.g];
    const int kblocks = a.K / BK;
    x.ks = 0;
    x.kb0 = 0;
    x.kb1 = kblocks;
    x.ntok = 0;
    if (MODE == TC_GATEUP_TOK || MODE == TC_DGATE_TOK) {
        const int mtiles = (x.rows + BM - 1) / BM;
        x.mt = local % mtiles;
        x.nb = local / mtiles;
    } else if (MODE == TC_WGRAD) {
        // the group's reduction range: its token rows, from the 64-aligned
        // segment start row0 on, rounded up to 64 (the rows past the group's
        // count are zero); the operand with fewer features is swept fastest
        // so that it stays in L2 while the other streams once
        const int mtiles = a.m_rows / BM;
        const int ntiles = a.n_feat / BN;
        if (a.n_fastest) {
            x.nb = local % ntiles;
            x.mt = local / ntiles;
        } else {
            x.mt = local % mtiles;
            x.nb = local / mtiles;
        }
        x.kb0 = x.row0 / BK;
        x.kb1 = x.kb0 + (x.rows + BK - 1) / BK;
    } else if (MODE == TC_DOWN_TOK) {
        // m tile fastest, then n tile, then K split
        const int mtiles = (x.rows + BM - 1) / BM;
        const int ntiles = a.n_feat / BN;
        x.mt = local % mtiles;
        const int rest = local / mtiles;
        x.nb = rest % ntiles;
        x.ks = rest / ntiles;
        const int per = kblocks / a.splits;
        x.kb0 = x.ks * per;
        x.kb1 = x.kb0 + per;
    } else if (MODE == TC_GATEUP_SWAP) {
        x.mt = 0;
        x.nb = local;
        x.ntok = (x.rows + 15) & ~15;
    } else {
        x.mt = 0;
        x.nb = local / a.splits;
        x.ks = local % a.splits;
        const int per = kblocks / a.splits;
        x.kb0 = x.ks * per;
        x.kb1 = x.kb0 + per;
        x.ntok = (x.rows + 15) & ~15;
    }
    return x;
}

template <int MODE, int BN>
__device__ __forceinline__ int units_of_group(int rows, const TcArgs& a) {
    // every weight-gradient tile is written, zeros for a group without tokens
    if (MODE == TC_WGRAD) return (a.m_rows / BM) * (a.n_feat / BN);
    if (rows <= 0) return 0;
    if (MODE == TC_DGATE_TOK) return ((rows + BM - 1) / BM) * (a.n_feat / BN);
    if (MODE == TC_GATEUP_TOK) return ((rows + BM - 1) / BM) * (a.n_feat / 128);
    if (MODE == TC_DOWN_TOK) return ((rows + BM - 1) / BM) * (a.n_feat / BN) * a.splits;
    if (MODE == TC_GATEUP_SWAP) return a.n_feat / 128;
    return (a.n_feat / 128) * a.splits;
}

// Stores 32 columns of fp32 for the warp's 32 rows: v holds row `lane`'s
// values; row r of the block goes to dst_row0 + r * ld (columns 0..31), rows
// at or past `valid` are skipped.  stg is the warp's staging buffer.  With
// `stream` the stores carry an L2 evict-first policy (outputs no kernel of the
// layer reads again, so that they do not push the operands out of L2).
__device__ __forceinline__ void store_rows_f32x32(float* stg, const float* v, int lane,
                                                  float* dst_row0, int64_t ld, int valid,
                                                  bool stream = false) {
    float4* srow = reinterpret_cast<float4*>(stg + lane * STG_LD);
#pragma unroll
    for (int j = 0; j < 8; ++j) srow[j] = make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
    __syncwarp();
    const int sub = lane >> 3, col = (lane & 7) * 4;
    const uint64_t pol = stream ? l2_policy_evict_first() : 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int r = 4 * i + sub;
        if (r < valid) {
            const float4 w = *reinterpret_cast<const float4*>(stg + r * STG_LD + col);
            if (stream)
                st_global_f32x4_hint(dst_row0 + r * ld + col, w, pol);
            else
                *reinterpret_cast<float4*>(dst_row0 + r * ld + col) = w;
        }
    }
    __syncwarp();
}

template <int MODE, int BN>
__global__ void __launch_bounds__(threads_of<MODE>(), 1)
    tc_gemm_kernel(const __grid_constant__ CUtensorMap tm_act,
                   const __grid_constant__ CUtensorMap tm_w, const TcArgs args) {
    constexpr bool TOK = (MODE == TC_GATEUP_TOK || MODE == TC_DOWN_TOK ||
                          MODE == TC_DGATE_TOK || MODE == TC_WGRAD);
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_addr(smem_raw);
    uint8_t* smem = smem_raw + (align_up(raw, 1024) - raw);

    const int groups = args.num_groups;
    const bool dsplit = down_split(MODE, args.lo_rows);
    const SharedLayout L = shared_layout(MODE, BN, args.nt_max, args.stages, groups, dsplit);
    const int S = args.stages;

    uint64_t* full = reinterpret_cast<uint64_t*>(smem + L.bar_off);
    uint64_t* empty = full + S;
    uint64_t* acc_full = empty + S;
    uint64_t* acc_empty = acc_full + 2;
    uint64_t* drain = acc_empty + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
    int* g_start = reinterpret_cast<int*>(smem + L.grp_off);
    int* g_rows = g_start + groups + 1;
    int* g_off = g_rows + groups;
    int* g_wi = g_off + groups;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    // accumulator geometry (TMEM columns)
    int acc_stride, n_acc;
    if (TOK) {
        acc_stride = BN;
        n_acc = 2;
    } else if (MODE == TC_GATEUP_SWAP) {
        acc_stride = 2 * args.nt_max;
        n_acc = (2 * acc_stride <= 512) ? 2 : 1;
    } else {
        // swapped down: with split H the low parts' columns follow the high
        // parts' in the same accumulator (one MMA of N = 2 ntok per K step)
        acc_stride = args.nt_max * (dsplit ? 2 : 1);
        n_acc = 2;
    }
    uint32_t tmem_cols = 32;
    while (tmem_cols < (uint32_t)(acc_stride * n_acc)) tmem_cols <<= 1;

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&acc_full[i], 1);
            mbar_init(&acc_empty[i], threads_of<MODE>() - 64);  // the epilogue threads
        }
        mbar_init(drain, 1);
        fence_mbar_init();
        prefetch_tmap(&tm_act);
        prefetch_tmap(&tm_w);
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, tmem_cols);
        tmem_relinquish();
    }
    if (MODE == TC_GATEUP_SWAP && args.prefetch_kb > 0 && warp == 0 && lane == 0) {
        // the predecessor (routing) may still run: prefetch into L2 the start of
        // the weight tile this CTA's first unit has when every expert has tokens
        // (a wrong guess only wastes the prefetch; weights are never written)
        const int ub = args.n_feat / 128;
        const int u = blockIdx.x;
        if (u < args.num_groups * ub) {
            const int wrow = (u / ub) * args.w_rows_per_group + (u % ub) * 256;
            const int nk = min(args.prefetch_kb, args.K / BK);
            for (int kb = 0; kb < nk; ++kb) {
                tma_prefetch_2d(&tm_w, kb * BK, wrow);
                tma_prefetch_2d(&tm_w, kb * BK, wrow + BM);
            }
        }
    }
    // everything below may read what the previous kernel in the stream wrote
    pdl_wait();
    pdl_trigger();
    if (warp == 2 && lane == 0) {
        int acc = 0;
        for (int g = 0; g < groups; ++g) {
            int r = args.group_rows ? args.group_rows[g] : args.dense_rows;
            int o = args.group_off ? args.group_off[g] : 0;
            if (!TOK && r > args.nt_max) {
                // a swapped tile holds at most nt_max token columns: clamp and
                // flag the oversized group rather than overrun shared memory
                if (args.status) atomicCAS(args.status, DEV_OK, DEV_SHAPE);
                r = args.nt_max;
            }
            g_rows[g] = r;
            g_wi[g] = args.group_w ? args.group_w[g] : g;
            g_off[g] = o;
            g_start[g] = acc;
            acc += units_of_group<MODE, BN>(r, args);
        }
        g_start[groups] = acc;
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    GroupTable tab{g_start, g_rows, g_off, g_wi, groups};
    const int total = g_start[groups];
    const uint64_t limit = args.wait_limit_ns;

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            uint64_t pol_w = 0, pol_a = 0;
            if (!TOK) {
                pol_w = l2_policy_evict_first();
                pol_a = l2_policy_evict_last();
            }
            // weight gradient: the operand swept fastest (fewer features) is
            // re-read for every tile of the other, which streams once: keep the
            // first in L2 ahead of the second
            uint64_t pol_wg_a = 0, pol_wg_b = 0;
            if (MODE == TC_WGRAD) {
                pol_wg_a = args.n_fastest ? l2_policy_evict_first() : l2_policy_evict_last();
                pol_wg_b = args.n_fastest ? l2_policy_evict_last() : l2_policy_evict_first();
            }
            int stage = 0;
            uint32_t phase = 0;
            uint32_t issued = 0, issued_par = 0;  // per-stage bits: loads issued / their parity
            bool ok = true;
            for (int u = blockIdx.x; u < total && ok; u += gridDim.x) {
                const Unit x = decode_unit<MODE, BN>(tab, u, args);
                for (int kb = x.kb0; kb < x.kb1; ++kb) {
                    if (!mbar_wait(&empty[stage], phase ^ 1, limit)) {
                        report_timeout(args.status);
                        ok = false;
                        break;
                    }
                    uint8_t* sa = smem + stage * L.stage_bytes;
                    uint8_t* sb = sa + L.a_bytes;
                    const int kc = kb * BK;
                    if (TOK) {
                        mbar_arrive_expect_tx(&full[stage],
                                              (BM * (dsplit ? 2 : 1) + BN) * BK * 2);
                        if (MODE == TC_WGRAD) {
                            // MN-major operands straight from the row-major
                            // activations: boxes of 64 features x 64 token rows
#pragma unroll
                            for (int i = 0; i < BM / 64; ++i)
                                tma_load_2d_hint(sa + i * 8192, &tm_act, &full[stage],
                                                 x.mt * BM + 64 * i, kc, pol_wg_a);
#pragma unroll
                            for (int i = 0; i < BN / 64; ++i)
                                tma_load_2d_hint(sb + i * 8192, &tm_w, &full[stage],
                                                 x.nb * BN + 64 * i, kc, pol_wg_b);
                        } else {
                            tma_load_2d(sa, &tm_act, &full[stage], kc, x.row0 + x.mt * BM);
                            if (dsplit)  // the same rows' low parts of H
                                tma_load_2d(sa + BM * BK * 2, &tm_act, &full[stage], kc,
                                            x.row0 + x.mt * BM + (int)args.lo_rows);
                            tma_load_2d(sb, &tm_w, &full[stage], kc,
                                        x.w * args.w_rows_per_group +
                                            x.nb * (MODE == TC_GATEUP_TOK ? 256 : BN));
                        }
                    } else {
                        const int wa = (MODE == TC_GATEUP_SWAP) ? 2 * BM : BM;
                        // token rows in boxes of tb: whole boxes land in shared memory
                        const int tb =
                            MODE == TC_GATEUP_SWAP ? swap_gateup_tok_box(args.nt_max) : 16;
                        const int trows = (x.ntok + tb - 1) / tb * tb;
                        mbar_arrive_expect_tx(&full[stage],
                                              (wa + trows * (dsplit ? 2 : 1)) * BK * 2);
                        const int wrow = x.w * args.w_rows_per_group +
                                         x.nb * (MODE == TC_GATEUP_SWAP ? 256 : BM);
                        tma_load_2d_hint(sa, &tm_w, &full[stage], kc, wrow, pol_w);
                        if (MODE == TC_GATEUP_SWAP)
                            tma_load_2d_hint(sa + BM * BK * 2, &tm_w, &full[stage], kc, wrow + BM,
                                             pol_w);
                        for (int r = 0; r < x.ntok; r += tb)
                            tma_load_2d_hint(sb + r * BK * 2, &tm_act, &full[stage], kc,
                                             x.row0 + r, pol_a);
                        if (dsplit)  // the low parts of H right behind the high ones
                            for (int r = 0; r < x.ntok; r += 16)
                                tma_load_2d_hint(sb + (x.ntok + r) * BK * 2, &tm_act,
                                                 &full[stage], kc,
                                                 x.row0 + r + (int)args.lo_rows, pol_a);
                    }
                    issued |= 1u << stage;
                    issued_par = (issued_par & ~(1u << stage)) | (phase << stage);
                    if (++stage == S) {
                        stage = 0;
                        phase ^= 1;
                    }
                }
            }
            // let every issued copy land before the CTA can release its memory
            for (int s = 0; s < S; ++s)
                if (issued & (1u << s)) mbar_wait(&full[s], (issued_par >> s) & 1, TEARDOWN_NS);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            int acc = 0;
            uint32_t acc_phase = 0;
            bool ok = true;
            const uint32_t idesc_tok =
                MODE == TC_WGRAD ? idesc_bf16_f32_mn(BM, BN) : idesc_bf16_f32(BM, BN);
            for (int u = blockIdx.x; u < total && ok; u += gridDim.x) {
                const Unit x = decode_unit<MODE, BN>(tab, u, args);
                if (!mbar_wait(&acc_empty[acc], acc_phase ^ 1, limit)) {
                    report_timeout(args.status);
                    break;
                }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + acc * acc_stride;
                // swapped down with split H: B = [H_hi; H_lo] rows, N = 2 ntok, so
                // that the weight tile is read once for both parts
                const uint32_t idesc =
                    TOK ? idesc_tok
                        : idesc_bf16_f32(BM, x.ntok * (MODE == TC_DOWN_SWAP && dsplit ? 2 : 1));
                for (int kb = x.kb0; kb < x.kb1; ++kb) {
                    if (!mbar_wait(&full[stage], phase, limit)) {
                        report_timeout(args.status);
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t sa = smem_addr(smem + stage * L.stage_bytes);
                    const uint32_t sb = sa + L.a_bytes;
#pragma unroll
                    for (int kk = 0; kk < BK / UK; ++kk) {
                        const uint32_t acc_flag = (kb > x.kb0 || kk > 0) ? 1u : 0u;
                        if (MODE == TC_WGRAD) {
                            // K steps of 16 rows of 128 B
                            umma_bf16(d_tmem, sdesc_mnmajor_sw128(sa + kk * UK * 128, 8192),
                                      sdesc_mnmajor_sw128(sb + kk * UK * 128, 8192), idesc,
                                      acc_flag);
                            continue;
                        }
                        const uint64_t bdesc = sdesc_kmajor_sw128(sb + kk * UK * 2);
                        const uint64_t adesc = sdesc_kmajor_sw128(sa + kk * UK * 2);
                        umma_bf16(d_tmem, adesc, bdesc, idesc, acc_flag);
                        if (MODE == TC_DOWN_TOK && dsplit)  // + H_lo . W
                            umma_bf16(d_tmem, sdesc_kmajor_sw128(sa + BM * BK * 2 + kk * UK * 2),
                                      bdesc, idesc, 1u);
                        if (MODE == TC_GATEUP_SWAP)
                            umma_bf16(d_tmem + args.nt_max,
                                      sdesc_kmajor_sw128(sa + BM * BK * 2 + kk * UK * 2), bdesc,
                                      idesc, acc_flag);
                    }
                    umma_commit(&empty[stage]);
                    if (++stage == S) {
                        stage = 0;
                        phase ^= 1;
                    }
                }
                if (!ok) break;
                // test hook: the first unit of CTA 0 never signals its epilogue,
                // whose bounded wait then runs out and reports a time-out
                const bool withhold = args.test_stall && blockIdx.x == 0 && u == (int)blockIdx.x;
                if (!withhold) umma_commit(&acc_full[acc]);
                if (++acc == n_acc) {
                    acc = 0;
                    acc_phase ^= 1;
                }
            }
            // every MMA issued by this thread completes before TMEM is released
            umma_commit(drain);
            mbar_wait(drain, 0, TEARDOWN_NS);
        }
    } else {
        // ------------------------------------------------------------ epilogue
        const int q = warp & 3;                 // TMEM lane quarter this warp may access
        const int part = (warp - 2) >> 2;       // which of the quarter's warps (swapped gate/up)
        constexpr int NPART = (threads_of<MODE>() - 64) / 128;
        const int row = q * 32 + lane;          // accumulator row (TMEM lane)
        const uint32_t lane_addr = tmem_base + ((uint32_t)(q * 32) << 16);
        int acc = 0;
        uint32_t acc_phase = 0;
        for (int u = blockIdx.x; u < total; u += gridDim.x) {
            const Unit x = decode_unit<MODE, BN>(tab, u, args);
            if (!mbar_wait(&acc_full[acc], acc_phase, limit)) {
                report_timeout(args.status);
                break;
            }
            tc_fence_after();
            const uint32_t t0 = lane_addr + acc * acc_stride;
            if (MODE == TC_GATEUP_TOK) {
                const int r = x.mt * BM + row;
                const bool valid = r < x.rows;
                __nv_bfloat16* dst = reinterpret_cast<__nv_bfloat16*>(args.out) +
                                     (int64_t)(x.row0 + r) * args.out_ld + x.nb * 128;
                __nv_bfloat16* abrow =
                    args.aux ? reinterpret_cast<__nv_bfloat16*>(args.aux) +
                                   (int64_t)(x.row0 + r) * args.aux_ld + x.nb * 256
                             : nullptr;
#pragma unroll 1
                for (int c = 0; c < 128; c += 16) {
                    float g[16], v[16];
                    tmem_ld16(t0 + c, g);
                    tmem_ld16(t0 + 128 + c, v);
                    tmem_ld_wait();
                    if (valid && abrow) {
                        // pre-activations kept for the backward pass
                        store_bf16x16(abrow + c, g);
                        store_bf16x16(abrow + 128 + c, v);
                    }
                    if (valid) {
                        float hv[16];
#pragma unroll
                        for (int i = 0; i < 16; ++i) hv[i] = silu_f(g[i]) * v[i];
                        if (args.lo_rows) {
                            // low parts: H - bf16(H) is exact in fp32, then rounded
                            float lo[16];
#pragma unroll
                            for (int i = 0; i < 16; ++i) lo[i] = hv[i] - bf16_round(hv[i]);
                            store_bf16x16(dst + args.lo_rows * args.out_ld + c, lo);
                        }
                        store_bf16x16(dst + c, hv);
                    }
                }
            } else if (MODE == TC_DOWN_TOK) {
                const int r0 = x.mt * BM + q * 32;  // first row of this warp's block
                const int valid = min(32, x.rows - r0);
                float* dst0 = reinterpret_cast<float*>(args.out) + x.ks * args.split_stride +
                              (int64_t)(x.row0 + r0) * args.out_ld + x.nb * BN;
                float* stg = reinterpret_cast<float*>(smem + L.stg_off) + q * (32 * STG_LD);
                if (args.out_cols > 0) {
                    // router GEMM: compact rows of out_cols columns (a multiple of
                    // 4), stored thread by thread; padding columns are skipped
                    const int ncol = min(BN, args.out_cols - x.nb * BN);
                    float* dst = dst0 + (int64_t)lane * args.out_ld;
#pragma unroll 1
                    for (int c = 0; c < ncol; c += 16) {
                        float v[16];
                        tmem_ld16(t0 + c, v);
                        tmem_ld_wait();
                        if (lane < valid) {
#pragma unroll
                            for (int i = 0; i < 16; i += 4)
                                if (c + i < ncol)
                                    *reinterpret_cast<float4*>(dst + c + i) =
                                        make_float4(v[i], v[i + 1], v[i + 2], v[i + 3]);
                        }
                    }
                } else {
#pragma unroll 1
                    for (int c = 0; c < BN; c += 32) {
                        float v[32];
                        tmem_ld16(t0 + c, v);
                        tmem_ld16(t0 + c + 16, v + 16);
                        tmem_ld_wait();
                        store_rows_f32x32(stg, v, lane, dst0 + c, args.out_ld, valid);
                    }
                }
            } else if (MODE == TC_DGATE_TOK) {
                // dH[r][f] for BN hidden features f; with a = x w1, b = x w3 of
                // the forward (AB, bf16): dA = dH b silu'(a), dB = dH silu(a),
                // stored interleaved per 128-wide block like AB itself
                const int r = x.mt * BM + row;
                const bool valid = r < x.rows;
                const int64_t rowoff = (int64_t)(x.row0 + r) * args.aux_ld;
                const __nv_bfloat16* ab = reinterpret_cast<const __nv_bfloat16*>(args.aux) + rowoff;
                __nv_bfloat16* dab = reinterpret_cast<__nv_bfloat16*>(args.out) + rowoff;
                // the pre-activations of the next 16 features are loaded while
                // the current ones are used (the loads are the epilogue's latency)
                auto ab_col = [&](int c) {
                    const int f = x.nb * BN + c;
                    return (int64_t)(f >> 7) * 256 + (f & 127);
                };
                uint4 na0 = make_uint4(0, 0, 0, 0), na1 = na0, nb0 = na0, nb1 = na0;
                if (valid) {
                    const uint4* pa = reinterpret_cast<const uint4*>(ab + ab_col(0));
                    na0 = pa[0];
                    na1 = pa[1];
                    nb0 = pa[16];
                    nb1 = pa[17];
                }
#pragma unroll 1
                for (int c = 0; c < BN; c += 16) {
                    float dh[16];
                    tmem_ld16(t0 + c, dh);
                    const uint4 ca0 = na0, ca1 = na1, cb0 = nb0, cb1 = nb1;
                    if (valid && c + 16 < BN) {
                        const uint4* pa = reinterpret_cast<const uint4*>(ab + ab_col(c + 16));
                        na0 = pa[0];
                        na1 = pa[1];
                        nb0 = pa[16];
                        nb1 = pa[17];
                    }
                    tmem_ld_wait();
                    if (valid) {
                        const int64_t col = ab_col(c);
                        float a[16], b[16], da[16], db[16];
                        const uint32_t wa[8] = {ca0.x, ca0.y, ca0.z, ca0.w, ca1.x, ca1.y, ca1.z, ca1.w};
                        const uint32_t wb[8] = {cb0.x, cb0.y, cb0.z, cb0.w, cb1.x, cb1.y, cb1.z, cb1.w};
#pragma unroll
                        for (int i = 0; i < 8; ++i) {
                            a[2 * i] = __uint_as_float(wa[i] << 16);
                            a[2 * i + 1] = __uint_as_float(wa[i] & 0xFFFF0000u);
                            b[2 * i] = __uint_as_float(wb[i] << 16);
                            b[2 * i + 1] = __uint_as_float(wb[i] & 0xFFFF0000u);
                        }
#pragma unroll
                        for (int i = 0; i < 16; ++i) {
                            const float sig = 1.0f / (1.0f + __expf(-a[i]));
                            da[i] = dh[i] * b[i] * sig * (1.0f + a[i] * (1.0f - sig));
                            db[i] = dh[i] * a[i] * sig;
                        }
                        store_bf16x16(dab + col, da);
                        store_bf16x16(dab + col + 128, db);
                    }
                }
            } else if (MODE == TC_WGRAD) {
                float* dst0 = reinterpret_cast<float*>(args.out) + x.g * args.group_stride +
                              (int64_t)(x.mt * BM + q * 32) * args.out_ld + x.nb * BN;
                float* stg = reinterpret_cast<float*>(smem + L.stg_off) + q * (32 * STG_LD);
                const bool empty = x.kb1 == x.kb0;
#pragma unroll 1
                for (int c = 0; c < BN; c += 32) {
                    float v[32];
                    if (!empty) {
                        tmem_ld16(t0 + c, v);
                        tmem_ld16(t0 + c + 16, v + 16);
                        tmem_ld_wait();
                    } else {
#pragma unroll
                        for (int i = 0; i < 32; ++i) v[i] = 0.0f;
                    }
                    // the weight gradients: read by no later kernel of the step
                    store_rows_f32x32(stg, v, lane, dst0 + c, args.out_ld, 32, true);
                }
            } else if (MODE == TC_GATEUP_SWAP) {
                __nv_bfloat16* dst = reinterpret_cast<__nv_bfloat16*>(args.out) +
                                     (int64_t)x.row0 * args.out_ld + x.nb * 128 + row;
#pragma unroll 1
                for (int c = 16 * part; c < x.ntok; c += 16 * NPART) {
                    float g[16], v[16];
                    tmem_ld16(t0 + c, g);
                    tmem_ld16(t0 + args.nt_max + c, v);
                    tmem_ld_wait();
#pragma unroll
                    for (int i = 0; i < 16; ++i)
                        if (c + i < x.rows) {
                            const float hv = silu_f(g[i]) * v[i];
                            dst[(int64_t)(c + i) * args.out_ld] = __float2bfloat16_rn(hv);
                            if (args.lo_rows)  // low part, lo_rows rows further
                                dst[(int64_t)(c + i + args.lo_rows) * args.out_ld] =
                                    __float2bfloat16_rn(hv - bf16_round(hv));
                        }
                    if (args.aux) {
                        __nv_bfloat16* ab = reinterpret_cast<__nv_bfloat16*>(args.aux) +
                                            (int64_t)x.row0 * args.aux_ld + x.nb * 256 + row;
#pragma unroll
                        for (int i = 0; i < 16; ++i)
                            if (c + i < x.rows) {
                                ab[(int64_t)(c + i) * args.aux_ld] = __float2bfloat16_rn(g[i]);
                                ab[(int64_t)(c + i) * args.aux_ld + 128] =
                                    __float2bfloat16_rn(v[i]);
                            }
                    }
                }
            } else {
                float* dst = reinterpret_cast<float*>(args.out) + x.ks * args.split_stride +
                             (int64_t)x.row0 * args.out_ld + x.nb * BM + row;
#pragma unroll 1
                for (int c = 0; c < x.ntok; c += 16) {
                    float v[16];
                    tmem_ld16(t0 + c, v);
                    if (dsplit) {
                        // + the low parts' columns: y = W.H_hi + W.H_lo
                        float w[16];
                        tmem_ld16(t0 + x.ntok + c, w);
                        tmem_ld_wait();
#pragma unroll
                        for (int i = 0; i < 16; ++i) v[i] += w[i];
                    }
                    tmem_ld_wait();
#pragma unroll
                    for (int i = 0; i < 16; ++i)
                        if (c + i < x.rows) dst[(int64_t)(c + i) * args.out_ld] = v[i];
                }
            }
            tc_fence_before();
            mbar_arrive(&acc_empty[acc]);
            if (++acc == n_acc) {
                acc = 0;
                acc_phase ^= 1;
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem_base, tmem_cols);
}

template <int MODE, int BN>
int launch_mode(const CUtensorMap& act, const CUtensorMap& w, const TcArgs& a, int grid,
                cudaStream_t st) {
    const SharedLayout L =
        shared_layout(MODE, BN, a.nt_max, a.stages, a.num_groups, down_split(MODE, a.lo_rows));
    auto kern = tc_gemm_kernel<MODE, BN>;
    // the shared-memory opt-in is a property of the kernel on each device: kept
    // per device (and per instantiation), under a lock for callers on several threads
    constexpr int kMaxDevices = 64;
    static std::mutex mu;
    static int configured_bytes[kMaxDevices] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return -1;
    {
        std::lock_guard<std::mutex> lk(mu);
        if ((int)L.total > configured_bytes[dev]) {
            if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     L.total) != cudaSuccess)
                return -1;
            configured_bytes[dev] = L.total;
        }
    }
    launch_ex(pdl_active(), kern, dim3(grid), dim3(threads_of<MODE>()), L.total, st, act, w, a);
    note_launch();
    return launch_result();
}

}  // namespace

int tc_max_stages(int mode, int bn, int nt_max, int groups, bool split, int smem_limit) {
    const bool ds = down_split(mode, split ? 1 : 0);
    for (int s = 8; s >= 2; --s)
        if ((int)shared_layout(mode, bn, nt_max, s, groups, ds).total <= smem_limit) return s;
    return 0;
}

int launch_tc_gemm(int mode, int bn, const CUtensorMap& act, const CUtensorMap& w,
                   const TcArgs& a, int grid, cudaStream_t st) {
    switch (mode) {
        case TC_GATEUP_TOK:
            return launch_mode<TC_GATEUP_TOK, 256>(act, w, a, grid, st);
        case TC_DOWN_TOK:
            return bn == 256 ? launch_mode<TC_DOWN_TOK, 256>(act, w, a, grid, st)
                             : launch_mode<TC_DOWN_TOK, 128>(act, w, a, grid, st);
        case TC_GATEUP_SWAP:
            return launch_mode<TC_GATEUP_SWAP, 128>(act, w, a, grid, st);
        case TC_DOWN_SWAP:
            return launch_mode<TC_DOWN_SWAP, 128>(act, w, a, grid, st);
        case TC_DGATE_TOK:
            return bn == 256 ? launch_mode<TC_DGATE_TOK, 256>(act, w, a, grid, st)
                             : launch_mode<TC_DGATE_TOK, 128>(act, w, a, grid, st);
        case TC_WGRAD:
            return bn == 256 ? launch_mode<TC_WGRAD, 256>(act, w, a, grid, st)
                             : launch_mode<TC_WGRAD, 128>(act, w, a, grid, st);
    }
    return -1;
}

}  // namespace moe
