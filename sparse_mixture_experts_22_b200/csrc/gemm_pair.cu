// gemm_pair.cu -- expert GEMMs with few tokens per expert, on CTA pairs.
//
// The expert FFN [Mixtral 8x7B and MoE explained, "Easy explanation" ¶2: each
// expert widens the embedding and narrows it back; ¶4: unselected experts are
// not computed] for layers whose experts each keep up to 256 tokens, such as
// the DeepSeek-V2-style layer [MoE routing fully explained, "Easy
// explanation" ¶4: many small routed experts].  The weights then dominate
// the bytes, so the tiles put weight rows on M and an expert's tokens on N
// ("swapped" tiles), and the kernel's job is to stream weights at HBM speed.
//
// Here each tile is one tcgen05 MMA over a pair of SMs (a cluster of two
// CTAs, cta_group::2): M = 256 weight rows, 128 in each CTA's shared memory,
// and the expert's N token rows split N/2 + N/2 between them.  Against a
// one-SM tile of the same weight rows each SM stages half the token rows, so
// about twice the pipeline stages fit and the accumulator of up to 256
// token columns fits twice in TMEM (the epilogue of one tile overlaps the
// MMAs of the next).
//
//   gate/up : unit = 128 hidden features of one expert; CTA v holds the gate
//             rows of features 64v..64v+63 (accumulator lanes 0-63) and
//             their up rows (lanes 64-127); the epilogue pairs each gate
//             warp with the up warp of the same features and exchanges
//             half of the columns through shared memory, so that each
//             computes H = silu(gate) * up for half of the tokens.
//   down    : unit = 256 output features; CTA v holds W2 rows 128v..128v+127
//             and receives y for them; with H in two bf16 parts a second
//             MMA per K step adds H_lo.
//
// The same pairing serves experts with thousands of tokens (token-major
// tiles, the large prefill layer): M = 256 tokens, 128 rows in each CTA, and
// N = 256 weight rows, 128 in each CTA -- for gate/up CTA 0 stages the 128
// gate rows of a hidden block and CTA 1 their up rows, so that each CTA's
// accumulator holds [gate | up] for its own 128 tokens, as the one-SM tile
// does.  Each SM then stages 32 KB per K step for a 256 x 256 x 64 MMA
// instead of 48 KB for 128 x 256 x 64: a third less shared-memory fill (L2
// traffic) per flop.
//
// Roles (each CTA): warp 0 loads this CTA's halves with TMA into its own
// stages, every copy signalling the even CTA's "stage full" barrier (the
// cta_group::2 form of the copy; no multicast), which the even CTA's producer
// arms with both CTAs' bytes; in the even CTA warp 1 issues the pair MMAs
// once a stage is full; the other warps are the epilogue.  The MMA's
// completion is signalled to both CTAs' barriers at once (tcgen05.commit
// multicast); the epilogues of both CTAs release an accumulator on the even
// CTA's barrier.  (A first version had the odd CTA's copies complete on its
// own barrier and a thread forward each stage to the even CTA with a
// cluster-scope release: that per-stage hop kept the tensor pipe 33% busy.)
// The pairs take their work units from a device counter (the even CTA's
// producer fetches the next unit and publishes it to every role of both CTAs
// through a small queue in shared memory), so the work spreads over however
// many pairs are resident at once.  Every wait is bounded; on a time-out the
// kernel records MOE_ERR_TIMEOUT, lets the copies it issued land and the MMAs
// drain, and both CTAs meet at a cluster barrier before TMEM is released.
#include <stdio.h>

#include <mutex>

#include "common.cuh"
#include "kernels.h"

namespace moe {

namespace {

constexpr int PBM = 128;   // weight rows per CTA (accumulator lanes)
constexpr int PBK = 64;    // K per stage: one 128-byte swizzle row of bf16
constexpr int PUK = 16;    // K per MMA
constexpr uint64_t P_TEARDOWN_NS = 200000000ull;
constexpr int P_STG_LD = 36;  // fp32 staging row (32 values + 4 of padding)
constexpr int P_QN = 4;       // slots of the unit queue

__host__ __device__ constexpr bool p_tok(int mode) {
    return mode == TC_PAIR_GATEUP_TOK || mode == TC_PAIR_DOWN_TOK || mode == TC_PAIR_DGATE_TOK;
}
// epilogue warps: two per TMEM lane quarter on swapped tiles (splitting the
// token columns), one per quarter on token-major tiles
__host__ __device__ constexpr int p_epi(int mode) { return p_tok(mode) ? 4 : 8; }
__host__ __device__ constexpr int p_threads(int mode) { return 64 + 32 * p_epi(mode); }

__host__ __device__ inline uint32_t p_align(uint32_t v, uint32_t a) { return (v + a - 1) / a * a; }

struct PairLayout {
    uint32_t a_bytes, b_bytes, b_lo, stage_bytes, xch_off, flag_off, bar_off, grp_off, total;
};

// Shared memory of one CTA.  Swapped: A = 128 weight rows, B = nt_max / 2
// token rows (the high parts of H, then as many low parts when split).
// Token-major: A = 128 token rows (then their low parts when split), B = 128
// weight rows.  Then the gate/up exchange buffers of the swapped epilogue (per
// pair of warps two directions x two chunks x 32 lanes x 8 floats) or the
// fp32 staging of the token-major down epilogue (32 x 36 floats per warp).
__host__ __device__ inline PairLayout pair_layout(int mode, int nt_max, int stages, int groups,
                                                  bool split) {
    PairLayout L;
    const uint32_t parts = split ? 2u : 1u;
    if (p_tok(mode)) {
        L.a_bytes = PBM * PBK * 2 * (mode == TC_PAIR_DOWN_TOK ? parts : 1u);
        L.b_lo = 0;
        L.b_bytes = PBM * PBK * 2;
    } else {
        // nt_max / 2 token rows rounded up to whole TMA boxes
        const int tb = pair_swap_tok_box(nt_max);
        L.a_bytes = PBM * PBK * 2;
        L.b_lo = (uint32_t)((nt_max / 2 + tb - 1) / tb * tb) * PBK * 2;
        L.b_bytes = p_align(L.b_lo * parts, 1024);
    }
    L.stage_bytes = L.a_bytes + L.b_bytes;
    L.xch_off = L.stage_bytes * stages;
    uint32_t xch = 0;
    if (mode == TC_PAIR_GATEUP) xch = (p_epi(mode) / 2) * 2 * 2 * 32 * 8 * 4;
    if (mode == TC_PAIR_DOWN_TOK) xch = p_epi(mode) * 32 * P_STG_LD * 4;
    L.flag_off = L.xch_off + xch;
    L.bar_off = p_align(L.flag_off + p_epi(mode) * 2 * 4, 16);
    // full[S], empty[S], acc_full[2], acc_empty[2], drain, q_full[QN], q_empty[QN],
    // tmem slot, q_unit[QN]
    L.grp_off = L.bar_off + p_align((2 * stages + 5 + 2 * P_QN) * 8 + 8 + 4 * P_QN, 16);
    L.total = L.grp_off + (4 * groups + 1) * 4 + 1024;
    return L;
}

struct PUnit {
    int g, w, rows, row0, nb, mt, ntok;
};

struct PGroups {
    const int* start;
    const int* rows;
    const int* off;
    const int* wi;
    int groups;
};

template <int MODE>
__device__ __forceinline__ PUnit p_decode(const PGroups& t, int u) {
    int lo = 0, hi = t.groups - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (t.start[mid] <= u) lo = mid; else hi = mid - 1;
    }
    PUnit x;
    x.g = lo;
    x.w = t.wi[lo];
    x.rows = t.rows[lo];
    x.row0 = t.off[lo];
    const int local = u - t.start[lo];
    if (p_tok(MODE)) {
        // m tile fastest: the units after one another share the weight tile
        const int mtiles = (x.rows + 255) / 256;
        x.mt = local % mtiles;
        x.nb = local / mtiles;
        x.ntok = 256;
    } else {
        x.mt = 0;
        x.nb = local;
        x.ntok = (x.rows + 15) & ~15;
    }
    return x;
}

// Stores 32 fp32 columns of the warp's 32 rows through the warp's staging
// buffer so that every store is a whole 128-byte row segment; rows at or
// past `valid` are skipped.
__device__ __forceinline__ void p_store_rows_f32x32(float* stg, const float* v, int lane,
                                                    float* dst_row0, int64_t ld, int valid) {
    float4* srow = reinterpret_cast<float4*>(stg + lane * P_STG_LD);
#pragma unroll
    for (int j = 0; j < 8; ++j)
        srow[j] = make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
    __syncwarp();
    const int sub = lane >> 3, col = (lane & 7) * 4;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int r = 4 * i + sub;
        if (r < valid)
            *reinterpret_cast<float4*>(dst_row0 + r * ld + col) =
                *reinterpret_cast<const float4*>(stg + r * P_STG_LD + col);
    }
    __syncwarp();
}

template <int MODE>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(p_threads(MODE), 1)
    tc_pair_kernel(const __grid_constant__ CUtensorMap tm_act,
                   const __grid_constant__ CUtensorMap tm_w, const TcArgs args) {
    constexpr bool GU = MODE == TC_PAIR_GATEUP;
    constexpr bool TOK = p_tok(MODE);
    constexpr int NEPI = p_epi(MODE);
    constexpr bool DOWN = MODE == TC_PAIR_DOWN || MODE == TC_PAIR_DOWN_TOK;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_addr(smem_raw);
    uint8_t* smem = smem_raw + (p_align(raw, 1024) - raw);

    const int groups = args.num_groups;
    const bool split = DOWN && args.lo_rows != 0;
    const int S = args.stages;
    const PairLayout L = pair_layout(MODE, args.nt_max, S, groups, split);

    uint64_t* full = reinterpret_cast<uint64_t*>(smem + L.bar_off);
    uint64_t* empty = full + S;
    uint64_t* acc_full = empty + S;
    uint64_t* acc_empty = acc_full + 2;
    uint64_t* drain = acc_empty + 2;
    uint64_t* q_full = drain + 1;        // unit published (both CTAs)
    uint64_t* q_empty = q_full + P_QN;   // unit read by every consumer (even CTA)
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(q_empty + P_QN);
    int* q_unit = reinterpret_cast<int*>(tmem_slot + 1);
    int* g_start = reinterpret_cast<int*>(smem + L.grp_off);
    int* g_rows = g_start + groups + 1;
    int* g_off = g_rows + groups;
    int* g_wi = g_off + groups;
    int* flags = reinterpret_cast<int*>(smem + L.flag_off);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t v = cluster_ctarank();       // 0: issues the MMAs

    // accumulator: 128 lanes x nt_max (token-major: 256) columns, twice when it fits
    const int acc_stride = TOK ? 256 : args.nt_max;
    const int n_acc = 2 * acc_stride <= 512 ? 2 : 1;
    uint32_t tmem_cols = 32;
    while (tmem_cols < (uint32_t)(acc_stride * n_acc)) tmem_cols <<= 1;

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(&full[s], 1);  // the even CTA's: armed once with both CTAs' bytes
            mbar_init(&empty[s], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&acc_full[i], 1);
            mbar_init(&acc_empty[i], 2 * NEPI);  // one arrive per epilogue warp of each CTA
        }
        mbar_init(drain, 1);
        for (int i = 0; i < P_QN; ++i) {
            mbar_init(&q_full[i], 1);
            // consumers: the MMA thread and epilogue warps of the even CTA, the
            // producer and epilogue warps of the odd one
            mbar_init(&q_empty[i], 2 + 2 * NEPI);
        }
        fence_mbar_init();
        prefetch_tmap(&tm_act);
        prefetch_tmap(&tm_w);
    }
    if (warp == 1) {
        tmem_alloc_pair(tmem_slot, tmem_cols);
        tmem_relinquish_pair();
    }
    pdl_wait();
    pdl_trigger();
    if (warp == 2 && lane == 0) {
        int acc = 0;
        for (int g = 0; g < groups; ++g) {
            int r = args.group_rows ? args.group_rows[g] : args.dense_rows;
            if (!TOK && r > args.nt_max) {
                // a tile holds at most nt_max token columns: clamp and flag
                if (args.status) atomicCAS(args.status, DEV_OK, DEV_SHAPE);
                r = args.nt_max;
            }
            g_rows[g] = r;
            g_off[g] = args.group_off ? args.group_off[g] : 0;
            g_wi[g] = args.group_w ? args.group_w[g] : g;
            g_start[g] = acc;
            const int per = args.n_feat / (GU || MODE == TC_PAIR_GATEUP_TOK ? 128 : 256);
            acc += r > 0 ? per * (TOK ? (r + 255) / 256 : 1) : 0;
        }
        g_start[groups] = acc;
    }
    tc_fence_before();
    __syncthreads();
    // barrier initialisation and TMEM allocation visible to the peer CTA
    cluster_sync_all();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    const PGroups tab{g_start, g_rows, g_off, g_wi, groups};
    const int total = g_start[groups];
    const uint64_t limit = args.wait_limit_ns;
    // the unit queue: slot j holds the j-th unit (mod P_QN) of this pair, or
    // `total` when there is no more work
    const uint32_t lead_q_empty0 = map_shared_rank(smem_addr(&q_empty[0]), 0);
    auto take_unit = [&](int& slot, uint32_t& qph, bool arrive, int* u) -> bool {
        if (!mbar_wait_cl(&q_full[slot], qph, limit)) return false;
        *u = *reinterpret_cast<volatile int*>(&q_unit[slot]);
        if (arrive) mbar_arrive_cluster(lead_q_empty0 + slot * 8);
        if (++slot == P_QN) {
            slot = 0;
            qph ^= 1;
        }
        return true;
    };

    if (warp == 0) {
        // ------------------------------------------------------------ producer (both CTAs)
        if (lane == 0) {
            // swapped: weights stream once (evict first), an expert's token rows
            // are read again for each of its units (evict last); token-major: the
            // default policy for both
            const uint64_t pol_w = l2_policy_evict_first();
            const uint64_t pol_a = TOK ? l2_policy_evict_normal() : l2_policy_evict_last();
            const uint64_t pol_n = l2_policy_evict_normal();
            int stage = 0;
            uint32_t phase = 0;
            uint32_t issued = 0, issued_par = 0;
            bool ok = true;
            const int kblocks = args.K / PBK;
            int qs = 0;
            uint32_t qph = 0;
            const uint32_t peer_unit0 = map_shared_rank(smem_addr(&q_unit[0]), 1);
            const uint32_t peer_full0 = map_shared_rank(smem_addr(&q_full[0]), 1);
            const uint32_t lead_full0 = map_shared_rank(smem_addr(&full[0]), 0);
            while (ok) {
                int u = total;
                if (v == 0) {
                    // the scheduler: next unit of this pair, published to both CTAs
                    if (!mbar_wait_cl(&q_empty[qs], qph ^ 1, limit)) {
                        report_timeout(args.status);
                        break;
                    }
                    u = atomicAdd(args.unit_ctr, 1);
                    if (u > total) u = total;
                    q_unit[qs] = u;
                    st_cluster_u32(peer_unit0 + qs * 4, (uint32_t)u);
                    mbar_arrive(&q_full[qs]);
                    mbar_arrive_cluster(peer_full0 + qs * 8);
                    if (++qs == P_QN) {
                        qs = 0;
                        qph ^= 1;
                    }
                } else if (!take_unit(qs, qph, true, &u)) {
                    report_timeout(args.status);
                    break;
                }
                if (u >= total) break;
                const PUnit x = p_decode<MODE>(tab, u);
                const int half = x.ntok / 2;          // token rows this CTA stages
                const int trow = TOK ? x.row0 + x.mt * 256 + (int)v * PBM : x.row0 + (int)v * half;
                // token rows per CTA and stage: token-major, half = 128 (the A
                // tile); swapped, half rounded up to whole boxes of tb rows (the
                // last box may run into the other CTA's or the next group's rows)
                const int tb = TOK ? 128 : pair_swap_tok_box(args.nt_max);
                const int hrows = (half + tb - 1) / tb * tb;
                const uint32_t bytes =
                    (uint32_t)PBM * PBK * 2 + (uint32_t)hrows * PBK * 2 * (split ? 2u : 1u);
                for (int kb = 0; kb < kblocks; ++kb) {
                    if (!mbar_wait(&empty[stage], phase ^ 1, limit)) {
                        report_timeout(args.status);
                        ok = false;
                        break;
                    }
                    uint8_t* sa = smem + stage * L.stage_bytes;
                    uint8_t* sb = sa + L.a_bytes;
                    const int kc = kb * PBK;
                    // the even CTA arms its barrier with both CTAs' bytes (the same
                    // for both); every copy below completes on that barrier
                    if (v == 0) mbar_arrive_expect_tx(&full[stage], 2 * bytes);
                    const uint32_t fb = lead_full0 + stage * 8;
                    if (TOK) {
                        // A: this CTA's 128 token rows (then their low parts); B: the
                        // weight rows of this CTA's half of N (gate/up: CTA 0 the gate
                        // rows of the hidden block, CTA 1 its up rows)
                        tma_load_2d_pair(sa, &tm_act, fb, kc, trow, pol_a);
                        if (split)
                            tma_load_2d_pair(sa + PBM * PBK * 2, &tm_act, fb, kc,
                                             trow + (int)args.lo_rows, pol_a);
                        tma_load_2d_pair(sb, &tm_w, fb, kc,
                                         x.w * args.w_rows_per_group + x.nb * 256 + (int)v * PBM,
                                         pol_n);
                    } else if (GU) {
                        // gate rows of features 64v.., then their up rows
                        const int wrow = x.w * args.w_rows_per_group + x.nb * 256 + (int)v * 64;
                        tma_load_2d_pair(sa, &tm_w, fb, kc, wrow, pol_w);
                        tma_load_2d_pair(sa + 64 * PBK * 2, &tm_w, fb, kc, wrow + 128, pol_w);
                    } else {
                        const int wrow = x.w * args.w_rows_per_group + x.nb * 256 + (int)v * PBM;
                        tma_load_2d_pair(sa, &tm_w, fb, kc, wrow, pol_w);
                    }
                    if (!TOK) {
                        for (int r = 0; r < half; r += tb)
                            tma_load_2d_pair(sb + r * PBK * 2, &tm_act, fb, kc, trow + r, pol_a);
                        if (split)  // the low parts of H behind the high ones
                            for (int r = 0; r < half; r += tb)
                                tma_load_2d_pair(sb + L.b_lo + r * PBK * 2, &tm_act, fb, kc,
                                                 trow + r + (int)args.lo_rows, pol_a);
                    }
                    issued |= 1u << stage;
                    issued_par = (issued_par & ~(1u << stage)) | (phase << stage);
                    if (++stage == S) {
                        stage = 0;
                        phase ^= 1;
                    }
                }
            }
            // every copy issued lands before either CTA may leave: the even CTA's
            // barrier counts both CTAs' bytes of every stage it armed; the odd CTA,
            // which cannot watch that barrier, gives copies it issued after a
            // time-out a moment to land (the two producers time out on the same
            // barriers, so the even CTA has armed all the others)
            if (v == 0) {
                for (int s = 0; s < S; ++s)
                    if (issued & (1u << s))
                        mbar_wait(&full[s], (issued_par >> s) & 1, P_TEARDOWN_NS);
            } else if (!ok && issued) {
                const uint64_t t0 = globaltimer_ns();
                while (globaltimer_ns() - t0 < 100000ull) {
                }
            }
        }
    } else if (warp == 1) {
        if (lane == 0 && v == 0) {
            // ------------------------------------------------------------ MMA issuer (even CTA)
            int stage = 0;
            uint32_t phase = 0;
            int acc = 0;
            uint32_t acc_phase = 0;
            bool ok = true;
            const int kblocks = args.K / PBK;
            int qs = 0;
            uint32_t qph = 0;
            while (ok) {
                int u = total;
                if (!take_unit(qs, qph, true, &u)) {
                    report_timeout(args.status);
                    break;
                }
                if (u >= total) break;
                const PUnit x = p_decode<MODE>(tab, u);
                if (!mbar_wait_cl(&acc_empty[acc], acc_phase ^ 1, limit)) {
                    report_timeout(args.status);
                    break;
                }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + acc * acc_stride;
                const uint32_t idesc = idesc_bf16_f32(256, x.ntok);
                for (int kb = 0; kb < kblocks; ++kb) {
                    if (!mbar_wait_cl(&full[stage], phase, limit)) {
                        report_timeout(args.status);
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t sa = smem_addr(smem + stage * L.stage_bytes);
                    const uint32_t sb = sa + L.a_bytes;
#pragma unroll
                    for (int kk = 0; kk < PBK / PUK; ++kk) {
                        const uint64_t adesc = sdesc_kmajor_sw128(sa + kk * PUK * 2);
                        const uint64_t bdesc = sdesc_kmajor_sw128(sb + kk * PUK * 2);
                        umma_bf16_pair(d_tmem, adesc, bdesc, idesc, (kb > 0 || kk > 0) ? 1u : 0u);
                        if (split && TOK)  // + H_lo . W
                            umma_bf16_pair(d_tmem,
                                           sdesc_kmajor_sw128(sa + PBM * PBK * 2 + kk * PUK * 2),
                                           bdesc, idesc, 1u);
                        if (split && !TOK)  // + W . H_lo
                            umma_bf16_pair(d_tmem, adesc,
                                           sdesc_kmajor_sw128(sb + L.b_lo + kk * PUK * 2), idesc,
                                           1u);
                    }
                    umma_commit_pair_both(&empty[stage]);
                    if (++stage == S) {
                        stage = 0;
                        phase ^= 1;
                    }
                }
                if (!ok) break;
                // test hook: the pair that takes unit 0 never signals its epilogues
                // for it (any pair may take it: the units come from a counter)
                const bool withhold = args.test_stall && u == 0;
                if (!withhold) umma_commit_pair_both(&acc_full[acc]);
                if (++acc == n_acc) {
                    acc = 0;
                    acc_phase ^= 1;
                }
            }
            // every pair MMA completes before either CTA releases memory
            umma_commit_pair(drain);
            mbar_wait(drain, 0, P_TEARDOWN_NS);
        }
    } else {
        // ------------------------------------------------------------ epilogue (both CTAs)
        const int ew = warp - 2;                 // 0..NEPI-1
        const int q = warp & 3;                  // TMEM lane quarter this warp may access
        const int part = ew >> 2;                // which half of the columns
        const uint32_t lane_addr = tmem_base + ((uint32_t)(q * 32) << 16);
        const uint32_t leader_acc_empty = map_shared_rank(smem_addr(&acc_empty[0]), 0);
        // gate/up: quarters 0,1 hold gate, 2,3 the up rows of the same features;
        // the warp pair (q, q + 2) of the same part exchanges through `xb`
        const int pidx = part * 2 + (q & 1);     // pair of warps 0..3
        float4* xb = reinterpret_cast<float4*>(smem + L.xch_off) + pidx * (2 * 2 * 2 * 32);
        const bool is_gate = q < 2;
        int acc = 0;
        uint32_t acc_phase = 0;
        int qs = 0;
        uint32_t qph = 0;
        for (int it = 0;; ++it) {
            int u = total;
            bool ok = take_unit(qs, qph, false, &u);
            __syncwarp();
            if (ok && lane == 0) mbar_arrive_cluster(lead_q_empty0 + ((qs + P_QN - 1) % P_QN) * 8);
            const bool done = ok && u >= total;
            if (ok && !done) ok = mbar_wait(&acc_full[acc], acc_phase, limit);
            if (GU) {
                // both warps of a pair go on, or stop, together: 0 a wait ran
                // out, 1 the accumulator is ready, 2 no more work
                if (lane == 0) flags[ew * 2 + (it & 1)] = !ok ? 0 : (done ? 2 : 1);
                named_sync(1 + pidx, 64);
                const int partner = is_gate ? ew - 2 : ew + 2;
                const int f0 = flags[ew * 2 + (it & 1)], f1 = flags[partner * 2 + (it & 1)];
                if (f0 == 0 || f1 == 0) {
                    report_timeout(args.status);
                    break;
                }
                if (f0 == 2 || f1 == 2) break;
            } else {
                if (!ok) {
                    report_timeout(args.status);
                    break;
                }
                if (done) break;
            }
            const PUnit x = p_decode<MODE>(tab, u);
            tc_fence_after();
            const uint32_t t0 = lane_addr + acc * acc_stride;
            if (MODE == TC_PAIR_GATEUP_TOK) {
                // [gate | up] of this CTA's 128 tokens: H = silu(gate) * up
                const int r = x.mt * 256 + (int)v * PBM + q * 32 + lane;
                const bool valid = r < x.rows;
                __nv_bfloat16* dst = reinterpret_cast<__nv_bfloat16*>(args.out) +
                                     (int64_t)(x.row0 + r) * args.out_ld + x.nb * 128;
                __nv_bfloat16* abrow =
                    args.aux ? reinterpret_cast<__nv_bfloat16*>(args.aux) +
                                   (int64_t)(x.row0 + r) * args.aux_ld + x.nb * 256
                             : nullptr;
#pragma unroll 1
                for (int c = 0; c < 128; c += 16) {
                    float g[16], up[16];
                    tmem_ld16(t0 + c, g);
                    tmem_ld16(t0 + 128 + c, up);
                    tmem_ld_wait();
                    if (valid && abrow) {
                        store_bf16x16(abrow + c, g);
                        store_bf16x16(abrow + 128 + c, up);
                    }
                    if (valid) {
                        float hv[16];
#pragma unroll
                        for (int i = 0; i < 16; ++i) hv[i] = silu_f(g[i]) * up[i];
                        if (args.lo_rows) {
                            float lo[16];
#pragma unroll
                            for (int i = 0; i < 16; ++i) lo[i] = hv[i] - bf16_round(hv[i]);
                            store_bf16x16(dst + args.lo_rows * args.out_ld + c, lo);
                        }
                        store_bf16x16(dst + c, hv);
                    }
                }
            } else if (MODE == TC_PAIR_DGATE_TOK) {
                // dH of this CTA's 128 tokens for 256 hidden features; with the
                // forward's pre-activations a, b (AB, bf16): dA = dH b silu'(a),
                // dB = dH silu(a), stored interleaved per 128-wide block like AB
                const int r = x.mt * 256 + (int)v * PBM + q * 32 + lane;
                const bool valid = r < x.rows;
                const int64_t rowoff = (int64_t)(x.row0 + r) * args.aux_ld;
                const __nv_bfloat16* ab =
                    reinterpret_cast<const __nv_bfloat16*>(args.aux) + rowoff;
                __nv_bfloat16* dab = reinterpret_cast<__nv_bfloat16*>(args.out) + rowoff;
                auto ab_col = [&](int c) {
                    const int f = x.nb * 256 + c;
                    return (int64_t)(f >> 7) * 256 + (f & 127);
                };
                // the pre-activations of the next 16 features load while the
                // current ones are used
                uint4 na0 = make_uint4(0, 0, 0, 0), na1 = na0, nb0 = na0, nb1 = na0;
                if (valid) {
                    const uint4* pa = reinterpret_cast<const uint4*>(ab + ab_col(0));
                    na0 = pa[0];
                    na1 = pa[1];
                    nb0 = pa[16];
                    nb1 = pa[17];
                }
#pragma unroll 1
                for (int c = 0; c < 256; c += 16) {
                    float dh[16];
                    tmem_ld16(t0 + c, dh);
                    const uint4 ca0 = na0, ca1 = na1, cb0 = nb0, cb1 = nb1;
                    if (valid && c + 16 < 256) {
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
                        const uint32_t wa[8] = {ca0.x, ca0.y, ca0.z, ca0.w,
                                                ca1.x, ca1.y, ca1.z, ca1.w};
                        const uint32_t wb[8] = {cb0.x, cb0.y, cb0.z, cb0.w,
                                                cb1.x, cb1.y, cb1.z, cb1.w};
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
            } else if (MODE == TC_PAIR_DOWN_TOK) {
                const int r0 = x.mt * 256 + (int)v * PBM + q * 32;  // this warp's first row
                const int valid = min(32, x.rows - r0);
                float* dst0 = reinterpret_cast<float*>(args.out) +
                              (int64_t)(x.row0 + r0) * args.out_ld + x.nb * 256;
                float* stg = reinterpret_cast<float*>(smem + L.xch_off) + ew * (32 * P_STG_LD);
#pragma unroll 1
                for (int c = 0; c < 256; c += 32) {
                    float val[32];
                    tmem_ld16(t0 + c, val);
                    tmem_ld16(t0 + c + 16, val + 16);
                    tmem_ld_wait();
                    if (valid > 0)
                        p_store_rows_f32x32(stg, val, lane, dst0 + c, args.out_ld, valid);
                }
            } else if (GU) {
                // feature of this lane and its H column
                const int f = x.nb * 128 + (int)v * 64 + (q & 1) * 32 + lane;
                __nv_bfloat16* hdst =
                    reinterpret_cast<__nv_bfloat16*>(args.out) + (int64_t)x.row0 * args.out_ld + f;
                __nv_bfloat16* abdst =
                    args.aux ? reinterpret_cast<__nv_bfloat16*>(args.aux) +
                                   (int64_t)x.row0 * args.aux_ld + (f >> 7) * 256 +
                                   (is_gate ? 0 : 128) + (f & 127)
                             : nullptr;
                int ci = 0;
#pragma unroll 1
                for (int c = 16 * part; c < x.ntok; c += 32, ++ci) {
                    float mine[16];
                    tmem_ld16(t0 + c, mine);
                    tmem_ld_wait();
                    if (abdst) {
#pragma unroll
                        for (int i = 0; i < 16; ++i)
                            if (c + i < x.rows)
                                abdst[(int64_t)(c + i) * args.aux_ld] = __float2bfloat16_rn(mine[i]);
                    }
                    // gate warps compute columns c..c+7, up warps c+8..c+15: each
                    // sends the other half of its values to its partner
                    float4* out_buf = xb + ((is_gate ? 0 : 1) * 2 + (ci & 1)) * 64;
                    float4* in_buf = xb + ((is_gate ? 1 : 0) * 2 + (ci & 1)) * 64;
                    float give[8], keepv[8];  // values sent / kept (static indices only)
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        give[i] = is_gate ? mine[8 + i] : mine[i];
                        keepv[i] = is_gate ? mine[i] : mine[8 + i];
                    }
                    out_buf[lane] = make_float4(give[0], give[1], give[2], give[3]);
                    out_buf[32 + lane] = make_float4(give[4], give[5], give[6], give[7]);
                    named_sync(1 + pidx, 64);
                    const float4 o0 = in_buf[lane], o1 = in_buf[32 + lane];
                    const float other[8] = {o0.x, o0.y, o0.z, o0.w, o1.x, o1.y, o1.z, o1.w};
                    const int keep = is_gate ? 0 : 8;  // this warp's columns within the chunk
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        const int col = c + keep + i;
                        if (col < x.rows) {
                            const float g = is_gate ? keepv[i] : other[i];
                            const float up = is_gate ? other[i] : keepv[i];
                            const float hv = silu_f(g) * up;
                            hdst[(int64_t)col * args.out_ld] = __float2bfloat16_rn(hv);
                            if (args.lo_rows)
                                hdst[(int64_t)(col + args.lo_rows) * args.out_ld] =
                                    __float2bfloat16_rn(hv - bf16_round(hv));
                        }
                    }
                }
            } else {
                const int f = x.nb * 256 + (int)v * PBM + q * 32 + lane;
                float* dst = reinterpret_cast<float*>(args.out) + (int64_t)x.row0 * args.out_ld + f;
#pragma unroll 1
                for (int c = 16 * part; c < x.ntok; c += 32) {
                    float val[16];
                    tmem_ld16(t0 + c, val);
                    tmem_ld_wait();
#pragma unroll
                    for (int i = 0; i < 16; ++i)
                        if (c + i < x.rows) dst[(int64_t)(c + i) * args.out_ld] = val[i];
                }
            }
            // this warp is done with the accumulator: release it on the even CTA
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(leader_acc_empty + acc * 8);
            if (++acc == n_acc) {
                acc = 0;
                acc_phase ^= 1;
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    // neither CTA leaves (or frees TMEM) while the other may still touch its
    // shared memory or TMEM
    cluster_sync_all();
    tc_fence_after();
    if (warp == 1) tmem_dealloc_pair(tmem_base, tmem_cols);
}

template <int MODE>
int launch_pair_mode(const CUtensorMap& act, const CUtensorMap& w, const TcArgs& a, int pairs,
                     cudaStream_t st) {
    const PairLayout L =
        pair_layout(MODE, a.nt_max, a.stages, a.num_groups,
                    (MODE == TC_PAIR_DOWN || MODE == TC_PAIR_DOWN_TOK) && a.lo_rows != 0);
    auto kern = tc_pair_kernel<MODE>;
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
    if (pairs < 1 || !a.unit_ctr) {
        last_launch_error() = cudaErrorInvalidConfiguration;
        return -1;
    }
    // the cluster shape is part of the kernel (__cluster_dims__)
    launch_ex(pdl_active(), kern, dim3(2 * pairs), dim3(p_threads(MODE)), L.total, st, act, w, a);
    note_launch();
    return launch_result();
}

}  // namespace

int tc_pair_max_stages(int mode, int nt_max, int groups, bool split, int smem_limit) {
    const bool ds = (mode == TC_PAIR_DOWN || mode == TC_PAIR_DOWN_TOK) && split;
    for (int s = 8; s >= 2; --s)
        if ((int)pair_layout(mode, nt_max, s, groups, ds).total <= smem_limit) return s;
    return 0;
}

int launch_tc_pair(int mode, const CUtensorMap& act, const CUtensorMap& w, const TcArgs& a,
                   int pairs, cudaStream_t st) {
    if (!p_tok(mode) && (a.nt_max < 16 || a.nt_max > 256 || a.nt_max % 16)) return -1;
    switch (mode) {
        case TC_PAIR_GATEUP:
            return launch_pair_mode<TC_PAIR_GATEUP>(act, w, a, pairs, st);
        case TC_PAIR_DOWN:
            return launch_pair_mode<TC_PAIR_DOWN>(act, w, a, pairs, st);
        case TC_PAIR_GATEUP_TOK:
            return launch_pair_mode<TC_PAIR_GATEUP_TOK>(act, w, a, pairs, st);
        case TC_PAIR_DOWN_TOK:
            return launch_pair_mode<TC_PAIR_DOWN_TOK>(act, w, a, pairs, st);
        case TC_PAIR_DGATE_TOK:
            if (a.n_feat % 256 || !a.aux) return -1;
            return launch_pair_mode<TC_PAIR_DGATE_TOK>(act, w, a, pairs, st);
    }
    return -1;
}

}  // namespace moe
