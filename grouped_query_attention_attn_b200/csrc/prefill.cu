// prefill.cu -- grouped-query attention forward on sm_100a tensor cores.
//
// Scores S = scale * Q K^T, causal -inf mask before the softmax, the
// max-subtracted softmax kept online in fp32, O = softmax(S) V (course
// "Неделя 7. Внимание", step 1; TT Lab "キー・バリューヘッドだけ減らしてみる",
// step 4).  Query head hq reads K/V head hq / G, G = Hq / Hkv (lab step 1).
//
// Tiling.  A 128-row M tile packs the G query heads of one KV group at
// P = floor(128 / G) consecutive positions: row r is (position t0 + r / G,
// head kvh * G + r % G).  In the [B, T, Hq, d] layout those rows are one 3-D
// box, so one TMA copy loads the tile, and every K/V tile the CTA stages in
// shared memory is used by all G heads of its group.  The causal mask depends
// on the position only.
//
// Per CTA: one (batch, KV head) and two adjacent M tiles (256 rows).
//   warp 0      TMA producer: Q tiles once, then a 2-deep ring of K tiles and
//               a 2-deep ring of V tiles (128 keys x d, 128-byte swizzle).
//   warp 1      one thread issues tcgen05.mma:  S_k = Q_k K_j^T into tensor
//               memory, then O_k += P_k V_j with P_k read from tensor memory.
//   warps 4-11  softmax + epilogue of M tile 0, two threads per row (the
//               .16x32bx2 tensor-memory shape), warps 12-19 the same for M
//               tile 1; with rotary embedding they also rotate their tile's Q
//               rows in shared memory at the start of each unit.
// Tensor memory (512 columns): S_0 | S_1 | O_0 | O_1; P_k (bf16) overwrites
// the first 64 columns of S_k.  The tensor pipe executes one thread's MMAs in
// issue order, so S_k(j+1) never overwrites P_k(j) before PV_k(j) has read it.
// Softmax warps rescale O_k by exp2(m_old - m_new) before the next PV, which
// is safe because the commit that signals S_k(j) also covers PV_k(j-1).
#include <cuda_bf16.h>
#include <atomic>
#include <climits>
#include <cmath>

#include "device.cuh"
#include "internal.h"

namespace gqa {

// Upper bound on the persistent grid set by gqa_set_prefill_grid_cap (0: none).
static std::atomic<int> g_prefill_grid_cap{0};

constexpr int kPfBM = 128;      // rows per M tile
constexpr int kPfBN = 128;      // keys per K/V tile
constexpr int kPfThreads = 640;   // 4 warps producer / MMA + 2 x 8 softmax warps
constexpr int kPfStages = 2;
// Register budget per warpgroup (setmaxnreg): 640 threads launch with 96
// registers each; warpgroup 0 (producer, MMA, rotation warps) and the
// softmax warpgroups (64 scores per thread) split them.
#ifndef GQA_PF_REGS_IO
#define GQA_PF_REGS_IO 80
#endif
constexpr int kPfRegsLaunch = 96;
constexpr int kPfRegsIo = GQA_PF_REGS_IO;
constexpr int kPfRegsSoftmax = ((kPfThreads * kPfRegsLaunch - 4 * 32 * kPfRegsIo) / (16 * 32)) / 8 * 8;
static_assert(4 * 32 * kPfRegsIo + 16 * 32 * kPfRegsSoftmax <= kPfThreads * kPfRegsLaunch,
              "register split");
constexpr float kRescaleLog2 = 8.0f;  // lazy rescale threshold (log2 units)
#ifndef GQA_POLY_PER4
#define GQA_POLY_PER4 1
#endif
constexpr int kPolyPer4 = GQA_POLY_PER4;  // pairs per 4 on the exp2 polynomial

template <int D>
struct PfLayout {
    static constexpr int kPanels = D / 64;
    static constexpr int kQPanel = kPfBM * 128;            // bytes of one 64-column panel
    static constexpr int kKPanel = kPfBN * 128;
    static constexpr int kQTile = kPanels * kQPanel;
    static constexpr int kKTile = kPanels * kKPanel;
    static constexpr int kOffQ = 0;                        // Q0, Q1
    static constexpr int kOffK = 2 * kQTile;               // K ring
    static constexpr int kOffV = kOffK + kPfStages * kKTile;  // V ring
    static constexpr int kBytes = kOffV + kPfStages * kKTile;
    static constexpr int kSmemBytes = kBytes + 1024;
    // tensor memory columns
    static constexpr uint32_t kColS0 = 0, kColS1 = 128;
    static constexpr uint32_t kColO0 = 256, kColO1 = 256 + D;
};

struct PfParams {
    int B, Tq, Tkv, Hq, Hkv, G, P;   // P = positions per M tile
    int tq_pitch;                     // rows between batches of o (>= Tq)
    int n_pairs;                      // M-tile pairs per (b, kvh)
    int causal;
    int window, sinks;                // sliding window (0 = none) and sink keys
    float scale_log2;                 // scale * log2(e)
    int q_pos0;                       // RoPE: query row t sits at position q_pos0 + t
    double log_theta;                 // RoPE: ln(theta)
    __nv_bfloat16 *o;
    float *lse;
    int *status;
};

// 32 scores of one row -> 16 packed bf16 probabilities (truncated) and their
// running sum over four accumulators.  With kPoly, kPolyPer4 of every 4 pairs
// use the exp2 polynomial to take load off the MUFU unit.
template <bool kPoly>
__device__ __forceinline__ void softmax_chunk(const uint32_t (&s)[32], float2 cc, float2 nm,
                                              uint32_t (&pk)[16], float (&acc)[4]) {
#pragma unroll
    for (int e = 0; e < 16; ++e) {
        const float2 x = fma2(make_float2(__uint_as_float(s[2 * e]), __uint_as_float(s[2 * e + 1])),
                              cc, nm);
        float2 pe;
        if (kPoly && (e & 3) < kPolyPer4)
            pe = exp2_poly2(x);
        else
            pe = make_float2(fast_exp2(x.x), fast_exp2(x.y));
        pk[e] = pack_hi16(pe.x, pe.y);
        acc[e & 3] = add_bf16x2(acc[e & 3], pk[e]);
    }
}

// One work unit: a (batch, KV head) and two adjacent M tiles (256 rows), with
// the KV tiles its rows can see.
struct PfUnit {
    int b, kvh, t0;             // t0: first position of M tile 0
    int n_kv;                   // KV tiles visited
    int n_sink_tiles, first_tile;
    // KV tiles are visited in order: the sink tiles, then the window tiles
    // (every tile below the causal limit when there is no window).
    __device__ __forceinline__ int tile(int j) const {
        return j < n_sink_tiles ? j : first_tile + (j - n_sink_tiles);
    }
};

// The i-th unit of this CTA.  Units are ranked by decreasing causal work
// (the last position pairs first); round i hands ranks [i g, (i + 1) g) to
// the g CTAs, in reverse order on odd rounds, which balances the rounds'
// decreasing costs across CTAs.  Returns false past the last unit.
__device__ __forceinline__ bool pf_unit(const PfParams &p, int i, PfUnit &u) {
    const int g = gridDim.x, c = blockIdx.x;
    const long long rank = static_cast<long long>(i) * g + ((i & 1) ? g - 1 - c : c);
    const int bhs = p.B * p.Hkv;
    if (rank >= static_cast<long long>(p.n_pairs) * bhs) return false;
    const int r = static_cast<int>(rank);
    const int bh = r % bhs;
    const int pair = p.n_pairs - 1 - r / bhs;
    u.b = bh / p.Hkv;
    u.kvh = bh % p.Hkv;
    u.t0 = pair * 2 * p.P;
    const int last_pos = min(u.t0 + 2 * p.P, p.Tq) - 1;    // last real position in the pair
    int kv_end = p.Tkv;                                      // keys [0, kv_end) can be visible
    if (p.causal) kv_end = min(p.Tkv, last_pos + (p.Tkv - p.Tq) + 1);
    u.n_sink_tiles = 0;
    u.first_tile = 0;
    if (p.window > 0 && kv_end > 0) {
        const int lo_min = u.t0 + (p.Tkv - p.Tq) - p.window + 1;   // window start, first row
        u.n_sink_tiles = (min(p.sinks, kv_end) + kPfBN - 1) / kPfBN;
        u.first_tile = max(u.n_sink_tiles, max(lo_min, 0) / kPfBN);
    }
    const int last_tile = kv_end > 0 ? (kv_end + kPfBN - 1) / kPfBN : 0;   // exclusive
    u.n_kv = u.n_sink_tiles + max(0, last_tile - u.first_tile);
    return true;
}

// Persistent kernel: one CTA per SM walks its units; the roles below stream
// across unit boundaries, so the next unit's Q load and first MMAs overlap
// the current unit's epilogue.  Iteration counters run over all units of the
// CTA (ring stages and barrier phases), unit counters over units with at
// least one KV tile.
// kRope: each tile's softmax warps rotate its Q rows in shared memory
// (rotary position embedding) after the TMA copy lands and before the first S
// product reads them.
template <int D, bool kRope>
__global__ void __launch_bounds__(kPfThreads, 1)
prefill_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
               const __grid_constant__ CUtensorMap tm_v, const PfParams p) {
    using Lay = PfLayout<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    __shared__ uint64_t q_full[2], q_empty[2], k_full[kPfStages], k_empty[kPfStages],
        v_full[kPfStages], v_empty[kPfStages], s_full[2], p_full[2][2], o_done[2], o_free[2],
        q_ready[2], mma_drain;
    __shared__ uint32_t tmem_base_sh;
    __shared__ int abort_flag;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kPfStages; ++s) {
            mbar_init(&k_full[s], 1);
            mbar_init(&k_empty[s], 1);
            mbar_init(&v_full[s], 1);
            mbar_init(&v_empty[s], 1);
        }
        for (int k = 0; k < 2; ++k) {
            mbar_init(&q_full[k], 1);
            mbar_init(&q_empty[k], 1);
            mbar_init(&s_full[k], 1);
            mbar_init(&p_full[k][0], 8);   // every softmax warp of the tile, per chunk
            mbar_init(&p_full[k][1], 8);
            mbar_init(&o_done[k], 1);
            mbar_init(&o_free[k], 8);
            mbar_init(&q_ready[k], 8);     // the tile's softmax warps, once rotated (kRope)
        }
        mbar_init(&mma_drain, 1);
        abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(&tmem_base_sh, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_base_sh;

    uint8_t *sQ = smem + Lay::kOffQ;
    uint8_t *sK = smem + Lay::kOffK;
    uint8_t *sV = smem + Lay::kOffV;

    if (warp < 4) {
    regs_dec<kPfRegsIo>();
    if (warp == 0) {
        // ------------------------------------------------ TMA producer ----
        // The whole warp runs the schedule (barrier waits stay warp-uniform);
        // one elected lane issues the copies.  The warp is not re-converged
        // after a copy (the next wait's vote does that): 1.3 % faster on a B200.
        const bool leader = elect_one();
        if (leader) {
            tma_prefetch_desc(&tm_q);
            tma_prefetch_desc(&tm_k);
            tma_prefetch_desc(&tm_v);
        }
        const uint32_t q_box_bytes = 64u * p.G * p.P * 2u;
        int gi = 0, ui = 0;         // iterations issued, active units started
        bool ok = true;
        PfUnit u;
        for (int i = 0; ok && pf_unit(p, i, u); ++i) {
            if (u.n_kv == 0) continue;
            for (int k = 0; k < 2; ++k) {           // Q tile k, once S_k of the last unit is done
                if (ui > 0 && !(ok = __all_sync(0xffffffffu, mbar_wait(&q_empty[k], (ui - 1) & 1,
                                                                        &abort_flag, p.status))))
                    break;
                if (leader) {
                    mbar_expect_tx(&q_full[k], Lay::kPanels * q_box_bytes);
                    for (int pn = 0; pn < Lay::kPanels; ++pn)
                        tma_load_4d(sQ + k * Lay::kQTile + pn * Lay::kQPanel, &tm_q, &q_full[k],
                                    pn * 64, u.kvh * p.G, u.t0 + k * p.P, u.b);
                }
            }
            ++ui;
            for (int j = 0; ok && j < u.n_kv; ++j) {
                const int st = gi % kPfStages;
                const uint32_t ph = (gi / kPfStages) & 1;
                const int row = u.tile(j) * kPfBN;
                if (!(ok = __all_sync(0xffffffffu,
                                      mbar_wait(&k_empty[st], ph ^ 1, &abort_flag, p.status))))
                    break;
                if (leader) {
                    mbar_expect_tx(&k_full[st], Lay::kKTile);
                    for (int pn = 0; pn < Lay::kPanels; ++pn)
                        tma_load_4d(sK + st * Lay::kKTile + pn * Lay::kKPanel, &tm_k, &k_full[st],
                                    pn * 64, u.kvh, row, u.b);
                }
                if (!(ok = __all_sync(0xffffffffu,
                                      mbar_wait(&v_empty[st], ph ^ 1, &abort_flag, p.status)))) {
                    ++gi;                           // K of this iteration is in flight
                    break;
                }
                if (leader) {
                    mbar_expect_tx(&v_full[st], Lay::kKTile);
                    for (int pn = 0; pn < Lay::kPanels; ++pn)
                        tma_load_4d(sV + st * Lay::kKTile + pn * Lay::kKPanel, &tm_v, &v_full[st],
                                    pn * 64, u.kvh, row, u.b);
                }
                ++gi;
            }
        }
        if (!ok) {
            // let copies that may be in flight land before the block exits
            for (int g = max(0, gi - kPfStages); g < gi; ++g) {
                const int st = g % kPfStages;
                const uint32_t ph = (g / kPfStages) & 1;
                mbar_wait(&k_full[st], ph, &abort_flag, p.status, 1000000ull);
                mbar_wait(&v_full[st], ph, &abort_flag, p.status, 1000000ull);
            }
            if (ui > 0)
                for (int k = 0; k < 2; ++k)
                    mbar_wait(&q_full[k], (ui - 1) & 1, &abort_flag, p.status, 1000000ull);
        }
    } else if (warp == 1) {
        // ------------------------------------------------- MMA issuer ----
        // The whole warp follows the schedule; one elected lane issues every
        // tcgen05.mma and tcgen05.commit (a commit tracks its own thread's MMAs).
        // Step g issues PV_0(g-1), S_0(g), PV_1(g-1), S_1(g) over the flattened
        // iterations of all units, so the two tiles keep alternating on the
        // tensor pipe across unit boundaries.
        const bool leader = elect_one();
        constexpr uint32_t idesc_s = umma_idesc_bf16(kPfBM, kPfBN, 0, 0);
        constexpr uint32_t idesc_o = umma_idesc_bf16(kPfBM, D, 0, 1);
        const uint32_t sQa = smem_u32(sQ), sKa = smem_u32(sK), sVa = smem_u32(sV);
        // Descriptors are built once; stepping along K only moves the start
        // address field (low bits, 16-byte units): +32 B per 16 elements
        // inside a 64-column panel of Q / K, +2048 B per 16 keys of V.
        static_assert(kPfStages == 2, "descriptor selects assume a 2-deep ring");
        const uint64_t dq0 = umma_smem_desc(sQa, 16, 1024);
        const uint64_t dq1 = umma_smem_desc(sQa + Lay::kQTile, 16, 1024);
        const uint64_t dk0 = umma_smem_desc(sKa, 16, 1024);
        const uint64_t dk1 = umma_smem_desc(sKa + Lay::kKTile, 16, 1024);
        const uint64_t dv0 = umma_smem_desc(sVa, Lay::kKPanel, 1024);
        const uint64_t dv1 = umma_smem_desc(sVa + Lay::kKTile, Lay::kKPanel, 1024);
        // S_k = Q_k K_st^T : K-major A and B, 16 elements of d per instruction
        auto issue_s = [&](int k, int st) {
            const uint32_t ts = tmem + (k ? Lay::kColS1 : Lay::kColS0);
            const uint64_t a = k ? dq1 : dq0, bk = st ? dk1 : dk0;
            if (leader) {
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = ((kk >> 2) * Lay::kQPanel + (kk & 3) * 32) >> 4;
                    umma_ss(ts, a + off, bk + off, idesc_s, kk > 0);
                }
            }
            __syncwarp();
        };
        // O_k (+)= P_k V_st over the keys of chunk `hf`: the softmax releases
        // P in two chunks, keys [32 hf, 32 hf + 32) and [64 + 32 hf, 96 + 32 hf)
        // (each thread of a row pair holds one 64-key half); 16 keys per
        // instruction.  P from tensor memory, V MN-major (d contiguous).
        auto issue_pv = [&](int k, int st, int hf, bool acc) {
            const uint32_t ts = tmem + (k ? Lay::kColS1 : Lay::kColS0);
            const uint32_t to = tmem + (k ? Lay::kColO1 : Lay::kColO0);
            const uint64_t bv = st ? dv1 : dv0;
            if (leader) {
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int kk = 2 * hf + (i & 1) + 4 * (i >> 1);
                    umma_ts(to, ts + kk * 8, bv + kk * (2048 >> 4), idesc_o,
                            (acc || i > 0) ? 1u : 0u);
                }
            }
            __syncwarp();
        };
        auto commit = [&](uint64_t *bar) {
            if (leader) tc_commit(bar);
            __syncwarp();
        };
        auto wait_all = [&](uint64_t *bar, uint32_t parity) {
            return __all_sync(0xffffffffu, mbar_wait(bar, parity, &abort_flag, p.status));
        };
        // PV_k of the previous step: its P, and for a unit's first PV (which
        // overwrites O_k) the previous unit's epilogue read of O_k.
        int pv_st = 0, pv_j = 0, pv_n = 0, pv_ui = 0, pv_gi = 0;
        bool pv_pending = false;
        // The softmax releases P_k in two key halves, so the first half's PV
        // runs while the second half's exponentials are computed.
        auto pv_step = [&](int k) {
            if (!wait_all(&p_full[k][0], pv_gi & 1)) return false;
            if (pv_j == 0 && pv_ui > 0 && !wait_all(&o_free[k], (pv_ui - 1) & 1)) return false;
            tc_fence_after();
            issue_pv(k, pv_st, 0, pv_j > 0);
            if (!wait_all(&p_full[k][1], pv_gi & 1)) return false;
            tc_fence_after();
            issue_pv(k, pv_st, 1, true);
            if (pv_j == pv_n - 1) commit(&o_done[k]);
            return true;
        };
        int gi = 0, ui = 0;
        bool ok = true;
        PfUnit u;
        for (int i = 0; ok && pf_unit(p, i, u); ++i) {
            if (u.n_kv == 0) continue;
            for (int j = 0; j < u.n_kv; ++j) {
                const int st = gi % kPfStages;
                const uint32_t ph = (gi / kPfStages) & 1;
                if (!(ok = wait_all(&k_full[st], ph))) break;
                if (pv_pending && !(ok = wait_all(&v_full[pv_st], (pv_gi / kPfStages) & 1))) break;
                if (pv_pending && !(ok = pv_step(0))) break;
                // at a unit boundary the last PV_1 goes first: it must not wait
                // for the new unit's Q tiles
                if (pv_pending && j == 0) {
                    if (!(ok = pv_step(1))) break;
                    commit(&v_empty[pv_st]);
                    pv_pending = false;
                }
                if (j == 0 && !(ok = wait_all(kRope ? &q_ready[0] : &q_full[0], ui & 1))) break;
                tc_fence_after();
                issue_s(0, st);
                commit(&s_full[0]);
                if (j == u.n_kv - 1) commit(&q_empty[0]);
                if (pv_pending) {
                    if (!(ok = pv_step(1))) break;
                    commit(&v_empty[pv_st]);
                }
                if (j == 0 && !(ok = wait_all(kRope ? &q_ready[1] : &q_full[1], ui & 1))) break;
                tc_fence_after();
                issue_s(1, st);
                commit(&s_full[1]);
                commit(&k_empty[st]);
                if (j == u.n_kv - 1) commit(&q_empty[1]);
                pv_st = st;
                pv_j = j;
                pv_n = u.n_kv;
                pv_ui = ui;
                pv_gi = gi;
                pv_pending = true;
                ++gi;
            }
            ++ui;
        }
        if (ok && pv_pending) {
            ok = wait_all(&v_full[pv_st], (pv_gi / kPfStages) & 1) && pv_step(0) && pv_step(1);
            if (ok) commit(&v_empty[pv_st]);
        }
        // every MMA this warp issued has finished before tensor memory is freed
        commit(&mma_drain);
        mbar_wait(&mma_drain, 0, &abort_flag, p.status, 1000000000ull);
    }
    } else {
        regs_inc<kPfRegsSoftmax>();      // marks the softmax code's budget for the compiler
        // -------------------------------------------- softmax + epilogue ----
        // Two threads per row, in one warp: warps 4-11 serve M tile 0, warps
        // 12-19 M tile 1.  Warp w reads tensor-memory lanes of its quarter
        // (w % 4), the lower or upper 16 of them; with the .16x32bx2 access
        // shape, threads t and t + 16 hold the same row, t the scores of keys
        // 0-63 and t + 16 those of keys 64-127, so the row max and the row sum
        // cross between the two with one shuffle.
        const int k = (warp - 4) >> 3;                  // M tile
        const int hh = ((warp - 4) >> 2) & 1;           // lower / upper 16 lanes of the quarter
        const int q4 = warp & 3;                        // lane quarter = SM sub-partition
        const int ch = lane >> 4;                       // column half: keys 64 ch .. 64 ch + 63
        const int r = q4 * 32 + hh * 16 + (lane & 15);  // row = tensor-memory lane
        const uint32_t lane_addr = tmem + ((static_cast<uint32_t>(q4 * 32 + hh * 16)) << 16);
        const uint32_t colS = k ? Lay::kColS1 : Lay::kColS0;
        const uint32_t colO = k ? Lay::kColO1 : Lay::kColO0;
        const float c2 = p.scale_log2;
        const int n_sinks = p.window > 0 ? p.sinks : 0;
        // Rotary embedding (kRope): the tile's 256 threads rotate its Q rows in
        // shared memory at the start of each unit, before its first S product.
        // Thread tt owns coordinate pair i (columns 2i, 2i+1) of a block of
        // consecutive rows; pairs never straddle a 16-byte chunk, so the
        // 128-byte swizzle moves whole pairs, and a warp's 32 pairs of one row
        // are 32 different banks.
        constexpr int kHalfD = D / 2, kPhases = 256 / kHalfD, kRowsPerPhase = kPfBM / kPhases;
        const int tt = ((warp - 4) & 7) * 32 + lane;   // thread of the tile, 0..255
        const int rope_i = tt % kHalfD, rope_ph = tt / kHalfD;
        const double rope_trn = kRope ? rope_turns(rope_i, kHalfD, p.log_theta) : 0.0;
        uint8_t *rope_base = sQ + k * Lay::kQTile + ((2 * rope_i) / 64) * Lay::kQPanel;
        const int rope_ck = ((2 * rope_i) % 64) / 8, rope_wd = ((2 * rope_i) % 8) / 2;
        // Rotates this tile's Q rows of unit uu (the unit's Q copy completes
        // phase `parity` of q_full[k]) and releases them to the S product.
        auto rotate_q = [&](const PfUnit &uu, uint32_t parity) {
            if (!__all_sync(0xffffffffu, mbar_wait(&q_full[k], parity, &abort_flag, p.status)))
                return false;
            auto word_of = [&](int row) {
                return reinterpret_cast<uint32_t *>(rope_base + row * 128 +
                                                    ((rope_ck ^ (row & 7)) << 4) + rope_wd * 4);
            };
            const int first = uu.t0 + k * p.P;                              // position of row 0
            const int real_rows = max(0, min(p.P, p.Tq - first)) * p.G;     // rest: zero fill
            const int r_end = min((rope_ph + 1) * kRowsPerPhase, real_rows);
            for (int r0 = rope_ph * kRowsPerPhase; r0 < r_end;) {
                const int pl = r0 / p.G;                                     // one position's rows
                const int r1 = min(r_end, (pl + 1) * p.G);
                float cs, sn;
                rope_cos_sin(p.q_pos0 + first + pl, rope_trn, cs, sn);
                for (int rr = r0; rr < r1; rr += 4) {                        // four loads in flight
                    uint32_t *w[4], v[4];
#pragma unroll
                    for (int x = 0; x < 4; ++x) w[x] = word_of(min(rr + x, r1 - 1));
#pragma unroll
                    for (int x = 0; x < 4; ++x) v[x] = *w[x];
#pragma unroll
                    for (int x = 0; x < 4; ++x)   // a clamped tail row repeats the last one
                        if (rr + x < r1) *w[x] = rope_rotate_pair(v[x], cs, sn);
                }
                r0 = r1;
            }
            // the tensor core reads the tile through the async proxy
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(&q_ready[k]);
            return true;
        };
        int gi = 0, ui = 0;
        bool ok = true;
        PfUnit u;
        for (int i = 0; ok && pf_unit(p, i, u); ++i) {
            const int pos = u.t0 + k * p.P + r / p.G;
            const bool row_real = (r < p.P * p.G) && (pos < p.Tq);
            // output row and lse slot, formed only where they are written
            auto out_row = [&]() {
                const int head = u.kvh * p.G + r % p.G;
                return p.o + ((static_cast<size_t>(u.b) * p.tq_pitch + pos) * p.Hq + head) * D +
                       (D / 2) * ch;
            };
            auto lse_slot = [&]() {
                const int head = u.kvh * p.G + r % p.G;
                return p.lse + (static_cast<size_t>(u.b) * p.Hq + head) * p.Tq + pos;
            };
            if (u.n_kv == 0) {
                // no visible key for any row of the unit: o = 0, lse = -inf
                if (row_real) {
                    __nv_bfloat16 *dst = out_row();
#pragma unroll
                    for (int e = 0; e < D / 16; ++e)
                        reinterpret_cast<uint4 *>(dst)[e] = make_uint4(0u, 0u, 0u, 0u);
                    if (p.lse && ch == 0) *lse_slot() = -INFINITY;
                }
                continue;
            }
            // the unit's Q rows are rotated before its first S product
            if constexpr (kRope) {
                if (!(ok = rotate_q(u, ui & 1))) break;
            }
            // visible keys of this row: key <= lim, and key >= lo or key < sinks
            // (keys past Tkv never count; lo / sinks only with a sliding window)
            int lim = p.Tkv - 1;
            if (p.causal && row_real) lim = min(lim, pos + (p.Tkv - p.Tq));
            const int lo =
                (p.window > 0 && row_real) ? pos + (p.Tkv - p.Tq) - p.window + 1 : INT_MIN;
            // Online softmax with a lazily moved reference max: O and l stay
            // scaled by exp2(-m_ref) and m_ref only moves when the row's max
            // exceeds it by more than kRescaleLog2 (P then stays <=
            // 2^kRescaleLog2).  Exact in real arithmetic: the epilogue divides
            // by l taken at the same m_ref.  Both threads of a row see the same
            // row max, so they take identical m_ref / alpha decisions; each
            // keeps the partial l of its keys.
            float m_ref = -INFINITY, l_run = 0.0f;
            for (int j = 0; j < u.n_kv; ++j, ++gi) {
                // warp-uniform outcome: the tensor-memory accesses below are .sync.aligned
                ok = __all_sync(0xffffffffu, mbar_wait(&s_full[k], gi & 1, &abort_flag, p.status));
                if (!ok) break;
                tc_fence_after();
                uint32_t sr[64];
                tmem_ld_16x32bx2_x64<64>(lane_addr + colS, sr);
                tmem_wait_ld();
                const int key0 = u.tile(j) * kPfBN + 64 * ch;   // key of my first column
                const bool masked = __any_sync(
                    0xffffffffu, key0 + 63 > lim || (key0 < lo && key0 + 63 >= n_sinks));
                if (masked) {
#pragma unroll
                    for (int e = 0; e < 64; ++e) {
                        const int key = key0 + e;
                        if (key > lim || (key < lo && key >= n_sinks))
                            sr[e] = __float_as_uint(-INFINITY);
                    }
                }
                // row max of the raw scores (scale > 0 keeps the order): 4
                // chains of 16 scores, then the partner thread's half
                float mx4[4];
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    const uint32_t *v = &sr[16 * c];
                    float m = __uint_as_float(v[0]);
#pragma unroll
                    for (int e = 1; e < 15; e += 2)
                        m = max3f(m, __uint_as_float(v[e]), __uint_as_float(v[e + 1]));
                    mx4[c] = fmaxf(m, __uint_as_float(v[15]));
                }
                float mx = fmaxf(fmaxf(mx4[0], mx4[1]), fmaxf(mx4[2], mx4[3]));
                mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
                const float mxs = mx * c2;
                const bool move = mxs > m_ref + kRescaleLog2;  // always true on the first key seen
                float alpha = 1.0f;
                if (move) {
                    alpha = fast_exp2(m_ref - mxs);     // 0 when nothing was seen before
                    m_ref = mxs;
                }
                // O holds tiles < j at the old reference: rescale rows whose
                // reference moved, before this tile's first P chunk is released
                if (j > 0 && __any_sync(0xffffffffu, move)) {
                    const float2 a2 = make_float2(alpha, alpha);
#pragma unroll 1
                    for (int c = 0; c < D / 32; ++c) {
                        uint32_t orr[16];
                        tmem_ld_16x32bx2_x16<D / 2>(lane_addr + colO + 16 * c, orr);
                        tmem_wait_ld();
#pragma unroll
                        for (int e = 0; e < 16; e += 2) {
                            const float2 v2 = mul2(make_float2(__uint_as_float(orr[e]),
                                                               __uint_as_float(orr[e + 1])), a2);
                            orr[e] = __float_as_uint(v2.x);
                            orr[e + 1] = __float_as_uint(v2.y);
                        }
                        tmem_st_16x32bx2_x16<D / 2>(lane_addr + colO + 16 * c, orr);
                    }
                }
                const float m_use = (m_ref == -INFINITY) ? 0.0f : m_ref;
                const float2 cc = make_float2(c2, c2), nm = make_float2(-m_use, -m_use);
                float acc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
                // P = exp2(s * scale * log2e - m_ref), truncated to bf16; P
                // overwrites the first 64 columns of S (keys 2c, 2c + 1 in packed
                // column c; this thread's keys 64 ch + [0, 64) in packed columns
                // 32 ch + [0, 32)).  l sums exactly the bf16 weights the PV
                // product uses, so O / l is a convex combination of V rows.
                // Tiles with masked (-inf) scores use the MUFU exp only; full
                // tiles send part of the pairs to the FMA-pipe polynomial.  The
                // chunk of 32 keys is released to the PV product once stored.
#pragma unroll
                for (int hf = 0; hf < 2; ++hf) {
                    uint32_t pk[16];
                    const uint32_t(&src)[32] = *reinterpret_cast<const uint32_t(*)[32]>(&sr[32 * hf]);
                    if (masked)
                        softmax_chunk<false>(src, cc, nm, pk, acc);
                    else
                        softmax_chunk<true>(src, cc, nm, pk, acc);
                    tmem_st_16x32bx2_x16<32>(lane_addr + colS + 16 * hf, pk);
                    tmem_wait_st();
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&p_full[k][hf]);
                }
                l_run = l_run * alpha + ((acc[0] + acc[1]) + (acc[2] + acc[3]));
            }
            if (!ok) break;
            // ---- epilogue: O / l -> bf16, lse (each thread writes its D/2 columns) ----
            // O_k is read out of tensor memory, then released to the next
            // unit's first PV before the conversion and the global stores.
            ok = __all_sync(0xffffffffu, mbar_wait(&o_done[k], ui & 1, &abort_flag, p.status));
            if (!ok) break;
            tc_fence_after();
            uint32_t orr[D / 32][16];
#pragma unroll
            for (int c = 0; c < D / 32; ++c)
                tmem_ld_16x32bx2_x16<D / 2>(lane_addr + colO + 16 * c, orr[c]);
            tmem_wait_ld();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&o_free[k]);
            ++ui;
            const float l_row = l_run + __shfl_xor_sync(0xffffffffu, l_run, 16);
            const float inv_l = (l_row > 0.0f) ? 1.0f / l_row : 0.0f;
            if (row_real) {
                __nv_bfloat16 *dst = out_row();
#pragma unroll
                for (int c = 0; c < D / 32; ++c) {
                    uint4 *d4 = reinterpret_cast<uint4 *>(dst + 16 * c);
#pragma unroll
                    for (int e = 0; e < 2; ++e) {
                        const uint32_t *v = &orr[c][8 * e];
                        d4[e] = make_uint4(
                            pack_bf16x2(__uint_as_float(v[0]) * inv_l, __uint_as_float(v[1]) * inv_l),
                            pack_bf16x2(__uint_as_float(v[2]) * inv_l, __uint_as_float(v[3]) * inv_l),
                            pack_bf16x2(__uint_as_float(v[4]) * inv_l, __uint_as_float(v[5]) * inv_l),
                            pack_bf16x2(__uint_as_float(v[6]) * inv_l, __uint_as_float(v[7]) * inv_l));
                    }
                }
                if (p.lse && ch == 0)
                    *lse_slot() = (l_row > 0.0f) ? (m_ref + __log2f(l_row)) * 0.69314718055994531f
                                                 : -INFINITY;
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

template <int D, bool kRope>
static int launch_prefill_d(const void *q, const void *k, const void *v, void *o, float *lse,
                            int B, int Tq, int Tkv, int Hq, int Hkv, int causal, int window,
                            int sinks, float scale, cudaStream_t stream, int tq_pitch,
                            int tkv_pitch, int q_pos0, float theta) {
    PfParams prm;
    prm.q_pos0 = q_pos0;
    prm.log_theta = kRope ? log(static_cast<double>(theta)) : 0.0;
    prm.tq_pitch = tq_pitch > 0 ? tq_pitch : Tq;
    prm.window = window;
    prm.sinks = sinks;
    prm.B = B;
    prm.Tq = Tq;
    prm.Tkv = Tkv;
    prm.Hq = Hq;
    prm.Hkv = Hkv;
    prm.G = Hq / Hkv;
    prm.P = kPfBM / prm.G;
    const int n_mt = (Tq + prm.P - 1) / prm.P;
    prm.n_pairs = (n_mt + 1) / 2;
    prm.causal = causal;
    prm.scale_log2 = scale * 1.4426950408889634f;
    prm.o = static_cast<__nv_bfloat16 *>(o);
    prm.lse = lse;
    prm.status = device_status_ptr();
    if (!prm.status) return GQA_ERR_CUDA;
    const long long units = static_cast<long long>(prm.n_pairs) * B * Hkv;
    if (units > 0x7fffffffLL) return set_error(GQA_ERR_UNSUPPORTED, "prefill grid too large");
    int n_sm = 0;
    if (int rc = sm_count(&n_sm)) return rc;
    long long blocks = units < n_sm ? units : n_sm;   // persistent: one CTA per SM
    const int cap = g_prefill_grid_cap.load(std::memory_order_relaxed);
    if (cap > 0 && cap < blocks) blocks = cap;

    CUtensorMap tq, tk, tv;
    const uint64_t kv_pitch = tkv_pitch > 0 ? tkv_pitch : Tkv;
    if (int rc = encode_tmap_bf16_4d(&tq, q, D, Hq, Tq, B, 64, prm.G, prm.P, 1, 1, prm.tq_pitch))
        return rc;
    if (int rc = encode_tmap_bf16_4d(&tk, k, D, Hkv, Tkv, B, 64, 1, kPfBN, 1, 1, kv_pitch))
        return rc;
    if (int rc = encode_tmap_bf16_4d(&tv, v, D, Hkv, Tkv, B, 64, 1, kPfBN, 1, 1, kv_pitch))
        return rc;

    auto kern = prefill_kernel<D, kRope>;
    const int smem = PfLayout<D>::kSmemBytes;
    // once per context: the register check and the shared-memory opt-in
    static CtxSlot setup;
    if (int rc = once_per_context(setup, [&](int) {
            // the setmaxnreg split adds up only at the launch budget it was sized
            // for: a build with fewer registers per thread would leave the softmax
            // warpgroups waiting for registers, so it is refused here
            cudaFuncAttributes fa;
            if (int e = check_cuda(cudaFuncGetAttributes(&fa, kern), "cudaFuncGetAttributes(prefill)"))
                return e;
            if (fa.numRegs != kPfRegsLaunch)
                return set_error(GQA_ERR_UNSUPPORTED,
                                 "prefill kernel built with %d registers per thread, %d expected",
                                 fa.numRegs, kPfRegsLaunch);
            return check_cuda(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                   smem), "cudaFuncSetAttribute(prefill)");
        }))
        return rc;
    kern<<<static_cast<unsigned>(blocks), kPfThreads, smem, stream>>>(tq, tk, tv, prm);
    return check_cuda(cudaGetLastError(), "prefill_kernel launch");
}

void set_prefill_grid_cap(int max_ctas) {
    g_prefill_grid_cap.store(max_ctas > 0 ? max_ctas : 0, std::memory_order_relaxed);
}

int launch_prefill(const void *q, const void *k, const void *v, void *o, float *lse, int B,
                   int Tq, int Tkv, int Hq, int Hkv, int d, int causal, int window, int sinks,
                   float scale, cudaStream_t stream, int tq_pitch, int tkv_pitch, float rope_theta,
                   int q_pos0) {
    const bool rope = rope_theta > 0.0f;
    if (d == 128)
        return rope ? launch_prefill_d<128, true>(q, k, v, o, lse, B, Tq, Tkv, Hq, Hkv, causal,
                                                  window, sinks, scale, stream, tq_pitch, tkv_pitch,
                                                  q_pos0, rope_theta)
                    : launch_prefill_d<128, false>(q, k, v, o, lse, B, Tq, Tkv, Hq, Hkv, causal,
                                                   window, sinks, scale, stream, tq_pitch,
                                                   tkv_pitch, 0, 0.0f);
    return rope ? launch_prefill_d<64, true>(q, k, v, o, lse, B, Tq, Tkv, Hq, Hkv, causal, window,
                                             sinks, scale, stream, tq_pitch, tkv_pitch, q_pos0,
                                             rope_theta)
                : launch_prefill_d<64, false>(q, k, v, o, lse, B, Tq, Tkv, Hq, Hkv, causal, window,
                                              sinks, scale, stream, tq_pitch, tkv_pitch, 0, 0.0f);
}

}  // namespace gqa
