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
//   warps 4-7   softmax + epilogue of M tile 0 (thread = row = TMEM lane),
//   warps 8-11  the same for M tile 1.
// Tensor memory (512 columns): S_0 | S_1 | O_0 | O_1; P_k (bf16) overwrites
// the first 64 columns of S_k.  The tensor pipe executes one thread's MMAs in
// issue order, so S_k(j+1) never overwrites P_k(j) before PV_k(j) has read it.
// Softmax warps rescale O_k by exp2(m_old - m_new) before the next PV, which
// is safe because the commit that signals S_k(j) also covers PV_k(j-1).
#include <cuda_bf16.h>

#include "device.cuh"
#include "internal.h"

namespace gqa {

constexpr int kPfBM = 128;      // rows per M tile
constexpr int kPfBN = 128;      // keys per K/V tile
constexpr int kPfThreads = 384;
constexpr int kPfStages = 2;

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
    int n_pairs;                      // M-tile pairs per (b, kvh)
    int causal;
    float scale_log2;                 // scale * log2(e)
    __nv_bfloat16 *o;
    float *lse;
    int *status;
};

template <int D>
__global__ void __launch_bounds__(kPfThreads, 1)
prefill_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
               const __grid_constant__ CUtensorMap tm_v, const PfParams p) {
    using Lay = PfLayout<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    __shared__ uint64_t q_full, k_full[kPfStages], k_empty[kPfStages], v_full[kPfStages],
        v_empty[kPfStages], s_full[2], p_full[2], o_done[2], mma_drain;
    __shared__ uint32_t tmem_base_sh;
    __shared__ int abort_flag;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    // ---- work unit: longest causal tiles first ----
    const int bh = blockIdx.x % (p.B * p.Hkv);
    const int pair = p.n_pairs - 1 - blockIdx.x / (p.B * p.Hkv);
    const int b = bh / p.Hkv, kvh = bh % p.Hkv;
    const int t0 = pair * 2 * p.P;                      // first position of M tile 0
    const int last_pos = min(t0 + 2 * p.P, p.Tq) - 1;   // last real position in the pair
    int kv_end = p.Tkv;                                 // keys [0, kv_end) can be visible
    if (p.causal) kv_end = min(p.Tkv, last_pos + (p.Tkv - p.Tq) + 1);
    const int n_kv = kv_end > 0 ? (kv_end + kPfBN - 1) / kPfBN : 0;

    if (threadIdx.x == 0) {
        mbar_init(&q_full, 1);
        for (int s = 0; s < kPfStages; ++s) {
            mbar_init(&k_full[s], 1);
            mbar_init(&k_empty[s], 1);
            mbar_init(&v_full[s], 1);
            mbar_init(&v_empty[s], 1);
        }
        for (int k = 0; k < 2; ++k) {
            mbar_init(&s_full[k], 1);
            mbar_init(&p_full[k], 4);
            mbar_init(&o_done[k], 1);
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

    if (warp == 0) {
        // ------------------------------------------------ TMA producer ----
        if (lane == 0 && n_kv > 0) {
            tma_prefetch_desc(&tm_q);
            tma_prefetch_desc(&tm_k);
            tma_prefetch_desc(&tm_v);
            const int q_box_bytes = 64 * p.G * p.P * 2;
            mbar_expect_tx(&q_full, 2 * Lay::kPanels * q_box_bytes);
            for (int mt = 0; mt < 2; ++mt)
                for (int pn = 0; pn < Lay::kPanels; ++pn)
                    tma_load_4d(sQ + mt * Lay::kQTile + pn * Lay::kQPanel, &tm_q, &q_full, pn * 64,
                                kvh * p.G, t0 + mt * p.P, b);
            int issued = 0;
            for (int j = 0; j < n_kv; ++j) {
                const int st = j % kPfStages;
                const uint32_t ph = (j / kPfStages) & 1;
                if (!mbar_wait(&k_empty[st], ph ^ 1, &abort_flag, p.status)) break;
                mbar_expect_tx(&k_full[st], Lay::kKTile);
                for (int pn = 0; pn < Lay::kPanels; ++pn)
                    tma_load_4d(sK + st * Lay::kKTile + pn * Lay::kKPanel, &tm_k, &k_full[st],
                                pn * 64, kvh, j * kPfBN, b);
                if (!mbar_wait(&v_empty[st], ph ^ 1, &abort_flag, p.status)) {
                    issued = j + 1;
                    break;
                }
                mbar_expect_tx(&v_full[st], Lay::kKTile);
                for (int pn = 0; pn < Lay::kPanels; ++pn)
                    tma_load_4d(sV + st * Lay::kKTile + pn * Lay::kKPanel, &tm_v, &v_full[st],
                                pn * 64, kvh, j * kPfBN, b);
                issued = j + 1;
            }
            if (abort_flag) {
                // let copies already in flight land before the block exits
                for (int j = max(0, issued - kPfStages); j < issued; ++j) {
                    const int st = j % kPfStages;
                    const uint32_t ph = (j / kPfStages) & 1;
                    mbar_wait(&k_full[st], ph, &abort_flag, p.status, 1000000ull);
                    mbar_wait(&v_full[st], ph, &abort_flag, p.status, 1000000ull);
                }
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------- MMA issuer ----
        if (lane == 0 && n_kv > 0) {
            constexpr uint32_t idesc_s = umma_idesc_bf16(kPfBM, kPfBN, 0, 0);
            constexpr uint32_t idesc_o = umma_idesc_bf16(kPfBM, D, 0, 1);
            const uint32_t sQa = smem_u32(sQ), sKa = smem_u32(sK), sVa = smem_u32(sV);
            bool ok = mbar_wait(&q_full, 0, &abort_flag, p.status);
            tc_fence_after();
            // S_k = Q_k K_st^T : K-major A and B, 16 keys of d per instruction
            auto issue_s = [&](int k, int st) {
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = (kk >> 2) * Lay::kQPanel + (kk & 3) * 32;
                    const uint64_t ad = umma_smem_desc(sQa + k * Lay::kQTile + off, 16, 1024);
                    const uint64_t bd = umma_smem_desc(sKa + st * Lay::kKTile + off, 16, 1024);
                    umma_ss(tmem + (k ? Lay::kColS1 : Lay::kColS0), ad, bd, idesc_s, kk > 0);
                }
            };
            // O_k (+)= P_k V_st : P from tensor memory, V MN-major (d contiguous)
            auto issue_pv = [&](int k, int st, bool acc) {
#pragma unroll
                for (int kk = 0; kk < kPfBN / 16; ++kk) {
                    const uint64_t bd = umma_smem_desc(sVa + st * Lay::kKTile + kk * 2048,
                                                       Lay::kKPanel, 1024);
                    umma_ts(tmem + (k ? Lay::kColO1 : Lay::kColO0),
                            tmem + (k ? Lay::kColS1 : Lay::kColS0) + kk * 8, bd, idesc_o,
                            (acc || kk > 0) ? 1u : 0u);
                }
            };
            for (int j = 0; ok && j < n_kv; ++j) {
                const int st = j % kPfStages;
                const uint32_t ph = (j / kPfStages) & 1;
                const int sp = (j + kPfStages - 1) % kPfStages;          // stage of tile j-1
                const uint32_t php = ((j - 1) / kPfStages) & 1;
                if (!(ok = mbar_wait(&k_full[st], ph, &abort_flag, p.status))) break;
                tc_fence_after();
                if (j > 0) {
                    if (!(ok = mbar_wait(&v_full[sp], php, &abort_flag, p.status))) break;
                    if (!(ok = mbar_wait(&p_full[0], (j - 1) & 1, &abort_flag, p.status))) break;
                    tc_fence_after();
                    issue_pv(0, sp, j > 1);
                }
                issue_s(0, st);
                tc_commit(&s_full[0]);
                if (j > 0) {
                    if (!(ok = mbar_wait(&p_full[1], (j - 1) & 1, &abort_flag, p.status))) break;
                    tc_fence_after();
                    issue_pv(1, sp, j > 1);
                    tc_commit(&v_empty[sp]);
                }
                issue_s(1, st);
                tc_commit(&s_full[1]);
                tc_commit(&k_empty[st]);
            }
            if (ok) {
                const int sl = (n_kv - 1) % kPfStages;
                const uint32_t phl = ((n_kv - 1) / kPfStages) & 1;
                ok = mbar_wait(&v_full[sl], phl, &abort_flag, p.status) &&
                     mbar_wait(&p_full[0], (n_kv - 1) & 1, &abort_flag, p.status);
                if (ok) {
                    tc_fence_after();
                    issue_pv(0, sl, n_kv > 1);
                    tc_commit(&o_done[0]);
                    ok = mbar_wait(&p_full[1], (n_kv - 1) & 1, &abort_flag, p.status);
                }
                if (ok) {
                    tc_fence_after();
                    issue_pv(1, sl, n_kv > 1);
                    tc_commit(&o_done[1]);
                    tc_commit(&v_empty[sl]);
                }
            }
            // every MMA this thread issued has finished before tensor memory is freed
            tc_commit(&mma_drain);
            mbar_wait(&mma_drain, 0, &abort_flag, p.status, 1000000000ull);
        }
    } else if (warp >= 4) {
        // -------------------------------------------- softmax + epilogue ----
        const int k = (warp - 4) >> 2;                  // M tile of this warpgroup
        const int r = ((warp & 3) << 5) + lane;         // row = tensor-memory lane
        const uint32_t lane_addr = tmem + ((static_cast<uint32_t>(warp & 3) * 32u) << 16);
        const uint32_t colS = k ? Lay::kColS1 : Lay::kColS0;
        const uint32_t colO = k ? Lay::kColO1 : Lay::kColO0;
        const int pos = t0 + k * p.P + r / p.G;
        const int head = kvh * p.G + r % p.G;
        const bool row_real = (r < p.P * p.G) && (pos < p.Tq);
        // last visible key of this row (keys past Tkv never count)
        int lim = p.Tkv - 1;
        if (p.causal && row_real) lim = min(lim, pos + (p.Tkv - p.Tq));
        float m_run = -INFINITY, l_run = 0.0f;
        bool ok = true;
        for (int j = 0; j < n_kv; ++j) {
            // warp-uniform outcome: the tensor-memory accesses below are .sync.aligned
            ok = __all_sync(0xffffffffu, mbar_wait(&s_full[k], j & 1, &abort_flag, p.status));
            if (!ok) break;
            tc_fence_after();
            uint32_t sr[4][32];
#pragma unroll
            for (int c = 0; c < 4; ++c) tmem_ld32(lane_addr + colS + 32 * c, sr[c]);
            tmem_wait_ld();
            const int cut = lim - j * kPfBN;            // columns > cut are masked
            float mx = -INFINITY;
            if (__any_sync(0xffffffffu, cut < kPfBN - 1)) {
#pragma unroll
                for (int c = 0; c < 4; ++c)
#pragma unroll
                    for (int e = 0; e < 32; ++e) {
                        float x = __uint_as_float(sr[c][e]) * p.scale_log2;
                        x = (32 * c + e <= cut) ? x : -INFINITY;
                        sr[c][e] = __float_as_uint(x);
                        mx = fmaxf(mx, x);
                    }
            } else {
#pragma unroll
                for (int c = 0; c < 4; ++c)
#pragma unroll
                    for (int e = 0; e < 32; ++e) {
                        const float x = __uint_as_float(sr[c][e]) * p.scale_log2;
                        sr[c][e] = __float_as_uint(x);
                        mx = fmaxf(mx, x);
                    }
            }
            const float m_new = fmaxf(m_run, mx);
            const float m_use = (m_new == -INFINITY) ? 0.0f : m_new;
            const float alpha = fast_exp2(m_run - m_use);   // 0 while nothing was seen
            // O holds tiles < j scaled by exp2(-m_run); bring it to m_new
            if (j > 0 && __any_sync(0xffffffffu, m_new > m_run)) {
#pragma unroll
                for (int c = 0; c < D / 32; ++c) {
                    uint32_t orr[32];
                    tmem_ld32(lane_addr + colO + 32 * c, orr);
                    tmem_wait_ld();
#pragma unroll
                    for (int e = 0; e < 32; ++e)
                        orr[e] = __float_as_uint(__uint_as_float(orr[e]) * alpha);
                    tmem_st32(lane_addr + colO + 32 * c, orr);
                }
            }
            m_run = m_new;
            float psum = 0.0f;
            uint32_t pp[2][32];
#pragma unroll
            for (int c = 0; c < 4; ++c)
#pragma unroll
                for (int e = 0; e < 32; e += 2) {
                    const float a = fast_exp2(__uint_as_float(sr[c][e]) - m_use);
                    const float bb = fast_exp2(__uint_as_float(sr[c][e + 1]) - m_use);
                    psum += a + bb;
                    pp[c >> 1][(c & 1) * 16 + (e >> 1)] = pack_bf16x2(a, bb);
                }
            l_run = l_run * alpha + psum;
            tmem_st32(lane_addr + colS, pp[0]);
            tmem_st32(lane_addr + colS + 32, pp[1]);
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&p_full[k]);
        }
        // ---- epilogue: O / l -> bf16, lse ----
        if (ok && n_kv > 0)
            ok = __all_sync(0xffffffffu, mbar_wait(&o_done[k], 0, &abort_flag, p.status));
        tc_fence_after();
        const float inv_l = (l_run > 0.0f) ? 1.0f / l_run : 0.0f;
        __nv_bfloat16 *dst =
            p.o + ((static_cast<size_t>(b) * p.Tq + pos) * p.Hq + head) * D;
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
            uint32_t orr[32];
            if (ok && n_kv > 0) {
                tmem_ld32(lane_addr + colO + 32 * c, orr);
                tmem_wait_ld();
            } else {
#pragma unroll
                for (int e = 0; e < 32; ++e) orr[e] = 0u;
            }
            uint32_t pk[16];
#pragma unroll
            for (int e = 0; e < 16; ++e)
                pk[e] = pack_bf16x2(__uint_as_float(orr[2 * e]) * inv_l,
                                    __uint_as_float(orr[2 * e + 1]) * inv_l);
            if (row_real) {
                uint4 *d4 = reinterpret_cast<uint4 *>(dst + 32 * c);
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    d4[e] = make_uint4(pk[4 * e], pk[4 * e + 1], pk[4 * e + 2], pk[4 * e + 3]);
            }
        }
        if (p.lse && row_real)
            p.lse[(static_cast<size_t>(b) * p.Hq + head) * p.Tq + pos] =
                (l_run > 0.0f) ? (m_run + __log2f(l_run)) * 0.69314718055994531f : -INFINITY;
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

template <int D>
static int launch_prefill_d(const void *q, const void *k, const void *v, void *o, float *lse,
                            int B, int Tq, int Tkv, int Hq, int Hkv, int causal, float scale,
                            cudaStream_t stream) {
    PfParams prm;
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
    const long long blocks = static_cast<long long>(prm.n_pairs) * B * Hkv;
    if (blocks > 0x7fffffffLL) return set_error(GQA_ERR_UNSUPPORTED, "prefill grid too large");

    CUtensorMap tq, tk, tv;
    if (int rc = encode_tmap_bf16_4d(&tq, q, D, Hq, Tq, B, 64, prm.G, prm.P, 1, 1)) return rc;
    if (int rc = encode_tmap_bf16_4d(&tk, k, D, Hkv, Tkv, B, 64, 1, kPfBN, 1, 1)) return rc;
    if (int rc = encode_tmap_bf16_4d(&tv, v, D, Hkv, Tkv, B, 64, 1, kPfBN, 1, 1)) return rc;

    auto kern = prefill_kernel<D>;
    const int smem = PfLayout<D>::kSmemBytes;
    if (int rc = check_cuda(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                 smem), "cudaFuncSetAttribute(prefill)"))
        return rc;
    kern<<<static_cast<unsigned>(blocks), kPfThreads, smem, stream>>>(tq, tk, tv, prm);
    return check_cuda(cudaGetLastError(), "prefill_kernel launch");
}

int launch_prefill(const void *q, const void *k, const void *v, void *o, float *lse, int B,
                   int Tq, int Tkv, int Hq, int Hkv, int d, int causal, float scale,
                   cudaStream_t stream) {
    if (d == 128)
        return launch_prefill_d<128>(q, k, v, o, lse, B, Tq, Tkv, Hq, Hkv, causal, scale, stream);
    return launch_prefill_d<64>(q, k, v, o, lse, B, Tq, Tkv, Hq, Hkv, causal, scale, stream);
}

}  // namespace gqa
