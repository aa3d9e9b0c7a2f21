// backward.cu -- gradients of grouped-query attention: dQ, dK, dV (bf16 in and
// out, fp32 accumulation).
//
// With P = softmax of the masked, scaled scores (recomputed from the forward's
// log-sum-exp) and D_i = <dO_i, O_i>:
//   dV_j = sum_i P_ij dO_i,   dP_ij = <dO_i, V_j>,   dS_ij = P_ij (dP_ij - D_i),
//   dQ_i = scale sum_j dS_ij K_j,   dK_j = scale sum_i dS_ij Q_i.
// Query head hq reads K/V head hq / G, so the gradient of a shared K/V head is
// the SUM over the G query heads of its group (K3 notes "GVA", "Backward:
// view + sum": the backward of a copy is a sum).  Three kernels:
//   rowdot  D = rowsum(dO * O)                                  (HBM-bound)
//   dkdv    tcgen05: one CTA per 128 keys of one KV head; loops over every
//           query row of the G heads of the group, so dK and dV accumulate
//           in tensor memory with no atomics
//   dq      tcgen05: one CTA per 128-row M tile (the group's heads packed by
//           position, as in the forward), looping over the visible keys
// dkdv and dq read the same inputs and write disjoint outputs, so after
// rowdot they run side by side: dkdv on a second stream, enqueued first so
// that its blocks (the longest first) are dispatched first, and dq on the
// caller's stream, its persistent CTAs taking the SMs that dkdv's tail frees.
#include <cuda_bf16.h>
#include <climits>
#include <mutex>

#include "device.cuh"
#include "internal.h"

namespace gqa {

// Visibility of key j to the query row at position i (causal bottom-right,
// optional sliding window with sinks).
struct Vis {
    int Tq, Tkv, causal, window, sinks;
    __device__ __forceinline__ bool operator()(int i, int j) const {
        if (i >= Tq || j >= Tkv) return false;
        const int p = i + (Tkv - Tq);
        if (causal && j > p) return false;
        if (window > 0 && j <= p - window && j >= sinks) return false;
        return true;
    }
};

// Every (query, key) pair of rows [i0, i0 + ni) x keys [j0, j0 + nj) visible?
__device__ __forceinline__ bool block_visible(const Vis &v, int i0, int ni, int j0, int nj) {
    if (i0 + ni > v.Tq || j0 + nj > v.Tkv) return false;
    const int p0 = i0 + (v.Tkv - v.Tq);                 // key position of the first row
    if (v.causal && j0 + nj - 1 > p0) return false;
    // window: the last row's window must still reach key j0 (sinks aside)
    if (v.window > 0 && j0 <= p0 + ni - 1 - v.window && j0 + nj > v.sinks) return false;
    return true;
}

// ------------------------------------------------------------- rowdot ---
// D = rowsum(dO o O) per (b, t, h), stored [B, H, T].  A group of D / 8 lanes
// owns kRowdotRows consecutive rows and reads them as 16-byte vectors (all
// loads in flight before the products), then reduces each row over the group.
constexpr int kRowdotRows = 2;

template <int D>
__global__ void __launch_bounds__(256)
rowdot_kernel(const __nv_bfloat16 *__restrict__ dout, const __nv_bfloat16 *__restrict__ o,
              float *__restrict__ Dsum, unsigned int *__restrict__ tile_counter, int B, int T,
              int H) {
    constexpr int kLanes = D / 8;                   // lanes per row: 8 or 16
    // the dQ kernel's tile counter starts from zero (it runs next on this stream)
    if (blockIdx.x == 0 && threadIdx.x == 0) *tile_counter = 0u;
    const long long rows = static_cast<long long>(B) * T * H;
    const long long gt = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
    const int c8 = threadIdx.x % kLanes;
    const long long row0 = gt / kLanes * kRowdotRows;
    uint4 x[kRowdotRows], y[kRowdotRows];
#pragma unroll
    for (int u = 0; u < kRowdotRows; ++u) {
        const long long r = row0 + u;
        if (r < rows) {
            x[u] = reinterpret_cast<const uint4 *>(dout + r * D)[c8];
            y[u] = reinterpret_cast<const uint4 *>(o + r * D)[c8];
        }
    }
#pragma unroll
    for (int u = 0; u < kRowdotRows; ++u) {
        const long long r = row0 + u;
        float acc = 0.0f;
        if (r < rows) {
            const uint32_t *xa = reinterpret_cast<const uint32_t *>(&x[u]);
            const uint32_t *ya = reinterpret_cast<const uint32_t *>(&y[u]);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float2 xf = bf16x2_to_float2(xa[e]), yf = bf16x2_to_float2(ya[e]);
                acc = fmaf(xf.x, yf.x, fmaf(xf.y, yf.y, acc));
            }
        }
        // every lane of the warp takes part in the shuffles (rows past the end add 0)
#pragma unroll
        for (int off = kLanes / 2; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
        if (c8 == 0 && r < rows) {
            const long long bt = r / H;
            const int h = static_cast<int>(r - bt * H);
            const long long b = bt / T, t = bt - b * T;
            Dsum[(b * H + h) * T + t] = acc;
        }
    }
}

// ------------------------------------------------------ dk dv (tcgen05) ---
// One CTA per 128 keys of one KV head (heaviest causal tiles first).  The K
// and V tiles stay in shared memory; for every 128-row query block of every
// query head of the group (an "item"):
//   tensor pipe   S^T = K Q^T and dP^T = V dO^T into tensor memory (M = 128
//                 keys, N = 128 queries);
//   16 warps      P^T = exp2(S^T * scale * log2e - lse_q * log2e) and
//                 dS^T = P^T (dP^T - D_q), bf16, written back over the first
//                 columns of each quarter's S^T / dP^T (four threads per key
//                 row, one per 32-query quarter);
//   tensor pipe   dV += P^T dO and dK += dS^T Q with P^T / dS^T read from
//                 tensor memory (dV and dK accumulate over all items).
// Issue order S(0) dP(0) | dV(0) S(1) | dK(0) dP(1) | dV(1) S(2) | ...: the
// next S^T is issued right behind the dV product that reads the P^T it
// overwrites (products run in issue order), so it runs while the warps form
// dS^T and is ready when they finish; dP^T(i+1) follows dK(i), which reads
// dS^T(i) from the region it overwrites.  S^T(i+1) therefore needs Q(i+1)
// about one elementwise phase after dK(i-1) has released a Q stage: Q has a
// 3-deep ring, dO (released by dV, earlier) a 2-deep one, each with its own
// barriers.  The item's lse travels with Q; its D (read by the warps after dV
// has released dO) has a 2-deep buffer of its own that the warps release.
// Tensor memory (512 columns): S^T | dP^T | dV | dK.  Shared memory (all of
// it dynamic, 1024-byte aligned, barriers at the end): K, V, the Q and dO
// rings, lse and D.
constexpr int kTcBK = 128;       // keys per CTA
constexpr int kTcBQ = 128;       // query rows per item
constexpr int kTcThreads = 640;  // producer, MMA, 2 idle, 16 elementwise warps
constexpr int kTcElemWarps = 16;   // 4 per tensor-memory lane group, 32 columns each
constexpr int kTcQStages = 3;
constexpr int kTcOStages = 2;

template <int D>
struct TcLayout {
    static constexpr int kPanels = D / 64;
    static constexpr int kPanel = 128 * 128;               // 128 rows x 64 bf16
    static constexpr int kTile = kPanels * kPanel;
    static constexpr int kOffK = 0, kOffV = kTile;
    static constexpr int kOffQ = 2 * kTile;                          // [kTcQStages]
    static constexpr int kOffO = kOffQ + kTcQStages * kTile;         // [kTcOStages]
    static constexpr int kOffL = kOffO + kTcOStages * kTile;         // [kTcQStages][128] f32
    static constexpr int kOffD = kOffL + kTcQStages * kTcBQ * 4;     // [2][128] f32
    // barriers: kv_full, q_full[3], q_empty[3], o_full[2], o_empty[2],
    // d_full[2], d_empty[2], s_full, dp_full, p_full, ds_full, acc_done
    static constexpr int kNumBars = 1 + 2 * kTcQStages + 2 * kTcOStages + 4 + 5;
    static constexpr int kOffBar = kOffD + 2 * kTcBQ * 4;
    static constexpr int kOffMisc = kOffBar + kNumBars * 8;          // tmem base, abort flag
    static constexpr int kSmemBytes = kOffMisc + 16;
    static constexpr uint32_t kColS = 0, kColP = 128, kColDV = 256, kColDK = 256 + D;
};
static_assert(TcLayout<128>::kSmemBytes <= 232448, "dK/dV shared memory");

struct TcParams {
    int B, Tq, Tkv, Hq, Hkv, G;
    int n_kt;                         // key tiles per (b, kvh)
    Vis vis;
    float scale, scale_log2;
    const float *lse, *Dsum;
    __nv_bfloat16 *dk, *dv;
    int *status;
};

template <int D>
__global__ void __launch_bounds__(kTcThreads, 1)
dkdv_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
               const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o,
               const TcParams p) {
    using Lay = TcLayout<D>;
    // the whole budget is used: the window must start 1024-byte aligned (the
    // 128-byte swizzle's requirement) with no room to align it here
    extern __shared__ __align__(1024) uint8_t smem[];
    if (smem_u32(smem) & 1023u) {
        if (threadIdx.x == 0) record_status(p.status, GQA_ERR_CUDA);
        return;
    }
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + Lay::kOffBar);
    uint64_t *kv_full = bars, *q_full = bars + 1, *q_empty = q_full + kTcQStages;
    uint64_t *o_full = q_empty + kTcQStages, *o_empty = o_full + kTcOStages;
    uint64_t *d_full = o_empty + kTcOStages, *d_empty = d_full + 2;
    uint64_t *s_full = d_empty + 2, *dp_full = s_full + 1, *p_full = s_full + 2;
    uint64_t *ds_full = s_full + 3, *acc_done = s_full + 4;
    uint32_t *tmem_base_sh = reinterpret_cast<uint32_t *>(smem + Lay::kOffMisc);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + Lay::kOffMisc + 4);
    float *sL = reinterpret_cast<float *>(smem + Lay::kOffL);
    float *sD = reinterpret_cast<float *>(smem + Lay::kOffD);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    const int bhs = p.Hkv * p.B, lin = blockIdx.x;
    const int kt = lin / bhs, kvh = lin % p.Hkv, b = (lin / p.Hkv) % p.B;
    const int k0 = kt * kTcBK;
    // query rows that can see a key of this tile
    const int off = p.Tkv - p.Tq;
    int q_lo = 0, q_hi = p.Tq;
    if (p.vis.causal) {
        q_lo = max(0, k0 - off);
        if (p.vis.window > 0 && k0 >= p.vis.sinks)
            q_hi = min(p.Tq, k0 + kTcBK - 1 + p.vis.window - off);
    }
    const int qb0 = q_lo / kTcBQ;
    const int n_qb = q_hi > q_lo ? (q_hi + kTcBQ - 1) / kTcBQ - qb0 : 0;
    const int n_items = p.G * n_qb;

    if (threadIdx.x == 0) {
        mbar_init(kv_full, 1);
        for (int s = 0; s < kTcQStages; ++s) {
            mbar_init(&q_full[s], 2);    // the copy's arrival and the lse stores'
            mbar_init(&q_empty[s], 1);
        }
        for (int s = 0; s < kTcOStages; ++s) {
            mbar_init(&o_full[s], 1);
            mbar_init(&o_empty[s], 1);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(&d_full[s], 1);
            mbar_init(&d_empty[s], kTcElemWarps);
        }
        mbar_init(s_full, 1);
        mbar_init(dp_full, 1);
        mbar_init(p_full, kTcElemWarps);
        mbar_init(ds_full, kTcElemWarps);
        mbar_init(acc_done, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(tmem_base_sh, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_base_sh;

    if (warp < 4) {
    if (warp == 0) {
        // ------------------------------------------------ TMA producer ----
        // Per item: Q and its lse (the copy is issued first and the lse stored
        // while it flies), dO, then D once the warps have released its buffer.
        const bool leader = elect_one();
        if (n_items > 0) {
            if (leader) {
                tma_prefetch_desc(&tm_q);
                tma_prefetch_desc(&tm_o);
                mbar_expect_tx(kv_full, 2 * Lay::kTile);
                for (int pn = 0; pn < Lay::kPanels; ++pn) {
                    tma_load_4d(smem + Lay::kOffK + pn * Lay::kPanel, &tm_k, kv_full, pn * 64,
                                kvh, k0, b);
                    tma_load_4d(smem + Lay::kOffV + pn * Lay::kPanel, &tm_v, kv_full, pn * 64,
                                kvh, k0, b);
                }
            }
            __syncwarp();
            int issued_q = 0, issued_o = 0;
            for (int it = 0; it < n_items; ++it) {
                const int g = it / n_qb, q0 = (qb0 + it % n_qb) * kTcBQ, hq = kvh * p.G + g;
                const size_t lrow = (static_cast<size_t>(b) * p.Hq + hq) * p.Tq;
                const int qs = it % kTcQStages, os = it % kTcOStages;
                if (!__all_sync(0xffffffffu, mbar_wait(&q_empty[qs], ((it / kTcQStages) & 1) ^ 1,
                                                       abort_flag, p.status)))
                    break;
                if (leader) {
                    mbar_expect_tx(&q_full[qs], Lay::kTile);
                    for (int pn = 0; pn < Lay::kPanels; ++pn)
                        tma_load_4d(smem + Lay::kOffQ + qs * Lay::kTile + pn * Lay::kPanel, &tm_q,
                                    &q_full[qs], pn * 64, hq, q0, b);
                }
                // lse in log2 units (rows past Tq: 0)
#pragma unroll
                for (int e = 0; e < kTcBQ / 32; ++e) {
                    const int r = lane + 32 * e, qi = q0 + r;
                    sL[qs * kTcBQ + r] = qi < p.Tq ? p.lse[lrow + qi] * 1.4426950408889634f : 0.0f;
                }
                __syncwarp();
                if (leader) mbar_arrive(&q_full[qs]);
                __syncwarp();
                issued_q = it + 1;
                if (!__all_sync(0xffffffffu, mbar_wait(&o_empty[os], ((it / kTcOStages) & 1) ^ 1,
                                                       abort_flag, p.status)))
                    break;
                if (leader) {
                    mbar_expect_tx(&o_full[os], Lay::kTile);
                    for (int pn = 0; pn < Lay::kPanels; ++pn)
                        tma_load_4d(smem + Lay::kOffO + os * Lay::kTile + pn * Lay::kPanel, &tm_o,
                                    &o_full[os], pn * 64, hq, q0, b);
                }
                __syncwarp();
                issued_o = it + 1;
                const int ds_ = it & 1;
                if (!__all_sync(0xffffffffu, mbar_wait(&d_empty[ds_], ((it >> 1) & 1) ^ 1,
                                                       abort_flag, p.status)))
                    break;
#pragma unroll
                for (int e = 0; e < kTcBQ / 32; ++e) {
                    const int r = lane + 32 * e, qi = q0 + r;
                    sD[ds_ * kTcBQ + r] = qi < p.Tq ? p.Dsum[lrow + qi] : 0.0f;
                }
                __syncwarp();
                if (leader) mbar_arrive(&d_full[ds_]);
                __syncwarp();
            }
            // copies still in flight land before the block exits
            mbar_wait(kv_full, 0, abort_flag, p.status, 1000000ull);
            for (int it = max(0, issued_q - kTcQStages); it < issued_q; ++it)
                mbar_wait(&q_full[it % kTcQStages], (it / kTcQStages) & 1, abort_flag, p.status,
                          1000000ull);
            for (int it = max(0, issued_o - kTcOStages); it < issued_o; ++it)
                mbar_wait(&o_full[it % kTcOStages], (it / kTcOStages) & 1, abort_flag, p.status,
                          1000000ull);
        }
    } else if (warp == 1) {
        // ------------------------------------------------- MMA issuer ----
        // The whole warp follows the schedule and waits on every barrier (the
        // vote in each wait re-converges it); one elected lane issues the
        // products and commits.  A lone thread running the same schedule (the
        // other lanes parked at the warp's end) made the backward 11 % slower on
        // a B200.
        if (n_items > 0) {
            const bool leader = elect_one();
            constexpr uint32_t idesc_s = umma_idesc_bf16(kTcBK, kTcBQ, 0, 0);
            constexpr uint32_t idesc_o = umma_idesc_bf16(kTcBK, D, 0, 1);
            const uint32_t base = smem_u32(smem);
            const uint64_t dK = umma_smem_desc(base + Lay::kOffK, 16, 1024);
            const uint64_t dV = umma_smem_desc(base + Lay::kOffV, 16, 1024);
            auto wait = [&](uint64_t *bar, uint32_t parity) {
                return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort_flag, p.status));
            };
            // S^T = K Q^T or dP^T = V dO^T into `col`: K-major A and B (+32 B per
            // 16 of d), committed to `bar`
            auto issue_s = [&](uint32_t col, uint64_t a, uint32_t off_b, uint64_t *bar) {
                const uint64_t bd = umma_smem_desc(base + off_b, 16, 1024);
                if (leader) {
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk) {
                        const uint32_t o = ((kk >> 2) * Lay::kPanel + (kk & 3) * 32) >> 4;
                        umma_ss(tmem + col, a + o, bd + o, idesc_s, kk > 0);
                    }
                    tc_commit(bar);
                }
            };
            // dV += P^T dO, dK += dS^T Q: A from tensor memory (quarter u of the
            // queries at columns 32 u .. 32 u + 15, 8 per 16 queries), B MN-major
            // (+2048 B per 16 queries)
            auto issue_acc = [&](bool first, uint32_t col_acc, uint32_t col_a, uint32_t off_b) {
                const uint64_t vb = umma_smem_desc(base + off_b, Lay::kPanel, 1024);
                if (leader) {
#pragma unroll
                    for (int kk = 0; kk < kTcBQ / 16; ++kk) {
                        const uint32_t ca = (kk >> 1) * 32 + (kk & 1) * 8;
                        umma_ts(tmem + col_acc, tmem + col_a + ca, vb + kk * (2048 >> 4), idesc_o,
                                (!first || kk > 0) ? 1u : 0u);
                    }
                }
            };
            auto q_off = [](int it) { return Lay::kOffQ + (it % kTcQStages) * Lay::kTile; };
            auto o_off = [](int it) { return Lay::kOffO + (it % kTcOStages) * Lay::kTile; };
            bool ok = wait(kv_full, 0) && wait(&q_full[0], 0);
            if (ok) {
                tc_fence_after();
                issue_s(Lay::kColS, dK, q_off(0), s_full);
                if ((ok = wait(&o_full[0], 0))) {
                    tc_fence_after();
                    issue_s(Lay::kColP, dV, o_off(0), dp_full);
                }
            }
            for (int it = 0; ok && it < n_items; ++it) {
                const bool more = it + 1 < n_items;
                if (!(ok = wait(p_full, it & 1))) break;
                tc_fence_after();
                issue_acc(it == 0, Lay::kColDV, Lay::kColS, o_off(it));
                if (leader) tc_commit(&o_empty[it % kTcOStages]);
                if (more) {
                    const int n = it + 1;
                    if (!(ok = wait(&q_full[n % kTcQStages], (n / kTcQStages) & 1))) break;
                    tc_fence_after();
                    issue_s(Lay::kColS, dK, q_off(n), s_full);
                }
                if (!(ok = wait(ds_full, it & 1))) break;
                tc_fence_after();
                issue_acc(it == 0, Lay::kColDK, Lay::kColP, q_off(it));
                if (leader) tc_commit(&q_empty[it % kTcQStages]);
                if (more) {
                    const int n = it + 1;
                    if (!(ok = wait(&o_full[n % kTcOStages], (n / kTcOStages) & 1))) break;
                    tc_fence_after();
                    issue_s(Lay::kColP, dV, o_off(n), dp_full);
                }
            }
            if (leader) tc_commit(acc_done);
            __syncwarp();
            mbar_wait(acc_done, 0, abort_flag, p.status, 1000000000ull);
        }
        __syncwarp();
    }
    } else {
        // ---------------------------------------- elementwise + epilogue ----
        const int u = (warp - 4) >> 2;                  // query quarter of an item
        const int g4 = warp & 3;                        // lane group
        const int r = (g4 << 5) + lane;                 // key row = tensor-memory lane
        const int key = k0 + r;
        const uint32_t lane_addr = tmem + ((static_cast<uint32_t>(g4) * 32u) << 16);
        const uint32_t col = 32 * u;
        bool ok = true;
        for (int it = 0; it < n_items; ++it) {
            const int q0 = (qb0 + it % n_qb) * kTcBQ;
            const int qs = it % kTcQStages, db = it & 1;
            // q_full also publishes the item's lse the producer stored
            if (!(ok = __all_sync(0xffffffffu,
                                  mbar_wait(&q_full[qs], (it / kTcQStages) & 1, abort_flag,
                                            p.status) &&
                                  mbar_wait(s_full, it & 1, abort_flag, p.status))))
                break;
            tc_fence_after();
            uint32_t sv[32];
            tmem_ld32(lane_addr + Lay::kColS + col, sv);
            const bool full = block_visible(p.vis, q0, kTcBQ, k0, kTcBK);
            // the quarter's lse / D: the same 32 values for every lane (broadcast)
            const float4 *L4 = reinterpret_cast<const float4 *>(sL + qs * kTcBQ + col);
            const float4 *D4 = reinterpret_cast<const float4 *>(sD + db * kTcBQ + col);
            tmem_wait_ld();
            // P^T, over columns this thread has already read (its own quarter);
            // one pair in four takes 2^x on the FMA pipe (the MUFU unit is the
            // busiest one here).  P^T is kept as the bf16 pairs the products use.
            uint32_t pk[16];
            const float2 cc = make_float2(p.scale_log2, p.scale_log2);
            auto p_quad = [&](int e4, float (&pr)[4]) {
                const float4 l4 = L4[e4];
                const float2 x0 = fma2(make_float2(__uint_as_float(sv[4 * e4]),
                                                   __uint_as_float(sv[4 * e4 + 1])),
                                       cc, make_float2(-l4.x, -l4.y));
                const float2 x1 = fma2(make_float2(__uint_as_float(sv[4 * e4 + 2]),
                                                   __uint_as_float(sv[4 * e4 + 3])),
                                       cc, make_float2(-l4.z, -l4.w));
                const float2 e1 = (e4 & 1) ? exp2_poly2(x1)
                                           : make_float2(fast_exp2(x1.x), fast_exp2(x1.y));
                pr[0] = fast_exp2(x0.x);
                pr[1] = fast_exp2(x0.y);
                pr[2] = e1.x;
                pr[3] = e1.y;
            };
            if (full) {
#pragma unroll
                for (int e4 = 0; e4 < 8; ++e4) {
                    float pr[4];
                    p_quad(e4, pr);
                    pk[2 * e4] = pack_bf16x2(pr[0], pr[1]);
                    pk[2 * e4 + 1] = pack_bf16x2(pr[2], pr[3]);
                }
            } else {
#pragma unroll
                for (int e4 = 0; e4 < 8; ++e4) {
                    float pr[4];
                    p_quad(e4, pr);
#pragma unroll
                    for (int t = 0; t < 4; ++t)
                        if (!p.vis(q0 + col + 4 * e4 + t, key)) pr[t] = 0.0f;
                    pk[2 * e4] = pack_bf16x2(pr[0], pr[1]);
                    pk[2 * e4 + 1] = pack_bf16x2(pr[2], pr[3]);
                }
            }
            tmem_st16(lane_addr + Lay::kColS + col, pk);
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(p_full);
            // dS^T = P^T (dP^T - D), over the same columns of the dP^T region
            if (!(ok = __all_sync(0xffffffffu,
                                  mbar_wait(dp_full, it & 1, abort_flag, p.status) &&
                                  mbar_wait(&d_full[db], (it >> 1) & 1, abort_flag, p.status))))
                break;
            tc_fence_after();
            uint32_t dp[32];
            tmem_ld32(lane_addr + Lay::kColP + col, dp);
            tmem_wait_ld();
            // dS^T from the bf16 P^T the dV product used (masked entries are 0)
            uint32_t dk[16];
#pragma unroll
            for (int e4 = 0; e4 < 8; ++e4) {
                const float4 d4 = D4[e4];
                const float2 ds0 = mul2(bf16x2_to_float2(pk[2 * e4]),
                                        add2(make_float2(__uint_as_float(dp[4 * e4]),
                                                         __uint_as_float(dp[4 * e4 + 1])),
                                             make_float2(-d4.x, -d4.y)));
                const float2 ds1 = mul2(bf16x2_to_float2(pk[2 * e4 + 1]),
                                        add2(make_float2(__uint_as_float(dp[4 * e4 + 2]),
                                                         __uint_as_float(dp[4 * e4 + 3])),
                                             make_float2(-d4.z, -d4.w)));
                dk[2 * e4] = pack_bf16x2(ds0.x, ds0.y);
                dk[2 * e4 + 1] = pack_bf16x2(ds1.x, ds1.y);
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&d_empty[db]);   // this warp is done with D
            tmem_st16(lane_addr + Lay::kColP + col, dk);
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(ds_full);
        }
        // ---- epilogue: dV, dK * scale -> bf16 (quarter u writes columns 32 u ..) ----
        if (ok && n_items > 0)
            ok = __all_sync(0xffffffffu, mbar_wait(acc_done, 0, abort_flag, p.status));
        tc_fence_after();
        // the tensor-memory loads are warp-collective: every lane loads, and
        // only rows of real keys are stored
        const bool have = ok && n_items > 0;            // warp-uniform
        const size_t rowoff = ((static_cast<size_t>(b) * p.Tkv + min(key, p.Tkv - 1)) * p.Hkv +
                               kvh) * D;
#pragma unroll
        for (int m = 0; m < 2; ++m) {                   // dV, then dK
            __nv_bfloat16 *dst = (m ? p.dk : p.dv) + rowoff + 32 * u;
            const float f = m ? p.scale : 1.0f;
            if (32 * u < D) {                           // warp-uniform
                uint32_t v[32];
                if (have) {
                    tmem_ld32(lane_addr + (m ? Lay::kColDK : Lay::kColDV) + 32 * u, v);
                    tmem_wait_ld();
                } else {
#pragma unroll
                    for (int e = 0; e < 32; ++e) v[e] = 0u;
                }
                if (key < p.Tkv) {
                    uint4 *d4 = reinterpret_cast<uint4 *>(dst);
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const uint32_t *w = &v[8 * e];
                        d4[e] = make_uint4(
                            pack_bf16x2(__uint_as_float(w[0]) * f, __uint_as_float(w[1]) * f),
                            pack_bf16x2(__uint_as_float(w[2]) * f, __uint_as_float(w[3]) * f),
                            pack_bf16x2(__uint_as_float(w[4]) * f, __uint_as_float(w[5]) * f),
                            pack_bf16x2(__uint_as_float(w[6]) * f, __uint_as_float(w[7]) * f));
                    }
                }
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

template <int D>
static int launch_dkdv_tc(const void *q, const void *k, const void *v, const void *dout,
                          const float *lse, const float *Dsum, void *dk, void *dv, int B, int Tq,
                          int Tkv, int Hq, int Hkv, Vis vis, float scale, cudaStream_t stream) {
    TcParams prm;
    prm.B = B;
    prm.Tq = Tq;
    prm.Tkv = Tkv;
    prm.Hq = Hq;
    prm.Hkv = Hkv;
    prm.G = Hq / Hkv;
    prm.n_kt = (Tkv + kTcBK - 1) / kTcBK;
    prm.vis = vis;
    prm.scale = scale;
    prm.scale_log2 = scale * 1.4426950408889634f;
    prm.lse = lse;
    prm.Dsum = Dsum;
    prm.dk = static_cast<__nv_bfloat16 *>(dk);
    prm.dv = static_cast<__nv_bfloat16 *>(dv);
    prm.status = device_status_ptr();
    if (!prm.status) return GQA_ERR_CUDA;
    const long long blocks = static_cast<long long>(prm.n_kt) * Hkv * B;
    if (blocks > 0x7fffffffLL) return set_error(GQA_ERR_UNSUPPORTED, "backward grid too large");
    CUtensorMap tq, tk, tv, to;
    if (int rc = encode_tmap_bf16_4d(&tq, q, D, Hq, Tq, B, 64, 1, kTcBQ, 1, 1)) return rc;
    if (int rc = encode_tmap_bf16_4d(&to, dout, D, Hq, Tq, B, 64, 1, kTcBQ, 1, 1)) return rc;
    if (int rc = encode_tmap_bf16_4d(&tk, k, D, Hkv, Tkv, B, 64, 1, kTcBK, 1, 1)) return rc;
    if (int rc = encode_tmap_bf16_4d(&tv, v, D, Hkv, Tkv, B, 64, 1, kTcBK, 1, 1)) return rc;
    auto kern = dkdv_tc_kernel<D>;
    const int smem = TcLayout<D>::kSmemBytes;
    static CtxSlot setup;   // the shared-memory opt-in, once per context
    if (int rc = once_per_context(setup, [&](int) {
            return check_cuda(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                   smem), "cudaFuncSetAttribute(dkdv_tc)");
        }))
        return rc;
    kern<<<static_cast<unsigned>(blocks), kTcThreads, smem, stream>>>(tq, tk, tv, to, prm);
    return check_cuda(cudaGetLastError(), "dkdv_tc_kernel launch");
}

// --------------------------------------------------------- dq (tcgen05) ---
// M tiles of 128 rows: the G query heads of one KV group at P = floor(128 / G)
// positions, as in the forward (one 3-D TMA box; every K / V tile serves the
// whole group).  For every visible 128-key tile of an M tile:
//   tensor pipe   S = Q K^T and dP = dO V^T into tensor memory;
//   16 warps      load S and dP (four threads per row, one per 32-key
//                 quarter), release them, and form dS = P (dP - D_row) with
//                 P = exp2(S * scale * log2e - lse_row * log2e), bf16, into a
//                 dS region of tensor memory;
//   tensor pipe   dQ += dS K with dS read from tensor memory.
// Once the warps hold S(j) and dP(j) in registers the next tile's S and dP are
// computed, overlapping the elementwise work; the warps write dS(j) after
// dQ(j-1) has read dS(j-1).  Tensor memory: S | dP | dQ | dS.  Shared memory:
// Q, dO, a 3-deep K ring (K(j) serves S(j) and, a tile later, dQ(j), so the
// copy of K(j+2) must not wait for dQ(j)) and a 2-deep V ring (V(j) is free
// once dP(j) has run).
//
// Persistent: one CTA per SM takes M tiles, heaviest first, from a counter in
// the workspace (zeroed by rowdot, which runs before on the same stream), so
// CTAs that start late -- the dK/dV kernel runs beside this one -- still share
// the work evenly.  Every barrier counts across M tiles: the next tile's Q / dO
// copy and its first S and dP run while the warps finish the current tile's
// last dS and read its dQ out of tensor memory.  Warp 0 fetches tile indices
// into a 2-slot ring in shared memory that the other roles read.
constexpr int kDqBN = 128;       // keys per tile
constexpr int kDqKStages = 3;
constexpr int kDqVStages = 2;
constexpr int kDqConsumers = 3 + kTcElemWarps;   // warps 1, 2, 3 and the elementwise warps

template <int D>
struct DqLayout {
    static constexpr int kPanels = D / 64;
    static constexpr int kPanel = 128 * 128;               // 128 rows x 64 bf16
    static constexpr int kTile = kPanels * kPanel;
    static constexpr int kOffQ = 0, kOffO = kTile;
    static constexpr int kOffK = 2 * kTile;                // [kDqKStages]
    static constexpr int kOffV = kOffK + kDqKStages * kTile;   // [kDqVStages]
    static constexpr int kBytes = kOffV + kDqVStages * kTile;
    static constexpr int kSmemBytes = kBytes + 1024;
    // S | dP | dQ | dS (bf16, keys 32 u .. 32 u + 31 at 384 + 16 u)
    static constexpr uint32_t kColS = 0, kColP = 128, kColDQ = 256, kColDS = 384;
};

struct DqParams {
    int B, Tq, Tkv, Hq, Hkv, G, P;    // P = positions per M tile
    int n_mt;                         // M tiles per (b, kvh)
    int n_tiles;                      // n_mt * Hkv * B
    Vis vis;
    float scale, scale_log2;
    const float *lse, *Dsum;
    __nv_bfloat16 *dq;
    unsigned int *tile_counter;       // zero on entry
    int *status;
};

// M tile number t (0 = heaviest) of a call: its rows and visible key tiles.
struct DqTile {
    int b, kvh, t0, n_kv, n_sink, first;
    __device__ __forceinline__ DqTile(const DqParams &p, int t) {
        const int bhs = p.Hkv * p.B;
        // M tiles in decreasing causal work (the last positions see the most keys)
        const int mt = p.n_mt - 1 - t / bhs;
        kvh = t % p.Hkv;
        b = (t / p.Hkv) % p.B;
        t0 = mt * p.P;
        const int last_pos = min(t0 + p.P, p.Tq) - 1;
        const int off = p.Tkv - p.Tq;
        int kv_end = p.Tkv;
        if (p.vis.causal) kv_end = min(p.Tkv, last_pos + off + 1);
        n_sink = 0;
        first = 0;
        if (p.vis.window > 0 && kv_end > 0) {
            n_sink = (min(p.vis.sinks, kv_end) + kDqBN - 1) / kDqBN;
            first = max(n_sink, max(t0 + off - p.vis.window + 1, 0) / kDqBN);
        }
        const int last = kv_end > 0 ? (kv_end + kDqBN - 1) / kDqBN : 0;
        n_kv = n_sink + max(0, last - first);
    }
    __device__ __forceinline__ int tile_of(int j) const { return j < n_sink ? j : first + (j - n_sink); }
};

template <int D>
__global__ void __launch_bounds__(kTcThreads, 1)
dq_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_o,
             const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
             const DqParams p) {
    using Lay = DqLayout<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    __shared__ uint64_t qo_full, qo_empty, k_full[kDqKStages], k_empty[kDqKStages],
        v_full[kDqVStages], v_empty[kDqVStages], s_full, s_free, p_full, dq_done, acc_done,
        dq_free, drain[2], t_full[2], t_empty[2];
    __shared__ int t_slot[2];
    __shared__ uint32_t tmem_base_sh;
    __shared__ int abort_flag;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        mbar_init(&qo_full, 1);
        mbar_init(&qo_empty, 1);
        for (int s = 0; s < kDqKStages; ++s) {
            mbar_init(&k_full[s], 1);
            mbar_init(&k_empty[s], 1);
        }
        for (int s = 0; s < kDqVStages; ++s) {
            mbar_init(&v_full[s], 1);
            mbar_init(&v_empty[s], 1);
        }
        mbar_init(&s_full, 1);
        mbar_init(&s_free, kTcElemWarps);
        mbar_init(&p_full, kTcElemWarps);
        mbar_init(&dq_done, 1);
        mbar_init(&acc_done, 1);
        mbar_init(&dq_free, kTcElemWarps);
        mbar_init(&drain[0], 1);
        mbar_init(&drain[1], 1);
        for (int s = 0; s < 2; ++s) {
            mbar_init(&t_full[s], 1);
            mbar_init(&t_empty[s], kDqConsumers);
        }
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
    auto wait = [&](uint64_t *bar, uint32_t parity) {
        return mbar_wait(bar, parity, &abort_flag, p.status);
    };
    // Tile number of iteration `it` (>= p.n_tiles: no more tiles), read by an
    // elementwise warp; lane 0 releases the slot.  -1 after an abort.
    auto take_tile = [&](int it) {
        const int slot = it & 1;
        if (!__all_sync(0xffffffffu, wait(&t_full[slot], (it >> 1) & 1))) return -1;
        const int t = *reinterpret_cast<volatile int *>(&t_slot[slot]);
        __syncwarp();
        if (lane == 0) mbar_arrive(&t_empty[slot]);
        return t;
    };

    if (warp == 0 && lane == 0) {
        // -------------------------- scheduler, Q / dO and K ring producer ----
        // Both producers run as one thread (measured a little faster here than
        // warp-wide with a re-convergence after each copy).
        tma_prefetch_desc(&tm_q);
        tma_prefetch_desc(&tm_o);
        tma_prefetch_desc(&tm_k);
        uint32_t kc = 0, qi = 0;   // K copies and Q / dO copies issued
        bool ok = true;
        for (int it = 0; ok; ++it) {
            const int slot = it & 1;
            if (it >= 2 && !(ok = wait(&t_empty[slot], ((it >> 1) & 1) ^ 1))) break;
            int t = static_cast<int>(atomicAdd(p.tile_counter, 1u));
            if (t > p.n_tiles) t = p.n_tiles;
            t_slot[slot] = t;
            mbar_arrive(&t_full[slot]);         // release: the index store comes first
            if (t >= p.n_tiles) break;
            const DqTile T(p, t);
            if (T.n_kv == 0) continue;
            // Q and dO of the previous tile are free once its last S / dP ran
            if (qi > 0 && !(ok = wait(&qo_empty, (qi - 1) & 1))) break;
            const uint32_t box = 64u * p.G * p.P * 2u;
            mbar_expect_tx(&qo_full, 2 * Lay::kPanels * box);
            for (int pn = 0; pn < Lay::kPanels; ++pn) {
                tma_load_4d(smem + Lay::kOffQ + pn * Lay::kPanel, &tm_q, &qo_full, pn * 64,
                            T.kvh * p.G, T.t0, T.b);
                tma_load_4d(smem + Lay::kOffO + pn * Lay::kPanel, &tm_o, &qo_full, pn * 64,
                            T.kvh * p.G, T.t0, T.b);
            }
            ++qi;
            for (int j = 0; j < T.n_kv; ++j, ++kc) {
                const uint32_t st = kc % kDqKStages, ph = (kc / kDqKStages) & 1;
                if (!(ok = wait(&k_empty[st], ph ^ 1))) break;
                mbar_expect_tx(&k_full[st], Lay::kTile);
                for (int pn = 0; pn < Lay::kPanels; ++pn)
                    tma_load_4d(smem + Lay::kOffK + st * Lay::kTile + pn * Lay::kPanel, &tm_k,
                                &k_full[st], pn * 64, T.kvh, T.tile_of(j) * kDqBN, T.b);
            }
        }
        // copies still in flight land before the block exits
        if (qi > 0) mbar_wait(&qo_full, (qi - 1) & 1, &abort_flag, p.status, 1000000ull);
        for (uint32_t c = kc > kDqKStages ? kc - kDqKStages : 0; c < kc; ++c)
            mbar_wait(&k_full[c % kDqKStages], (c / kDqKStages) & 1, &abort_flag, p.status,
                      1000000ull);
    } else if (warp == 2 && lane == 0) {
        // ------------------------------------------------ V ring producer ----
        tma_prefetch_desc(&tm_v);
        uint32_t vc = 0;
        bool ok = true;
        for (int it = 0; ok; ++it) {
            const int slot = it & 1;
            if (!(ok = wait(&t_full[slot], (it >> 1) & 1))) break;
            const int t = *reinterpret_cast<volatile int *>(&t_slot[slot]);
            mbar_arrive(&t_empty[slot]);
            if (t >= p.n_tiles) break;
            const DqTile T(p, t);
            for (int j = 0; j < T.n_kv; ++j, ++vc) {
                const uint32_t st = vc % kDqVStages, ph = (vc / kDqVStages) & 1;
                if (!(ok = wait(&v_empty[st], ph ^ 1))) break;
                mbar_expect_tx(&v_full[st], Lay::kTile);
                for (int pn = 0; pn < Lay::kPanels; ++pn)
                    tma_load_4d(smem + Lay::kOffV + st * Lay::kTile + pn * Lay::kPanel, &tm_v,
                                &v_full[st], pn * 64, T.kvh, T.tile_of(j) * kDqBN, T.b);
            }
        }
        for (uint32_t c = vc > kDqVStages ? vc - kDqVStages : 0; c < vc; ++c)
            mbar_wait(&v_full[c % kDqVStages], (c / kDqVStages) & 1, &abort_flag, p.status,
                      1000000ull);
    } else if (warp == 1 || warp == 3) {
        // ------------------------------------------------ MMA issuers ----
        // Warp 1 issues S and dP, warp 3 issues dQ.  The two streams touch
        // disjoint tensor-memory regions (S | dP against dQ, reading dS) and
        // release shared-memory stages through their own barriers, so they need
        // no order between them; with one issuer a dQ(j) whose dS was ready sat
        // behind the whole S / dP(j+1) group (tcgen05.mma blocks the issuing
        // thread once its queue is full), and S / dP(j+2) behind dQ(j).
        // Each warp waits on every barrier as a whole (a vote) and one elected
        // lane issues; the warp is not re-converged after a group, since the
        // next wait's vote does that.  Measured on a B200 against a lone thread
        // per issuer: 0.4280 against 0.4465 ms for the backward.
        const bool leader = elect_one();
        auto wwait = [&](uint64_t *bar, uint32_t parity) {
            return __all_sync(0xffffffffu, wait(bar, parity));
        };
        constexpr uint32_t idesc_s = umma_idesc_bf16(128, kDqBN, 0, 0);
        constexpr uint32_t idesc_o = umma_idesc_bf16(128, D, 0, 1);
        const uint32_t base = smem_u32(smem);
        const uint64_t dQt = umma_smem_desc(base + Lay::kOffQ, 16, 1024);
        const uint64_t dOt = umma_smem_desc(base + Lay::kOffO, 16, 1024);
        uint32_t g = 0, qi = 0;   // key tiles and M tiles with keys, over the whole block
        bool ok = true;
        for (int it = 0; ok; ++it) {
            const int slot = it & 1;
            if (!(ok = wwait(&t_full[slot], (it >> 1) & 1))) break;
            const int t = *reinterpret_cast<volatile int *>(&t_slot[slot]);
            __syncwarp();
            if (leader) mbar_arrive(&t_empty[slot]);
            if (t >= p.n_tiles) break;
            const DqTile T(p, t);
            if (T.n_kv == 0) continue;
            if (warp == 1) {
                // S = Q K_j^T, dP = dO V_j^T: K-major A and B (+32 B per 16 of d);
                // V_j's stage is released as soon as dP has run
                if (!(ok = wwait(&qo_full, qi & 1))) break;
                for (int j = 0; j < T.n_kv; ++j, ++g) {
                    // the warps hold S, dP of the previous key tile in registers
                    if (g > 0 && !(ok = wwait(&s_free, (g - 1) & 1))) break;
                    const uint32_t ks = g % kDqKStages, vs = g % kDqVStages;
                    if (!(ok = wwait(&k_full[ks], (g / kDqKStages) & 1))) break;
                    tc_fence_after();
                    const uint64_t bk = umma_smem_desc(base + Lay::kOffK + ks * Lay::kTile, 16, 1024);
                    if (leader) {
#pragma unroll
                        for (int kk = 0; kk < D / 16; ++kk) {
                            const uint32_t o16 = ((kk >> 2) * Lay::kPanel + (kk & 3) * 32) >> 4;
                            umma_ss(tmem + Lay::kColS, dQt + o16, bk + o16, idesc_s, kk > 0);
                        }
                    }
                    if (!(ok = wwait(&v_full[vs], (g / kDqVStages) & 1))) break;
                    tc_fence_after();
                    const uint64_t bv = umma_smem_desc(base + Lay::kOffV + vs * Lay::kTile, 16, 1024);
                    if (leader) {
#pragma unroll
                        for (int kk = 0; kk < D / 16; ++kk) {
                            const uint32_t o16 = ((kk >> 2) * Lay::kPanel + (kk & 3) * 32) >> 4;
                            umma_ss(tmem + Lay::kColP, dOt + o16, bv + o16, idesc_s, kk > 0);
                        }
                        tc_commit(&s_full);
                        tc_commit(&v_empty[vs]);
                    }
                }
                if (!ok) break;
                // this tile's Q and dO are free once its last products have run
                if (leader) tc_commit(&qo_empty);
            } else {
                // the previous tile's dQ has been read out of tensor memory
                if (qi > 0 && !(ok = wwait(&dq_free, (qi - 1) & 1))) break;
                for (int j = 0; j < T.n_kv; ++j, ++g) {
                    const uint32_t ks = g % kDqKStages;
                    // dS is in tensor memory; K has landed (S read it)
                    if (!(ok = wwait(&p_full, g & 1) && wwait(&k_full[ks], (g / kDqKStages) & 1))) break;
                    tc_fence_after();
                    // dQ += dS K: dS from tensor memory (keys 32 u .. at 384 + 16 u,
                    // 8 columns per 16 keys), K MN-major (+2048 B per 16 keys)
                    const uint64_t km =
                        umma_smem_desc(base + Lay::kOffK + ks * Lay::kTile, Lay::kPanel, 1024);
                    if (leader) {
#pragma unroll
                        for (int kk = 0; kk < kDqBN / 16; ++kk)
                            umma_ts(tmem + Lay::kColDQ, tmem + Lay::kColDS + kk * 8,
                                    km + kk * (2048 >> 4), idesc_o, (j > 0 || kk > 0) ? 1u : 0u);
                        tc_commit(&dq_done);
                        tc_commit(&k_empty[ks]);
                    }
                }
                if (!ok) break;
                if (leader) tc_commit(&acc_done);
            }
            ++qi;
        }
        // the last products have finished before the block exits
        uint64_t *dr = &drain[warp == 1 ? 0 : 1];
        if (leader) tc_commit(dr);
        __syncwarp();
        mbar_wait(dr, 0, &abort_flag, p.status, 1000000000ull);
    } else if (warp >= 4) {
        // ---------------------------------------- elementwise + epilogue ----
        const int u = (warp - 4) >> 2;                  // key quarter of a tile
        const int g4 = warp & 3;                        // lane group
        const int r = (g4 << 5) + lane;                 // row = tensor-memory lane
        const uint32_t lane_addr = tmem + ((static_cast<uint32_t>(g4) * 32u) << 16);
        const uint32_t col = 32 * u;
        const float2 cc = make_float2(p.scale_log2, p.scale_log2);
        // row r of M tile t: position, head, and whether it is a real row
        auto row_pos = [&](int t) { return DqTile(p, t).t0 + r / p.G; };
        auto row_real = [&](int t) { return r < p.P * p.G && row_pos(t) < p.Tq; };
        auto row_index = [&](int t) {   // (b, head, pos) -> index of the row's lse / D
            const DqTile T(p, t);
            return (static_cast<size_t>(T.b) * p.Hq + T.kvh * p.G + r % p.G) * p.Tq + row_pos(t);
        };
        uint32_t g = 0, qi = 0;
        bool ok = true;
        int t = take_tile(0);
        // lse and D of the row, loaded a tile ahead so that their latency overlaps
        // the previous tile's epilogue
        float Lr = 0.0f, Dr = 0.0f;
        if (t >= 0 && t < p.n_tiles && row_real(t)) {
            const size_t li = row_index(t);
            Lr = p.lse[li] * 1.4426950408889634f;
            Dr = p.Dsum[li];
        }
        for (int it = 0; ok && t >= 0 && t < p.n_tiles; ++it) {
            bool have = false;                          // warp-uniform
            {
                const DqTile T(p, t);
                const int pos = T.t0 + r / p.G;
                const bool real = r < p.P * p.G && pos < p.Tq;
                const float2 nl = make_float2(-Lr, -Lr), nd = make_float2(-Dr, -Dr);
                have = T.n_kv > 0;
                for (int j = 0; j < T.n_kv; ++j, ++g) {
                    if (!(ok = __all_sync(0xffffffffu, wait(&s_full, g & 1)))) break;
                    tc_fence_after();
                    uint32_t sv[32], dp[32];
                    tmem_ld32(lane_addr + Lay::kColS + col, sv);
                    tmem_ld32(lane_addr + Lay::kColP + col, dp);
                    tmem_wait_ld();
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&s_free);        // S and dP may be overwritten
                    const int key0 = T.tile_of(j) * kDqBN + col;
                    const bool full = block_visible(p.vis, T.t0, p.P, T.tile_of(j) * kDqBN, kDqBN) &&
                                      __all_sync(0xffffffffu, real || r >= p.P * p.G);
                    // dS = P (dP - D); one pair in four takes 2^x on the FMA pipe (the
                    // MUFU unit is the busiest one here).  Tiles the mask leaves whole
                    // skip the per-element test.
                    uint32_t pk[16];
                    auto ds_pair = [&](int e) {
                        const float2 x = fma2(make_float2(__uint_as_float(sv[e]), __uint_as_float(sv[e + 1])),
                                              cc, nl);
                        const float2 pr = ((e >> 1) & 3) == 3 ? exp2_poly2(x)
                                                              : make_float2(fast_exp2(x.x), fast_exp2(x.y));
                        return mul2(pr, add2(make_float2(__uint_as_float(dp[e]), __uint_as_float(dp[e + 1])),
                                             nd));
                    };
                    if (full) {
#pragma unroll
                        for (int e = 0; e < 32; e += 2) {
                            const float2 ds = ds_pair(e);
                            pk[e / 2] = pack_bf16x2(ds.x, ds.y);
                        }
                        // rows past the tile's real ones hold stale operands: exact zeros
                        if (!real) {
#pragma unroll
                            for (int e = 0; e < 16; ++e) pk[e] = 0u;
                        }
                    } else {
#pragma unroll
                        for (int e = 0; e < 32; e += 2) {
                            float2 ds = ds_pair(e);
                            if (!(real && p.vis(pos, key0 + e))) ds.x = 0.0f;
                            if (!(real && p.vis(pos, key0 + e + 1))) ds.y = 0.0f;
                            pk[e / 2] = pack_bf16x2(ds.x, ds.y);
                        }
                    }
                    // the previous dQ product has read the dS region
                    if (g > 0 && !(ok = __all_sync(0xffffffffu, wait(&dq_done, (g - 1) & 1)))) break;
                    tc_fence_after();
                    tmem_st16(lane_addr + Lay::kColDS + 16 * u, pk);   // keys 32 u .. 32 u + 31
                    tmem_wait_st();
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&p_full);
                }
            }
            if (!ok) break;
            // the next tile's index and row statistics, loaded before this tile's
            // epilogue so that their latency overlaps it
            const int t_next = take_tile(it + 1);
            if (t_next >= 0 && t_next < p.n_tiles && row_real(t_next)) {
                const size_t li = row_index(t_next);
                Lr = p.lse[li] * 1.4426950408889634f;
                Dr = p.Dsum[li];
            }
            // ---- epilogue: dQ * scale -> bf16 (quarter u writes columns 32 u ..) ----
            // read 16 columns at a time and pack them at once, to keep few
            // registers live across the tile loop
            uint32_t pk[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) pk[e] = 0u;
            if (have) {
                if (!(ok = __all_sync(0xffffffffu, wait(&acc_done, qi & 1)))) break;
                tc_fence_after();
                if (col < D) {                          // warp-uniform
                    const float f = p.scale;
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        uint32_t v[16];
                        tmem_ld16(lane_addr + Lay::kColDQ + col + 16 * h, v);
                        tmem_wait_ld();
#pragma unroll
                        for (int e = 0; e < 8; ++e)
                            pk[8 * h + e] = pack_bf16x2(__uint_as_float(v[2 * e]) * f,
                                                        __uint_as_float(v[2 * e + 1]) * f);
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&dq_free);   // the next tile's dQ may start
                ++qi;
            }
            if (col < D && row_real(t)) {
                const DqTile T(p, t);
                uint4 *d4 = reinterpret_cast<uint4 *>(
                    p.dq + ((static_cast<size_t>(T.b) * p.Tq + row_pos(t)) * p.Hq + T.kvh * p.G +
                            r % p.G) * D + col);
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    d4[e] = make_uint4(pk[4 * e], pk[4 * e + 1], pk[4 * e + 2], pk[4 * e + 3]);
            }
            t = t_next;
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

template <int D>
static int launch_dq_tc(const void *q, const void *k, const void *v, const void *dout,
                        const float *lse, const float *Dsum, unsigned int *tile_counter, void *dq,
                        int B, int Tq, int Tkv, int Hq, int Hkv, Vis vis, float scale,
                        cudaStream_t stream) {
    DqParams prm;
    prm.B = B;
    prm.Tq = Tq;
    prm.Tkv = Tkv;
    prm.Hq = Hq;
    prm.Hkv = Hkv;
    prm.G = Hq / Hkv;
    prm.P = 128 / prm.G;
    prm.n_mt = (Tq + prm.P - 1) / prm.P;
    prm.vis = vis;
    prm.scale = scale;
    prm.scale_log2 = scale * 1.4426950408889634f;
    prm.lse = lse;
    prm.Dsum = Dsum;
    prm.dq = static_cast<__nv_bfloat16 *>(dq);
    prm.tile_counter = tile_counter;
    prm.status = device_status_ptr();
    if (!prm.status) return GQA_ERR_CUDA;
    const long long tiles = static_cast<long long>(prm.n_mt) * Hkv * B;
    if (tiles > 0x7fffffffLL) return set_error(GQA_ERR_UNSUPPORTED, "backward grid too large");
    prm.n_tiles = static_cast<int>(tiles);
    if (tiles == 0) return GQA_OK;
    int n_sm = 0;
    if (int rc = sm_count(&n_sm)) return rc;
    const int blocks = static_cast<int>(tiles < n_sm ? tiles : n_sm);
    CUtensorMap tq, to, tk, tv;
    if (int rc = encode_tmap_bf16_4d(&tq, q, D, Hq, Tq, B, 64, prm.G, prm.P, 1, 1)) return rc;
    if (int rc = encode_tmap_bf16_4d(&to, dout, D, Hq, Tq, B, 64, prm.G, prm.P, 1, 1)) return rc;
    if (int rc = encode_tmap_bf16_4d(&tk, k, D, Hkv, Tkv, B, 64, 1, kDqBN, 1, 1)) return rc;
    if (int rc = encode_tmap_bf16_4d(&tv, v, D, Hkv, Tkv, B, 64, 1, kDqBN, 1, 1)) return rc;
    auto kern = dq_tc_kernel<D>;
    const int smem = DqLayout<D>::kSmemBytes;
    static CtxSlot setup;   // the shared-memory opt-in, once per context
    if (int rc = once_per_context(setup, [&](int) {
            return check_cuda(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                   smem), "cudaFuncSetAttribute(dq_tc)");
        }))
        return rc;
    kern<<<static_cast<unsigned>(blocks), kTcThreads, smem, stream>>>(tq, to, tk, tv, prm);
    return check_cuda(cudaGetLastError(), "dq_tc_kernel launch");
}

// D (one float per query row, rounded up to 256 bytes), then the dQ kernel's
// tile counter (256 bytes).
static size_t bwd_dsum_bytes(int B, int Tq, int Hq) {
    return ((static_cast<size_t>(B) * Tq * Hq * sizeof(float)) + 255) & ~static_cast<size_t>(255);
}

size_t bwd_workspace_bytes(int B, int Tq, int Hq) { return bwd_dsum_bytes(B, Tq, Hq) + 256; }

namespace {

// The second stream and the fork / join events, created once per CUDA context
// (again when another context is current, e.g. after a cudaDeviceReset).  The
// record / wait sequence runs under the lock, so concurrent host threads cannot
// interleave their records of the shared events.
struct SideRes {
    cudaStream_t s = nullptr;
    cudaEvent_t fork = nullptr, join = nullptr;
    unsigned long long ctx_id = 0;
    bool ready = false;
};

std::mutex g_side_mu;
SideRes g_side[kMaxDevices];

int side_res(SideRes **out) {
    int dev = 0;
    unsigned long long ctx_id = 0;
    if (int rc = current_ctx_key(&dev, &ctx_id)) return rc;
    SideRes &r = g_side[dev];
    if (!r.ready || (ctx_id != 0 && r.ctx_id != ctx_id)) {
        r.ready = false;
        int least = 0, greatest = 0;
        if (int rc = check_cuda(cudaDeviceGetStreamPriorityRange(&least, &greatest),
                                "cudaDeviceGetStreamPriorityRange"))
            return rc;
        if (int rc = check_cuda(cudaStreamCreateWithPriority(&r.s, cudaStreamNonBlocking, greatest),
                                "cudaStreamCreateWithPriority"))
            return rc;
        if (int rc = check_cuda(cudaEventCreateWithFlags(&r.fork, cudaEventDisableTiming),
                                "cudaEventCreateWithFlags"))
            return rc;
        if (int rc = check_cuda(cudaEventCreateWithFlags(&r.join, cudaEventDisableTiming),
                                "cudaEventCreateWithFlags"))
            return rc;
        int dev2 = 0;
        unsigned long long id2 = 0;
        r.ctx_id = (current_ctx_key(&dev2, &id2) == GQA_OK && dev2 == dev) ? id2 : 0;
        r.ready = true;
    }
    *out = &r;
    return GQA_OK;
}

}  // namespace

template <int D>
static int launch_bwd_d(const void *q, const void *k, const void *v, const void *o,
                        const void *dout, const float *lse, void *dq, void *dk, void *dv, int B,
                        int Tq, int Tkv, int Hq, int Hkv, int causal, int window, int sinks,
                        float scale, void *workspace, cudaStream_t stream) {
    using bf = __nv_bfloat16;
    float *Dsum = static_cast<float *>(workspace);
    auto *tile_counter = reinterpret_cast<unsigned int *>(static_cast<uint8_t *>(workspace) +
                                                          bwd_dsum_bytes(B, Tq, Hq));
    const long long rows = static_cast<long long>(B) * Tq * Hq;
    const long long threads = (rows + kRowdotRows - 1) / kRowdotRows * (D / 8);
    if ((threads + 255) / 256 > 0x7fffffffLL)
        return set_error(GQA_ERR_UNSUPPORTED, "backward: too many rows");
    if (rows > 0)
        rowdot_kernel<D><<<static_cast<unsigned>((threads + 255) / 256), 256, 0, stream>>>(
            static_cast<const bf *>(dout), static_cast<const bf *>(o), Dsum, tile_counter, B, Tq,
            Hq);
    if (int rc = check_cuda(cudaGetLastError(), "rowdot_kernel launch")) return rc;
    Vis vis{Tq, Tkv, causal, causal ? window : 0, sinks};
    if (Tkv == 0)   // no key: every query gradient is zero
        return check_cuda(cudaMemsetAsync(dq, 0, static_cast<size_t>(B) * Tq * Hq * D * 2, stream),
                          "cudaMemsetAsync(dq)");
    std::lock_guard<std::mutex> lock(g_side_mu);
    SideRes *r = nullptr;
    if (int rc = side_res(&r)) return rc;
    // fork: the side stream waits for rowdot; dkdv is enqueued before dq
    if (int rc = check_cuda(cudaEventRecord(r->fork, stream), "cudaEventRecord(fork)")) return rc;
    if (int rc = check_cuda(cudaStreamWaitEvent(r->s, r->fork, 0), "cudaStreamWaitEvent(fork)"))
        return rc;
    int rc = launch_dkdv_tc<D>(q, k, v, dout, lse, Dsum, dk, dv, B, Tq, Tkv, Hq, Hkv, vis, scale,
                               r->s);
    if (rc == GQA_OK)
        rc = launch_dq_tc<D>(q, k, v, dout, lse, Dsum, tile_counter, dq, B, Tq, Tkv, Hq, Hkv, vis,
                             scale, stream);
    // join, on every path: the caller's stream (and a capture in progress on
    // it) then covers all the side stream's work
    const int rj = check_cuda(cudaEventRecord(r->join, r->s), "cudaEventRecord(join)");
    const int rw = rj ? rj : check_cuda(cudaStreamWaitEvent(stream, r->join, 0),
                                        "cudaStreamWaitEvent(join)");
    return rc ? rc : rw;
}

int launch_bwd(const void *q, const void *k, const void *v, const void *o, const void *dout,
               const float *lse, void *dq, void *dk, void *dv, int B, int Tq, int Tkv, int Hq,
               int Hkv, int d, int causal, int window, int sinks, float scale, void *workspace,
               cudaStream_t stream) {
    if (d == 128)
        return launch_bwd_d<128>(q, k, v, o, dout, lse, dq, dk, dv, B, Tq, Tkv, Hq, Hkv, causal,
                                 window, sinks, scale, workspace, stream);
    return launch_bwd_d<64>(q, k, v, o, dout, lse, dq, dk, dv, B, Tq, Tkv, Hq, Hkv, causal, window,
                            sinks, scale, workspace, stream);
}

}  // namespace gqa
