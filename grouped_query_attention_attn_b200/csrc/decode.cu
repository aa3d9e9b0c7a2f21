// decode.cu -- split-KV grouped-query decode (one query token per sequence)
// with the log-sum-exp merge of the splits in the same kernel.
//
// Work unit: one CTA per (split, KV head, sequence).  A split is `chunk`
// consecutive cache rows; the CTA streams its K and V rows from HBM exactly
// once through a TMA ring in shared memory and uses each row for all
// G = Hq / Hkv query heads of the group, which sit as the M rows of warp-level
// bf16 tensor-core tiles (m16n8k16; G <= 16 per tile, padding rows are zero).
//   - warp 4 (one thread) issues the TMA copies: per stage 64 keys of K and V
//     (four 64-column panels with 128-byte swizzle for d = 128);
//   - warps 0-3 each take 16 keys of every stage: S = Q K^T, the running-max
//     softmax of course "Неделя 7. Внимание", step 1 (mask of keys past the
//     sequence end, max subtracted, exp2 with scale * log2 e folded in), then
//     O += P V; row max / sum reductions are warp shuffles inside each quad;
//   - at the end the four warps' (m, l, O) are merged through shared memory
//     and the split's normalised O and natural-log lse go to the workspace.
// The last split of a (sequence, KV head) to finish -- found with an arrival
// counter in the workspace -- then merges the splits of the group's G heads:
//   O = sum_s e^(lse_s - M) O_s / sum_s e^(lse_s - M),  M = max_s lse_s,
// so the merge of one group overlaps the other groups' streaming and no
// second kernel waits for the whole grid.
#include <cuda_bf16.h>
#include <atomic>
#include <chrono>
#include <cmath>

#include "device.cuh"
#include "internal.h"

namespace gqa {

constexpr int kDecBK = 64;                         // keys per pipeline stage
constexpr int kDecWarps = 4;                       // consumer warps, 16 keys each per stage
constexpr int kDecThreads = (kDecWarps + 1) * 32;  // + one producer warp
#ifndef GQA_DEC_STAGES
#define GQA_DEC_STAGES 2
#endif
#ifndef GQA_DEC_CHUNK
#define GQA_DEC_CHUNK 1024
#endif
constexpr int kDecStages = GQA_DEC_STAGES;         // TMA ring depth
constexpr int kDecChunk = GQA_DEC_CHUNK;           // keys per split (multiple of kDecBK)
// CTAs per SM the register budget must allow (3 x 66.6 KB of shared memory
// also fit): more stages in flight per SM.  Groups of more than 16 heads
// (MB = 2) hold twice the accumulators and keep the full register budget.
template <int MB>
constexpr int dec_min_blocks() { return MB == 1 ? 3 : 1; }

template <int D, int MB = 1>
struct DecLayout {
    static constexpr int kPanels = D / 64;                 // 64 bf16 = one 128-byte row
    static constexpr int kPanelBytes = kDecBK * 128;
    static constexpr int kTileBytes = kPanels * kPanelBytes;
    static constexpr int kStageBytes = 2 * kTileBytes;     // K tile then V tile
    static constexpr int kRingBytes = kDecStages * kStageBytes;
    // the end-of-split merge reuses the ring: per warp 16*MB rows of O, m and l
    static constexpr int kMergeBytes = kDecWarps * 16 * MB * (D + 2) * 4;
    static constexpr int kBytes = kRingBytes > kMergeBytes ? kRingBytes : kMergeBytes;
    static constexpr int kSmemBytes = kBytes + 1024;       // + alignment slack
};

__device__ __forceinline__ uint32_t ld_b32(const __nv_bfloat16 *p) {
    return *reinterpret_cast<const uint32_t *>(p);
}

// Byte offset of 16-byte chunk `cg` (0 .. D/8-1) of tile row `row` in a tile
// made of 64-column panels written by TMA with 128-byte swizzle.
template <int D>
__device__ __forceinline__ uint32_t swz_off(int row, int cg) {
    return (cg >> 3) * DecLayout<D>::kPanelBytes + row * 128 + (((cg & 7) ^ (row & 7)) << 4);
}

// kRope: the query is rotated (rotary position embedding) in registers as it
// is loaded, at position max(seqlens[b] - 1, 0); the cached keys are rotated.
template <int D, int MB, bool kRope>
__global__ void __launch_bounds__(kDecThreads, dec_min_blocks<MB>())
decode_split_kernel(const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v,
                    const __nv_bfloat16 *__restrict__ q, const int32_t *__restrict__ seqlens,
                    float *__restrict__ part_o, float *__restrict__ part_lse,
                    unsigned long long *__restrict__ arrivals, unsigned long long call_id,
                    __nv_bfloat16 *__restrict__ o, int B, int Hq, int Hkv, int Lmax, int chunk,
                    int window, int sinks, float scale_log2, double log_theta, int *status) {
    using Lay = DecLayout<D, MB>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    __shared__ uint64_t full_bar[kDecStages], empty_bar[kDecStages];
    __shared__ int abort_flag, merger;

    const int split = blockIdx.x, kvh = blockIdx.y, b = blockIdx.z;
    int L = seqlens[b];
    if (L > Lmax || L < 0) {
        if (threadIdx.x == 0 && split == 0 && kvh == 0) record_status(status, GQA_ERR_INVALID_ARG);
        L = L < 0 ? 0 : Lmax;
    }
    // Sliding window: key j is visible iff j >= lo or j < sinks (and j < L).
    // The splits cover [lo, L) from lo on, chunk keys each, so none of them
    // holds only invisible keys; split 0 first takes the sink keys below the
    // window, [0, s_end), as whole stages.  Without a window lo = s_end = 0.
    const int lo = window > 0 ? max(0, L - window) : 0;
    const int s_end = window > 0 ? min(sinks, lo) : 0;
    const int n_splits = (L - lo + chunk - 1) / chunk;   // splits that hold visible keys
    const int G = Hq / Hkv;
    if (split >= n_splits) {
        // nothing in this split; with no visible key at all (an empty
        // sequence) split 0 writes the group's output rows as zeros
        if (split == 0 && threadIdx.x < kDecWarps * 32) {
            __nv_bfloat16 *og = o + (static_cast<size_t>(b) * Hq + static_cast<size_t>(kvh) * G) * D;
            for (int idx = threadIdx.x; idx < G * D / 8; idx += kDecWarps * 32)
                reinterpret_cast<uint4 *>(og)[idx] = make_uint4(0u, 0u, 0u, 0u);
        }
        return;
    }
    const int start = lo + split * chunk;
    const int end = min(start + chunk, L);
    const int t_s = split == 0 ? (s_end + kDecBK - 1) / kDecBK : 0;   // sink stages
    const int n_iter = t_s + (end - start + kDecBK - 1) / kDecBK;
    const int off_w = start - t_s * kDecBK;         // window stage t starts at key off_w + 64 t
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kDecStages; ++s) {
            mbar_init(&full_bar[s], 1);
            mbar_init(&empty_bar[s], kDecWarps);
        }
        abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();

    if (warp == kDecWarps) {                        // ---- TMA producer ----
        if (lane == 0) {
            tma_prefetch_desc(&tm_k);
            tma_prefetch_desc(&tm_v);
            for (int t = 0; t < n_iter; ++t) {
                const int st = t % kDecStages;
                const uint32_t ph = (t / kDecStages) & 1;
                if (!mbar_wait(&empty_bar[st], ph ^ 1, &abort_flag, status)) break;
                uint8_t *kt = smem + st * Lay::kStageBytes;
                uint8_t *vt = kt + Lay::kTileBytes;
                mbar_expect_tx(&full_bar[st], Lay::kStageBytes);
                const int j0 = t * kDecBK + (t < t_s ? 0 : off_w);
#pragma unroll
                for (int p = 0; p < Lay::kPanels; ++p) {
                    tma_load_4d(kt + p * Lay::kPanelBytes, &tm_k, &full_bar[st], p * 64, kvh, j0, b);
                    tma_load_4d(vt + p * Lay::kPanelBytes, &tm_v, &full_bar[st], p * 64, kvh, j0, b);
                }
            }
        }
        return;                                     // consumers sync with named barrier 1 only
    }

    // ---- consumers: query fragments of the G heads of this group ----
    const int gq = lane >> 2, tq = lane & 3;        // quad row, lane in quad
    const __nv_bfloat16 *qg = q + (static_cast<size_t>(b) * Hq + static_cast<size_t>(kvh) * G) * D;
    uint32_t qa[MB][D / 16][4];
#pragma unroll
    for (int mb = 0; mb < MB; ++mb) {
        const int r0 = mb * 16 + gq, r1 = r0 + 8;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
            const int c0 = kk * 16 + 2 * tq, c1 = c0 + 8;
            qa[mb][kk][0] = r0 < G ? ld_b32(qg + r0 * D + c0) : 0u;
            qa[mb][kk][1] = r1 < G ? ld_b32(qg + r1 * D + c0) : 0u;
            qa[mb][kk][2] = r0 < G ? ld_b32(qg + r0 * D + c1) : 0u;
            qa[mb][kk][3] = r1 < G ? ld_b32(qg + r1 * D + c1) : 0u;
        }
    }
    if constexpr (kRope) {
        // one cosine / sine per coordinate pair, shared by the G heads
        __shared__ float2 rope_cs[D / 2];
        const int m = max(seqlens[b] - 1, 0);
        for (int i = threadIdx.x; i < D / 2; i += kDecWarps * 32) {
            float cs, sn;
            rope_cos_sin(m, rope_turns(i, D / 2, log_theta), cs, sn);
            rope_cs[i] = make_float2(cs, sn);
        }
        named_barrier_sync(1, kDecWarps * 32);
#pragma unroll
        for (int mb = 0; mb < MB; ++mb)
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
                // words 0 / 1 hold pair kk * 8 + tq of rows r0 / r1, words 2 / 3 pair + 4
                const float2 c0 = rope_cs[kk * 8 + tq], c1 = rope_cs[kk * 8 + tq + 4];
                qa[mb][kk][0] = rope_rotate_pair(qa[mb][kk][0], c0.x, c0.y);
                qa[mb][kk][1] = rope_rotate_pair(qa[mb][kk][1], c0.x, c0.y);
                qa[mb][kk][2] = rope_rotate_pair(qa[mb][kk][2], c1.x, c1.y);
                qa[mb][kk][3] = rope_rotate_pair(qa[mb][kk][3], c1.x, c1.y);
            }
    }
    float oacc[MB][D / 8][4];
    float m_run[MB][2], l_run[MB][2];
#pragma unroll
    for (int mb = 0; mb < MB; ++mb) {
#pragma unroll
        for (int nd = 0; nd < D / 8; ++nd)
#pragma unroll
            for (int e = 0; e < 4; ++e) oacc[mb][nd][e] = 0.0f;
        m_run[mb][0] = m_run[mb][1] = -INFINITY;
        l_run[mb][0] = l_run[mb][1] = 0.0f;
    }

    for (int t = 0; t < n_iter; ++t) {
        const int st = t % kDecStages;
        const uint32_t ph = (t / kDecStages) & 1;
        // warp-uniform outcome: ldmatrix and mma.sync below are warp-collective
        if (!__all_sync(0xffffffffu, mbar_wait(&full_bar[st], ph, &abort_flag, status))) break;
        uint8_t *kt = smem + st * Lay::kStageBytes;
        uint8_t *vt = kt + Lay::kTileBytes;
        // first key of this warp's slice, and how many keys of it are visible:
        // a sink stage's run ends at s_end, a window stage's at the split end
        const bool sink = t < t_s;
        const int key0 = t * kDecBK + (sink ? 0 : off_w) + warp * 16;
        const int n_valid = (sink ? s_end : end) - key0;
        const bool partial = n_valid > 0 && n_valid < 16;
        if (partial) {
            // Rows past the split end may be another split's keys or the
            // caller's padding (anything, NaN included): zero their V rows so
            // P = 0 there multiplies exact zeros.
            for (int idx = lane; idx < (16 - n_valid) * (D / 8); idx += 32) {
                const int r = warp * 16 + n_valid + idx / (D / 8);
                *reinterpret_cast<uint4 *>(vt + swz_off<D>(r, idx % (D / 8))) =
                    make_uint4(0u, 0u, 0u, 0u);
            }
            __syncwarp();
        }
        if (n_valid > 0) {
            float sacc[MB][2][4];
#pragma unroll
            for (int mb = 0; mb < MB; ++mb)
#pragma unroll
                for (int nb = 0; nb < 2; ++nb)
#pragma unroll
                    for (int e = 0; e < 4; ++e) sacc[mb][nb][e] = 0.0f;
            const uint32_t kbase = smem_u32(kt);
            const int krow = warp * 16 + (lane & 7) + ((lane >> 4) << 3);
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
                uint32_t kb[4];
                ldsm_x4(kb, kbase + swz_off<D>(krow, 2 * kk + ((lane >> 3) & 1)));
#pragma unroll
                for (int mb = 0; mb < MB; ++mb) {
                    mma_16816(sacc[mb][0], qa[mb][kk], kb[0], kb[1]);
                    mma_16816(sacc[mb][1], qa[mb][kk], kb[2], kb[3]);
                }
            }
            uint32_t pa[MB][4];
#pragma unroll
            for (int mb = 0; mb < MB; ++mb) {
                float s[2][4], mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
                for (int nb = 0; nb < 2; ++nb)
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int kl = nb * 8 + 2 * tq + (e & 1);
                        const bool vis = kl < n_valid;
                        s[nb][e] = vis ? sacc[mb][nb][e] * scale_log2 : -INFINITY;
                        mx[e >> 1] = fmaxf(mx[e >> 1], s[nb][e]);
                    }
                float alpha[2], m_use[2];
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    mx[h] = fmaxf(mx[h], __shfl_xor_sync(0xffffffffu, mx[h], 1));
                    mx[h] = fmaxf(mx[h], __shfl_xor_sync(0xffffffffu, mx[h], 2));
                    const float m_new = fmaxf(m_run[mb][h], mx[h]);
                    m_use[h] = (m_new == -INFINITY) ? 0.0f : m_new;
                    alpha[h] = fast_exp2(m_run[mb][h] - m_use[h]);
                    m_run[mb][h] = m_new;
                }
#pragma unroll
                for (int nb = 0; nb < 2; ++nb)
#pragma unroll
                    for (int e = 0; e < 4; ++e) s[nb][e] = fast_exp2(s[nb][e] - m_use[e >> 1]);
                pa[mb][0] = pack_bf16x2(s[0][0], s[0][1]);   // row gq
                pa[mb][1] = pack_bf16x2(s[0][2], s[0][3]);   // row gq + 8
                pa[mb][2] = pack_bf16x2(s[1][0], s[1][1]);   // row gq
                pa[mb][3] = pack_bf16x2(s[1][2], s[1][3]);   // row gq + 8
                // l sums the bf16 weights the PV product uses (see prefill.cu)
                const float2 w0 = bf16x2_to_float2(pa[mb][0]), w1 = bf16x2_to_float2(pa[mb][1]);
                const float2 w2 = bf16x2_to_float2(pa[mb][2]), w3 = bf16x2_to_float2(pa[mb][3]);
                l_run[mb][0] = l_run[mb][0] * alpha[0] + ((w0.x + w0.y) + (w2.x + w2.y));
                l_run[mb][1] = l_run[mb][1] * alpha[1] + ((w1.x + w1.y) + (w3.x + w3.y));
#pragma unroll
                for (int nd = 0; nd < D / 8; ++nd) {
                    oacc[mb][nd][0] *= alpha[0];
                    oacc[mb][nd][1] *= alpha[0];
                    oacc[mb][nd][2] *= alpha[1];
                    oacc[mb][nd][3] *= alpha[1];
                }
            }
            const uint32_t vbase = smem_u32(vt);
            const int vrow = warp * 16 + (lane & 7) + (((lane >> 3) & 1) << 3);
#pragma unroll
            for (int dd = 0; dd < D / 16; ++dd) {
                uint32_t vb[4];
                ldsm_x4_trans(vb, vbase + swz_off<D>(vrow, 2 * dd + (lane >> 4)));
#pragma unroll
                for (int mb = 0; mb < MB; ++mb) {
                    mma_16816(oacc[mb][2 * dd], pa[mb], vb[0], vb[1]);
                    mma_16816(oacc[mb][2 * dd + 1], pa[mb], vb[2], vb[3]);
                }
            }
        }
        if (partial) fence_proxy_async_smem();      // zeroing before the ring slot is refilled
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty_bar[st]);
    }

    // ---- merge the four warps' partial softmax states ----
#pragma unroll
    for (int mb = 0; mb < MB; ++mb)
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            l_run[mb][h] += __shfl_xor_sync(0xffffffffu, l_run[mb][h], 1);
            l_run[mb][h] += __shfl_xor_sync(0xffffffffu, l_run[mb][h], 2);
        }
    named_barrier_sync(1, kDecWarps * 32);          // every stage consumed: reuse the ring
    constexpr int kRows = MB * 16;
    float *s_o = reinterpret_cast<float *>(smem);             // [warp][row][D]
    float *s_m = s_o + kDecWarps * kRows * D;                 // [warp][row]
    float *s_l = s_m + kDecWarps * kRows;                     // [warp][row]
#pragma unroll
    for (int mb = 0; mb < MB; ++mb) {
#pragma unroll
        for (int nd = 0; nd < D / 8; ++nd)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int r = mb * 16 + gq + ((e >> 1) << 3);
                const int c = nd * 8 + 2 * tq + (e & 1);
                s_o[(warp * kRows + r) * D + c] = oacc[mb][nd][e];
            }
        if (tq == 0) {
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int r = mb * 16 + gq + h * 8;
                s_m[warp * kRows + r] = m_run[mb][h];
                s_l[warp * kRows + r] = l_run[mb][h];
            }
        }
    }
    named_barrier_sync(1, kDecWarps * 32);
    const size_t row0 = (static_cast<size_t>(split) * B + b) * Hq + static_cast<size_t>(kvh) * G;
    for (int idx = threadIdx.x; idx < G * D; idx += kDecWarps * 32) {
        const int r = idx / D, c = idx % D;
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < kDecWarps; ++w) M = fmaxf(M, s_m[w * kRows + r]);
        float wsum = 0.0f, acc = 0.0f;
#pragma unroll
        for (int w = 0; w < kDecWarps; ++w) {
            const float f = fast_exp2(s_m[w * kRows + r] - M);   // 0 for a warp with no key
            wsum += f * s_l[w * kRows + r];
            acc += f * s_o[(w * kRows + r) * D + c];
        }
        part_o[(row0 + r) * D + c] = acc / wsum;
        if (c == 0) part_lse[row0 + r] = (M + __log2f(wsum)) * 0.69314718055994531f;
    }

    // ---- the last split of this (sequence, KV head) merges all of them ----
    // Arrival word: call id in the high 48 bits, arrivals of that call in the
    // low 16.  A word left by another call (or uninitialised memory) restarts
    // the count at this call; the merging CTA leaves (call id, 0), so a replay
    // of the same launch (a CUDA graph) counts from zero again.  The CAS loop
    // ends: every failed attempt means another split's attempt succeeded.
    __threadfence();                                 // my partial rows, device-wide
    named_barrier_sync(1, kDecWarps * 32);
    if (threadIdx.x == 0) {
        unsigned long long *word = arrivals + static_cast<size_t>(b) * Hkv + kvh;
        unsigned long long cur = *reinterpret_cast<volatile unsigned long long *>(word), seen;
        unsigned long long next;
        do {
            seen = cur;
            next = (seen >> 16) == call_id ? seen + 1 : ((call_id << 16) | 1ull);
            cur = atomicCAS(word, seen, next);
        } while (cur != seen);
        const bool last = static_cast<int>(next & 0xFFFFu) == n_splits;
        if (last) *reinterpret_cast<volatile unsigned long long *>(word) = call_id << 16;
        merger = last;
    }
    named_barrier_sync(1, kDecWarps * 32);
    if (!merger) return;
    __threadfence();                                 // every split's partial rows are visible
    const size_t plane = static_cast<size_t>(B) * Hq;
    const size_t grow0 = static_cast<size_t>(b) * Hq + static_cast<size_t>(kvh) * G;
    // Batches of 8 splits keep their loads in flight together (the partial
    // rows sit in L2); the running max is taken first, then the sums.
    constexpr int kBatch = 8;
    for (int idx = threadIdx.x; idx < G * D / 2; idx += kDecWarps * 32) {
        const int r = idx / (D / 2), c = (idx % (D / 2)) * 2;
        const float *lse_r = part_lse + grow0 + r;
        const float *o_r = part_o + (grow0 + r) * D + c;
        float M = -INFINITY;
        for (int sp0 = 0; sp0 < n_splits; sp0 += kBatch) {
            float l[kBatch];
#pragma unroll
            for (int e = 0; e < kBatch; ++e)
                l[e] = sp0 + e < n_splits ? __ldcg(lse_r + (sp0 + e) * plane) : -INFINITY;
#pragma unroll
            for (int e = 0; e < kBatch; ++e) M = fmaxf(M, l[e]);
        }
        float wsum = 0.0f, a0 = 0.0f, a1 = 0.0f;
        for (int sp0 = 0; sp0 < n_splits; sp0 += kBatch) {
            float l[kBatch];
            float2 v[kBatch];
#pragma unroll
            for (int e = 0; e < kBatch; ++e) {
                const bool in = sp0 + e < n_splits;
                l[e] = in ? __ldcg(lse_r + (sp0 + e) * plane) : -INFINITY;
                v[e] = in ? __ldcg(reinterpret_cast<const float2 *>(o_r + (sp0 + e) * plane * D))
                          : make_float2(0.0f, 0.0f);
            }
#pragma unroll
            for (int e = 0; e < kBatch; ++e) {
                const float w = __expf(l[e] - M);          // 0 for the padding entries
                wsum += w;
                a0 += w * v[e].x;
                a1 += w * v[e].y;
            }
        }
        const float inv = 1.0f / wsum;
        *reinterpret_cast<__nv_bfloat162 *>(o + (grow0 + r) * D + c) =
            __floats2bfloat162_rn(a0 * inv, a1 * inv);
    }
}

// Keys per split: kDecChunk.  A windowed call (at most `window` keys after the
// window start) splits the window span in about three: ceil(span / 3) rounded up
// to 128 keys, between kDecChunk / 2 and kDecChunk, when the workspace (sized
// for the plain chunk over Lmax) has room for that many splits.  Measured on 64
// sequences x 8 KV heads with a 2048-key window: 512-key splits 5.18-5.28 TB/s,
// 768 (this rule) 5.42, 1024 5.23, 2048 4.70 -- fewer CTAs pay less per-CTA
// setup and merge work, until the grid is too short to fill its last wave.
static int decode_chunk(int Lmax, int window) {
    const long long plain_splits = (static_cast<long long>(Lmax) + kDecChunk - 1) / kDecChunk;
    if (window > 0) {
        const long long span = window < Lmax ? window : Lmax;
        long long c = ((span + 2) / 3 + 127) / 128 * 128;
        c = c < kDecChunk / 2 ? kDecChunk / 2 : (c > kDecChunk ? kDecChunk : c);
        if ((span + c - 1) / c <= plain_splits) return static_cast<int>(c);
    }
    return kDecChunk;
}

static size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

// Workspace: partial O [splits, B, Hq, d] fp32 | partial lse [splits, B, Hq]
// fp32 | arrival words [B, Hkv] u64, splits = ceil(Lmax / kDecChunk).
struct DecWorkspace {
    size_t splits, rows, off_lse, off_arrivals, bytes;
    DecWorkspace(int B, int Hq, int Hkv, int d, int Lmax) {
        splits = (static_cast<size_t>(Lmax) + kDecChunk - 1) / kDecChunk;
        rows = splits * B * Hq;
        off_lse = align256(rows * d * sizeof(float));
        off_arrivals = off_lse + align256(rows * sizeof(float));
        bytes = splits ? off_arrivals + align256(static_cast<size_t>(B) * Hkv * 8) : 0;
    }
};

size_t decode_workspace_bytes(int B, int Hq, int Hkv, int d, int Lmax) {
    return DecWorkspace(B, Hq, Hkv, d, Lmax).bytes;
}

// Per-call ids for the arrival words: 48 bits, never 0, different for every
// launch of the process (the start is drawn from the clock, so a workspace
// reused by another process is unlikely to hold a matching word either).
static unsigned long long next_call_id() {
    static std::atomic<unsigned long long> counter{
        static_cast<unsigned long long>(
            std::chrono::steady_clock::now().time_since_epoch().count()) * 0x9E3779B97F4A7C15ull};
    for (;;) {
        const unsigned long long id = counter.fetch_add(1) & 0xFFFFFFFFFFFFull;
        if (id != 0) return id;
    }
}

template <int D, int MB, bool kRope>
static int launch_split(const CUtensorMap &tk, const CUtensorMap &tv, const void *q,
                        const int32_t *seqlens, float *part_o, float *part_lse,
                        unsigned long long *arrivals, void *o, int B, int Hq, int Hkv, int Lmax,
                        int chunk, int window, int sinks, float scale_log2, double log_theta,
                        int *status, cudaStream_t stream) {
    auto kern = decode_split_kernel<D, MB, kRope>;
    const int smem = DecLayout<D, MB>::kSmemBytes;
    static CtxSlot setup;   // one per instantiation: the opt-in is set once per context
    if (int rc = once_per_context(setup, [&](int) {
            return check_cuda(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                   smem), "cudaFuncSetAttribute(decode)");
        }))
        return rc;
    const int span = window > 0 ? min(Lmax, window) : Lmax;   // keys after the window start
    dim3 grid((span + chunk - 1) / chunk, Hkv, B);
    kern<<<grid, kDecThreads, smem, stream>>>(tk, tv, static_cast<const __nv_bfloat16 *>(q),
                                              seqlens, part_o, part_lse, arrivals, next_call_id(),
                                              static_cast<__nv_bfloat16 *>(o), B, Hq, Hkv, Lmax,
                                              chunk, window, sinks, scale_log2, log_theta,
                                              status);
    return check_cuda(cudaGetLastError(), "decode_split_kernel launch");
}

int launch_decode(const void *q, const void *k_cache, const void *v_cache,
                  const int32_t *seqlens, void *o, int B, int Hq, int Hkv, int d, int Lmax,
                  int window, int sinks, float scale, void *workspace, cudaStream_t stream,
                  float rope_theta) {
    if (B > 65535 || Hkv > 65535)
        return set_error(GQA_ERR_UNSUPPORTED, "decode: B and Hkv must be <= 65535");
    const DecWorkspace ws(B, Hq, Hkv, d, Lmax);
    if (ws.splits > 0xFFFF)
        return set_error(GQA_ERR_UNSUPPORTED, "decode: Lmax=%d gives more than 65535 splits", Lmax);
    // an empty cache: every output row is zero
    if (ws.splits == 0) return launch_empty_rows(o, nullptr, 2, B, 1, Hq, d, stream);
    int *status = device_status_ptr();
    if (!status) return GQA_ERR_CUDA;
    const int chunk = decode_chunk(Lmax, window);
    uint8_t *base = static_cast<uint8_t *>(workspace);
    float *part_o = reinterpret_cast<float *>(base);
    float *part_lse = reinterpret_cast<float *>(base + ws.off_lse);
    auto *arrivals = reinterpret_cast<unsigned long long *>(base + ws.off_arrivals);
    const int G = Hq / Hkv;
    const float scale_log2 = scale * 1.4426950408889634f;
    CUtensorMap tk, tv;
    if (int rc = encode_tmap_bf16_4d(&tk, k_cache, d, Hkv, Lmax, B, 64, 1, kDecBK, 1, 1)) return rc;
    if (int rc = encode_tmap_bf16_4d(&tv, v_cache, d, Hkv, Lmax, B, 64, 1, kDecBK, 1, 1)) return rc;
    const bool rope = rope_theta > 0.0f;
    const double log_theta = rope ? log(static_cast<double>(rope_theta)) : 0.0;
#define GQA_DEC_LAUNCH(DD, MBB, RR)                                                             \
    launch_split<DD, MBB, RR>(tk, tv, q, seqlens, part_o, part_lse, arrivals, o, B, Hq, Hkv, Lmax, \
                              chunk, window, sinks, scale_log2, log_theta, status, stream)
    if (d == 128) {
        if (G <= 16) return rope ? GQA_DEC_LAUNCH(128, 1, true) : GQA_DEC_LAUNCH(128, 1, false);
        return rope ? GQA_DEC_LAUNCH(128, 2, true) : GQA_DEC_LAUNCH(128, 2, false);
    }
    if (G <= 16) return rope ? GQA_DEC_LAUNCH(64, 1, true) : GQA_DEC_LAUNCH(64, 1, false);
    return rope ? GQA_DEC_LAUNCH(64, 2, true) : GQA_DEC_LAUNCH(64, 2, false);
#undef GQA_DEC_LAUNCH
}

}  // namespace gqa
