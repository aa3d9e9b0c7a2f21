// backward.cu -- gradients of grouped-query attention: dQ, dK, dV (bf16 in and
// out, fp32 accumulation, warp-level bf16 tensor-core tiles).
//
// With P = softmax of the masked, scaled scores (recomputed from the forward's
// log-sum-exp) and D_i = <dO_i, O_i>:
//   dV_j = sum_i P_ij dO_i,   dP_ij = <dO_i, V_j>,   dS_ij = P_ij (dP_ij - D_i),
//   dQ_i = scale sum_j dS_ij K_j,   dK_j = scale sum_i dS_ij Q_i.
// Query head hq reads K/V head hq / G, so the gradient of a shared K/V head is
// the SUM over the G query heads of its group (K3 notes "GVA", "Backward:
// view + sum": the backward of a copy is a sum).  Three kernels:
//   rowdot  D = rowsum(dO * O)                                  (HBM-bound)
//   dkdv    one CTA per 64 keys of one KV head; loops over every query row
//           of the G heads of the group, so dK and dV accumulate in
//           registers with no atomics
//   dq      one CTA per 64 query rows of one head; loops over the keys
// Tiles reach shared memory through double-buffered cp.async with padded
// rows (ldmatrix is then free of bank conflicts).
#include <cuda_bf16.h>
#include <climits>

#include "device.cuh"
#include "internal.h"

namespace gqa {

constexpr int kBwThreads = 128;   // 4 warps x 16 rows of the MMA M dimension
constexpr int kKvTile = 64;       // keys per dkdv CTA
constexpr int kQBlk = 32;         // query rows per dkdv iteration
constexpr int kQTile = 64;        // query rows per dq CTA
constexpr int kKBlk = 32;         // keys per dq iteration

__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src, bool valid) {
    // src-size 0 writes zeros (rows past the end of the tensor)
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;"
                 ::"r"(dst), "l"(src), "r"(valid ? 16 : 0) : "memory");
}
__device__ __forceinline__ void cp_async4(uint32_t dst, const void *src, bool valid) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;"
                 ::"r"(dst), "l"(src), "r"(valid ? 4 : 0) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

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
__global__ void __launch_bounds__(256)
rowdot_kernel(const __nv_bfloat16 *__restrict__ dout, const __nv_bfloat16 *__restrict__ o,
              float *__restrict__ Dsum, int B, int T, int H, int d) {
    const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, lane = threadIdx.x & 31;
    const long long rows = static_cast<long long>(B) * T * H;
    if (warp >= rows) return;
    const int h = warp % H, t = (warp / H) % T, b = warp / (H * T);
    const __nv_bfloat16 *a = dout + static_cast<size_t>(warp) * d;
    const __nv_bfloat16 *c = o + static_cast<size_t>(warp) * d;
    float acc = 0.0f;
    for (int e = lane * 2; e < d; e += 64) {
        const float2 x = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(a + e));
        const float2 y = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(c + e));
        acc = fmaf(x.x, y.x, fmaf(x.y, y.y, acc));
    }
    for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
    if (lane == 0) Dsum[(static_cast<size_t>(b) * H + h) * T + t] = acc;
}

// Copy `rows` rows of D bf16 (global row stride gstride elements) starting at
// row r0 into shared memory with row pitch D + 8; rows >= nrows are zeros.
template <int D>
__device__ __forceinline__ void load_tile(uint32_t sdst, const __nv_bfloat16 *g, size_t gstride,
                                          int r0, int rows, int nrows) {
    constexpr int kChunks = D / 8;
    for (int idx = threadIdx.x; idx < rows * kChunks; idx += kBwThreads) {
        const int r = idx / kChunks, c = idx % kChunks;
        const bool ok = r0 + r < nrows;
        const __nv_bfloat16 *src = g + static_cast<size_t>(ok ? r0 + r : 0) * gstride + c * 8;
        cp_async16(sdst + (r * (D + 8) + c * 8) * 2, src, ok);
    }
}

template <int D>
__device__ __forceinline__ uint32_t tile_addr(uint32_t base, int row, int chunk) {
    return base + (row * (D + 8) + chunk * 8) * 2;
}

// --------------------------------------------------------------- dk dv ---
template <int D>
__global__ void __launch_bounds__(kBwThreads)
dkdv_kernel(const __nv_bfloat16 *__restrict__ q, const __nv_bfloat16 *__restrict__ k,
            const __nv_bfloat16 *__restrict__ v, const __nv_bfloat16 *__restrict__ dout,
            const float *__restrict__ lse, const float *__restrict__ Dsum,
            __nv_bfloat16 *__restrict__ dk, __nv_bfloat16 *__restrict__ dv, int B, int Tq,
            int Tkv, int Hq, int Hkv, Vis vis, float scale) {
    constexpr int P = D + 8;
    extern __shared__ __align__(16) uint8_t smem[];
    __nv_bfloat16 *sK = reinterpret_cast<__nv_bfloat16 *>(smem);
    __nv_bfloat16 *sV = sK + kKvTile * P;
    __nv_bfloat16 *sQ = sV + kKvTile * P;                // [2][kQBlk][P]
    __nv_bfloat16 *sO = sQ + 2 * kQBlk * P;              // dO, [2][kQBlk][P]
    float *sL = reinterpret_cast<float *>(sO + 2 * kQBlk * P);   // lse, [2][kQBlk]
    float *sD = sL + 2 * kQBlk;                                  // D,   [2][kQBlk]
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int gq = lane >> 2, tq = lane & 3;
    // key tiles in decreasing causal work (the first tiles see the most queries)
    const int bhs = Hkv * B;
    const int lin = blockIdx.x;
    const int kb = lin / bhs, kvh = lin % Hkv, b = (lin / Hkv) % B;
    const int G = Hq / Hkv;
    const int k0 = kb * kKvTile;
    const float c2 = scale * 1.4426950408889634f;

    // query rows that can see any key of this tile
    const int off = Tkv - Tq;
    int q_lo = 0, q_hi = Tq;
    if (vis.causal) {
        q_lo = max(0, k0 - off);
        if (vis.window > 0 && k0 >= vis.sinks) q_hi = min(Tq, k0 + kKvTile - 1 + vis.window - off);
    }
    const int qb0 = q_lo / kQBlk;
    const int n_qb = q_hi > q_lo ? (q_hi + kQBlk - 1) / kQBlk - qb0 : 0;
    const int n_items = G * n_qb;

    const size_t kstride = static_cast<size_t>(Hkv) * D, qstride = static_cast<size_t>(Hq) * D;
    const uint32_t aK = smem_u32(sK), aV = smem_u32(sV), aQ = smem_u32(sQ), aO = smem_u32(sO);
    load_tile<D>(aK, k + (static_cast<size_t>(b) * Tkv * Hkv + kvh) * D, kstride, k0, kKvTile, Tkv);
    load_tile<D>(aV, v + (static_cast<size_t>(b) * Tkv * Hkv + kvh) * D, kstride, k0, kKvTile, Tkv);
    const uint32_t aL = smem_u32(sL), aD = smem_u32(sD);
    auto issue_item = [&](int it) {
        const int g = it / n_qb, qb = qb0 + it % n_qb, buf = it & 1;
        const size_t base = (static_cast<size_t>(b) * Tq * Hq + kvh * G + g) * D;
        load_tile<D>(aQ + buf * kQBlk * P * 2, q + base, qstride, qb * kQBlk, kQBlk, Tq);
        load_tile<D>(aO + buf * kQBlk * P * 2, dout + base, qstride, qb * kQBlk, kQBlk, Tq);
        // the block's softmax statistics: lse and D of its kQBlk query rows
        const int t = threadIdx.x;
        if (t < 2 * kQBlk) {
            const int r = t % kQBlk, qi = qb * kQBlk + r;
            const size_t li = (static_cast<size_t>(b) * Hq + kvh * G + g) * Tq + min(qi, Tq - 1);
            cp_async4((t < kQBlk ? aL : aD) + (buf * kQBlk + r) * 4,
                      (t < kQBlk ? lse : Dsum) + li, qi < Tq);
        }
    };
    if (n_items > 0) issue_item(0);
    cp_async_commit();

    float dka[D / 8][4], dva[D / 8][4];
#pragma unroll
    for (int n = 0; n < D / 8; ++n)
#pragma unroll
        for (int e = 0; e < 4; ++e) dka[n][e] = dva[n][e] = 0.0f;
    const int krow = 16 * warp;                          // this warp's keys in the tile

    for (int it = 0; it < n_items; ++it) {
        if (it + 1 < n_items) issue_item(it + 1);
        cp_async_commit();
        cp_async_wait<1>();
        __syncthreads();
        const int qb = qb0 + it % n_qb, buf = it & 1;
        const uint32_t bQ = aQ + buf * kQBlk * P * 2, bO = aO + buf * kQBlk * P * 2;
        // S^T (16 keys x 32 queries) and dP^T = V dO^T
        float st[4][4], dpt[4][4];
#pragma unroll
        for (int n = 0; n < 4; ++n)
#pragma unroll
            for (int e = 0; e < 4; ++e) st[n][e] = dpt[n][e] = 0.0f;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
            uint32_t ka[4], va[4];
            const int ar = krow + (lane & 7) + (((lane >> 3) & 1) << 3), ac = 2 * kk + (lane >> 4);
            ldsm_x4(ka, tile_addr<D>(aK, ar, ac));
            ldsm_x4(va, tile_addr<D>(aV, ar, ac));
#pragma unroll
            for (int np = 0; np < 2; ++np) {
                uint32_t qbf[4], obf[4];
                const int br = np * 16 + (lane & 7) + ((lane >> 4) << 3), bc = 2 * kk + ((lane >> 3) & 1);
                ldsm_x4(qbf, tile_addr<D>(bQ, br, bc));
                ldsm_x4(obf, tile_addr<D>(bO, br, bc));
                mma_16816(st[2 * np], ka, qbf[0], qbf[1]);
                mma_16816(st[2 * np + 1], ka, qbf[2], qbf[3]);
                mma_16816(dpt[2 * np], va, obf[0], obf[1]);
                mma_16816(dpt[2 * np + 1], va, obf[2], obf[3]);
            }
        }
        // P^T and dS^T, packed as A fragments over the 32 queries (2 k-steps).
        // Blocks inside the visible region skip the per-element test.
        const bool full = block_visible(vis, qb * kQBlk, kQBlk, k0, kKvTile);
        const float *bL = sL + buf * kQBlk, *bD = sD + buf * kQBlk;
        uint32_t pa[2][4], sa[2][4];
#pragma unroll
        for (int n = 0; n < 4; ++n) {
            float pv[4], sv[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int key = k0 + krow + gq + ((e >> 1) << 3);
                const int ql = n * 8 + 2 * tq + (e & 1);
                float pr = 0.0f, dsv = 0.0f;
                if (full || vis(qb * kQBlk + ql, key)) {
                    pr = fast_exp2(fmaf(st[n][e], c2, -bL[ql] * 1.4426950408889634f));
                    dsv = pr * (dpt[n][e] - bD[ql]);
                }
                pv[e] = pr;
                sv[e] = dsv;
            }
            const int ks = n >> 1, hi = n & 1;
            pa[ks][2 * hi] = pack_bf16x2(pv[0], pv[1]);
            pa[ks][2 * hi + 1] = pack_bf16x2(pv[2], pv[3]);
            sa[ks][2 * hi] = pack_bf16x2(sv[0], sv[1]);
            sa[ks][2 * hi + 1] = pack_bf16x2(sv[2], sv[3]);
        }
        // dV += P^T dO,  dK += dS^T Q   (B operands: dO / Q rows = queries, trans)
#pragma unroll
        for (int ks = 0; ks < 2; ++ks) {
#pragma unroll
            for (int dp = 0; dp < D / 16; ++dp) {
                uint32_t ob[4], qbt[4];
                const int r = ks * 16 + (lane & 7) + (((lane >> 3) & 1) << 3), c = 2 * dp + (lane >> 4);
                ldsm_x4_trans(ob, tile_addr<D>(bO, r, c));
                ldsm_x4_trans(qbt, tile_addr<D>(bQ, r, c));
                mma_16816(dva[2 * dp], pa[ks], ob[0], ob[1]);
                mma_16816(dva[2 * dp + 1], pa[ks], ob[2], ob[3]);
                mma_16816(dka[2 * dp], sa[ks], qbt[0], qbt[1]);
                mma_16816(dka[2 * dp + 1], sa[ks], qbt[2], qbt[3]);
            }
        }
        __syncthreads();                                 // buffer `buf` is refilled next
    }
    cp_async_wait<0>();

    // write dK (scaled) and dV for this warp's 16 keys
#pragma unroll
    for (int h2 = 0; h2 < 2; ++h2) {
        const int key = k0 + krow + gq + 8 * h2;
        if (key >= Tkv) continue;
        const size_t rowoff = ((static_cast<size_t>(b) * Tkv + key) * Hkv + kvh) * D;
#pragma unroll
        for (int n = 0; n < D / 8; ++n) {
            const int c = n * 8 + 2 * tq;
            *reinterpret_cast<__nv_bfloat162 *>(dk + rowoff + c) =
                __floats2bfloat162_rn(dka[n][2 * h2] * scale, dka[n][2 * h2 + 1] * scale);
            *reinterpret_cast<__nv_bfloat162 *>(dv + rowoff + c) =
                __floats2bfloat162_rn(dva[n][2 * h2], dva[n][2 * h2 + 1]);
        }
    }
}

// ------------------------------------------------------------------ dq ---
template <int D>
__global__ void __launch_bounds__(kBwThreads)
dq_kernel(const __nv_bfloat16 *__restrict__ q, const __nv_bfloat16 *__restrict__ k,
          const __nv_bfloat16 *__restrict__ v, const __nv_bfloat16 *__restrict__ dout,
          const float *__restrict__ lse, const float *__restrict__ Dsum,
          __nv_bfloat16 *__restrict__ dq, int B, int Tq, int Tkv, int Hq, int Hkv, Vis vis,
          float scale) {
    constexpr int P = D + 8;
    extern __shared__ __align__(16) uint8_t smem[];
    __nv_bfloat16 *sQ = reinterpret_cast<__nv_bfloat16 *>(smem);   // [kQTile][P]
    __nv_bfloat16 *sO = sQ + kQTile * P;                            // dO
    __nv_bfloat16 *sK = sO + kQTile * P;                            // [2][kKBlk][P]
    __nv_bfloat16 *sV = sK + 2 * kKBlk * P;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int gq = lane >> 2, tq = lane & 3;
    // query tiles in decreasing causal work (the last tiles see the most keys)
    const int bhs = Hq * B, n_qt = (Tq + kQTile - 1) / kQTile;
    const int lin = blockIdx.x;
    const int qt = n_qt - 1 - lin / bhs, hq = lin % Hq, b = (lin / Hq) % B;
    const int G = Hq / Hkv, kvh = hq / G;
    const int q0 = qt * kQTile;
    const float c2 = scale * 1.4426950408889634f;
    const int off = Tkv - Tq;

    // key blocks: the sink blocks, then the window / causal range
    const int q_last = min(Tq, q0 + kQTile) - 1;
    int kend = Tkv;
    if (vis.causal) kend = min(Tkv, q_last + off + 1);
    int n_sink = 0, first = 0;
    if (vis.causal && vis.window > 0 && kend > 0) {
        n_sink = (min(vis.sinks, kend) + kKBlk - 1) / kKBlk;
        first = max(n_sink, max(q0 + off - vis.window + 1, 0) / kKBlk);
    }
    const int last = kend > 0 ? (kend + kKBlk - 1) / kKBlk : 0;
    const int n_kb = n_sink + max(0, last - first);
    auto block_of = [&](int j) { return j < n_sink ? j : first + (j - n_sink); };

    const size_t kstride = static_cast<size_t>(Hkv) * D, qstride = static_cast<size_t>(Hq) * D;
    const size_t qbase = (static_cast<size_t>(b) * Tq * Hq + hq) * D;
    const size_t kbase = (static_cast<size_t>(b) * Tkv * Hkv + kvh) * D;
    const uint32_t aQ = smem_u32(sQ), aO = smem_u32(sO), aK = smem_u32(sK), aV = smem_u32(sV);
    load_tile<D>(aQ, q + qbase, qstride, q0, kQTile, Tq);
    load_tile<D>(aO, dout + qbase, qstride, q0, kQTile, Tq);
    auto issue = [&](int j) {
        const int buf = j & 1, kb = block_of(j);
        load_tile<D>(aK + buf * kKBlk * P * 2, k + kbase, kstride, kb * kKBlk, kKBlk, Tkv);
        load_tile<D>(aV + buf * kKBlk * P * 2, v + kbase, kstride, kb * kKBlk, kKBlk, Tkv);
    };
    if (n_kb > 0) issue(0);
    cp_async_commit();

    const int qrow = 16 * warp;
    float dqa[D / 8][4];
#pragma unroll
    for (int n = 0; n < D / 8; ++n)
#pragma unroll
        for (int e = 0; e < 4; ++e) dqa[n][e] = 0.0f;
    // per-row softmax statistics of this lane's two rows
    float lrow[2], drow[2];
#pragma unroll
    for (int h2 = 0; h2 < 2; ++h2) {
        const int qi = q0 + qrow + gq + 8 * h2;
        const size_t li = (static_cast<size_t>(b) * Hq + hq) * Tq + min(qi, Tq - 1);
        lrow[h2] = lse[li] * 1.4426950408889634f;
        drow[h2] = Dsum[li];
    }

    for (int j = 0; j < n_kb; ++j) {
        if (j + 1 < n_kb) issue(j + 1);
        cp_async_commit();
        cp_async_wait<1>();
        __syncthreads();
        const int buf = j & 1, kb = block_of(j);
        const uint32_t bK = aK + buf * kKBlk * P * 2, bV = aV + buf * kKBlk * P * 2;
        float s[4][4], dp[4][4];
#pragma unroll
        for (int n = 0; n < 4; ++n)
#pragma unroll
            for (int e = 0; e < 4; ++e) s[n][e] = dp[n][e] = 0.0f;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
            uint32_t qa[4], oa[4];
            const int ar = qrow + (lane & 7) + (((lane >> 3) & 1) << 3), ac = 2 * kk + (lane >> 4);
            ldsm_x4(qa, tile_addr<D>(aQ, ar, ac));
            ldsm_x4(oa, tile_addr<D>(aO, ar, ac));
#pragma unroll
            for (int np = 0; np < 2; ++np) {
                uint32_t kbf[4], vbf[4];
                const int br = np * 16 + (lane & 7) + ((lane >> 4) << 3), bc = 2 * kk + ((lane >> 3) & 1);
                ldsm_x4(kbf, tile_addr<D>(bK, br, bc));
                ldsm_x4(vbf, tile_addr<D>(bV, br, bc));
                mma_16816(s[2 * np], qa, kbf[0], kbf[1]);
                mma_16816(s[2 * np + 1], qa, kbf[2], kbf[3]);
                mma_16816(dp[2 * np], oa, vbf[0], vbf[1]);
                mma_16816(dp[2 * np + 1], oa, vbf[2], vbf[3]);
            }
        }
        // blocks inside the visible region skip the per-element test
        const bool full = block_visible(vis, q0, kQTile, kb * kKBlk, kKBlk);
        uint32_t sa[2][4];
#pragma unroll
        for (int n = 0; n < 4; ++n) {
            float sv[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int qi = q0 + qrow + gq + ((e >> 1) << 3);
                const int key = kb * kKBlk + n * 8 + 2 * tq + (e & 1);
                float dsv = 0.0f;
                if (full || vis(qi, key)) {
                    const float pr = fast_exp2(s[n][e] * c2 - lrow[e >> 1]);
                    dsv = pr * (dp[n][e] - drow[e >> 1]);
                }
                sv[e] = dsv;
            }
            const int ks = n >> 1, hi = n & 1;
            sa[ks][2 * hi] = pack_bf16x2(sv[0], sv[1]);
            sa[ks][2 * hi + 1] = pack_bf16x2(sv[2], sv[3]);
        }
        // dQ += dS K   (B operand: K rows = keys, trans)
#pragma unroll
        for (int ks = 0; ks < 2; ++ks)
#pragma unroll
            for (int dp2 = 0; dp2 < D / 16; ++dp2) {
                uint32_t kb2[4];
                const int r = ks * 16 + (lane & 7) + (((lane >> 3) & 1) << 3), c = 2 * dp2 + (lane >> 4);
                ldsm_x4_trans(kb2, tile_addr<D>(bK, r, c));
                mma_16816(dqa[2 * dp2], sa[ks], kb2[0], kb2[1]);
                mma_16816(dqa[2 * dp2 + 1], sa[ks], kb2[2], kb2[3]);
            }
        __syncthreads();
    }
    cp_async_wait<0>();
#pragma unroll
    for (int h2 = 0; h2 < 2; ++h2) {
        const int qi = q0 + qrow + gq + 8 * h2;
        if (qi >= Tq) continue;
        const size_t rowoff = ((static_cast<size_t>(b) * Tq + qi) * Hq + hq) * D;
#pragma unroll
        for (int n = 0; n < D / 8; ++n)
            *reinterpret_cast<__nv_bfloat162 *>(dq + rowoff + n * 8 + 2 * tq) =
                __floats2bfloat162_rn(dqa[n][2 * h2] * scale, dqa[n][2 * h2 + 1] * scale);
    }
}

size_t bwd_workspace_bytes(int B, int Tq, int Hq) {
    return ((static_cast<size_t>(B) * Tq * Hq * sizeof(float)) + 255) & ~static_cast<size_t>(255);
}

template <int D>
static int launch_bwd_d(const void *q, const void *k, const void *v, const void *o,
                        const void *dout, const float *lse, void *dq, void *dk, void *dv, int B,
                        int Tq, int Tkv, int Hq, int Hkv, int causal, int window, int sinks,
                        float scale, void *workspace, cudaStream_t stream) {
    using bf = __nv_bfloat16;
    float *Dsum = static_cast<float *>(workspace);
    const long long rows = static_cast<long long>(B) * Tq * Hq;
    rowdot_kernel<<<static_cast<unsigned>((rows * 32 + 255) / 256), 256, 0, stream>>>(
        static_cast<const bf *>(dout), static_cast<const bf *>(o), Dsum, B, Tq, Hq, D);
    if (int rc = check_cuda(cudaGetLastError(), "rowdot_kernel launch")) return rc;
    Vis vis{Tq, Tkv, causal, causal ? window : 0, sinks};
    constexpr int P = D + 8;
    const int smem_kv = (2 * kKvTile + 4 * kQBlk) * P * 2 + 4 * kQBlk * 4;
    const int smem_q = (2 * kQTile + 4 * kKBlk) * P * 2;
    auto kkv = dkdv_kernel<D>;
    auto kq = dq_kernel<D>;
    if (int rc = check_cuda(cudaFuncSetAttribute(kkv, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                 smem_kv), "cudaFuncSetAttribute(dkdv)"))
        return rc;
    if (int rc = check_cuda(cudaFuncSetAttribute(kq, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                 smem_q), "cudaFuncSetAttribute(dq)"))
        return rc;
    if (Tkv > 0) {
        const long long n1 = static_cast<long long>((Tkv + kKvTile - 1) / kKvTile) * Hkv * B;
        if (n1 > 0x7fffffffLL) return set_error(GQA_ERR_UNSUPPORTED, "backward grid too large");
        kkv<<<static_cast<unsigned>(n1), kBwThreads, smem_kv, stream>>>(
            static_cast<const bf *>(q), static_cast<const bf *>(k), static_cast<const bf *>(v),
            static_cast<const bf *>(dout), lse, Dsum, static_cast<bf *>(dk), static_cast<bf *>(dv),
            B, Tq, Tkv, Hq, Hkv, vis, scale);
        if (int rc = check_cuda(cudaGetLastError(), "dkdv_kernel launch")) return rc;
    }
    const long long n2 = static_cast<long long>((Tq + kQTile - 1) / kQTile) * Hq * B;
    if (n2 > 0x7fffffffLL) return set_error(GQA_ERR_UNSUPPORTED, "backward grid too large");
    kq<<<static_cast<unsigned>(n2), kBwThreads, smem_q, stream>>>(
        static_cast<const bf *>(q), static_cast<const bf *>(k), static_cast<const bf *>(v),
        static_cast<const bf *>(dout), lse, Dsum, static_cast<bf *>(dq), B, Tq, Tkv, Hq, Hkv, vis,
        scale);
    return check_cuda(cudaGetLastError(), "dq_kernel launch");
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
