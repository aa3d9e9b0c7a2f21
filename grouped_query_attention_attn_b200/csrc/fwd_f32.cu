// fwd_f32.cu -- fp32 grouped-query attention on the FP32 pipe (no tensor
// cores), and the fill of rows that see no key.
//
// One warp owns one query row (b, i, hq).  It walks the visible keys 32 at a
// time: lane j scores key j0 + j, the warp takes the block max, rescales its
// running output by exp(m_old - m_new) (the max-subtracted softmax kept
// online), then accumulates p_j * v_j with lanes splitting the head dim.
// Query head hq reads K/V head hq / (Hq / Hkv).
#include <cuda_bf16.h>

#include "device.cuh"
#include "internal.h"

namespace gqa {

constexpr int kF32RowsPerBlock = 4;
constexpr int kF32MaxCols = 8;     // d <= 256 = 32 lanes x 8 columns

__device__ __forceinline__ float warp_max(float x) {
    for (int o = 16; o > 0; o >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, o));
    return x;
}

__device__ __forceinline__ float warp_sum(float x) {
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}

__global__ void __launch_bounds__(32 * kF32RowsPerBlock)
fwd_f32_kernel(const float *__restrict__ q, const float *__restrict__ k,
               const float *__restrict__ v, float *__restrict__ o, float *__restrict__ lse,
               int Tq, int Tkv, int Hq, int Hkv, int d, int causal, float scale) {
    extern __shared__ float s_q[];                 // kF32RowsPerBlock x d
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int i = blockIdx.x * kF32RowsPerBlock + warp;
    const int hq = blockIdx.y, b = blockIdx.z;
    if (i >= Tq) return;                           // whole warp leaves together
    const int kvh = hq / (Hq / Hkv);
    const size_t q_off = ((static_cast<size_t>(b) * Tq + i) * Hq + hq) * d;
    float *my_q = s_q + warp * d;
    for (int c = lane; c < d; c += 32) my_q[c] = q[q_off + c];
    __syncwarp();

    int n_vis = Tkv;
    if (causal) {
        const long long n = static_cast<long long>(i) + (Tkv - Tq) + 1;
        n_vis = n < 0 ? 0 : (n > Tkv ? Tkv : static_cast<int>(n));
    }
    const size_t row_stride = static_cast<size_t>(Hkv) * d;
    const float *k0 = k + (static_cast<size_t>(b) * Tkv * Hkv + kvh) * d;
    const float *v0 = v + (static_cast<size_t>(b) * Tkv * Hkv + kvh) * d;

    float m = -INFINITY, l = 0.0f;
    float acc[kF32MaxCols];
#pragma unroll
    for (int cc = 0; cc < kF32MaxCols; ++cc) acc[cc] = 0.0f;

    for (int j0 = 0; j0 < n_vis; j0 += 32) {
        const int j = j0 + lane;
        float s = -INFINITY;
        if (j < n_vis) {
            const float *kj = k0 + static_cast<size_t>(j) * row_stride;
            float dot = 0.0f;
            for (int c = 0; c < d; ++c) dot = fmaf(my_q[c], kj[c], dot);
            s = dot * scale;
        }
        const float m_new = fmaxf(m, warp_max(s));  // finite: lane 0's key is visible
        const float alpha = expf(m - m_new);        // 0 on the first block (m = -inf)
        const float p = (j < n_vis) ? expf(s - m_new) : 0.0f;
        l = l * alpha + warp_sum(p);
#pragma unroll
        for (int cc = 0; cc < kF32MaxCols; ++cc) acc[cc] *= alpha;
        const int n_here = min(32, n_vis - j0);
        for (int t = 0; t < n_here; ++t) {
            const float pt = __shfl_sync(0xffffffffu, p, t);
            const float *vt = v0 + static_cast<size_t>(j0 + t) * row_stride;
#pragma unroll
            for (int cc = 0; cc < kF32MaxCols; ++cc) {
                const int c = lane + 32 * cc;
                if (c < d) acc[cc] = fmaf(pt, vt[c], acc[cc]);
            }
        }
        m = m_new;
    }

    const float inv_l = (n_vis > 0) ? 1.0f / l : 0.0f;
#pragma unroll
    for (int cc = 0; cc < kF32MaxCols; ++cc) {
        const int c = lane + 32 * cc;
        if (c < d) o[q_off + c] = acc[cc] * inv_l;
    }
    if (lse && lane == 0)
        lse[(static_cast<size_t>(b) * Hq + hq) * Tq + i] = (n_vis > 0) ? m + logf(l) : -INFINITY;
}

int launch_fwd_f32(const float *q, const float *k, const float *v, float *o, float *lse,
                   int B, int Tq, int Tkv, int Hq, int Hkv, int d, int causal, float scale,
                   cudaStream_t stream) {
    if (Hq > 65535 || B > 65535)
        return set_error(GQA_ERR_UNSUPPORTED, "fp32 path: Hq and B must be <= 65535");
    dim3 grid((Tq + kF32RowsPerBlock - 1) / kF32RowsPerBlock, Hq, B);
    const size_t smem = sizeof(float) * kF32RowsPerBlock * d;
    fwd_f32_kernel<<<grid, 32 * kF32RowsPerBlock, smem, stream>>>(q, k, v, o, lse, Tq, Tkv, Hq,
                                                                  Hkv, d, causal, scale);
    return check_cuda(cudaGetLastError(), "fwd_f32_kernel launch");
}

// Rows that see no key (Tkv == 0): o = 0 and lse = -inf.
__global__ void empty_rows_kernel(uint8_t *o, size_t o_bytes, float *lse, size_t n_lse) {
    const size_t stride = static_cast<size_t>(gridDim.x) * blockDim.x;
    for (size_t t = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; t < o_bytes;
         t += stride)
        o[t] = 0;
    if (lse)
        for (size_t t = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; t < n_lse;
             t += stride)
            lse[t] = -INFINITY;
}

int launch_empty_rows(void *o, float *lse, int elem_bytes, int B, int Tq, int Hq, int d,
                      cudaStream_t stream) {
    const size_t rows = static_cast<size_t>(B) * Tq * Hq;
    empty_rows_kernel<<<296, 256, 0, stream>>>(static_cast<uint8_t *>(o),
                                               rows * d * elem_bytes, lse, rows);
    return check_cuda(cudaGetLastError(), "empty_rows_kernel launch");
}

}  // namespace gqa
