// rope.cu -- rotary position embedding of q or k, in place, bf16.
//
// Course "Неделя 7. Внимание", step 3: coordinate pair (2i, 2i+1) of the row at
// position m is rotated by the angle m * theta_i, theta_i = theta^(-2i/d); only q
// and k rotate.  HBM-bound: each thread moves 16-byte vectors (4 pairs).  The
// angle m * theta_i reaches ~10^4 rad at long context, so it is formed and
// reduced modulo 2 pi in double before the fp32 sine and cosine.
#include <cuda_bf16.h>

#include "device.cuh"
#include "internal.h"

namespace gqa {

constexpr int kRopeMaxHalf = 128;    // d <= 256

// x viewed as [B, T, H, d]; row (b, t) sits at position pos0 + t, or at
// seqlens[b] - 1 when seqlens is given (decode queries, T = 1).
__global__ void __launch_bounds__(256)
rope_kernel(uint4 *__restrict__ x, size_t n_vec, int T, int H, int d, int pos0,
            const int32_t *__restrict__ seqlens, double log_theta) {
    __shared__ double inv_freq[kRopeMaxHalf];
    for (int i = threadIdx.x; i < d / 2; i += blockDim.x)
        inv_freq[i] = exp(-2.0 * i / d * log_theta);
    __syncthreads();
    const int d8 = d / 8;
    const double two_pi = 6.283185307179586476925286766559;
    const size_t stride = static_cast<size_t>(gridDim.x) * blockDim.x;
    for (size_t v = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; v < n_vec;
         v += stride) {
        const int c8 = static_cast<int>(v % d8);
        const size_t row = v / d8;                 // (b * T + t) * H + h
        const size_t bt = row / H;
        const int t = static_cast<int>(bt % T);
        const int b = static_cast<int>(bt / T);
        const int m = seqlens ? max(seqlens[b] - 1, 0) : pos0 + t;
        uint4 w = x[v];
        uint32_t *wp = reinterpret_cast<uint32_t *>(&w);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int i = c8 * 4 + e;              // pair index
            const double ang = static_cast<double>(m) * inv_freq[i];
            const double red = ang - two_pi * rint(ang / two_pi);
            float sn, cs;
            sincosf(static_cast<float>(red), &sn, &cs);
            const float2 a = bf16x2_to_float2(wp[e]);
            wp[e] = pack_bf16x2(a.x * cs - a.y * sn, a.x * sn + a.y * cs);
        }
        x[v] = w;
    }
}

static int launch_rope(void *x, int B, int T, int H, int d, int pos0, const int32_t *seqlens,
                       float theta, cudaStream_t stream) {
    const size_t n_vec = static_cast<size_t>(B) * T * H * (d / 8);
    int blocks = static_cast<int>((n_vec + 255) / 256);
    if (blocks > 148 * 16) blocks = 148 * 16;
    rope_kernel<<<blocks, 256, 0, stream>>>(static_cast<uint4 *>(x), n_vec, T, H, d, pos0, seqlens,
                                            log(static_cast<double>(theta)));
    return check_cuda(cudaGetLastError(), "rope_kernel launch");
}

static int check_rope_args(const void *x, int B, int T, int H, int d, float theta) {
    if (B < 0 || T < 0 || H < 1)
        return set_error(GQA_ERR_INVALID_ARG, "B=%d, T=%d must be >= 0 and H=%d >= 1", B, T, H);
    if (d < 8 || d % 8 != 0 || d > 2 * kRopeMaxHalf)
        return set_error(GQA_ERR_INVALID_ARG, "head dim d=%d must be a multiple of 8 in [8, 256]",
                         d);
    if (!(theta > 0.0f) || !isfinite(theta))
        return set_error(GQA_ERR_INVALID_ARG, "theta=%g must be finite and > 0", (double)theta);
    if (B > 0 && T > 0) {
        if (!x) return set_error(GQA_ERR_INVALID_ARG, "x is NULL");
        if (reinterpret_cast<uintptr_t>(x) % 16)
            return set_error(GQA_ERR_INVALID_ARG, "x is not 16-byte aligned");
    }
    return GQA_OK;
}

}  // namespace gqa

using namespace gqa;

extern "C" int gqa_rope(void *x, int B, int T, int H, int d, int pos0, float theta,
                        gqa_stream_t stream) {
    clear_error();
    if (int rc = check_rope_args(x, B, T, H, d, theta)) return rc;
    if (B == 0 || T == 0) return GQA_OK;
    if (int rc = require_sm100()) return rc;
    return launch_rope(x, B, T, H, d, pos0, nullptr, theta, reinterpret_cast<cudaStream_t>(stream));
}

extern "C" int gqa_rope_decode_q(void *q, const int32_t *seqlens, int B, int H, int d, float theta,
                                 gqa_stream_t stream) {
    clear_error();
    if (int rc = check_rope_args(q, B, 1, H, d, theta)) return rc;
    if (B == 0) return GQA_OK;
    if (!seqlens || reinterpret_cast<uintptr_t>(seqlens) % 4)
        return set_error(GQA_ERR_INVALID_ARG, "seqlens is NULL or misaligned");
    if (int rc = require_sm100()) return rc;
    return launch_rope(q, B, 1, H, d, 0, seqlens, theta, reinterpret_cast<cudaStream_t>(stream));
}
