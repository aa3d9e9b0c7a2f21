// fold_kv.cu -- MHA -> GQA mean pooling of K or V heads, and the self-test
// kernel of the bounded device waits.
//
// fold: out[b, t, grp, :] = (sum over the contiguous group members, in head
// order, in fp32) / (H / g), rounded to bf16 -- the position-wise mean over
// heads[start:start+size] of TT Lab "キー・バリューヘッドだけ減らしてみる",
// step 2.  HBM-bound: each thread moves 16-byte vectors and has all loads of
// a group in flight before it adds them.
#include <cuda_bf16.h>

#include "device.cuh"
#include "internal.h"

namespace gqa {

constexpr int kFoldBatch = 4;   // group members loaded before any is added

// Index type I: 32-bit when every vector index fits, so the per-vector
// divisions stay cheap.  kD8: d / 8 known at compile time (d = 64, 128: the
// index math becomes shifts), 0 for any other d.
template <typename I, int kD8>
__global__ void __launch_bounds__(256, 5)
fold_kv_kernel(const uint4 *__restrict__ in, uint4 *__restrict__ out, I n_vec, int H, int g,
               int d8_arg) {
    const int d8 = kD8 > 0 ? kD8 : d8_arg;
    const int size = H / g;
    const float divisor = static_cast<float>(size);
    // dividing by a power of two is exact, so it is a multiplication by the
    // reciprocal; any other group size takes the correctly rounded division
    const bool pow2 = (size & (size - 1)) == 0;
    const float inv = 1.0f / divisor;
    const I stride = static_cast<I>(gridDim.x) * blockDim.x;
    for (I t = static_cast<I>(blockIdx.x) * blockDim.x + threadIdx.x; t < n_vec; t += stride) {
        const I c8 = t % d8, rest = t / d8;
        const I grp = rest % g, bt = rest / g;
        const uint4 *src = in + (static_cast<size_t>(bt) * H + static_cast<size_t>(grp) * size) *
                                    d8 + c8;
        float acc[8];
        for (int m0 = 0; m0 < size; m0 += kFoldBatch) {
            // all loads of the batch in flight, then the adds in head order
            uint4 x[kFoldBatch];
#pragma unroll
            for (int j = 0; j < kFoldBatch; ++j)
                if (m0 + j < size) x[j] = src[static_cast<size_t>(m0 + j) * d8];
#pragma unroll
            for (int j = 0; j < kFoldBatch; ++j) {
                if (m0 + j < size) {
                    const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&x[j]);
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float2 f = __bfloat1622float2(h[e]);
                        acc[2 * e] = m0 + j == 0 ? f.x : __fadd_rn(acc[2 * e], f.x);
                        acc[2 * e + 1] = m0 + j == 0 ? f.y : __fadd_rn(acc[2 * e + 1], f.y);
                    }
                }
            }
        }
        uint4 r;
        uint32_t *rw = reinterpret_cast<uint32_t *>(&r);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const float lo = pow2 ? acc[2 * e] * inv : __fdiv_rn(acc[2 * e], divisor);
            const float hi = pow2 ? acc[2 * e + 1] * inv : __fdiv_rn(acc[2 * e + 1], divisor);
            __nv_bfloat162 pr = __floats2bfloat162_rn(lo, hi);
            rw[e] = *reinterpret_cast<uint32_t *>(&pr);
        }
        out[t] = r;
    }
}

int launch_fold_kv(const void *in, void *out, int B, int T, int H, int g, int d,
                   cudaStream_t stream) {
    const int d8 = d / 8;
    const size_t n_vec = static_cast<size_t>(B) * T * g * d8;
    // one output vector per thread (the loop in the kernel covers larger inputs)
    size_t blocks = (n_vec + 255) / 256;
    if (blocks > 0x7fffffffull) blocks = 0x7fffffffull;
    const uint4 *src = static_cast<const uint4 *>(in);
    uint4 *dst = static_cast<uint4 *>(out);
    const unsigned nb = static_cast<unsigned>(blocks);
    if (n_vec + static_cast<size_t>(blocks) * 256 <= 0xffffffffull) {
        const uint32_t n32 = static_cast<uint32_t>(n_vec);
        if (d8 == 16)
            fold_kv_kernel<uint32_t, 16><<<nb, 256, 0, stream>>>(src, dst, n32, H, g, d8);
        else if (d8 == 8)
            fold_kv_kernel<uint32_t, 8><<<nb, 256, 0, stream>>>(src, dst, n32, H, g, d8);
        else
            fold_kv_kernel<uint32_t, 0><<<nb, 256, 0, stream>>>(src, dst, n32, H, g, d8);
    } else {
        fold_kv_kernel<size_t, 0><<<nb, 256, 0, stream>>>(src, dst, n_vec, H, g, d8);
    }
    return check_cuda(cudaGetLastError(), "fold_kv_kernel launch");
}

// One warp waits on a barrier that nothing arrives at; the bounded wait must
// give up after limit_ns and record GQA_ERR_TIMEOUT in *status.
__global__ void selftest_wait_kernel(uint64_t limit_ns, int *status) {
    __shared__ uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        abort_flag = 0;
        fence_mbar_init();
    }
    __syncwarp();
    mbar_wait(&bar, 0, &abort_flag, status, limit_ns);
}

// Launches the self-test and waits for it.  The caller reads the status word.
int selftest_wait_timeout(int timeout_us) {
    int *status = device_status_ptr();
    if (!status) return GQA_ERR_CUDA;
    if (int rc = check_cuda(cudaMemset(status, 0, sizeof(int)), "cudaMemset")) return rc;
    selftest_wait_kernel<<<1, 32>>>(static_cast<uint64_t>(timeout_us) * 1000ull, status);
    if (int rc = check_cuda(cudaGetLastError(), "selftest_wait_kernel launch")) return rc;
    return check_cuda(cudaDeviceSynchronize(), "selftest sync");
}

}  // namespace gqa
