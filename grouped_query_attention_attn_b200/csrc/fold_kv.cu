// fold_kv.cu -- MHA -> GQA mean pooling of K or V heads, and the self-test
// kernel of the bounded device waits.
//
// fold: out[b, t, grp, :] = (sum over the contiguous group members, in head
// order, in fp32) / (H / g), rounded to bf16 -- the position-wise mean over
// heads[start:start+size] of TT Lab "キー・バリューヘッドだけ減らしてみる",
// step 2.  HBM-bound: each thread moves 16-byte vectors.
#include <cuda_bf16.h>

#include "device.cuh"
#include "internal.h"

namespace gqa {

__global__ void __launch_bounds__(256)
fold_kv_kernel(const uint4 *__restrict__ in, uint4 *__restrict__ out, size_t n_vec, int H,
               int g, int d8) {
    const int size = H / g;
    const float divisor = static_cast<float>(size);
    const size_t stride = static_cast<size_t>(gridDim.x) * blockDim.x;
    for (size_t t = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; t < n_vec;
         t += stride) {
        const size_t c8 = t % d8;
        const size_t grp = (t / d8) % g;
        const size_t bt = t / (static_cast<size_t>(d8) * g);
        const uint4 *src = in + (bt * H + grp * size) * d8 + c8;
        float acc[8];
        {
            const uint4 x = src[0];
            const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&x);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float2 f = __bfloat1622float2(h[e]);
                acc[2 * e] = f.x;
                acc[2 * e + 1] = f.y;
            }
        }
        for (int m = 1; m < size; ++m) {
            const uint4 x = src[static_cast<size_t>(m) * d8];
            const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&x);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float2 f = __bfloat1622float2(h[e]);
                acc[2 * e] = __fadd_rn(acc[2 * e], f.x);
                acc[2 * e + 1] = __fadd_rn(acc[2 * e + 1], f.y);
            }
        }
        uint4 r;
        uint32_t *rw = reinterpret_cast<uint32_t *>(&r);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            __nv_bfloat162 pr = __floats2bfloat162_rn(__fdiv_rn(acc[2 * e], divisor),
                                                      __fdiv_rn(acc[2 * e + 1], divisor));
            rw[e] = *reinterpret_cast<uint32_t *>(&pr);
        }
        out[t] = r;
    }
}

int launch_fold_kv(const void *in, void *out, int B, int T, int H, int g, int d,
                   cudaStream_t stream) {
    const int d8 = d / 8;
    const size_t n_vec = static_cast<size_t>(B) * T * g * d8;
    int blocks = static_cast<int>((n_vec + 255) / 256);
    if (blocks > 148 * 16) blocks = 148 * 16;
    fold_kv_kernel<<<blocks, 256, 0, stream>>>(static_cast<const uint4 *>(in),
                                               static_cast<uint4 *>(out), n_vec, H, g, d8);
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
