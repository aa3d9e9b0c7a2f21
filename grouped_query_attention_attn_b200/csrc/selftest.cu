// selftest.cu -- device self-test of a numerical building block of the
// kernels: the FMA-pipe 2^x polynomial (exp2_poly2 in device.cuh) that the
// prefill softmax uses for part of its exponentials.  The test evaluates it
// on caller-chosen points so its error can be checked against 2^x in double.
#include "device.cuh"
#include "internal.h"

namespace gqa {

__global__ void __launch_bounds__(256) exp2_poly_kernel(const float *__restrict__ x,
                                                        float *__restrict__ y, int n_pairs) {
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= n_pairs) return;
    const float2 r = exp2_poly2(make_float2(x[2 * i], x[2 * i + 1]));
    y[2 * i] = r.x;
    y[2 * i + 1] = r.y;
}

}  // namespace gqa

extern "C" int gqa_selftest_exp2_poly(const float *x, float *y, int n, gqa_stream_t stream) {
    using namespace gqa;
    clear_error();
    if (n < 0 || n % 2 != 0)
        return set_error(GQA_ERR_INVALID_ARG, "n=%d must be even and >= 0 (points go in pairs)", n);
    if (n == 0) return GQA_OK;
    if (!x || !y) return set_error(GQA_ERR_INVALID_ARG, "x or y is NULL");
    if (reinterpret_cast<uintptr_t>(x) % 4 || reinterpret_cast<uintptr_t>(y) % 4)
        return set_error(GQA_ERR_INVALID_ARG, "x and y must be 4-byte aligned");
    if (int rc = require_sm100()) return rc;
    const int pairs = n / 2;
    exp2_poly_kernel<<<(pairs + 255) / 256, 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
        x, y, pairs);
    return check_cuda(cudaGetLastError(), "exp2_poly_kernel launch");
}
