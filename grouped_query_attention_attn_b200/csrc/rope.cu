// rope.cu -- rotary position embedding of q and k, in place, bf16.
//
// Course "Неделя 7. Внимание", step 3: coordinate pair (2i, 2i+1) of the row at
// position m is rotated by the angle m * theta_i, theta_i = theta^(-2i/d); only q
// and k rotate.  HBM-bound (one read and one write of each element), so the
// arithmetic is arranged to stay far below the memory time:
//   * thread (c8, slot) of a block owns 16-byte column c8 (pairs 4 c8 .. 4 c8 + 3)
//     of up to kRopeBatch head rows of one token (a batch: q's heads, then k's,
//     in groups of kRopeBatch), computes those four sine / cosine pairs and
//     applies them to that column of every row of the batch;
//   * the angle and the rotation are device.cuh's rope_cos_sin and
//     rope_rotate_pair (turns reduced in double, fp32 sine / cosine), shared
//     with the attention kernels that rotate q as they load it;
//   * all loads of a batch are issued before any store, and the batches of a
//     token are spread over threads so that enough loads are in flight;
//   * a thread issues its loads first, and the block builds its table of
//     double-precision turns while they fly (12 % faster than building the
//     table first; 79 registers, 3 blocks per SM -- capped at 64 registers it
//     spills and loses the gain).
#include <cuda_bf16.h>

#include "device.cuh"
#include "internal.h"

namespace gqa {

constexpr int kRopeMaxHalf = 128;    // d <= 256
constexpr int kRopeThreads = 256;
constexpr int kRopeBatch = 8;

// x0 [n_tok, H0, d], x1 [n_tok, H1, d] (x1 may be absent, H1 = 0); token tok =
// b * T + t sits at position pos0 + t, or at max(seqlens[b] - 1, 0) when seqlens
// is given (decode queries, T = 1).  blockDim = (d8, slots): one batch of
// kRopeBatch head rows of one token per slot; a token has n_batch =
// ceil(H0 / kRopeBatch) + ceil(H1 / kRopeBatch) batches.
__global__ void __launch_bounds__(kRopeThreads)
rope_kernel(uint4 *__restrict__ x0, int H0, uint4 *__restrict__ x1, int H1, long long n_work,
            int n_batch, int T, int pos0, const int32_t *__restrict__ seqlens, double log_theta) {
    __shared__ double turns[kRopeMaxHalf];         // theta_i / (2 pi)
    const int d8 = blockDim.x, half = 4 * d8;
    const int tid = threadIdx.y * d8 + threadIdx.x;
    const long long w = static_cast<long long>(blockIdx.x) * blockDim.y + threadIdx.y;
    const bool active = w < n_work;
    const int c8 = threadIdx.x;
    // this thread's rows: loads issued before the block builds its angle table
    int tok = 0, n = 0;
    uint4 *row0 = nullptr;
    if (active) {
        tok = static_cast<int>(w / n_batch);
        const int bi = static_cast<int>(w % n_batch);
        const int b0 = (H0 + kRopeBatch - 1) / kRopeBatch;
        if (bi < b0) {
            const int h = bi * kRopeBatch;
            row0 = x0 + (static_cast<size_t>(tok) * H0 + h) * d8 + c8;
            n = min(kRopeBatch, H0 - h);
        } else {
            const int h = (bi - b0) * kRopeBatch;
            row0 = x1 + (static_cast<size_t>(tok) * H1 + h) * d8 + c8;
            n = min(kRopeBatch, H1 - h);
        }
    }
    uint4 v[kRopeBatch];
#pragma unroll
    for (int j = 0; j < kRopeBatch; ++j)
        if (j < n) v[j] = row0[static_cast<size_t>(j) * d8];
    for (int i = tid; i < half; i += d8 * blockDim.y) turns[i] = rope_turns(i, half, log_theta);
    __syncthreads();
    if (!active) return;
    const int b = tok / T;
    const int m = seqlens ? max(seqlens[b] - 1, 0) : pos0 + (tok - b * T);
    float cs[4], sn[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) rope_cos_sin(m, turns[c8 * 4 + e], cs[e], sn[e]);
#pragma unroll
    for (int j = 0; j < kRopeBatch; ++j) {
        if (j < n) {
            v[j].x = rope_rotate_pair(v[j].x, cs[0], sn[0]);
            v[j].y = rope_rotate_pair(v[j].y, cs[1], sn[1]);
            v[j].z = rope_rotate_pair(v[j].z, cs[2], sn[2]);
            v[j].w = rope_rotate_pair(v[j].w, cs[3], sn[3]);
            row0[static_cast<size_t>(j) * d8] = v[j];
        }
    }
}

static int launch_rope(void *x0, int H0, void *x1, int H1, int B, int T, int d, int pos0,
                       const int32_t *seqlens, float theta, cudaStream_t stream) {
    const int d8 = d / 8;
    const int slots = kRopeThreads / d8;
    const int n_batch = (H0 + kRopeBatch - 1) / kRopeBatch + (H1 + kRopeBatch - 1) / kRopeBatch;
    const long long n_work = static_cast<long long>(B) * T * n_batch;
    const long long blocks = (n_work + slots - 1) / slots;
    if (blocks > 0x7fffffffLL) return set_error(GQA_ERR_UNSUPPORTED, "rope grid too large");
    rope_kernel<<<static_cast<unsigned>(blocks), dim3(d8, slots), 0, stream>>>(
        static_cast<uint4 *>(x0), H0, static_cast<uint4 *>(x1), H1, n_work, n_batch, T, pos0,
        seqlens, log(static_cast<double>(theta)));
    return check_cuda(cudaGetLastError(), "rope_kernel launch");
}

static int check_rope_args(const void *x, const char *name, int B, int T, int H, int d,
                           float theta) {
    if (B < 0 || T < 0 || H < 1)
        return set_error(GQA_ERR_INVALID_ARG, "B=%d, T=%d must be >= 0 and %s heads=%d >= 1", B,
                         T, name, H);
    if (static_cast<long long>(B) * T > 0x7fffffffLL)
        return set_error(GQA_ERR_INVALID_ARG, "B*T=%lld tokens exceeds 2^31 - 1",
                         static_cast<long long>(B) * T);
    if (d < 8 || d % 8 != 0 || d > 2 * kRopeMaxHalf)
        return set_error(GQA_ERR_INVALID_ARG, "head dim d=%d must be a multiple of 8 in [8, 256]",
                         d);
    if (!(theta > 0.0f) || !isfinite(theta))
        return set_error(GQA_ERR_INVALID_ARG, "theta=%g must be finite and > 0", (double)theta);
    if (B > 0 && T > 0) {
        if (!x) return set_error(GQA_ERR_INVALID_ARG, "%s is NULL", name);
        if (reinterpret_cast<uintptr_t>(x) % 16)
            return set_error(GQA_ERR_INVALID_ARG, "%s is not 16-byte aligned", name);
    }
    return GQA_OK;
}

}  // namespace gqa

using namespace gqa;

extern "C" int gqa_rope(void *x, int B, int T, int H, int d, int pos0, float theta,
                        gqa_stream_t stream) {
    clear_error();
    if (int rc = check_rope_args(x, "x", B, T, H, d, theta)) return rc;
    if (B == 0 || T == 0) return GQA_OK;
    if (int rc = require_sm100()) return rc;
    return launch_rope(x, H, nullptr, 0, B, T, d, pos0, nullptr, theta,
                       reinterpret_cast<cudaStream_t>(stream));
}

extern "C" int gqa_rope_qk(void *q, void *k, int B, int T, int Hq, int Hkv, int d, int pos0,
                           float theta, gqa_stream_t stream) {
    clear_error();
    if (int rc = check_rope_args(q, "q", B, T, Hq, d, theta)) return rc;
    if (int rc = check_rope_args(k, "k", B, T, Hkv, d, theta)) return rc;
    if (B == 0 || T == 0) return GQA_OK;
    if (q == k) return set_error(GQA_ERR_INVALID_ARG, "q and k are the same buffer");
    if (int rc = require_sm100()) return rc;
    return launch_rope(q, Hq, k, Hkv, B, T, d, pos0, nullptr, theta,
                       reinterpret_cast<cudaStream_t>(stream));
}

extern "C" int gqa_rope_decode_q(void *q, const int32_t *seqlens, int B, int H, int d, float theta,
                                 gqa_stream_t stream) {
    clear_error();
    if (int rc = check_rope_args(q, "q", B, 1, H, d, theta)) return rc;
    if (B == 0) return GQA_OK;
    if (!seqlens || reinterpret_cast<uintptr_t>(seqlens) % 4)
        return set_error(GQA_ERR_INVALID_ARG, "seqlens is NULL or misaligned");
    if (int rc = require_sm100()) return rc;
    return launch_rope(q, H, nullptr, 0, B, 1, d, 0, seqlens, theta,
                       reinterpret_cast<cudaStream_t>(stream));
}
