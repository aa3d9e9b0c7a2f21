// gqa_api.cu -- the extern "C" boundary: argument validation, error
// reporting, device status, tensor-map encoding and dispatch to the kernels.
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>

#include "device.cuh"
#include "internal.h"

namespace gqa {

// First error any kernel of the library recorded on this device (GQA_OK when none).
__device__ int g_device_status = 0;

using CtxGetCurrentFn = CUresult (*)(CUcontext *);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long *);

template <class Fn>
static Fn driver_fn(const char *name) {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint(name, &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
        return reinterpret_cast<Fn>(p);
    return nullptr;
}

int current_ctx_key(int *dev, unsigned long long *ctx_id) {
    static CtxGetCurrentFn get_current = nullptr;
    static CtxGetIdFn get_id = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        get_current = driver_fn<CtxGetCurrentFn>("cuCtxGetCurrent");
        get_id = driver_fn<CtxGetIdFn>("cuCtxGetId");
    });
    if (int rc = check_cuda(cudaGetDevice(dev), "cudaGetDevice")) return rc;
    if (*dev < 0 || *dev >= kMaxDevices)
        return set_error(GQA_ERR_UNSUPPORTED, "device ordinal %d >= %d", *dev, kMaxDevices);
    *ctx_id = 0;
    if (!get_current || !get_id) return GQA_OK;
    CUcontext ctx = nullptr;
    if (get_current(&ctx) == CUDA_SUCCESS && !ctx) {
        // no context yet (first call, or after cudaDeviceReset): cudaSetDevice
        // makes the device's primary context current
        if (int rc = check_cuda(cudaSetDevice(*dev), "cudaSetDevice")) return rc;
        get_current(&ctx);
    }
    unsigned long long id = 0;
    if (ctx && get_id(ctx, &id) == CUDA_SUCCESS) *ctx_id = id;
    return GQA_OK;
}

void *symbol_address(const void *symbol, SymbolSlot &slot, const char *what) {
    int dev = 0;
    unsigned long long id = 0;
    if (current_ctx_key(&dev, &id)) return nullptr;
    std::lock_guard<std::mutex> lock(slot.ctx.mu);
    if (id != 0 && slot.ctx.ctx_id[dev] == id && slot.addr[dev]) return slot.addr[dev];
    void *p = nullptr;
    if (check_cuda(cudaGetSymbolAddress(&p, symbol), what)) return nullptr;
    // the lookup may have made the primary context current: key on it
    int dev2 = 0;
    unsigned long long id2 = 0;
    const bool keyed = current_ctx_key(&dev2, &id2) == GQA_OK && dev2 == dev;
    slot.ctx.ctx_id[dev] = keyed ? id2 : 0;
    slot.addr[dev] = p;
    return p;
}

int *device_status_ptr() {
    static SymbolSlot slot;
    return static_cast<int *>(symbol_address(reinterpret_cast<const void *>(&g_device_status),
                                             slot, "cudaGetSymbolAddress(status)"));
}

static thread_local char t_last_error[512] = "";

int set_error(int code, const char *fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(t_last_error, sizeof(t_last_error), fmt, ap);
    va_end(ap);
    return code;
}

void clear_error() { t_last_error[0] = 0; }

int check_cuda(cudaError_t e, const char *what) {
    if (e == cudaSuccess) return GQA_OK;
    return set_error(GQA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

int require_sm100() {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return check_cuda(e, "cudaGetDevice");
    int major = 0, minor = 0;
    cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
    cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
    if (major != 10 || minor != 0)
        return set_error(GQA_ERR_UNSUPPORTED,
                         "device %d is sm_%d%d; this library is built for sm_100a only", dev,
                         major, minor);
    return GQA_OK;
}

int sm_count(int *n) {
    static int cache[64] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return check_cuda(e, "cudaGetDevice");
    if (dev < 0 || dev >= 64) return set_error(GQA_ERR_UNSUPPORTED, "device index %d", dev);
    if (!cache[dev]) {
        int v = 0;
        if (int rc = check_cuda(cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev),
                                "cudaDeviceGetAttribute(SM count)"))
            return rc;
        cache[dev] = v;
    }
    *n = cache[dev];
    return GQA_OK;
}

using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                   const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                   const cuuint32_t *, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion,
                                   CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

int encode_tmap_bf16_4d(CUtensorMap *map, const void *base, uint64_t n0, uint64_t n1,
                        uint64_t n2, uint64_t n3, uint32_t b0, uint32_t b1, uint32_t b2,
                        uint32_t b3, int swizzle128, uint64_t n2_pitch) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return set_error(GQA_ERR_CUDA, "cuTensorMapEncodeTiled is not available");
    cuuint64_t dims[4] = {n0, n1, n2, n3};
    cuuint64_t strides[3] = {n0 * 2, n0 * n1 * 2, n0 * n1 * (n2_pitch ? n2_pitch : n2) * 2};
    cuuint32_t box[4] = {b0, b1, b2, b3};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(base), dims,
                    strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                    swizzle128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS)
        return set_error(GQA_ERR_CUDA,
                         "cuTensorMapEncodeTiled failed (%d) for dims %llu x %llu x %llu x %llu",
                         (int)r, (unsigned long long)n0, (unsigned long long)n1,
                         (unsigned long long)n2, (unsigned long long)n3);
    return GQA_OK;
}

// ------------------------------------------------------------ validation --
static bool aligned(const void *p, size_t a) {
    return (reinterpret_cast<uintptr_t>(p) % a) == 0;
}

static int check_heads(int Hq, int Hkv, int d) {
    if (Hq < 1 || Hkv < 1) return set_error(GQA_ERR_INVALID_ARG, "Hq=%d, Hkv=%d must be >= 1", Hq, Hkv);
    if (Hq % Hkv != 0)
        return set_error(GQA_ERR_INVALID_ARG,
                         "Hq=%d query heads do not split evenly into Hkv=%d groups", Hq, Hkv);
    if (d < 1) return set_error(GQA_ERR_INVALID_ARG, "head dim d=%d must be >= 1", d);
    return GQA_OK;
}

static int check_scale(float scale) {
    if (!(scale > 0.0f) || !std::isfinite(scale))
        return set_error(GQA_ERR_INVALID_ARG, "scale=%g must be finite and > 0", (double)scale);
    return GQA_OK;
}

static int check_ptr(const void *p, size_t align, const char *name) {
    if (!p) return set_error(GQA_ERR_INVALID_ARG, "%s is NULL", name);
    if (!aligned(p, align))
        return set_error(GQA_ERR_INVALID_ARG, "%s is not %zu-byte aligned", name, align);
    return GQA_OK;
}

static int check_fwd_common(int B, int Tq, int Tkv, int Hq, int Hkv, int d, int causal,
                            float scale) {
    if (B < 0 || Tq < 0 || Tkv < 0)
        return set_error(GQA_ERR_INVALID_ARG, "B=%d, Tq=%d, Tkv=%d must be >= 0", B, Tq, Tkv);
    if (int rc = check_heads(Hq, Hkv, d)) return rc;
    if (causal != 0 && causal != 1)
        return set_error(GQA_ERR_INVALID_ARG, "causal=%d must be 0 or 1", causal);
    if (int rc = check_scale(scale)) return rc;
    // the element count of each tensor must fit the index arithmetic
    const double nq = (double)B * Tq * Hq * d, nk = (double)B * Tkv * Hkv * d;
    if (nq > 9.0e15 || nk > 9.0e15)
        return set_error(GQA_ERR_INVALID_ARG, "tensor too large");
    return GQA_OK;
}

}  // namespace gqa

using namespace gqa;

extern "C" {

const char *gqa_last_error(void) { return t_last_error; }

// Shared by the plain and the sliding-window forward (window = 0: none).
static int attn_fwd_bf16(const void *q, const void *k, const void *v, void *o, float *lse,
                         int B, int Tq, int Tkv, int Hq, int Hkv, int d, int causal, int window,
                         int sinks, float scale, gqa_stream_t stream, float rope_theta = 0.0f,
                         int q_pos0 = 0) {
    if (int rc = check_fwd_common(B, Tq, Tkv, Hq, Hkv, d, causal, scale)) return rc;
    if (d != 64 && d != 128)
        return set_error(GQA_ERR_UNSUPPORTED, "head dim d=%d: the bf16 path supports 64 and 128", d);
    if (Hq / Hkv > 128)
        return set_error(GQA_ERR_UNSUPPORTED, "group size Hq/Hkv=%d exceeds 128", Hq / Hkv);
    if (B == 0 || Tq == 0) return GQA_OK;
    if (int rc = check_ptr(q, 16, "q")) return rc;
    if (int rc = check_ptr(o, 16, "o")) return rc;
    if (lse && !aligned(lse, 4)) return set_error(GQA_ERR_INVALID_ARG, "lse is not 4-byte aligned");
    if (int rc = require_sm100()) return rc;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (Tkv == 0) return launch_empty_rows(o, lse, 2, B, Tq, Hq, d, s);
    if (int rc = check_ptr(k, 16, "k")) return rc;
    if (int rc = check_ptr(v, 16, "v")) return rc;
    return launch_prefill(q, k, v, o, lse, B, Tq, Tkv, Hq, Hkv, d, causal, window, sinks, scale,
                          s, 0, 0, rope_theta, q_pos0);
}

static int check_theta(float theta) {
    if (!(theta > 0.0f) || !std::isfinite(theta))
        return set_error(GQA_ERR_INVALID_ARG, "theta=%g must be finite and > 0", (double)theta);
    return GQA_OK;
}

int gqa_attn_fwd_host(const void *q_host, const void *k_host, const void *v_host, void *o_host,
                      void *q_dev, void *k_dev, void *v_dev, void *o_dev, int B, int Tq, int Tkv,
                      int Hq, int Hkv, int d, int causal, float scale, gqa_stream_t stream,
                      void *done_event) {
    t_last_error[0] = 0;
    if (int rc = check_fwd_common(B, Tq, Tkv, Hq, Hkv, d, causal, scale)) return rc;
    if (d != 64 && d != 128)
        return set_error(GQA_ERR_UNSUPPORTED, "head dim d=%d: the bf16 path supports 64 and 128", d);
    if (Hq / Hkv > 128)
        return set_error(GQA_ERR_UNSUPPORTED, "group size Hq/Hkv=%d exceeds 128", Hq / Hkv);
    if (B == 0 || Tq == 0) return GQA_OK;
    if (int rc = check_ptr(q_host, 2, "q_host")) return rc;
    if (int rc = check_ptr(o_host, 2, "o_host")) return rc;
    if (int rc = check_ptr(q_dev, 16, "q_dev")) return rc;
    if (int rc = check_ptr(o_dev, 16, "o_dev")) return rc;
    if (Tkv > 0) {
        if (int rc = check_ptr(k_host, 2, "k_host")) return rc;
        if (int rc = check_ptr(v_host, 2, "v_host")) return rc;
        if (int rc = check_ptr(k_dev, 16, "k_dev")) return rc;
        if (int rc = check_ptr(v_dev, 16, "v_dev")) return rc;
    }
    if (int rc = require_sm100()) return rc;
    return launch_fwd_host_pipeline(q_host, k_host, v_host, o_host, q_dev, k_dev, v_dev, o_dev, B,
                                    Tq, Tkv, Hq, Hkv, d, causal, scale,
                                    reinterpret_cast<cudaStream_t>(stream),
                                    static_cast<cudaEvent_t>(done_event));
}

int gqa_attn_fwd_lse(const void *q, const void *k, const void *v, void *o, float *lse,
                     int B, int Tq, int Tkv, int Hq, int Hkv, int d, int causal, float scale,
                     gqa_stream_t stream) {
    t_last_error[0] = 0;
    return attn_fwd_bf16(q, k, v, o, lse, B, Tq, Tkv, Hq, Hkv, d, causal, 0, 0, scale, stream);
}

int gqa_attn_fwd_window(const void *q, const void *k, const void *v, void *o, float *lse,
                        int B, int Tq, int Tkv, int Hq, int Hkv, int d, int window, int sinks,
                        float scale, gqa_stream_t stream) {
    t_last_error[0] = 0;
    if (window < 1 || sinks < 0)
        return set_error(GQA_ERR_INVALID_ARG, "window=%d must be >= 1 and sinks=%d >= 0", window,
                         sinks);
    return attn_fwd_bf16(q, k, v, o, lse, B, Tq, Tkv, Hq, Hkv, d, 1, window, sinks, scale, stream);
}

int gqa_attn_fwd_rope(const void *q, const void *k, const void *v, void *o, float *lse, int B,
                      int Tq, int Tkv, int Hq, int Hkv, int d, int causal, float scale, int q_pos0,
                      float theta, gqa_stream_t stream) {
    t_last_error[0] = 0;
    if (int rc = check_theta(theta)) return rc;
    if (q_pos0 < 0 || static_cast<long long>(q_pos0) + Tq > 0x7fffffffLL)
        return set_error(GQA_ERR_INVALID_ARG, "q_pos0=%d must be >= 0 and q_pos0 + Tq fit an int",
                         q_pos0);
    return attn_fwd_bf16(q, k, v, o, lse, B, Tq, Tkv, Hq, Hkv, d, causal, 0, 0, scale, stream, theta,
                         q_pos0);
}

int gqa_attn_fwd(const void *q, const void *k, const void *v, void *o, int B, int Tq, int Tkv,
                 int Hq, int Hkv, int d, int causal, float scale, gqa_stream_t stream) {
    return gqa_attn_fwd_lse(q, k, v, o, nullptr, B, Tq, Tkv, Hq, Hkv, d, causal, scale, stream);
}

int gqa_attn_fwd_f32(const float *q, const float *k, const float *v, float *o, float *lse,
                     int B, int Tq, int Tkv, int Hq, int Hkv, int d, int causal, float scale,
                     gqa_stream_t stream) {
    t_last_error[0] = 0;
    if (int rc = check_fwd_common(B, Tq, Tkv, Hq, Hkv, d, causal, scale)) return rc;
    if (d > 256) return set_error(GQA_ERR_UNSUPPORTED, "head dim d=%d: the fp32 path supports d <= 256", d);
    if (B == 0 || Tq == 0) return GQA_OK;
    if (int rc = check_ptr(q, 4, "q")) return rc;
    if (int rc = check_ptr(o, 4, "o")) return rc;
    if (lse && !aligned(lse, 4)) return set_error(GQA_ERR_INVALID_ARG, "lse is not 4-byte aligned");
    if (int rc = require_sm100()) return rc;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (Tkv == 0) return launch_empty_rows(o, lse, 4, B, Tq, Hq, d, s);
    if (int rc = check_ptr(k, 4, "k")) return rc;
    if (int rc = check_ptr(v, 4, "v")) return rc;
    return launch_fwd_f32(q, k, v, o, lse, B, Tq, Tkv, Hq, Hkv, d, causal, scale, s);
}

size_t gqa_decode_workspace_size(int B, int Hq, int Hkv, int d, int Lmax) {
    if (B < 0 || Lmax < 0 || Hq < 1 || Hkv < 1 || Hq % Hkv != 0 || d < 1) return 0;
    return decode_workspace_bytes(B, Hq, Hkv, d, Lmax);
}

} // extern "C"

namespace gqa {

int validate_decode(const void *q, const void *k_cache, const void *v_cache,
                    const int32_t *seqlens, const void *o, int B, int Hq, int Hkv, int d,
                    int Lmax, float scale) {
    if (B < 0 || Lmax < 0) return set_error(GQA_ERR_INVALID_ARG, "B=%d, Lmax=%d must be >= 0", B, Lmax);
    if (int rc = check_heads(Hq, Hkv, d)) return rc;
    if (int rc = check_scale(scale)) return rc;
    if (d != 64 && d != 128)
        return set_error(GQA_ERR_UNSUPPORTED, "head dim d=%d: decode supports 64 and 128", d);
    if (Hq / Hkv > 32)
        return set_error(GQA_ERR_UNSUPPORTED, "decode group size Hq/Hkv=%d exceeds 32", Hq / Hkv);
    if ((double)B * Lmax * Hkv * d > 9.0e15) return set_error(GQA_ERR_INVALID_ARG, "cache too large");
    if (B == 0) return GQA_OK;
    if (int rc = check_ptr(q, 16, "q")) return rc;
    if (int rc = check_ptr(o, 16, "o")) return rc;
    if (int rc = check_ptr(seqlens, 4, "seqlens")) return rc;
    if (Lmax > 0) {
        if (int rc = check_ptr(k_cache, 16, "k_cache")) return rc;
        if (int rc = check_ptr(v_cache, 16, "v_cache")) return rc;
    }
    return GQA_OK;
}

}  // namespace gqa

extern "C" {

static int decode_bf16(const void *q, const void *k_cache, const void *v_cache,
                       const int32_t *seqlens, void *o, int B, int Hq, int Hkv, int d, int Lmax,
                       int window, int sinks, float scale, void *workspace,
                       size_t workspace_bytes, gqa_stream_t stream, float rope_theta = 0.0f) {
    if (int rc = validate_decode(q, k_cache, v_cache, seqlens, o, B, Hq, Hkv, d, Lmax, scale))
        return rc;
    if (B == 0) return GQA_OK;
    const size_t need = decode_workspace_bytes(B, Hq, Hkv, d, Lmax);
    if (need > 0) {
        if (!workspace) return set_error(GQA_ERR_WORKSPACE, "workspace is NULL (%zu bytes needed)", need);
        if (!aligned(workspace, 256))
            return set_error(GQA_ERR_WORKSPACE, "workspace is not 256-byte aligned");
        if (workspace_bytes < need)
            return set_error(GQA_ERR_WORKSPACE, "workspace has %zu bytes, %zu needed",
                             workspace_bytes, need);
    }
    if (int rc = require_sm100()) return rc;
    return launch_decode(q, k_cache, v_cache, seqlens, o, B, Hq, Hkv, d, Lmax, window, sinks,
                         scale, workspace, reinterpret_cast<cudaStream_t>(stream), rope_theta);
}

int gqa_decode(const void *q, const void *k_cache, const void *v_cache, const int32_t *seqlens,
               void *o, int B, int Hq, int Hkv, int d, int Lmax, float scale, void *workspace,
               size_t workspace_bytes, gqa_stream_t stream) {
    t_last_error[0] = 0;
    return decode_bf16(q, k_cache, v_cache, seqlens, o, B, Hq, Hkv, d, Lmax, 0, 0, scale,
                       workspace, workspace_bytes, stream);
}

int gqa_decode_rope(const void *q, const void *k_cache, const void *v_cache,
                    const int32_t *seqlens, void *o, int B, int Hq, int Hkv, int d, int Lmax,
                    float scale, float theta, void *workspace, size_t workspace_bytes,
                    gqa_stream_t stream) {
    t_last_error[0] = 0;
    if (int rc = check_theta(theta)) return rc;
    return decode_bf16(q, k_cache, v_cache, seqlens, o, B, Hq, Hkv, d, Lmax, 0, 0, scale,
                       workspace, workspace_bytes, stream, theta);
}

int gqa_decode_window(const void *q, const void *k_cache, const void *v_cache,
                      const int32_t *seqlens, void *o, int B, int Hq, int Hkv, int d, int Lmax,
                      int window, int sinks, float scale, void *workspace,
                      size_t workspace_bytes, gqa_stream_t stream) {
    t_last_error[0] = 0;
    if (window < 1 || sinks < 0)
        return set_error(GQA_ERR_INVALID_ARG, "window=%d must be >= 1 and sinks=%d >= 0", window,
                         sinks);
    return decode_bf16(q, k_cache, v_cache, seqlens, o, B, Hq, Hkv, d, Lmax, window, sinks, scale,
                       workspace, workspace_bytes, stream);
}

size_t gqa_attn_bwd_workspace_size(int B, int Tq, int Hq) {
    if (B < 0 || Tq < 0 || Hq < 1) return 0;
    return bwd_workspace_bytes(B, Tq, Hq);
}

int gqa_attn_bwd(const void *q, const void *k, const void *v, const void *o, const void *dout,
                 const float *lse, void *dq, void *dk, void *dv, int B, int Tq, int Tkv, int Hq,
                 int Hkv, int d, int causal, int window, int sinks, float scale, void *workspace,
                 size_t workspace_bytes, gqa_stream_t stream) {
    t_last_error[0] = 0;
    if (int rc = check_fwd_common(B, Tq, Tkv, Hq, Hkv, d, causal, scale)) return rc;
    if (d != 64 && d != 128)
        return set_error(GQA_ERR_UNSUPPORTED, "head dim d=%d: the backward supports 64 and 128", d);
    if (window < 0 || sinks < 0 || (window > 0 && !causal))
        return set_error(GQA_ERR_INVALID_ARG,
                         "window=%d, sinks=%d must be >= 0 (a window needs causal=1)", window, sinks);
    if (B == 0 || (Tq == 0 && Tkv == 0)) return GQA_OK;
    // query-side tensors are needed when Tq > 0, key-side ones when Tkv > 0
    const struct { const void *p; const char *n; bool kv_side; } ptrs[] = {
        {q, "q", false}, {o, "o", false}, {dout, "dout", false}, {dq, "dq", false},
        {k, "k", true},  {v, "v", true},  {dk, "dk", true},      {dv, "dv", true}};
    for (const auto &e : ptrs)
        if (e.kv_side ? Tkv > 0 : Tq > 0)
            if (int rc = check_ptr(e.p, 16, e.n)) return rc;
    if (Tq > 0 && !lse) return set_error(GQA_ERR_INVALID_ARG, "lse is NULL");
    if (lse && !aligned(lse, 4)) return set_error(GQA_ERR_INVALID_ARG, "lse is not 4-byte aligned");
    const size_t need = bwd_workspace_bytes(B, Tq, Hq);
    if (need > 0) {
        if (!workspace) return set_error(GQA_ERR_WORKSPACE, "workspace is NULL (%zu bytes needed)", need);
        if (!aligned(workspace, 256))
            return set_error(GQA_ERR_WORKSPACE, "workspace is not 256-byte aligned");
        if (workspace_bytes < need)
            return set_error(GQA_ERR_WORKSPACE, "workspace has %zu bytes, %zu needed",
                             workspace_bytes, need);
    }
    if (int rc = require_sm100()) return rc;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (Tq == 0) {
        // no query sees any key: the K / V gradients are zero
        const size_t bytes = static_cast<size_t>(B) * Tkv * Hkv * d * 2;
        if (int rc = check_cuda(cudaMemsetAsync(dk, 0, bytes, s), "cudaMemsetAsync(dk)")) return rc;
        return check_cuda(cudaMemsetAsync(dv, 0, bytes, s), "cudaMemsetAsync(dv)");
    }
    return launch_bwd(q, k, v, o, dout, lse, dq, dk, dv, B, Tq, Tkv, Hq, Hkv, d, causal, window,
                      sinks, scale, workspace, s);
}

int gqa_fold_kv(const void *in, void *out, int B, int T, int H, int g, int d,
                gqa_stream_t stream) {
    t_last_error[0] = 0;
    if (B < 0 || T < 0) return set_error(GQA_ERR_INVALID_ARG, "B=%d, T=%d must be >= 0", B, T);
    if (H < 1 || g < 1 || H % g != 0)
        return set_error(GQA_ERR_INVALID_ARG, "%d groups do not divide %d heads evenly", g, H);
    if (d < 8 || d % 8 != 0)
        return set_error(GQA_ERR_INVALID_ARG, "head dim d=%d must be a positive multiple of 8", d);
    if (B == 0 || T == 0) return GQA_OK;
    if (int rc = check_ptr(in, 16, "in")) return rc;
    if (int rc = check_ptr(out, 16, "out")) return rc;
    if (int rc = require_sm100()) return rc;
    return launch_fold_kv(in, out, B, T, H, g, d, reinterpret_cast<cudaStream_t>(stream));
}

int gqa_device_status(int reset) {
    t_last_error[0] = 0;
    if (int rc = check_cuda(cudaDeviceSynchronize(), "cudaDeviceSynchronize")) return rc;
    int status = 0;
    if (int rc = check_cuda(cudaMemcpyFromSymbol(&status, g_device_status, sizeof(int)),
                            "cudaMemcpyFromSymbol"))
        return rc;
    if (reset) {
        const int zero = 0;
        if (int rc = check_cuda(cudaMemcpyToSymbol(g_device_status, &zero, sizeof(int)),
                                "cudaMemcpyToSymbol"))
            return rc;
    }
    if (status == GQA_ERR_TIMEOUT)
        return set_error(GQA_ERR_TIMEOUT, "a bounded device wait timed out");
    if (status != 0) return set_error(status, "a kernel recorded status %d", status);
    return GQA_OK;
}

void gqa_set_prefill_grid_cap(int max_ctas) { set_prefill_grid_cap(max_ctas); }

int gqa_selftest_wait_timeout(int timeout_us) {
    t_last_error[0] = 0;
    if (timeout_us < 1 || timeout_us > 10 * 1000 * 1000)
        return set_error(GQA_ERR_INVALID_ARG, "timeout_us=%d must be in [1, 1e7]", timeout_us);
    if (int rc = require_sm100()) return rc;
    if (int rc = selftest_wait_timeout(timeout_us)) {
        if (rc != GQA_ERR_TIMEOUT) return rc;
    }
    // the kernel recorded GQA_ERR_TIMEOUT in the status word: report and clear it
    return gqa_device_status(1);
}

}  // extern "C"
