// decode_static.cu -- gqa_decode_static: the decode entry point for callers
// that cannot allocate device memory.
//
// Some callers cannot call cudaMalloc at the point where they decode: code
// running inside a memory pool or arena that owns all device memory, plugins
// of runtimes that forbid allocation on their hot path, or code that must not
// synchronise the device (cudaMalloc/cudaFree can).  gqa_decode needs scratch
// for the partial outputs of its KV splits; this entry point uses a scratch
// array built into the library instead of a caller workspace.
//
// The scratch is a file-scope __device__ array of kStaticScratchBytes.  Every
// GPU that loads this code holds it until the process exits.  In host code the
// array's name is only a host-side stand-in, so its device address is looked
// up with cudaGetSymbolAddress once per device (on the first call made with
// that device current) and that address is what the kernels receive.
#include <mutex>

#include "internal.h"

namespace gqa {

// Built-in decode scratch: 32 MiB, enough for B=64, Hq=32, d=128, Lmax=8192.
constexpr size_t kStaticScratchBytes = 32u << 20;

static __device__ __align__(256) unsigned char g_decode_scratch[kStaticScratchBytes];

// Device address of g_decode_scratch on the current device, looked up once per
// device; nullptr (message set) on failure.
static void *static_scratch_ptr() {
    static void *cache[64] = {};
    static std::mutex mu;
    int dev = 0;
    if (int rc = check_cuda(cudaGetDevice(&dev), "cudaGetDevice")) {
        (void)rc;
        return nullptr;
    }
    if (dev < 0 || dev >= 64) {
        set_error(GQA_ERR_UNSUPPORTED, "gqa_decode_static: device ordinal %d >= 64", dev);
        return nullptr;
    }
    std::lock_guard<std::mutex> lock(mu);
    if (!cache[dev]) {
        void *ptr = nullptr;
        if (check_cuda(cudaGetSymbolAddress(&ptr, g_decode_scratch),
                       "gqa_decode_static: cudaGetSymbolAddress"))
            return nullptr;
        cache[dev] = ptr;
    }
    return cache[dev];
}

}  // namespace gqa

extern "C" int gqa_decode_static(const void *q, const void *k_cache, const void *v_cache,
                                 const int32_t *seqlens, void *o, int B, int Hq, int Hkv, int d,
                                 int Lmax, float scale, gqa_stream_t stream) {
    using namespace gqa;
    // Sizes are checked before the scratch is touched, so an oversize request
    // fails cleanly (and nothing is launched).
    const size_t need = gqa_decode_workspace_size(B, Hq, Hkv, d, Lmax);
    if (need > kStaticScratchBytes)
        return set_error(GQA_ERR_WORKSPACE,
                         "gqa_decode_static: B=%d, Hq=%d, d=%d, Lmax=%d need %zu bytes of "
                         "scratch; the built-in scratch holds %zu (use gqa_decode with a "
                         "caller workspace)",
                         B, Hq, d, Lmax, need, kStaticScratchBytes);
    // No scratch needed (empty batch, empty cache) or invalid sizes: gqa_decode
    // validates and answers without touching any scratch.
    if (need == 0) return gqa_decode(q, k_cache, v_cache, seqlens, o, B, Hq, Hkv, d, Lmax, scale,
                                     nullptr, 0, stream);
    void *scratch = static_scratch_ptr();
    if (!scratch) return GQA_ERR_CUDA;
    // Nothing in the scratch has to start at zero: every partial result the
    // combine kernel reads is written earlier in the same call.
    return gqa_decode(q, k_cache, v_cache, seqlens, o, B, Hq, Hkv, d, Lmax, scale, scratch,
                      kStaticScratchBytes, stream);
}
