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
// up with cudaGetSymbolAddress and that address is what the kernels receive.
// The lookup runs on the first call made in a CUDA context (the first call on
// each device, and again after a cudaDeviceReset, which loads the module anew)
// and is cached for that context.
#include "internal.h"

namespace gqa {

// Built-in decode scratch: 32 MiB, enough for B=64, Hq=32, d=128, Lmax=8192.
constexpr size_t kStaticScratchBytes = 32u << 20;

static __device__ __align__(256) unsigned char g_decode_scratch[kStaticScratchBytes];

// Device address of g_decode_scratch in the current context; nullptr (message
// set) on failure.
static void *static_scratch_ptr() {
    static SymbolSlot slot;
    return symbol_address(reinterpret_cast<const void *>(&g_decode_scratch), slot,
                          "gqa_decode_static: cudaGetSymbolAddress");
}

}  // namespace gqa

extern "C" int gqa_decode_static(const void *q, const void *k_cache, const void *v_cache,
                                 const int32_t *seqlens, void *o, int B, int Hq, int Hkv, int d,
                                 int Lmax, float scale, gqa_stream_t stream) {
    using namespace gqa;
    clear_error();
    // The same argument checks and errors as gqa_decode, before anything else.
    if (int rc = validate_decode(q, k_cache, v_cache, seqlens, o, B, Hq, Hkv, d, Lmax, scale))
        return rc;
    // Then the size check, before the scratch is touched: an oversize request
    // fails cleanly and nothing is launched.
    const size_t need = decode_workspace_bytes(B, Hq, Hkv, d, Lmax);
    if (need > kStaticScratchBytes)
        return set_error(GQA_ERR_WORKSPACE,
                         "gqa_decode_static: B=%d, Hq=%d, d=%d, Lmax=%d need %zu bytes of "
                         "scratch; the built-in scratch holds %zu (use gqa_decode with a "
                         "caller workspace)",
                         B, Hq, d, Lmax, need, kStaticScratchBytes);
    if (B == 0) return GQA_OK;
    if (int rc = require_sm100()) return rc;
    void *scratch = nullptr;
    if (need > 0) {
        scratch = static_scratch_ptr();
        if (!scratch) return GQA_ERR_CUDA;
    }
    // Nothing in the scratch has to start at zero: every partial result the
    // merge reads is written earlier in the same call.
    return launch_decode(q, k_cache, v_cache, seqlens, o, B, Hq, Hkv, d, Lmax, 0, 0, scale,
                         scratch, reinterpret_cast<cudaStream_t>(stream));
}
