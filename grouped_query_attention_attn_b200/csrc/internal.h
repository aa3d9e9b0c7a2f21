// internal.h -- declarations shared by the library's translation units.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <cstddef>
#include <cstdint>
#include <mutex>

#include "gqa.h"

namespace gqa {

// Record a message for gqa_last_error() on this host thread; returns `code`.
int set_error(int code, const char *fmt, ...);

// Clear that message (every entry point starts with it).
void clear_error();

// Map a CUDA runtime error to GQA_ERR_CUDA with a message; GQA_OK on success.
int check_cuda(cudaError_t e, const char *what);

// GQA_OK when the current device is an sm_100 part, else GQA_ERR_UNSUPPORTED.
int require_sm100();
// Number of SMs of the current device (cached per device).
int sm_count(int *n);

// ---- per-context host caches ---------------------------------------------
// A device address of a __device__ variable, or an attribute set on a kernel,
// belongs to one CUDA context: after cudaDeviceReset (or with another context
// current) the module is loaded again, possibly elsewhere.  Caches are
// therefore keyed on the current context's unique id (cuCtxGetId), not on
// the device ordinal alone.
constexpr int kMaxDevices = 64;

// Device ordinal and unique id of the context current on this host thread
// (id 0: no context is current yet, or the driver cannot say).
int current_ctx_key(int *dev, unsigned long long *ctx_id);

// Remembers, per device, the context for which an initialisation ran.
struct CtxSlot {
    std::mutex mu;
    unsigned long long ctx_id[kMaxDevices] = {};
};

// Runs init(dev) unless it already succeeded for the current context;
// returns GQA_OK or init's error (nothing recorded then).
template <class F>
int once_per_context(CtxSlot &slot, F &&init) {
    int dev = 0;
    unsigned long long id = 0;
    if (int rc = current_ctx_key(&dev, &id)) return rc;
    std::lock_guard<std::mutex> lock(slot.mu);
    if (id != 0 && slot.ctx_id[dev] == id) return GQA_OK;
    if (int rc = init(dev)) return rc;
    // init may have made the primary context current: key on the context now current
    int dev2 = 0;
    unsigned long long id2 = 0;
    if (current_ctx_key(&dev2, &id2) == GQA_OK && dev2 == dev) slot.ctx_id[dev] = id2;
    return GQA_OK;
}

// Device address of a __device__ variable in the current context, looked up
// once per context; nullptr with a message set on failure.
struct SymbolSlot {
    CtxSlot ctx;
    void *addr[kMaxDevices] = {};
};
void *symbol_address(const void *symbol, SymbolSlot &slot, const char *what);

// Device address of the library's status word in the current context;
// nullptr with a message set on failure.
int *device_status_ptr();

// 4-D bf16 tensor map over a [n3][n2][n1][n0] array (n0 innermost, the first
// three dimensions contiguous), box (b0, b1, b2, b3), 128-byte swizzle when
// swizzle128 != 0, zero fill out of bounds.  Consecutive n3 indices lie
// n2_pitch rows of n1 * n0 elements apart (n2_pitch = 0: n2, i.e. contiguous),
// so a window of rows of a longer tensor can be mapped.  Returns GQA_OK or
// GQA_ERR_CUDA.
int encode_tmap_bf16_4d(CUtensorMap *map, const void *base, uint64_t n0, uint64_t n1,
                        uint64_t n2, uint64_t n3, uint32_t b0, uint32_t b1, uint32_t b2,
                        uint32_t b3, int swizzle128, uint64_t n2_pitch = 0);

// ---- launchers (arguments already validated by the C-ABI layer) ----------
int launch_fwd_f32(const float *q, const float *k, const float *v, float *o, float *lse,
                   int B, int Tq, int Tkv, int Hq, int Hkv, int d, int causal, float scale,
                   cudaStream_t stream);

int launch_empty_rows(void *o, float *lse, int elem_bytes, int B, int Tq, int Hq, int d,
                      cudaStream_t stream);

int launch_fold_kv(const void *in, void *out, int B, int T, int H, int g, int d,
                   cudaStream_t stream);

// Host-side checks of gqa_decode's arguments (sizes, head dims, pointers);
// GQA_OK or the error gqa_decode returns for them.  B == 0 passes with no
// pointer checked.
int validate_decode(const void *q, const void *k_cache, const void *v_cache,
                    const int32_t *seqlens, const void *o, int B, int Hq, int Hkv, int d,
                    int Lmax, float scale);

// Bytes of workspace gqa_decode needs (partial results of the KV splits and
// one arrival word per (sequence, KV head)).
size_t decode_workspace_bytes(int B, int Hq, int Hkv, int d, int Lmax);
// window = 0: no sliding window (sinks ignored)
// rope_theta > 0: q is rotated as it is loaded, at position max(seqlens[b] - 1, 0).
int launch_decode(const void *q, const void *k_cache, const void *v_cache,
                  const int32_t *seqlens, void *o, int B, int Hq, int Hkv, int d, int Lmax,
                  int window, int sinks, float scale, void *workspace, cudaStream_t stream,
                  float rope_theta = 0.0f);

// q / o are views of Tq rows of [B, tq_pitch, Hq, d] buffers and k / v of Tkv rows
// of [B, tkv_pitch, Hkv, d] buffers (pitch 0: the view is the whole tensor).
// rope_theta > 0: q is rotated as it is loaded, row t at position q_pos0 + t.
int launch_prefill(const void *q, const void *k, const void *v, void *o, float *lse,
                   int B, int Tq, int Tkv, int Hq, int Hkv, int d, int causal, int window,
                   int sinks, float scale, cudaStream_t stream, int tq_pitch = 0,
                   int tkv_pitch = 0, float rope_theta = 0.0f, int q_pos0 = 0);

// Caps the persistent prefill grid at max_ctas CTAs (<= 0: no cap).
void set_prefill_grid_cap(int max_ctas);

// Forward on host-resident tensors through device staging buffers, with the
// copies pipelined against the attention in chunks of query rows.
int launch_fwd_host_pipeline(const void *q_host, const void *k_host, const void *v_host,
                             void *o_host, void *q_dev, void *k_dev, void *v_dev, void *o_dev,
                             int B, int Tq, int Tkv, int Hq, int Hkv, int d, int causal,
                             float scale, cudaStream_t stream, cudaEvent_t done);

size_t bwd_workspace_bytes(int B, int Tq, int Hq);
int launch_bwd(const void *q, const void *k, const void *v, const void *o, const void *dout,
               const float *lse, void *dq, void *dk, void *dv, int B, int Tq, int Tkv, int Hq,
               int Hkv, int d, int causal, int window, int sinks, float scale, void *workspace,
               cudaStream_t stream);

int selftest_wait_timeout(int timeout_us);

}  // namespace gqa
