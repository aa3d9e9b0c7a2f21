/*
 * gqa.h -- C ABI of libgqa.so, grouped-query scaled-dot-product attention for
 * NVIDIA B200 (sm_100a).
 *
 * The operation (TT Lab "キー・バリューヘッドだけ減らしてみる", steps 1-5; course
 * "Неделя 7. Внимание", steps 1-2):
 *
 *   Hq query heads are split into Hkv contiguous groups of G = Hq / Hkv heads;
 *   query head hq reads K/V head hq / G (the repeat_interleave expansion of
 *   the K3 notes "GVA", subsection "Forward: repeat_interleave", never
 *   materialised).  For query row i of head hq:
 *       s_j = scale * <q_i, k_j>                      (scale = 1/sqrt(d) usually)
 *       s_j = -inf  if causal and j > i + (Tkv - Tq)  (mask before the softmax)
 *       o_i = sum_j softmax(s)_j v_j                  (max subtracted first)
 *   MHA (Hkv = Hq) and MQA (Hkv = 1) are the end cases.
 *
 * Conventions shared by every entry point
 *   - Layouts are row-major and contiguous: q, o [B, Tq, Hq, d];
 *     k, v [B, Tkv, Hkv, d]; lse [B, Hq, Tq].
 *   - All tensor pointers are DEVICE pointers owned by the caller.  The
 *     library keeps no pointer after a call returns and allocates no device
 *     memory; scratch space is the caller's `workspace`.
 *   - Work is enqueued asynchronously on `stream` (a cudaStream_t; NULL is the
 *     legacy default stream).  A GQA_OK return means "validated and
 *     launched"; kernel-side problems are reported by gqa_device_status().
 *   - Arguments are validated on the host before anything is launched; a
 *     non-zero status is returned and gqa_last_error() gives a message.
 *     Nothing is launched when a call fails validation.
 *   - Causal alignment is bottom-right: with Tq != Tkv, query row i sees keys
 *     j <= i + (Tkv - Tq).  A row that sees no key gets o = 0, lse = -inf.
 *   - Empty problems (B == 0 or Tq == 0) are valid and launch nothing.
 */
#ifndef GQA_H
#define GQA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

struct CUstream_st;                     /* the type behind cudaStream_t */
typedef struct CUstream_st *gqa_stream_t;

typedef enum {
    GQA_OK = 0,
    GQA_ERR_INVALID_ARG = 1,   /* bad shape, Hq % Hkv != 0, null/misaligned pointer, bad scale */
    GQA_ERR_UNSUPPORTED = 2,   /* valid but not built: head dim or group size, no sm_100 GPU */
    GQA_ERR_CUDA = 3,          /* a CUDA runtime/driver call failed (launch, tensor map) */
    GQA_ERR_WORKSPACE = 4,     /* decode workspace missing or too small */
    GQA_ERR_TIMEOUT = 5        /* a bounded device-side wait ran out (see gqa_device_status) */
} gqa_status;

/*
 * gqa_attn_fwd -- prefill / full-sequence forward, bf16 in, bf16 out, fp32
 * accumulation and fp32 online softmax on tcgen05 tensor cores.
 *
 *   q  [B, Tq,  Hq,  d] bf16      k, v [B, Tkv, Hkv, d] bf16
 *   o  [B, Tq,  Hq,  d] bf16 (written)
 *   B, Tq, Tkv >= 0; Hq, Hkv >= 1 with Hq % Hkv == 0 (the lab's ValueError
 *   becomes GQA_ERR_INVALID_ARG); G = Hq/Hkv <= 128 (else UNSUPPORTED);
 *   d in {64, 128} (else UNSUPPORTED); causal 0/1; scale > 0 and finite
 *   (callers normally pass 1/sqrt(d)).  Pointers must be 16-byte aligned
 *   (tensor-memory-access copies need it).
 * The kernel is persistent: min(#work units, #SMs) CTAs, a unit being two
 * 128-row tiles of one (batch, KV head); gqa_set_prefill_grid_cap can lower
 * that bound.  Host work per call: argument checks and three tensor-map
 * encodings; the kernel's attributes are set once per CUDA context.
 */
int gqa_attn_fwd(const void *q, const void *k, const void *v, void *o,
                 int B, int Tq, int Tkv, int Hq, int Hkv, int d,
                 int causal, float scale, gqa_stream_t stream);

/*
 * gqa_attn_fwd_lse -- as gqa_attn_fwd, and also writes the natural-log
 * log-sum-exp of each row's scaled, masked scores:
 *   lse [B, Hq, Tq] fp32, lse = m + ln(sum_j exp(s_j - m)); -inf for a row
 *   with no visible key.  lse may be NULL (then identical to gqa_attn_fwd).
 */
int gqa_attn_fwd_lse(const void *q, const void *k, const void *v, void *o, float *lse,
                     int B, int Tq, int Tkv, int Hq, int Hkv, int d,
                     int causal, float scale, gqa_stream_t stream);

/*
 * gqa_attn_fwd_rope -- gqa_attn_fwd_lse with rotary position embedding applied
 * to q as it is loaded (course "Неделя 7. Внимание", step 3: pair (2i, 2i+1)
 * of the row at position m turns by m * theta^(-2i/d); only q and k rotate).
 * Query row t sits at position q_pos0 + t (q_pos0 >= 0; for self-attention
 * over a whole sequence q_pos0 = Tkv - Tq, the key positions being 0..Tkv-1).
 * q in memory is NOT modified; k must already be rotated (gqa_rope, once,
 * when the keys enter the cache: a key tile is read by every query tile of
 * its group, so rotating it on each load would repeat the work).  The
 * rotation is the same arithmetic as gqa_rope's, so the result equals
 * gqa_rope(q) followed by gqa_attn_fwd_lse bit for bit.  theta > 0 and
 * finite; everything else as gqa_attn_fwd_lse.
 */
int gqa_attn_fwd_rope(const void *q, const void *k, const void *v, void *o, float *lse,
                      int B, int Tq, int Tkv, int Hq, int Hkv, int d, int causal, float scale,
                      int q_pos0, float theta, gqa_stream_t stream);

/*
 * gqa_attn_fwd_host -- gqa_attn_fwd for host-resident tensors (same operation,
 * layouts and arguments; no lse).  q_host, k_host, v_host are read and o_host
 * written (pinned host memory for the copies to run asynchronously; pageable
 * memory works, slower); q_dev, k_dev, v_dev, o_dev are caller-owned device
 * staging buffers of the full tensor sizes (16-byte aligned), overwritten.
 * k and v are copied up whole first, then the query rows in 4 chunks of
 * >= 256 rows, last rows first, on a library-owned copy stream; each chunk's
 * attention runs on `stream` once its rows have landed, while the previous
 * chunk's o is copied down on a second library-owned stream.  Asynchronous: with
 * done_event == NULL, o_host is complete when the work enqueued on `stream` so
 * far is; otherwise done_event (a cudaEvent_t created by the caller) is
 * recorded when o_host is complete and `stream` is not held for the copies
 * down, so a following call's copies up overlap them.  A call orders its
 * copies up after the work on `stream` at the time of the call and its first
 * attention chunk after the previous call's copies down (on this device).
 * The host buffers must stay allocated and unchanged until the call completes.
 * The copy streams and their events are created on first use in each CUDA
 * context and kept (no device memory is allocated); concurrent calls from several
 * host threads are serialised while they enqueue.  Errors as
 * gqa_attn_fwd_lse, plus GQA_ERR_CUDA for a failed copy.
 */
int gqa_attn_fwd_host(const void *q_host, const void *k_host, const void *v_host, void *o_host,
                      void *q_dev, void *k_dev, void *v_dev, void *o_dev, int B, int Tq, int Tkv,
                      int Hq, int Hkv, int d, int causal, float scale, gqa_stream_t stream,
                      void *done_event);

/*
 * gqa_attn_fwd_window -- causal forward with a sliding window and attention
 * sinks (course "Неделя 7. Внимание", step 3: the window bounds what a token
 * sees -- and the cache -- to the most recent keys, while the first tokens,
 * where the softmax parks its mass, stay visible).
 *
 * Row i (key position p = i + Tkv - Tq) sees key j iff j <= p and
 * (j > p - window or j < sinks).  window >= 1 (window >= Tkv + Tq is plain
 * causal attention), sinks >= 0; other arguments, layouts, lse (may be NULL)
 * and errors as gqa_attn_fwd_lse.  Only the KV tiles a CTA's rows can see are
 * read: the sink tiles and the tiles of the window.
 */
int gqa_attn_fwd_window(const void *q, const void *k, const void *v, void *o, float *lse,
                        int B, int Tq, int Tkv, int Hq, int Hkv, int d,
                        int window, int sinks, float scale, gqa_stream_t stream);

/*
 * gqa_attn_fwd_f32 -- the same operation in fp32 end to end (fp32 FFMA,
 * no tensor cores).  Same layouts; fp32 tensors; any 1 <= d <= 256; pointers
 * 4-byte aligned; lse may be NULL.  A correctness path for fp32 callers, not
 * a throughput path.
 */
int gqa_attn_fwd_f32(const float *q, const float *k, const float *v, float *o, float *lse,
                     int B, int Tq, int Tkv, int Hq, int Hkv, int d,
                     int causal, float scale, gqa_stream_t stream);

/*
 * gqa_decode_workspace_size -- bytes of device scratch gqa_decode needs for
 * these sizes (partial outputs and log-sum-exp of every KV split).  Returns 0
 * for invalid sizes.  Pure host function, no CUDA call.
 */
size_t gqa_decode_workspace_size(int B, int Hq, int Hkv, int d, int Lmax);

/*
 * gqa_decode -- one new query token per sequence against a KV cache
 * (the course's KV-cache motivation, step 2; the causal mask leaves every
 * cached key visible to the newest token).
 *
 *   q        [B, Hq, d] bf16
 *   k_cache, v_cache [B, Lmax, Hkv, d] bf16; rows >= seqlens[b] are never read
 *   seqlens  [B] int32 DEVICE array, 0 <= seqlens[b] <= Lmax
 *   o        [B, Hq, d] bf16 (written; a sequence of length 0 gets zeros)
 *   workspace: device scratch of at least gqa_decode_workspace_size(...)
 *   bytes, 256-byte aligned; its contents on entry do not matter.
 *   d in {64, 128}; Hq % Hkv == 0; G = Hq/Hkv <= 32 (else UNSUPPORTED).
 * Each split of the KV length is streamed from HBM once for all G query heads
 * of its group, and the splits are merged with the log-sum-exp identity by a
 * second kernel on the same stream.  A seqlens[b] above Lmax is clamped to
 * Lmax and flagged in gqa_device_status (GQA_ERR_INVALID_ARG).
 */
int gqa_decode(const void *q, const void *k_cache, const void *v_cache,
               const int32_t *seqlens, void *o,
               int B, int Hq, int Hkv, int d, int Lmax, float scale,
               void *workspace, size_t workspace_bytes, gqa_stream_t stream);

/*
 * gqa_decode_rope -- gqa_decode with rotary position embedding applied to the
 * query as it is loaded (course "Неделя 7. Внимание", step 3): sequence b's new token sits at
 * position max(seqlens[b] - 1, 0), as for gqa_rope_decode_q; q in memory is
 * not modified and the cached keys must already be rotated.  The result
 * equals gqa_rope_decode_q followed by gqa_decode bit for bit.  theta > 0 and
 * finite; everything else (layouts, workspace, errors) as gqa_decode.
 */
int gqa_decode_rope(const void *q, const void *k_cache, const void *v_cache,
                    const int32_t *seqlens, void *o,
                    int B, int Hq, int Hkv, int d, int Lmax, float scale, float theta,
                    void *workspace, size_t workspace_bytes, gqa_stream_t stream);

/*
 * gqa_decode_window -- gqa_decode with a sliding window and attention sinks
 * (course "Неделя 7. Внимание", step 3): the newest token of sequence b sees cache rows
 * j >= seqlens[b] - window and rows j < sinks.  window >= 1, sinks >= 0;
 * everything else (layouts, workspace and its size, errors) as gqa_decode.
 * The KV splits start at the window's first row, and split 0 also reads the
 * sink rows below the window; reads are whole 64-row stages, so apart from
 * that rounding no invisible row is read.
 */
int gqa_decode_window(const void *q, const void *k_cache, const void *v_cache,
                      const int32_t *seqlens, void *o,
                      int B, int Hq, int Hkv, int d, int Lmax, int window, int sinks,
                      float scale, void *workspace, size_t workspace_bytes,
                      gqa_stream_t stream);

/*
 * gqa_decode_static -- gqa_decode for callers that cannot allocate device
 * memory.  (The pages have no counterpart: this is a library convenience.)
 *
 * Who needs it: code that may not call cudaMalloc where it decodes -- a
 * runtime whose memory pool or arena owns all device memory, a plugin whose
 * host framework forbids allocation on its hot path, or code that must not
 * risk the device-wide synchronisation cudaMalloc/cudaFree can cause.
 * gqa_decode needs scratch for the partial results of its KV splits; this
 * entry point uses a scratch array built into the library instead of a
 * caller `workspace`.  Inputs and outputs are the caller's, exactly as for
 * gqa_decode (same arguments minus workspace, same validation and errors).
 *
 * Limits and behaviour:
 *   - The built-in scratch is 32 MiB per GPU, held by every GPU that loads
 *     the library's code until the process exits.  Sizes whose
 *     gqa_decode_workspace_size(...) exceeds it are rejected with
 *     GQA_ERR_WORKSPACE and nothing is launched (B=64, Hq=32, d=128,
 *     Lmax=8192 fits).
 *   - The first call in a CUDA context (the first call with a device
 *     current, and the first one after a cudaDeviceReset of that device)
 *     looks up the scratch's device address (cudaGetSymbolAddress) and
 *     caches it for that context; make that first call before any stream
 *     capture.  Arguments are checked exactly as gqa_decode checks them, and
 *     before the lookup.
 *   - All calls on a device share the one scratch array, which keeps the last
 *     call's contents.  Nothing in it needs to start at zero, but calls whose
 *     kernels overlap on the GPU (different streams, or several host threads)
 *     race on it: serialise them, e.g. on one stream.
 *   - No cudaMalloc, cudaFree or other allocating routine is called.
 */
int gqa_decode_static(const void *q, const void *k_cache, const void *v_cache,
                      const int32_t *seqlens, void *o,
                      int B, int Hq, int Hkv, int d, int Lmax, float scale,
                      gqa_stream_t stream);

/*
 * gqa_attn_bwd_workspace_size -- bytes of device scratch gqa_attn_bwd needs
 * (one fp32 row statistic per query row: B * Hq * Tq floats, rounded up to
 * 256, then 256 bytes for the dQ kernel's work counter).  0 for invalid
 * sizes.  Pure host function.
 */
size_t gqa_attn_bwd_workspace_size(int B, int Tq, int Hq);

/*
 * gqa_attn_bwd -- gradients of the forward (gqa_attn_fwd_lse or, with
 * window > 0, gqa_attn_fwd_window) with respect to q, k and v.
 *
 *   q, o, dout [B, Tq, Hq, d] bf16 (o and lse from the forward; dout = dL/do)
 *   k, v       [B, Tkv, Hkv, d] bf16
 *   lse        [B, Hq, Tq] fp32 from the forward
 *   dq [B, Tq, Hq, d], dk, dv [B, Tkv, Hkv, d] bf16 (written)
 *   causal, window (0 = none, else needs causal), sinks, scale: as the forward.
 * The gradient of a K/V head shared by G query heads is the sum of the G
 * heads' gradients (K3 notes "GVA", "Backward: view + sum": a copy's
 * backward is a sum, not a mean); dq carries the chain-rule factor `scale`
 * (same notes, "scale 的处理").  P is recomputed from lse; fp32 accumulation.
 * workspace: >= gqa_attn_bwd_workspace_size(B, Tq, Hq) bytes, 256-byte
 * aligned, contents on entry irrelevant; it holds D and the dQ kernel's work
 * counter until the call's kernels finish, so calls in flight at the same time
 * need workspaces of their own.  The dK/dV kernel runs on a second stream of
 * the library's, forked from `stream` after D is formed and joined back before
 * the call's work on `stream` ends (CUDA-graph capture on `stream` holds both).
 * The first call in a CUDA context creates that stream and two events, so make
 * one call before capturing (stream and event creation may be refused during a
 * global-mode capture; the call then returns GQA_ERR_CUDA).
 * d in {64, 128}.  Errors as the forward plus GQA_ERR_WORKSPACE.
 */
int gqa_attn_bwd(const void *q, const void *k, const void *v, const void *o, const void *dout,
                 const float *lse, void *dq, void *dk, void *dv,
                 int B, int Tq, int Tkv, int Hq, int Hkv, int d,
                 int causal, int window, int sinks, float scale,
                 void *workspace, size_t workspace_bytes, gqa_stream_t stream);

/*
 * gqa_rope -- rotary position embedding, in place (course "Неделя 7.
 * Внимание", step 3): coordinate pair (2i, 2i+1) of the row at position m is
 * rotated by m * theta^(-2i/d).  Apply it to q and to k (never to v) before
 * attention; the scores then depend on position differences only.
 *   x [B, T, H, d] bf16, rewritten in place; row t sits at position pos0 + t
 *   (for causal prefill with Tq != Tkv: q uses pos0 + Tkv - Tq, k uses pos0).
 *   d a multiple of 8 in [8, 256]; theta > 0 (10000 is usual); x 16-byte
 *   aligned.  Angles are reduced in double, then fp32 sine / cosine; the
 *   result is rounded to bf16 (nearest even).  Reading of the page: adjacent
 *   coordinates form a pair.
 */
int gqa_rope(void *x, int B, int T, int H, int d, int pos0, float theta, gqa_stream_t stream);

/*
 * gqa_rope_qk -- gqa_rope of q [B, T, Hq, d] and k [B, T, Hkv, d] in one launch
 * (self-attention prefill: row t of both at position pos0 + t).  Each angle is
 * evaluated once per token and column and applied to all Hq + Hkv heads.
 * Same argument rules as gqa_rope for each tensor; q and k must be distinct
 * buffers (GQA_ERR_INVALID_ARG otherwise).
 */
int gqa_rope_qk(void *q, void *k, int B, int T, int Hq, int Hkv, int d, int pos0, float theta,
                gqa_stream_t stream);

/*
 * gqa_rope_decode_q -- gqa_rope of decode queries q [B, H, d] (bf16, in place):
 * sequence b's new token sits at position max(seqlens[b] - 1, 0) (seqlens:
 * device int32 [B]; an empty cache makes it the first token).  The cached keys are expected to be rotated already, each at
 * its own position when it was appended.
 */
int gqa_rope_decode_q(void *q, const int32_t *seqlens, int B, int H, int d, float theta,
                      gqa_stream_t stream);

/*
 * gqa_fold_kv -- MHA -> GQA conversion of a K or V tensor by mean pooling
 * (TT Lab "キー・バリューヘッドだけ減らしてみる", step 2; course "Неделя 7. Внимание",
 * step 2: average the heads of each contiguous group).
 *   in  [B, T, H, d] bf16, out [B, T, g, d] bf16 (written), H % g == 0.
 * Members of a group are added in head order in fp32, divided by H/g in fp32
 * and rounded to bf16 (nearest even).  d must be a multiple of 8 and both
 * pointers 16-byte aligned.
 */
int gqa_fold_kv(const void *in, void *out, int B, int T, int H, int g, int d,
                gqa_stream_t stream);

/*
 * gqa_last_error -- message for the last non-OK status returned on the
 * calling host thread ("" if none).  Valid until the next call on the thread.
 */
const char *gqa_last_error(void);

/*
 * gqa_device_status -- synchronises the current device, then reports the
 * first error a kernel recorded since the last reset (GQA_OK if none):
 * GQA_ERR_TIMEOUT when a bounded wait inside a kernel ran out (the kernel
 * then stopped early and its output is incomplete), GQA_ERR_INVALID_ARG for a
 * decode length above Lmax.  reset != 0 clears the record.
 */
int gqa_device_status(int reset);

/*
 * gqa_selftest_wait_timeout -- launches a one-warp kernel that waits on a
 * shared-memory barrier nothing will ever arrive at, bounded by timeout_us
 * microseconds, and returns what that kernel recorded: GQA_ERR_TIMEOUT when
 * the bound works.  Exercises the failure path of every bounded wait without
 * hanging or faulting the GPU; synchronises the device; resets the record.
 */
int gqa_selftest_wait_timeout(int timeout_us);

/*
 * gqa_selftest_exp2_poly -- evaluates, on the GPU, the FMA-pipe 2^x
 * polynomial the prefill softmax uses for part of its exponentials (the
 * max-subtracted softmax of the TT Lab page, step 4, and the course page, step 1, needs
 * exp(s - m) = 2^((s - m) log2 e)): y[i] = poly 2^x[i] for n points (n even,
 * x and y device float arrays, 4-byte aligned).  Range reduction
 * x = n + f, f in [-1/2, 1/2], a degree-3 minimax fit of 2^f (relative error
 * <= 7.5e-5), 2^n added to the exponent field; x is clamped to >= -125
 * (which keeps every result a normal float), so every x <= -125 gives 2^-125
 * (to the same relative error).  Asynchronous on `stream`.  For tests of that
 * bound.
 */
int gqa_selftest_exp2_poly(const float *x, float *y, int n, gqa_stream_t stream);

/*
 * gqa_set_prefill_grid_cap -- testing aid: caps the persistent prefill grid
 * (gqa_attn_fwd and its variants) at max_ctas CTAs for every later launch in
 * the process, so each CTA walks many work units; max_ctas <= 0 removes the
 * cap.  The output does not depend on the grid.  Not needed in normal use.
 */
void gqa_set_prefill_grid_cap(int max_ctas);

#ifdef __cplusplus
}
#endif

#endif /* GQA_H */
