"""Tensor-level calls on top of the C ABI.

PyTorch supplies device memory, shapes and the current stream; every step of
the computation runs in libgqa.so.  Non-OK statuses become exceptions:
``ValueError`` for invalid arguments and workspace problems,
``NotImplementedError`` for unsupported shapes, ``RuntimeError`` otherwise.
"""

import math

import torch

from . import _binding as _b

_EXC = {
    _b.GQA_ERR_INVALID_ARG: ValueError,
    _b.GQA_ERR_WORKSPACE: ValueError,
    _b.GQA_ERR_UNSUPPORTED: NotImplementedError,
}


def _check(rc, what):
    if rc != _b.GQA_OK:
        raise _EXC.get(rc, RuntimeError)(f"{what}: {_b.gqa_last_error()} (status {rc})")


def _stream(t):
    return torch.cuda.current_stream(t.device).cuda_stream


def _need(t, name, dtype, ndim):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dims, got shape {tuple(t.shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _shapes(q, k, v):
    B, Tq, Hq, d = q.shape
    Bk, Tkv, Hkv, dk = k.shape
    if Bk != B or dk != d or tuple(v.shape) != tuple(k.shape):
        raise ValueError(f"shape mismatch: q {tuple(q.shape)}, k {tuple(k.shape)}, v {tuple(v.shape)}")
    return B, Tq, Tkv, Hq, Hkv, d


def attn(q, k, v, causal=True, scale=None, out=None, return_lse=False, window=None, sinks=0,
         rope_theta=None, q_pos0=None):
    """Grouped-query attention forward, bf16.

    q [B, Tq, Hq, d], k/v [B, Tkv, Hkv, d] (bf16, contiguous, on one GPU);
    query head h reads K/V head h // (Hq // Hkv).  Returns o [B, Tq, Hq, d]
    (and lse [B, Hq, Tq] fp32 when ``return_lse``).  ``window`` (an int >= 1)
    selects causal sliding-window attention with ``sinks`` always-visible
    leading keys.  ``rope_theta`` rotates q as it is loaded (query row t at
    position ``q_pos0`` + t, default Tkv - Tq); k must already be rotated.
    """
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _need(t, n, torch.bfloat16, 4)
    B, Tq, Tkv, Hq, Hkv, d = _shapes(q, k, v)
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    o = torch.empty_like(q) if out is None else out
    _need(o, "out", torch.bfloat16, 4)
    lse = torch.empty((B, Hq, Tq), dtype=torch.float32, device=q.device) if return_lse else None
    lp = lse.data_ptr() if lse is not None else None
    if rope_theta is not None:
        if window is not None:
            raise NotImplementedError("rope_theta with a sliding window")
        pos0 = Tkv - Tq if q_pos0 is None else int(q_pos0)
        rc = _b.gqa_attn_fwd_rope(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lp,
                                  B, Tq, Tkv, Hq, Hkv, d, int(bool(causal)), scale, pos0,
                                  float(rope_theta), _stream(q))
    elif window is None:
        rc = _b.gqa_attn_fwd_lse(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lp,
                                 B, Tq, Tkv, Hq, Hkv, d, int(bool(causal)), scale, _stream(q))
    else:
        if not causal:
            raise ValueError("a sliding window needs causal=True")
        rc = _b.gqa_attn_fwd_window(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lp,
                                    B, Tq, Tkv, Hq, Hkv, d, int(window), int(sinks), scale,
                                    _stream(q))
    _check(rc, "gqa_attn_fwd")
    return (o, lse) if return_lse else o


def _need_host(t, name, ndim):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.is_cuda:
        raise ValueError(f"{name} must be a host (CPU) tensor")
    if t.dtype != torch.bfloat16:
        raise ValueError(f"{name} must be torch.bfloat16, got {t.dtype}")
    if t.dim() != ndim or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous {ndim}-d tensor, got {tuple(t.shape)}")


def host_staging(q, k, device=None):
    """Device staging buffers (q, k, v, o) for ``attn_host`` on host tensors shaped like q, k."""
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else device
    return (torch.empty(q.shape, dtype=torch.bfloat16, device=dev),
            torch.empty(k.shape, dtype=torch.bfloat16, device=dev),
            torch.empty(k.shape, dtype=torch.bfloat16, device=dev),
            torch.empty(q.shape, dtype=torch.bfloat16, device=dev))


def attn_host(q, k, v, out=None, causal=True, scale=None, staging=None, done=None):
    """``attn`` on host (CPU, preferably pinned) bf16 tensors: the copies up and down
    run in the library, overlapped with the attention chunk by chunk.  ``staging``
    is a (q, k, v, o) tuple of device buffers (``host_staging``).  The call is
    asynchronous on the staging device's current stream and returns ``out``: valid
    once that stream has reached this point, or, with ``done`` (a torch.cuda.Event),
    once ``done`` has completed (the stream is then not held for the copies down, so
    consecutive calls overlap).  The host tensors must stay alive and unchanged until
    then: the copies run after this function returns."""
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _need_host(t, n, 4)
    B, Tq, Tkv, Hq, Hkv, d = _shapes(q, k, v)
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    o = torch.empty(q.shape, dtype=torch.bfloat16, pin_memory=q.is_pinned()) if out is None else out
    _need_host(o, "out", 4)
    if tuple(o.shape) != tuple(q.shape):
        raise ValueError(f"out shape {tuple(o.shape)} != q shape {tuple(q.shape)}")
    st = host_staging(q, k) if staging is None else staging
    for t, ref, n in zip(st, (q, k, k, q), ("q_dev", "k_dev", "v_dev", "o_dev")):
        _need(t, n, torch.bfloat16, 4)
        if tuple(t.shape) != tuple(ref.shape):
            raise ValueError(f"{n} shape {tuple(t.shape)} != {tuple(ref.shape)}")
    ev = None
    if done is not None:
        done.record(torch.cuda.current_stream(st[0].device))   # makes sure the event exists
        ev = done.cuda_event
    rc = _b.gqa_attn_fwd_host(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                              *(t.data_ptr() for t in st), B, Tq, Tkv, Hq, Hkv, d,
                              int(bool(causal)), scale, _stream(st[0]), ev)
    _check(rc, "gqa_attn_fwd_host")
    return o


def attn_f32(q, k, v, causal=True, scale=None, return_lse=False):
    """The same operation in fp32 (FP32 pipe); q/k/v fp32 in the same layouts."""
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _need(t, n, torch.float32, 4)
    B, Tq, Tkv, Hq, Hkv, d = _shapes(q, k, v)
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    o = torch.empty_like(q)
    lse = torch.empty((B, Hq, Tq), dtype=torch.float32, device=q.device) if return_lse else None
    rc = _b.gqa_attn_fwd_f32(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                             lse.data_ptr() if lse is not None else None,
                             B, Tq, Tkv, Hq, Hkv, d, int(bool(causal)), scale, _stream(q))
    _check(rc, "gqa_attn_fwd_f32")
    return (o, lse) if return_lse else o


def decode_workspace_size(B, Hq, Hkv, d, Lmax):
    return int(_b.gqa_decode_workspace_size(B, Hq, Hkv, d, Lmax))


def decode(q, k_cache, v_cache, seqlens, scale=None, workspace=None, out=None, window=None,
           sinks=0, rope_theta=None):
    """One query token per sequence against a bf16 KV cache.

    q [B, Hq, d], caches [B, Lmax, Hkv, d], seqlens int32 [B] on the device.
    ``workspace``: a uint8 CUDA tensor of at least decode_workspace_size(...)
    bytes (allocated here when None).  ``rope_theta`` rotates q as it is loaded
    (position max(seqlens[b] - 1, 0)); the cached keys must already be rotated.
    """
    _need(q, "q", torch.bfloat16, 3)
    _need(k_cache, "k_cache", torch.bfloat16, 4)
    _need(v_cache, "v_cache", torch.bfloat16, 4)
    _need(seqlens, "seqlens", torch.int32, 1)
    B, Hq, d = q.shape
    Bc, Lmax, Hkv, dc = k_cache.shape
    if Bc != B or dc != d or tuple(v_cache.shape) != tuple(k_cache.shape) or seqlens.shape[0] != B:
        raise ValueError("decode shape mismatch")
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    need = decode_workspace_size(B, Hq, Hkv, d, Lmax)
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=q.device)
    o = torch.empty_like(q) if out is None else out
    if rope_theta is not None:
        if window is not None:
            raise NotImplementedError("rope_theta with a sliding window")
        rc = _b.gqa_decode_rope(q.data_ptr(), k_cache.data_ptr(), v_cache.data_ptr(),
                                seqlens.data_ptr(), o.data_ptr(), B, Hq, Hkv, d, Lmax, scale,
                                float(rope_theta), workspace.data_ptr(), workspace.numel(),
                                _stream(q))
    elif window is None:
        rc = _b.gqa_decode(q.data_ptr(), k_cache.data_ptr(), v_cache.data_ptr(),
                           seqlens.data_ptr(), o.data_ptr(), B, Hq, Hkv, d, Lmax, scale,
                           workspace.data_ptr(), workspace.numel(), _stream(q))
    else:
        rc = _b.gqa_decode_window(q.data_ptr(), k_cache.data_ptr(), v_cache.data_ptr(),
                                  seqlens.data_ptr(), o.data_ptr(), B, Hq, Hkv, d, Lmax,
                                  int(window), int(sinks), scale, workspace.data_ptr(),
                                  workspace.numel(), _stream(q))
    _check(rc, "gqa_decode")
    return o


def fold_kv(kv, g):
    """Mean-pool the heads of a bf16 [B, T, H, d] K or V tensor into g contiguous groups."""
    _need(kv, "kv", torch.bfloat16, 4)
    B, T, H, d = kv.shape
    out = torch.empty((B, T, g, d), dtype=kv.dtype, device=kv.device)
    rc = _b.gqa_fold_kv(kv.data_ptr(), out.data_ptr(), B, T, H, g, d, _stream(kv))
    _check(rc, "gqa_fold_kv")
    return out


def attn_bwd_workspace_size(B, Tq, Hq):
    return int(_b.gqa_attn_bwd_workspace_size(B, Tq, Hq))


def attn_bwd(q, k, v, o, lse, dout, causal=True, scale=None, window=None, sinks=0,
             workspace=None):
    """Gradients (dq, dk, dv) of attn(q, k, v) for the upstream gradient dout.

    o and lse are the forward's outputs (attn(..., return_lse=True)).  dk / dv
    of a K/V head are summed over the G query heads that share it.
    """
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (o, "o"), (dout, "dout")):
        _need(t, n, torch.bfloat16, 4)
    _need(lse, "lse", torch.float32, 3)
    B, Tq, Tkv, Hq, Hkv, d = _shapes(q, k, v)
    if tuple(o.shape) != tuple(q.shape) or tuple(dout.shape) != tuple(q.shape):
        raise ValueError("o and dout must have q's shape")
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    need = int(_b.gqa_attn_bwd_workspace_size(B, Tq, Hq))
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=q.device)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    rc = _b.gqa_attn_bwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), dout.data_ptr(),
                         lse.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(),
                         B, Tq, Tkv, Hq, Hkv, d, int(bool(causal)),
                         0 if window is None else int(window), int(sinks), scale,
                         workspace.data_ptr(), workspace.numel(), _stream(q))
    _check(rc, "gqa_attn_bwd")
    return dq, dk, dv


def rope_(x, pos0=0, theta=10000.0):
    """Rotary position embedding of a bf16 [B, T, H, d] q or k tensor, in place
    (row t at position pos0 + t).  Returns x."""
    _need(x, "x", torch.bfloat16, 4)
    B, T, H, d = x.shape
    _check(_b.gqa_rope(x.data_ptr(), B, T, H, d, int(pos0), float(theta), _stream(x)), "gqa_rope")
    return x


def rope_qk_(q, k, pos0=0, theta=10000.0):
    """RoPE of bf16 q [B, T, Hq, d] and k [B, T, Hkv, d] in place, in one launch
    (row t of both at position pos0 + t).  Returns (q, k)."""
    _need(q, "q", torch.bfloat16, 4)
    _need(k, "k", torch.bfloat16, 4)
    B, T, Hq, d = q.shape
    if k.shape[0] != B or k.shape[1] != T or k.shape[3] != d:
        raise ValueError(f"k shape {tuple(k.shape)} does not match q {tuple(q.shape)}")
    _check(_b.gqa_rope_qk(q.data_ptr(), k.data_ptr(), B, T, Hq, k.shape[2], d, int(pos0),
                          float(theta), _stream(q)), "gqa_rope_qk")
    return q, k


def rope_decode_q_(q, seqlens, theta=10000.0):
    """RoPE of bf16 decode queries [B, H, d] in place, sequence b at position seqlens[b] - 1."""
    _need(q, "q", torch.bfloat16, 3)
    _need(seqlens, "seqlens", torch.int32, 1)
    B, H, d = q.shape
    _check(_b.gqa_rope_decode_q(q.data_ptr(), seqlens.data_ptr(), B, H, d, float(theta),
                                _stream(q)), "gqa_rope_decode_q")
    return q


def device_status(reset=True):
    """Synchronise, then raise if a kernel recorded an error (e.g. a wait timeout)."""
    _check(_b.gqa_device_status(int(bool(reset))), "gqa_device_status")
