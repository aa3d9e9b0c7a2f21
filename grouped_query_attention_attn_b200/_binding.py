"""ctypes binding of libgqa.so: one Python function per C entry point, same
names and argument order, argument marshalling only.

Pointers are passed as Python ints (device addresses, e.g. ``tensor.data_ptr()``
or 0 for NULL) and the stream as an int (``torch.cuda.Stream.cuda_stream``).
The functions return the C status code unchanged; ``api.py`` turns codes into
exceptions.  There is no fallback: if the shared library is missing or fails
to load, every call raises.
"""

import ctypes
import os

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libgqa.so")

GQA_OK = 0
GQA_ERR_INVALID_ARG = 1
GQA_ERR_UNSUPPORTED = 2
GQA_ERR_CUDA = 3
GQA_ERR_WORKSPACE = 4
GQA_ERR_TIMEOUT = 5

_lib = None

_I = ctypes.c_int
_P = ctypes.c_void_p
_F = ctypes.c_float
_SIGNATURES = {
    "gqa_attn_fwd": (_I, [_P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _F, _P]),
    "gqa_attn_fwd_lse": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _F, _P]),
    "gqa_attn_fwd_host": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _F, _P,
                               _P]),
    "gqa_attn_fwd_window": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _I, _F, _P]),
    "gqa_attn_fwd_f32": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _F, _P]),
    "gqa_decode_workspace_size": (ctypes.c_size_t, [_I, _I, _I, _I, _I]),
    "gqa_decode": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _F, _P, ctypes.c_size_t, _P]),
    "gqa_decode_window": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _F, _P,
                               ctypes.c_size_t, _P]),
    "gqa_decode_static": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _F, _P]),
    "gqa_fold_kv": (_I, [_P, _P, _I, _I, _I, _I, _I, _P]),
    "gqa_attn_bwd_workspace_size": (ctypes.c_size_t, [_I, _I, _I]),
    "gqa_attn_bwd": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _I, _I,
                          _F, _P, ctypes.c_size_t, _P]),
    "gqa_rope": (_I, [_P, _I, _I, _I, _I, _I, _F, _P]),
    "gqa_rope_qk": (_I, [_P, _P, _I, _I, _I, _I, _I, _I, _F, _P]),
    "gqa_rope_decode_q": (_I, [_P, _P, _I, _I, _I, _F, _P]),
    "gqa_last_error": (ctypes.c_char_p, []),
    "gqa_device_status": (_I, [_I]),
    "gqa_selftest_wait_timeout": (_I, [_I]),
    "gqa_set_prefill_grid_cap": (None, [_I]),
    "gqa_selftest_exp2_poly": (_I, [_P, _P, _I, _P]),
    "gqa_attn_fwd_rope": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _F, _I, _F, _P]),
    "gqa_decode_rope": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _F, _F, _P, ctypes.c_size_t,
                             _P]),
}


def lib():
    """The loaded libgqa.so (raises RuntimeError if it is not built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"{LIB_PATH} is not built: run `python -m grouped_query_attention_attn_b200.build`")
        handle = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGNATURES.items():
            fn = getattr(handle, name)
            fn.restype = res
            fn.argtypes = args
        _lib = handle
    return _lib


def gqa_attn_fwd(q, k, v, o, B, Tq, Tkv, Hq, Hkv, d, causal, scale, stream):
    return lib().gqa_attn_fwd(q, k, v, o, B, Tq, Tkv, Hq, Hkv, d, causal, scale, stream)


def gqa_attn_fwd_lse(q, k, v, o, lse, B, Tq, Tkv, Hq, Hkv, d, causal, scale, stream):
    return lib().gqa_attn_fwd_lse(q, k, v, o, lse, B, Tq, Tkv, Hq, Hkv, d, causal, scale, stream)


def gqa_attn_fwd_window(q, k, v, o, lse, B, Tq, Tkv, Hq, Hkv, d, window, sinks, scale, stream):
    return lib().gqa_attn_fwd_window(q, k, v, o, lse, B, Tq, Tkv, Hq, Hkv, d, window, sinks,
                                     scale, stream)


def gqa_attn_fwd_rope(q, k, v, o, lse, B, Tq, Tkv, Hq, Hkv, d, causal, scale, q_pos0, theta,
                      stream):
    return lib().gqa_attn_fwd_rope(q, k, v, o, lse, B, Tq, Tkv, Hq, Hkv, d, causal, scale, q_pos0,
                                   theta, stream)


def gqa_attn_fwd_f32(q, k, v, o, lse, B, Tq, Tkv, Hq, Hkv, d, causal, scale, stream):
    return lib().gqa_attn_fwd_f32(q, k, v, o, lse, B, Tq, Tkv, Hq, Hkv, d, causal, scale, stream)


def gqa_decode_workspace_size(B, Hq, Hkv, d, Lmax):
    return lib().gqa_decode_workspace_size(B, Hq, Hkv, d, Lmax)


def gqa_decode(q, k_cache, v_cache, seqlens, o, B, Hq, Hkv, d, Lmax, scale, workspace,
               workspace_bytes, stream):
    return lib().gqa_decode(q, k_cache, v_cache, seqlens, o, B, Hq, Hkv, d, Lmax, scale,
                            workspace, workspace_bytes, stream)


def gqa_decode_rope(q, k_cache, v_cache, seqlens, o, B, Hq, Hkv, d, Lmax, scale, theta, workspace,
                    workspace_bytes, stream):
    return lib().gqa_decode_rope(q, k_cache, v_cache, seqlens, o, B, Hq, Hkv, d, Lmax, scale,
                                 theta, workspace, workspace_bytes, stream)


def gqa_decode_window(q, k_cache, v_cache, seqlens, o, B, Hq, Hkv, d, Lmax, window, sinks, scale,
                      workspace, workspace_bytes, stream):
    return lib().gqa_decode_window(q, k_cache, v_cache, seqlens, o, B, Hq, Hkv, d, Lmax, window,
                                   sinks, scale, workspace, workspace_bytes, stream)


def gqa_decode_static(q, k_cache, v_cache, seqlens, o, B, Hq, Hkv, d, Lmax, scale, stream):
    """Decode with the library's built-in scratch, for callers that cannot allocate."""
    return lib().gqa_decode_static(q, k_cache, v_cache, seqlens, o, B, Hq, Hkv, d, Lmax, scale,
                                   stream)


def gqa_fold_kv(inp, out, B, T, H, g, d, stream):
    return lib().gqa_fold_kv(inp, out, B, T, H, g, d, stream)


def gqa_attn_bwd_workspace_size(B, Tq, Hq):
    return lib().gqa_attn_bwd_workspace_size(B, Tq, Hq)


def gqa_attn_bwd(q, k, v, o, dout, lse, dq, dk, dv, B, Tq, Tkv, Hq, Hkv, d, causal, window, sinks,
                 scale, workspace, workspace_bytes, stream):
    return lib().gqa_attn_bwd(q, k, v, o, dout, lse, dq, dk, dv, B, Tq, Tkv, Hq, Hkv, d, causal,
                              window, sinks, scale, workspace, workspace_bytes, stream)


def gqa_rope(x, B, T, H, d, pos0, theta, stream):
    return lib().gqa_rope(x, B, T, H, d, pos0, theta, stream)


def gqa_attn_fwd_host(q_host, k_host, v_host, o_host, q_dev, k_dev, v_dev, o_dev, B, Tq, Tkv, Hq,
                      Hkv, d, causal, scale, stream, done_event):
    return lib().gqa_attn_fwd_host(q_host, k_host, v_host, o_host, q_dev, k_dev, v_dev, o_dev, B,
                                   Tq, Tkv, Hq, Hkv, d, causal, scale, stream, done_event)


def gqa_rope_qk(q, k, B, T, Hq, Hkv, d, pos0, theta, stream):
    return lib().gqa_rope_qk(q, k, B, T, Hq, Hkv, d, pos0, theta, stream)


def gqa_rope_decode_q(q, seqlens, B, H, d, theta, stream):
    return lib().gqa_rope_decode_q(q, seqlens, B, H, d, theta, stream)


def gqa_last_error():
    msg = lib().gqa_last_error()
    return msg.decode() if msg else ""


def gqa_device_status(reset):
    return lib().gqa_device_status(reset)


def gqa_selftest_wait_timeout(timeout_us):
    return lib().gqa_selftest_wait_timeout(timeout_us)


def gqa_set_prefill_grid_cap(max_ctas):
    """Cap the persistent prefill grid (testing aid; 0 removes the cap)."""
    lib().gqa_set_prefill_grid_cap(max_ctas)


def gqa_selftest_exp2_poly(x, y, n, stream):
    return lib().gqa_selftest_exp2_poly(x, y, n, stream)
