"""ctypes wrappers around the double-precision C oracle, plus the tensor fold.

TEST INFRASTRUCTURE ONLY: imported by ``tests/``, ``__graft_entry__.smoke()``
and the CPU-baseline leg of ``bench.py``; never by the product path.

The C source (``gqa_oracle.c``) is compiled with the host gcc into
``oracle/_build/liboracle.so`` on first use (or by ``build_oracle()``).
No fast-math flags: the oracle keeps IEEE double semantics.
"""

import ctypes
import math
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gqa_oracle.c")
_OUT_DIR = os.path.join(_HERE, "_build")
_LIB_PATH = os.path.join(_OUT_DIR, "liboracle.so")
_lib = None


def build_oracle(force=False):
    """Compile the C oracle with gcc -O2 -fopenmp (no fast-math).  Returns the .so path."""
    os.makedirs(_OUT_DIR, exist_ok=True)
    stale = (not os.path.exists(_LIB_PATH)
             or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC))
    if force or stale:
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-fno-fast-math", "-fopenmp", "-fPIC", "-shared",
               "-std=c11", "-Wall", "-Wextra", "-o", tmp, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is not None:
        return _lib
    lib = ctypes.CDLL(build_oracle())
    dp = ctypes.POINTER(ctypes.c_double)
    fp = ctypes.POINTER(ctypes.c_float)
    L = ctypes.c_long
    lib.oracle_attn_fwd.argtypes = [fp, fp, fp, dp, dp, L, L, L, L, L, L,
                                    ctypes.c_int, ctypes.c_double, ctypes.c_int]
    lib.oracle_attn_fwd_rows.argtypes = [fp, fp, fp, ctypes.POINTER(ctypes.c_int64), L,
                                         dp, dp, L, L, L, L, L, L,
                                         ctypes.c_int, ctypes.c_double, ctypes.c_int]
    lib.oracle_decode.argtypes = [fp, fp, fp, ctypes.POINTER(ctypes.c_int32), dp, dp,
                                  L, L, L, L, L, ctypes.c_double, ctypes.c_int]
    lib.oracle_decode_split.argtypes = [fp, fp, fp, ctypes.POINTER(ctypes.c_int32), dp, dp,
                                        L, L, L, L, L, ctypes.c_double, L, ctypes.c_int]
    lib.oracle_attn_fwd_window.argtypes = [fp, fp, fp, dp, dp, L, L, L, L, L, L, L, L,
                                           ctypes.c_double, ctypes.c_int]
    lib.oracle_decode_window.argtypes = [fp, fp, fp, ctypes.POINTER(ctypes.c_int32), dp, dp,
                                         L, L, L, L, L, L, L, ctypes.c_double, ctypes.c_int]
    for f in (lib.oracle_attn_fwd, lib.oracle_attn_fwd_rows, lib.oracle_decode,
              lib.oracle_decode_split, lib.oracle_num_threads, lib.oracle_attn_fwd_window,
              lib.oracle_decode_window):
        f.restype = ctypes.c_int
    _lib = lib
    return lib


def num_threads():
    """OpenMP threads the oracle uses by default on this host."""
    return int(_load().oracle_num_threads())


def _f32(x):
    """Exact float32 copy of a torch tensor (bf16/fp32) or array, C-contiguous."""
    if hasattr(x, "detach"):
        x = x.detach().to("cpu")
        import torch
        x = x.to(torch.float32).numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.float32))


def _ptr(a, ctype):
    return a.ctypes.data_as(ctypes.POINTER(ctype))


def _default_scale(d, scale):
    return 1.0 / math.sqrt(d) if scale is None else float(scale)


def attn_fwd(q, k, v, causal, scale=None, threads=0):
    """Full forward.  q:[B,Tq,Hq,d], k,v:[B,Tkv,Hkv,d] -> (o [B,Tq,Hq,d] f64, lse [B,Hq,Tq] f64)."""
    q, k, v = _f32(q), _f32(k), _f32(v)
    B, Tq, Hq, d = q.shape
    _, Tkv, Hkv, _ = k.shape
    o = np.empty((B, Tq, Hq, d), np.float64)
    lse = np.empty((B, Hq, Tq), np.float64)
    rc = _load().oracle_attn_fwd(_ptr(q, ctypes.c_float), _ptr(k, ctypes.c_float),
                                 _ptr(v, ctypes.c_float), _ptr(o, ctypes.c_double),
                                 _ptr(lse, ctypes.c_double), B, Tq, Tkv, Hq, Hkv, d,
                                 int(bool(causal)), _default_scale(d, scale), threads)
    if rc != 0:
        raise ValueError("invalid shape for the oracle (Hq must be a multiple of Hkv)")
    return o, lse


def attn_fwd_window(q, k, v, window, sinks=0, scale=None, threads=0):
    """Causal forward with a sliding window and sink keys -> (o, lse) as attn_fwd."""
    q, k, v = _f32(q), _f32(k), _f32(v)
    B, Tq, Hq, d = q.shape
    _, Tkv, Hkv, _ = k.shape
    o = np.empty((B, Tq, Hq, d), np.float64)
    lse = np.empty((B, Hq, Tq), np.float64)
    rc = _load().oracle_attn_fwd_window(_ptr(q, ctypes.c_float), _ptr(k, ctypes.c_float),
                                        _ptr(v, ctypes.c_float), _ptr(o, ctypes.c_double),
                                        _ptr(lse, ctypes.c_double), B, Tq, Tkv, Hq, Hkv, d,
                                        int(window), int(sinks), _default_scale(d, scale), threads)
    if rc != 0:
        raise ValueError("invalid shape, window or sinks for the oracle")
    return o, lse


def decode_window(q, k_cache, v_cache, seqlens, window, sinks=0, scale=None, threads=0):
    """Decode with a sliding window and sink keys -> (o [B,Hq,d], lse [B,Hq])."""
    q, kc, vc = _f32(q), _f32(k_cache), _f32(v_cache)
    if hasattr(seqlens, "detach"):
        seqlens = seqlens.detach().cpu().numpy()
    sl = np.ascontiguousarray(np.asarray(seqlens, dtype=np.int32))
    B, Hq, d = q.shape
    _, Lmax, Hkv, _ = kc.shape
    o = np.empty((B, Hq, d), np.float64)
    lse = np.empty((B, Hq), np.float64)
    rc = _load().oracle_decode_window(_ptr(q, ctypes.c_float), _ptr(kc, ctypes.c_float),
                                      _ptr(vc, ctypes.c_float), _ptr(sl, ctypes.c_int32),
                                      _ptr(o, ctypes.c_double), _ptr(lse, ctypes.c_double),
                                      B, Hq, Hkv, d, Lmax, int(window), int(sinks),
                                      _default_scale(d, scale), threads)
    if rc != 0:
        raise ValueError("invalid shape, length, window or sinks for the oracle")
    return o, lse


def attn_fwd_rows(q, k, v, rows, causal, scale=None, threads=0):
    """Rows given as flat indices (b*Hq + hq)*Tq + i -> (o [n,d] f64, lse [n] f64)."""
    q, k, v = _f32(q), _f32(k), _f32(v)
    B, Tq, Hq, d = q.shape
    _, Tkv, Hkv, _ = k.shape
    rows = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
    o = np.empty((rows.size, d), np.float64)
    lse = np.empty((rows.size,), np.float64)
    rc = _load().oracle_attn_fwd_rows(_ptr(q, ctypes.c_float), _ptr(k, ctypes.c_float),
                                      _ptr(v, ctypes.c_float), _ptr(rows, ctypes.c_int64),
                                      rows.size, _ptr(o, ctypes.c_double),
                                      _ptr(lse, ctypes.c_double), B, Tq, Tkv, Hq, Hkv, d,
                                      int(bool(causal)), _default_scale(d, scale), threads)
    if rc != 0:
        raise ValueError("invalid shape or row index for the oracle")
    return o, lse


def decode(q, k_cache, v_cache, seqlens, scale=None, threads=0, chunk=None):
    """q:[B,Hq,d], caches:[B,Lmax,Hkv,d], seqlens:[B] -> (o [B,Hq,d] f64, lse [B,Hq] f64).

    With ``chunk`` the result is computed split by split and merged through
    the log-sum-exp identity instead of in one pass.
    """
    q, kc, vc = _f32(q), _f32(k_cache), _f32(v_cache)
    if hasattr(seqlens, "detach"):
        seqlens = seqlens.detach().cpu().numpy()
    sl = np.ascontiguousarray(np.asarray(seqlens, dtype=np.int32))
    B, Hq, d = q.shape
    _, Lmax, Hkv, _ = kc.shape
    o = np.empty((B, Hq, d), np.float64)
    lse = np.empty((B, Hq), np.float64)
    args = [_ptr(q, ctypes.c_float), _ptr(kc, ctypes.c_float), _ptr(vc, ctypes.c_float),
            _ptr(sl, ctypes.c_int32), _ptr(o, ctypes.c_double), _ptr(lse, ctypes.c_double),
            B, Hq, Hkv, d, Lmax, _default_scale(d, scale)]
    if chunk is None:
        rc = _load().oracle_decode(*args, threads)
    else:
        rc = _load().oracle_decode_split(*args, int(chunk), threads)
    if rc != 0:
        raise ValueError("invalid shape or sequence length for the oracle")
    return o, lse


def fold_kv_tensor(kv, g):
    """Fold the head axis of a [B,T,H,d] bf16 K or V tensor to ``g`` heads.

    TT Lab "キー・バリューヘッドだけ減らしてみる", step 2: position-wise mean over
    contiguous slices of H/g heads.  Reading for bf16 tensors: the members of
    a group are added in head order in float32, the sum divided by the group
    size in float32, and the result rounded to bf16 (round to nearest even).
    Returns a bf16 torch tensor [B,T,g,d].
    """
    import torch
    x = _f32(kv)
    B, T, H, d = x.shape
    if g <= 0 or H % g != 0:
        raise ValueError(f"{g} groups do not divide {H} heads evenly")
    size = H // g
    out = np.empty((B, T, g, d), np.float32)
    for grp in range(g):
        acc = x[:, :, grp * size, :].copy()
        for m in range(1, size):
            acc = acc + x[:, :, grp * size + m, :]        # float32 adds, head order
        out[:, :, grp, :] = acc / np.float32(size)
    return torch.from_numpy(out).to(torch.bfloat16)


def rope_tensor(x, pos0, theta=10000.0):
    """RoPE of a [B, T, H, d] tensor with row t at position pos0 + t, in double.

    Course "Неделя 7. Внимание", step 3: pair (2i, 2i+1) rotated by
    m * theta ** (-2i / d).  Returns a float64 numpy array."""
    x = _f32(x).astype(np.float64)
    B, T, H, d = x.shape
    if d % 2:
        raise ValueError("head dim must be even for RoPE")
    m = (pos0 + np.arange(T, dtype=np.float64))[:, None]          # [T, 1]
    inv = theta ** (-2.0 * np.arange(d // 2, dtype=np.float64) / d)  # [d/2]
    ang = m * inv[None, :]                                          # [T, d/2]
    c = np.cos(ang)[None, :, None, :]
    s = np.sin(ang)[None, :, None, :]
    a, b = x[..., 0::2], x[..., 1::2]
    out = np.empty_like(x)
    out[..., 0::2] = a * c - b * s
    out[..., 1::2] = a * s + b * c
    return out


def rope_decode_q(q, seqlens, theta=10000.0):
    """RoPE of decode queries [B, H, d]: sequence b's token sits at position
    max(seqlens[b] - 1, 0) (reading: with an empty cache the new token is the
    first one, position 0)."""
    q = _f32(q).astype(np.float64)
    if hasattr(seqlens, "detach"):
        seqlens = seqlens.detach().cpu().numpy()
    out = np.empty_like(q)
    for b in range(q.shape[0]):
        out[b] = rope_tensor(q[b][None, None], max(int(seqlens[b]) - 1, 0), theta)[0, 0]
    return out


def attn_bwd(q, k, v, do, causal, scale=None, window=0, sinks=0):
    """Gradients of the attention output with respect to q, k and v, in float64.

    The forward is the plain definition, written with torch CPU ops: K and V
    expanded to the query heads by repeat_interleave (K3 notes, "GVA",
    "Forward: repeat_interleave"), scores scaled by ``scale``, masked with -inf
    before the softmax, weighted sum of V.  torch autograd supplies the chain
    rule, so the expanded heads' gradients are summed back into each shared K/V
    head ("Backward: view + sum": the gradient of a copy is a sum, not a mean).
    Returns (dq [B,Tq,Hq,d], dk, dv [B,Tkv,Hkv,d]) as float64 numpy arrays.
    """
    import torch
    qd = torch.from_numpy(_f32(q).astype(np.float64)).requires_grad_(True)
    kd = torch.from_numpy(_f32(k).astype(np.float64)).requires_grad_(True)
    vd = torch.from_numpy(_f32(v).astype(np.float64)).requires_grad_(True)
    dod = torch.from_numpy(_f32(do).astype(np.float64))
    B, Tq, Hq, d = qd.shape
    Tkv, Hkv = kd.shape[1], kd.shape[2]
    if Hq % Hkv != 0:
        raise ValueError("Hq must be a multiple of Hkv")
    G = Hq // Hkv
    sc = 1.0 / math.sqrt(d) if scale is None else float(scale)
    ke = kd.repeat_interleave(G, dim=2)                     # [B, Tkv, Hq, d]
    ve = vd.repeat_interleave(G, dim=2)
    s = torch.einsum("bihc,bjhc->bhij", qd, ke) * sc
    i = torch.arange(Tq)[:, None]
    j = torch.arange(Tkv)[None, :]
    p_pos = i + (Tkv - Tq)
    vis = torch.ones(Tq, Tkv, dtype=torch.bool)
    if causal:
        vis &= j <= p_pos
        if window > 0:
            vis &= (j > p_pos - window) | (j < sinks)
    s = s.masked_fill(~vis, float("-inf"))
    m = s.amax(dim=-1, keepdim=True)
    m = torch.where(torch.isfinite(m), m, torch.zeros_like(m))   # rows with no key
    e = torch.exp(s - m)
    den = e.sum(dim=-1, keepdim=True)
    p = e / torch.where(den > 0, den, torch.ones_like(den))
    o = torch.einsum("bhij,bjhc->bihc", p, ve)
    o.backward(dod)
    return qd.grad.numpy(), kd.grad.numpy(), vd.grad.numpy()
