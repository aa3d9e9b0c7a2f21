"""Seeded synthetic inputs for the attention workloads.

This module only draws numbers and lays them out; it holds none of the
method's arithmetic (no scores, softmax or head folding).  Both the CUDA path
and the CPU oracle consume exactly the tensors it returns.

Recipes
-------
* tiny_f32 -- B=1, Hq=8, Hkv=2, T=16, d=16, fp32, no mask.  Values come from
  the integer-state linear congruential generator of TT Lab
  "キー・バリューヘッドだけ減らしてみる" (step 1: state = (a*state + c) % m, value
  state/m - 0.5) with the published constants a=1664525, c=1013904223,
  m=2**32 (the page prints none), seeds 101/202/303 for q/k/v as in the lab's
  sample (step 8), drawn head by head, row by row, column by column and then
  placed in the [B, T, H, d] layout.  The huge-logit variant multiplies q and
  k by 1000 in float32.
* every bf16 workload -- torch's CPU generator, seeded per tensor (q=1, k=2,
  v=3, lengths=4), N(0,1) drawn in float32, optionally scaled, then rounded to
  bf16 (round to nearest even).
* decode -- per-sequence lengths uniform on the closed range [Lmin, Lmax]; the
  cache rows of sequence b at positions >= L_b are NaN so that any read past
  the end poisons the result.  Valid rows are drawn sequence by sequence.
"""

import numpy as np
import torch

LCG_A = 1664525
LCG_C = 1013904223
LCG_M = 2 ** 32

SEED_Q, SEED_K, SEED_V, SEED_LEN = 1, 2, 3, 4

# name -> shape parameters (the five workloads the benchmark and tests use)
WORKLOADS = {
    "tiny_f32": dict(B=1, Hq=8, Hkv=2, T=16, d=16, causal=False, dtype="f32"),
    "prefill_causal_llama3_8b_t4096": dict(B=1, Hq=32, Hkv=8, T=4096, d=128,
                                           causal=True, dtype="bf16"),
    "head_sharing_sweep_t2048": dict(B=4, Hq=32, Hkv=(32, 8, 1), T=2048, d=128,
                                     causal=True, dtype="bf16"),
    "decode_b64_l1024_8192": dict(B=64, Hq=32, Hkv=8, d=128, Lmin=1024, Lmax=8192,
                                  dtype="bf16"),
    "prefill_causal_long_t32768": dict(B=1, Hq=64, Hkv=8, T=32768, d=128, causal=True,
                                       qk_std=8.0, dtype="bf16"),
}


def lcg_heads(count, rows, dim, seed):
    """[count, rows, dim] float64 values state/m - 0.5 from the lab's LCG."""
    out = np.empty(count * rows * dim, dtype=np.float64)
    state = seed % LCG_M
    for n in range(out.size):
        state = (LCG_A * state + LCG_C) % LCG_M
        out[n] = state / LCG_M - 0.5
    return out.reshape(count, rows, dim)


def tiny_f32_inputs(qk_factor=1.0, B=1, Hq=8, Hkv=2, T=16, d=16, seeds=(101, 202, 303)):
    """fp32 q [B,T,Hq,d], k/v [B,T,Hkv,d] from the LCG; q and k times ``qk_factor`` in fp32."""
    def draw(count, seed):
        heads = lcg_heads(count * B, T, d, seed).reshape(B, count, T, d)
        return torch.from_numpy(np.ascontiguousarray(heads.transpose(0, 2, 1, 3))).float()
    q, k, v = draw(Hq, seeds[0]), draw(Hkv, seeds[1]), draw(Hkv, seeds[2])
    if qk_factor != 1.0:
        f = torch.tensor(qk_factor, dtype=torch.float32)
        q, k = q * f, k * f
    return q.contiguous(), k.contiguous(), v.contiguous()


def randn(shape, seed, std=1.0, dtype=torch.bfloat16):
    """N(0, std^2) drawn in float32 from a seeded CPU generator, then cast."""
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    x = torch.randn(shape, generator=g, dtype=torch.float32)
    if std != 1.0:
        x = x * torch.tensor(std, dtype=torch.float32)
    return x.to(dtype)


def prefill_inputs(B, T, Hq, Hkv, d, qk_std=1.0, Tkv=None, dtype=torch.bfloat16,
                   seeds=(SEED_Q, SEED_K, SEED_V)):
    """q [B,T,Hq,d], k/v [B,Tkv,Hkv,d] on the CPU."""
    Tkv = T if Tkv is None else Tkv
    q = randn((B, T, Hq, d), seeds[0], qk_std, dtype)
    k = randn((B, Tkv, Hkv, d), seeds[1], qk_std, dtype)
    v = randn((B, Tkv, Hkv, d), seeds[2], 1.0, dtype)
    return q, k, v


def decode_lengths(B, Lmin, Lmax, seed=SEED_LEN):
    """int32 [B], uniform on the closed range [Lmin, Lmax]."""
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    return torch.randint(Lmin, Lmax + 1, (B,), generator=g, dtype=torch.int64).to(torch.int32)


def decode_inputs(B, Hq, Hkv, d, Lmin, Lmax, pad=float("nan"), dtype=torch.bfloat16,
                  seeds=(SEED_Q, SEED_K, SEED_V, SEED_LEN), lengths=None):
    """q [B,Hq,d], k_cache/v_cache [B,Lmax,Hkv,d] (rows >= L_b hold ``pad``), seqlens int32 [B]."""
    seqlens = decode_lengths(B, Lmin, Lmax, seeds[3]) if lengths is None else \
        torch.as_tensor(lengths, dtype=torch.int32)
    q = randn((B, Hq, d), seeds[0], 1.0, dtype)
    caches = []
    for seed in (seeds[1], seeds[2]):
        cache = torch.full((B, Lmax, Hkv, d), pad, dtype=dtype)
        g = torch.Generator(device="cpu")
        g.manual_seed(seed)
        for b in range(B):
            L = int(seqlens[b])
            if L > 0:
                cache[b, :L] = torch.randn((L, Hkv, d), generator=g,
                                           dtype=torch.float32).to(dtype)
        caches.append(cache)
    return q, caches[0], caches[1], seqlens
