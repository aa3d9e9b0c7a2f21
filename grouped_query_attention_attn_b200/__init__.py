"""Grouped-query scaled-dot-product attention for NVIDIA B200 (sm_100a).

The computation lives in the C-ABI library ``libgqa.so`` (declared in
``include/gqa.h``): a tcgen05/TMEM/TMA prefill kernel (causal, full, sliding
window with sinks, and a host-buffer entry point that pipelines the copies),
a split-KV decode kernel whose last split per group merges the splits (log-sum-exp), the tcgen05 backward
(dQ, dK, dV), in-place RoPE, an fp32 path and a head-folding kernel.
This package is its Python binding; PyTorch is used for device memory and
streams only.  The library is loaded on first use and there is no CPU
fallback: a missing or unloadable library raises.
"""

from .api import (attn, attn_bwd, attn_bwd_workspace_size, attn_f32, attn_host, decode, decode_workspace_size, device_status, fold_kv,  # noqa: F401
                  host_staging, rope_, rope_decode_q_, rope_qk_)
