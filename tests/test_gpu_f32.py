"""fp32 path against the double oracle (tolerance 1e-4 max-abs)."""

import numpy as np
import pytest
import torch

import grouped_query_attention_attn_b200 as gqa
from grouped_query_attention_attn_b200 import workloads
from oracle import ref
from parity import F32_TOL, max_abs

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("factor", [1.0, 1000.0])
def test_tiny_lcg_workload(gqa_lib, factor):
    # B=1, Hq=8, Hkv=2, T=16, d=16, no mask; LCG inputs; rerun with q, k x 1000
    q, k, v = workloads.tiny_f32_inputs(qk_factor=factor)
    o_ref, lse_ref = ref.attn_fwd(q, k, v, causal=False)
    o, lse = gqa.attn_f32(q.cuda(), k.cuda(), v.cuda(), causal=False, return_lse=True)
    assert max_abs(o, o_ref) <= F32_TOL
    if factor == 1.0:
        assert max_abs(lse, lse_ref) <= F32_TOL
    else:
        # lse ~ 1e5 here: compare relative to its magnitude
        assert np.allclose(lse.cpu().numpy(), lse_ref, rtol=1e-6, atol=0)


@pytest.mark.parametrize("B,Tq,Tkv,Hq,Hkv,d", [
    (2, 33, 33, 8, 2, 16), (1, 70, 70, 4, 4, 128), (2, 65, 130, 6, 3, 33),
    (1, 130, 65, 4, 1, 256), (1, 1, 77, 2, 1, 64), (3, 17, 17, 12, 4, 8)])
@pytest.mark.parametrize("causal", [False, True])
def test_random_shapes(gqa_lib, B, Tq, Tkv, Hq, Hkv, d, causal):
    g = torch.Generator().manual_seed(B * 1000 + Tq + Hq + d)
    q = torch.randn((B, Tq, Hq, d), generator=g)
    k = torch.randn((B, Tkv, Hkv, d), generator=g)
    v = torch.randn((B, Tkv, Hkv, d), generator=g)
    o_ref, lse_ref = ref.attn_fwd(q, k, v, causal)
    o, lse = gqa.attn_f32(q.cuda(), k.cuda(), v.cuda(), causal=causal, return_lse=True)
    assert max_abs(o, o_ref) <= F32_TOL
    fin = np.isfinite(lse_ref)
    l = lse.cpu().numpy()
    assert np.array_equal(np.isneginf(l), ~fin)
    assert np.max(np.abs(l[fin] - lse_ref[fin])) <= F32_TOL


def test_empty_keys(gqa_lib):
    q = torch.randn(1, 5, 4, 16, device="cuda")
    k = torch.empty(1, 0, 2, 16, device="cuda")
    o, lse = gqa.attn_f32(q, k, k.clone(), causal=False, return_lse=True)
    assert torch.all(o == 0) and torch.all(torch.isneginf(lse))
