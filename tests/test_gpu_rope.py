"""RoPE kernel against the oracle rotation, and attention on rotated inputs."""

import numpy as np
import pytest
import torch

import grouped_query_attention_attn_b200 as gqa
from grouped_query_attention_attn_b200 import workloads
from oracle import ref
from parity import BF16_TOL, max_abs

pytestmark = pytest.mark.gpu


def bf16_round(a):
    return torch.from_numpy(np.ascontiguousarray(a)).to(torch.bfloat16)


@pytest.mark.parametrize("B,T,H,d,pos0,theta", [(2, 100, 4, 128, 0, 10000.0),
                                                (1, 33, 8, 64, 4000, 10000.0),
                                                (1, 16, 2, 8, 7, 500.0),
                                                (1, 64, 1, 256, 32000, 1e6)])
def test_rope_matches_oracle(gqa_lib, B, T, H, d, pos0, theta):
    x = workloads.randn((B, T, H, d), T + d)
    want = ref.rope_tensor(x, pos0, theta)
    got = gqa.rope_(x.cuda(), pos0, theta)
    # the GPU rounds its fp32 rotation to bf16; the oracle is exact: half a bf16 ulp
    rel = np.abs(got.float().cpu().numpy() - want) / np.maximum(np.abs(want), 1e-30)
    assert np.max(np.where(np.abs(want) > 1e-3, rel, 0.0)) <= 2.0 ** -8
    # and the bf16 roundings agree almost everywhere
    assert (got.cpu() == bf16_round(want)).float().mean() > 0.99


@pytest.mark.parametrize("B,T,Hq,Hkv,d,pos0", [(2, 77, 8, 2, 128, 0), (1, 300, 32, 8, 128, 9000),
                                              (3, 5, 3, 1, 24, 11), (1, 9, 20, 4, 64, 3)])
def test_rope_qk_matches_oracle(gqa_lib, B, T, Hq, Hkv, d, pos0):
    q = workloads.randn((B, T, Hq, d), 40 + T)
    k = workloads.randn((B, T, Hkv, d), 41 + T)
    gq, gk = gqa.rope_qk_(q.cuda(), k.cuda(), pos0)
    for got, x in ((gq, q), (gk, k)):
        want = ref.rope_tensor(x, pos0, 10000.0)
        rel = np.abs(got.float().cpu().numpy() - want) / np.maximum(np.abs(want), 1e-30)
        assert np.max(np.where(np.abs(want) > 1e-3, rel, 0.0)) <= 2.0 ** -8
    # one launch over q and k gives the same bits as two separate rotations
    assert torch.equal(gq.cpu(), gqa.rope_(q.cuda(), pos0).cpu())
    assert torch.equal(gk.cpu(), gqa.rope_(k.cuda(), pos0).cpu())


def test_rope_position_zero_is_identity(gqa_lib):
    x = workloads.randn((1, 1, 4, 128), 3)
    assert torch.equal(gqa.rope_(x.cuda(), 0).cpu(), x)


def test_rope_decode_q(gqa_lib):
    q = workloads.randn((4, 8, 128), 5)
    sl = torch.tensor([1, 100, 4096, 0], dtype=torch.int32)
    want = ref.rope_decode_q(q, sl)
    got = gqa.rope_decode_q_(q.cuda(), sl.cuda()).float().cpu().numpy()
    assert np.max(np.abs(got - want)) <= 0.02


def test_attention_with_rope(gqa_lib):
    # q, k rotated on the GPU, then the tcgen05 prefill; the oracle rotates in
    # double, stores bf16 (as the GPU does) and runs its attention
    B, T, Hq, Hkv, d = 1, 500, 8, 2, 128
    q, k, v = workloads.prefill_inputs(B, T, Hq, Hkv, d, seeds=(91, 92, 93))
    qr, kr = bf16_round(ref.rope_tensor(q, 0)), bf16_round(ref.rope_tensor(k, 0))
    o_ref, _ = ref.attn_fwd(qr, kr, v, causal=True)
    qg, kg = gqa.rope_(q.cuda(), 0), gqa.rope_(k.cuda(), 0)
    o = gqa.attn(qg, kg, v.cuda(), causal=True)
    assert max_abs(o, o_ref) <= BF16_TOL


def test_rope_qk_headline_shape(gqa_lib):
    # q and k of the B=1, T=4096, 32 / 8 head workload, one launch, positions 0..4095
    q, k, _ = workloads.prefill_inputs(1, 4096, 32, 8, 128)
    gq, gk = gqa.rope_qk_(q.cuda(), k.cuda(), 0)
    for got, x in ((gq, q), (gk, k)):
        want = ref.rope_tensor(x, 0)
        rel = np.abs(got.float().cpu().numpy() - want) / np.maximum(np.abs(want), 1e-30)
        assert np.max(np.where(np.abs(want) > 1e-3, rel, 0.0)) <= 2.0 ** -8
