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


# ---- RoPE fused into the attention kernels' loads ---------------------------

FUSED_PREFILL = [
    # B, Tq, Tkv, Hq, Hkv, d, causal, q_pos0 (None: Tkv - Tq)
    (1, 500, 500, 8, 2, 128, True, None),
    (2, 300, 300, 32, 8, 128, True, None),
    (1, 200, 700, 8, 1, 64, True, None),          # chunk of a longer sequence
    (1, 129, 129, 4, 4, 128, False, 0),           # MHA: one position per row
    (1, 260, 260, 32, 1, 128, True, 1000),        # MQA, offset positions
    (1, 100, 100, 6, 2, 64, True, 31000),         # G = 3 (ragged M tile), long positions
]


@pytest.mark.parametrize("B,Tq,Tkv,Hq,Hkv,d,causal,q_pos0", FUSED_PREFILL)
def test_fused_rope_prefill(gqa_lib, B, Tq, Tkv, Hq, Hkv, d, causal, q_pos0):
    # q rotated as each tile is loaded equals rotating q first (the same bits),
    # and both match the oracle's rotation + attention
    q, k, v = workloads.prefill_inputs(B, Tq, Hq, Hkv, d, Tkv=Tkv, seeds=(Tq, Tkv, Hq + d))
    pos0 = Tkv - Tq if q_pos0 is None else q_pos0
    kr = gqa.rope_(k.cuda(), 0)                           # keys at positions 0..Tkv-1
    qd = q.cuda()
    o, lse = gqa.attn(qd, kr, v.cuda(), causal=causal, return_lse=True, rope_theta=10000.0,
                      q_pos0=pos0)
    gqa.device_status()
    assert torch.equal(qd.cpu(), q)                       # q in memory is not modified
    o2, lse2 = gqa.attn(gqa.rope_(q.cuda(), pos0), kr, v.cuda(), causal=causal, return_lse=True)
    assert torch.equal(o, o2) and torch.equal(lse, lse2)
    qr = bf16_round(ref.rope_tensor(q, pos0))
    kro = bf16_round(ref.rope_tensor(k, 0))
    o_ref, lse_ref = ref.attn_fwd(qr, kro, v, causal=causal)
    assert max_abs(o, o_ref) <= BF16_TOL
    l = lse.cpu().numpy().astype(np.float64)
    fin = np.isfinite(lse_ref)
    assert np.array_equal(np.isneginf(l), ~fin)
    assert np.max(np.abs(l[fin] - lse_ref[fin]), initial=0.0) <= BF16_TOL


def test_fused_rope_prefill_headline_shape(gqa_lib):
    # the B=1, T=4096, 32 / 8 head workload: fused rotation of q against rotating
    # first (bit for bit) and against the oracle on every row
    q, k, v = workloads.prefill_inputs(1, 4096, 32, 8, 128)
    kr = gqa.rope_(k.cuda(), 0)
    o, lse = gqa.attn(q.cuda(), kr, v.cuda(), causal=True, return_lse=True, rope_theta=10000.0)
    gqa.device_status()
    qg = gqa.rope_(q.cuda(), 0)
    o2 = gqa.attn(qg, kr, v.cuda(), causal=True)
    assert torch.equal(o, o2)
    o_ref, lse_ref = ref.attn_fwd(qg.cpu(), kr.cpu(), v, causal=True)
    assert max_abs(o, o_ref) <= BF16_TOL
    assert np.max(np.abs(lse.cpu().numpy() - lse_ref)) <= BF16_TOL


@pytest.mark.parametrize("Hq,Hkv,d", [(32, 8, 128), (8, 1, 64), (32, 1, 128)])
def test_fused_rope_decode(gqa_lib, Hq, Hkv, d):
    lengths = [1, 700, 0, 1025, 3000, 64]
    q, kc, vc, sl = workloads.decode_inputs(len(lengths), Hq, Hkv, d, 1, 3000, lengths=lengths,
                                            seeds=(Hq, Hkv, d, 0))
    qd = q.cuda()
    o = gqa.decode(qd, kc.cuda(), vc.cuda(), sl.cuda(), rope_theta=10000.0)
    gqa.device_status()
    assert torch.equal(qd.cpu(), q)
    o2 = gqa.decode(gqa.rope_decode_q_(q.cuda(), sl.cuda()), kc.cuda(), vc.cuda(), sl.cuda())
    assert torch.equal(o, o2)
    o_ref, _ = ref.decode(bf16_round(ref.rope_decode_q(q, sl)), kc, vc, sl)
    assert max_abs(o, o_ref) <= BF16_TOL
