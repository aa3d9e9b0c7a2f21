"""Split-KV decode with the in-kernel log-sum-exp merge of the splits, against the double oracle (2e-2 max-abs).

Cache rows past each sequence's length are NaN, so any read of them poisons
the output and fails the comparison."""

import numpy as np
import pytest
import torch

import grouped_query_attention_attn_b200 as gqa
from grouped_query_attention_attn_b200 import _binding, workloads
from oracle import ref
from parity import BF16_TOL, max_abs

pytestmark = pytest.mark.gpu


def run_case(B, Hq, Hkv, d, Lmax, lengths, seed=0):
    q, kc, vc, sl = workloads.decode_inputs(B, Hq, Hkv, d, 1, Lmax, lengths=lengths,
                                            seeds=(seed + 1, seed + 2, seed + 3, seed + 4))
    o_ref, _ = ref.decode(q, kc, vc, sl)
    o = gqa.decode(q.cuda(), kc.cuda(), vc.cuda(), sl.cuda())
    gqa.device_status()
    return o, o_ref


@pytest.mark.parametrize("Hq,Hkv,d", [(8, 2, 128), (32, 8, 128), (8, 8, 128), (8, 1, 64),
                                      (16, 1, 128), (32, 1, 128), (12, 4, 64), (24, 1, 128)])
def test_small_ragged(gqa_lib, Hq, Hkv, d):
    # lengths hit: 1 key, a partial 16-key slice, exact stage / split multiples,
    # split boundaries +-1, the full cache and an empty sequence
    lengths = [1, 15, 64, 511, 512, 513, 700, 0, 1025, 129]
    o, o_ref = run_case(len(lengths), Hq, Hkv, d, 1100, lengths, seed=Hq + Hkv + d)
    assert max_abs(o, o_ref) <= BF16_TOL
    assert torch.all(o[7] == 0)


def test_full_size_batched_decode(gqa_lib):
    # B=64, Hq=32, Hkv=8, d=128, L_b uniform on [1024, 8192]: every output row
    q, kc, vc, sl = workloads.decode_inputs(64, 32, 8, 128, 1024, 8192)
    o_ref, _ = ref.decode(q, kc, vc, sl)
    o = gqa.decode(q.cuda(), kc.cuda(), vc.cuda(), sl.cuda())
    gqa.device_status()
    assert max_abs(o, o_ref) <= BF16_TOL


def test_decode_equals_last_row_of_prefill_oracle(gqa_lib):
    # decode of a sequence = the causal forward's newest row over the cache
    B, Hq, Hkv, d, L = 2, 8, 2, 128, 300
    q, kc, vc, sl = workloads.decode_inputs(B, Hq, Hkv, d, L, L, lengths=[L, L])
    o = gqa.decode(q.cuda(), kc.cuda(), vc.cuda(), sl.cuda())
    of, _ = ref.attn_fwd(q[:, None], kc, vc, causal=True)
    assert max_abs(o, of[:, 0]) <= BF16_TOL


def test_repeat_is_deterministic(gqa_lib):
    lengths = [700, 3, 1024]
    q, kc, vc, sl = workloads.decode_inputs(3, 8, 2, 128, 1, 1100, lengths=lengths)
    args = (q.cuda(), kc.cuda(), vc.cuda(), sl.cuda())
    assert torch.equal(gqa.decode(*args), gqa.decode(*args))


def test_length_above_capacity_is_flagged(gqa_lib):
    q, kc, vc, sl = workloads.decode_inputs(2, 8, 2, 128, 1, 200, lengths=[200, 50])
    sl_bad = torch.tensor([250, 50], dtype=torch.int32)
    gqa.decode(q.cuda(), kc.cuda(), vc.cuda(), sl_bad.cuda())
    assert _binding.gqa_device_status(1) == _binding.GQA_ERR_INVALID_ARG
    assert _binding.gqa_device_status(0) == _binding.GQA_OK


def test_undersized_workspace_rejected(gqa_lib):
    q, kc, vc, sl = workloads.decode_inputs(2, 8, 2, 128, 1, 600, lengths=[600, 10])
    need = gqa.decode_workspace_size(2, 8, 2, 128, 600)
    ws = torch.empty(need - 256, dtype=torch.uint8, device="cuda")
    with pytest.raises(ValueError):
        gqa.decode(q.cuda(), kc.cuda(), vc.cuda(), sl.cuda(), workspace=ws)


# ---- the in-kernel merge: arrival words in the workspace --------------------

def test_workspace_garbage_and_reuse_across_shapes(gqa_lib):
    # The last split of each (sequence, KV head) is found with an arrival word
    # in the workspace.  Neither leftover words of other calls (other shapes,
    # other splits counts) nor arbitrary bytes on entry may change the result.
    cases = [(8, 32, 8, 128, 3000, [3000, 1, 2048, 0, 1025, 513, 2999, 64]),
             (5, 8, 2, 64, 1100, [1100, 700, 0, 1, 1024]),
             (3, 32, 1, 128, 5000, [4097, 5000, 1])]
    need = max(gqa.decode_workspace_size(B, Hq, Hkv, d, L) for B, Hq, Hkv, d, L, _ in cases)
    ws = torch.full((need,), 0xFF, dtype=torch.uint8, device="cuda")
    for rep in range(2):
        for i, (B, Hq, Hkv, d, Lmax, lengths) in enumerate(cases):
            q, kc, vc, sl = workloads.decode_inputs(B, Hq, Hkv, d, 1, Lmax, lengths=lengths,
                                                    seeds=(50 + i, 60 + i, 70 + i, 0))
            o_ref, _ = ref.decode(q, kc, vc, sl)
            o = gqa.decode(q.cuda(), kc.cuda(), vc.cuda(), sl.cuda(), workspace=ws)
            gqa.device_status()
            assert max_abs(o, o_ref) <= BF16_TOL, (rep, i)
        if rep == 0:
            ws.random_(0, 256)                   # arbitrary bytes before the second round


def test_cuda_graph_replays_of_one_launch(gqa_lib):
    # A captured launch replays with the same call id; the merging split leaves
    # the word counting from zero, so every replay merges correctly.
    B, Hq, Hkv, d, Lmax = 6, 32, 8, 128, 2100
    lengths = [2100, 1, 1024, 1025, 0, 2048]
    q, kc, vc, sl = workloads.decode_inputs(B, Hq, Hkv, d, 1, Lmax, lengths=lengths)
    qd, kd, vd, sd = q.cuda(), kc.cuda(), vc.cuda(), sl.cuda()
    ws = torch.empty(gqa.decode_workspace_size(B, Hq, Hkv, d, Lmax), dtype=torch.uint8,
                     device="cuda")
    o = torch.empty_like(qd)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        gqa.decode(qd, kd, vd, sd, workspace=ws, out=o)          # warm-up outside capture
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=s):
            gqa.decode(qd, kd, vd, sd, workspace=ws, out=o)
    for rep in range(3):
        qn = workloads.randn((B, Hq, d), 900 + rep)
        qd.copy_(qn)
        o.fill_(float("nan"))
        g.replay()
        torch.cuda.synchronize()
        o_ref, _ = ref.decode(qn, kc, vc, sl)
        assert max_abs(o, o_ref) <= BF16_TOL, rep
    gqa.device_status()


def test_empty_cache_gives_zeros(gqa_lib):
    q = workloads.randn((3, 8, 128), 5).cuda()
    kc = torch.empty((3, 0, 2, 128), dtype=torch.bfloat16, device="cuda")
    sl = torch.zeros(3, dtype=torch.int32, device="cuda")
    o = gqa.decode(q, kc, kc.clone(), sl)
    gqa.device_status()
    assert torch.all(o == 0)
