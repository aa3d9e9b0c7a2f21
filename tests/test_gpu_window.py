"""Sliding window + attention sinks on the GPU against the double oracle (2e-2 max-abs)."""

import numpy as np
import pytest
import torch

import grouped_query_attention_attn_b200 as gqa
from grouped_query_attention_attn_b200 import workloads
from oracle import ref
from parity import BF16_TOL, max_abs

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("B,Tq,Tkv,Hq,Hkv,d,window,sinks", [
    (1, 300, 300, 8, 2, 128, 64, 0),       # window narrower than a key tile
    (1, 700, 700, 8, 2, 128, 200, 4),      # window across tiles, a few sinks
    (2, 520, 520, 8, 8, 128, 128, 130),    # MHA, sinks spanning more than a tile
    (1, 400, 400, 32, 1, 64, 300, 1),      # MQA, d = 64
    (1, 250, 600, 12, 4, 128, 100, 16),    # Tq < Tkv, G = 3
    (1, 600, 250, 8, 2, 128, 50, 8),       # Tq > Tkv: early rows see nothing
    (1, 1, 900, 4, 2, 128, 129, 3),        # a single query row
    (1, 130, 130, 4, 1, 128, 1, 0),        # window 1: each row sees itself
])
def test_prefill_window(gqa_lib, B, Tq, Tkv, Hq, Hkv, d, window, sinks):
    q, k, v = workloads.prefill_inputs(B, Tq, Hq, Hkv, d, Tkv=Tkv, seeds=(window, sinks + 1, Tq))
    o_ref, lse_ref = ref.attn_fwd_window(q, k, v, window, sinks)
    o, lse = gqa.attn(q.cuda(), k.cuda(), v.cuda(), causal=True, return_lse=True,
                      window=window, sinks=sinks)
    gqa.device_status()
    assert max_abs(o, o_ref) <= BF16_TOL
    fin = np.isfinite(lse_ref)
    l = lse.cpu().numpy().astype(np.float64)
    assert np.array_equal(np.isneginf(l), ~fin)
    assert np.max(np.abs(l[fin] - lse_ref[fin]), initial=0.0) <= BF16_TOL


def test_prefill_window_long(gqa_lib):
    # a long sequence with a realistic window: only window / sink tiles are read
    q, k, v = workloads.prefill_inputs(1, 8192, 8, 2, 128, seeds=(71, 72, 73))
    o_ref, _ = ref.attn_fwd_window(q, k, v, 1024, 4)
    o = gqa.attn(q.cuda(), k.cuda(), v.cuda(), causal=True, window=1024, sinks=4)
    assert max_abs(o, o_ref) <= BF16_TOL


def test_wide_window_equals_causal(gqa_lib):
    q, k, v = workloads.prefill_inputs(1, 333, 8, 2, 128, seeds=(81, 82, 83))
    args = (q.cuda(), k.cuda(), v.cuda())
    assert torch.equal(gqa.attn(*args, causal=True), gqa.attn(*args, causal=True, window=333))


# windows that take 512-, 768- and 1024-key splits (Lmax = 3000)
@pytest.mark.parametrize("Hq,Hkv,window,sinks", [(8, 2, 300, 0), (32, 8, 1000, 4),
                                                 (8, 1, 64, 2000), (16, 2, 1, 1), (8, 2, 2100, 3),
                                                 (8, 2, 4000, 2)])
def test_decode_window(gqa_lib, Hq, Hkv, window, sinks):
    lengths = [1, 15, 700, 1023, 1024, 1025, 2500, 0, 3000, 129]
    q, kc, vc, sl = workloads.decode_inputs(len(lengths), Hq, Hkv, 128, 1, 3000, lengths=lengths,
                                            seeds=(window, sinks + 3, Hq, 0))
    o_ref, _ = ref.decode_window(q, kc, vc, sl, window, sinks)
    o = gqa.decode(q.cuda(), kc.cuda(), vc.cuda(), sl.cuda(), window=window, sinks=sinks)
    gqa.device_status()
    assert max_abs(o, o_ref) <= BF16_TOL


# ----------------------------------------------------- bench workload sizes --

def test_prefill_window_bench_workload(gqa_lib):
    # B=1, Hq=32, Hkv=8, T=16384, W=4096, 4 sinks, the inputs the bench times.
    # The oracle computes blocks of query rows [i0, i1) against keys [0, i1):
    # with bottom-right alignment those rows see exactly what they see in the
    # full problem (the start, the first rows past the window, the middle, the end).
    T, W, S = 16384, 4096, 4
    q, k, v = workloads.prefill_inputs(1, T, 32, 8, 128, seeds=(11, 12, 13))
    o, lse = gqa.attn(q.cuda(), k.cuda(), v.cuda(), causal=True, return_lse=True, window=W,
                      sinks=S)
    gqa.device_status()
    assert bool(torch.isfinite(o).all())
    for i0, i1 in ((0, 128), (W - 64, W + 128), (8128, 8256), (T - 128, T)):
        o_ref, lse_ref = ref.attn_fwd_window(q[:, i0:i1], k[:, :i1], v[:, :i1], W, S)
        assert max_abs(o[:, i0:i1], o_ref) <= BF16_TOL
        assert max_abs(lse[:, :, i0:i1], lse_ref) <= BF16_TOL


def test_decode_window_bench_workload(gqa_lib):
    # the batched-decode workload (B=64, Hq=32, Hkv=8, L ~ U{1024..8192}, NaN
    # padding) with W=2048 and 4 sinks: every output row
    q, kc, vc, sl = workloads.decode_inputs(64, 32, 8, 128, 1024, 8192)
    o_ref, _ = ref.decode_window(q, kc, vc, sl, 2048, 4)
    o = gqa.decode(q.cuda(), kc.cuda(), vc.cuda(), sl.cuda(), window=2048, sinks=4)
    gqa.device_status()
    assert max_abs(o, o_ref) <= BF16_TOL
