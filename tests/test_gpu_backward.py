"""Backward kernels (dq, dk, dv) against the float64 autograd oracle.

Tolerance: the kernels round P and dS to bf16 before the tensor-core products
(2^-9 relative each) and write bf16 gradients; gradients grow with the number
of rows summed, so the bound is relative to the tensor's largest magnitude:
max |gpu - ref| <= 2e-2 * max(1, max |ref|).
"""

import numpy as np
import pytest
import torch

import grouped_query_attention_attn_b200 as gqa
from grouped_query_attention_attn_b200 import workloads
from oracle import ref

pytestmark = pytest.mark.gpu


def rel_err(gpu, want):
    g = gpu.float().cpu().numpy().astype(np.float64)
    assert np.all(np.isfinite(g))
    return float(np.max(np.abs(g - want))) / max(1.0, float(np.max(np.abs(want))))


@pytest.mark.parametrize("B,Tq,Tkv,Hq,Hkv,d,causal,window,sinks", [
    (1, 128, 128, 4, 1, 128, True, 0, 0),
    (2, 200, 200, 8, 2, 128, True, 0, 0),       # ragged tails, G = 4
    (1, 150, 150, 8, 8, 64, False, 0, 0),       # MHA, non-causal, d = 64
    (1, 100, 260, 6, 2, 128, True, 0, 0),       # Tq < Tkv
    (1, 260, 100, 4, 2, 128, True, 0, 0),       # Tq > Tkv: rows with no key
    (1, 300, 300, 8, 2, 128, True, 64, 3),      # sliding window with sinks
    (1, 96, 96, 32, 1, 128, True, 0, 0),        # MQA
    (2, 333, 333, 16, 2, 64, True, 100, 2),     # d = 64, G = 8, window + sinks, ragged
    (1, 513, 700, 12, 4, 128, True, 0, 0),      # G = 3: 126 real rows per M tile, Tq < Tkv
    (3, 64, 64, 4, 1, 64, False, 0, 0),         # B = 3, one M tile each, non-causal
])
def test_backward_matches_oracle(gqa_lib, B, Tq, Tkv, Hq, Hkv, d, causal, window, sinks):
    q, k, v = workloads.prefill_inputs(B, Tq, Hq, Hkv, d, Tkv=Tkv, seeds=(Tq, Tkv + 1, Hq + d))
    dout = workloads.randn((B, Tq, Hq, d), 77)
    qc, kc, vc = q.cuda(), k.cuda(), v.cuda()
    if window:
        o, lse = gqa.attn(qc, kc, vc, causal=True, return_lse=True, window=window, sinks=sinks)
    else:
        o, lse = gqa.attn(qc, kc, vc, causal=causal, return_lse=True)
    dq, dk, dv = gqa.attn_bwd(qc, kc, vc, o, lse, dout.cuda(), causal=causal,
                              window=window or None, sinks=sinks)
    gqa.device_status()
    rq, rk, rv = ref.attn_bwd(q, k, v, dout, causal, window=window, sinks=sinks)
    assert rel_err(dq, rq) <= 2e-2
    assert rel_err(dk, rk) <= 2e-2
    assert rel_err(dv, rv) <= 2e-2


def test_backward_shared_head_sum(gqa_lib):
    # GQA gradients equal the expanded-MHA gradients summed over each group
    B, T, Hq, Hkv, d = 1, 256, 8, 2, 128
    G = Hq // Hkv
    q, k, v = workloads.prefill_inputs(B, T, Hq, Hkv, d, seeds=(5, 6, 7))
    dout = workloads.randn((B, T, Hq, d), 8).cuda()
    qc, kc, vc = q.cuda(), k.cuda(), v.cuda()
    o, lse = gqa.attn(qc, kc, vc, causal=True, return_lse=True)
    dq, dk, dv = gqa.attn_bwd(qc, kc, vc, o, lse, dout)
    ke, ve = kc.repeat_interleave(G, 2).contiguous(), vc.repeat_interleave(G, 2).contiguous()
    oe, lsee = gqa.attn(qc, ke, ve, causal=True, return_lse=True)
    dqe, dke, dve = gqa.attn_bwd(qc, ke, ve, oe, lsee, dout)
    sk = dke.float().view(B, T, Hkv, G, d).sum(3)
    sv = dve.float().view(B, T, Hkv, G, d).sum(3)
    assert float((dk.float() - sk).abs().max()) <= 2e-2 * max(1.0, float(sk.abs().max()))
    assert float((dv.float() - sv).abs().max()) <= 2e-2 * max(1.0, float(sv.abs().max()))


def test_backward_without_keys_is_zero(gqa_lib):
    B, Tq, Hq, Hkv, d = 1, 64, 4, 2, 128
    q = workloads.randn((B, Tq, Hq, d), 1).cuda()
    k = torch.empty((B, 0, Hkv, d), dtype=torch.bfloat16, device="cuda")
    o = torch.zeros_like(q)
    lse = torch.full((B, Hq, Tq), float("-inf"), device="cuda")
    dq, dk, dv = gqa.attn_bwd(q, k, k, o, lse, workloads.randn((B, Tq, Hq, d), 2).cuda())
    torch.cuda.synchronize()
    assert dq.shape == q.shape and bool((dq == 0).all())


@pytest.mark.parametrize("g", [0, 7])
def test_backward_headline_shape(gqa_lib, g):
    # The causal T=4096, 32 / 8 head workload the bench times, full launch on
    # the GPU.  KV groups are independent problems, so the oracle takes group g
    # alone (query heads 4g .. 4g+3, K/V head g).  The output of a query row
    # depends on that row and K/V only, so the oracle runs over blocks of 512
    # query rows against keys [0, i1): dq of a block is exact, and dk / dv are
    # the sums of the blocks' contributions.
    T, Hq, Hkv, d, G = 4096, 32, 8, 128, 4
    q, k, v = workloads.prefill_inputs(1, T, Hq, Hkv, d)
    dout = workloads.randn((1, T, Hq, d), 77)
    qc, kc, vc = q.cuda(), k.cuda(), v.cuda()
    o, lse = gqa.attn(qc, kc, vc, causal=True, return_lse=True)
    dq, dk, dv = gqa.attn_bwd(qc, kc, vc, o, lse, dout.cuda())
    gqa.device_status()
    hs = slice(g * G, (g + 1) * G)
    rq = np.zeros((1, T, G, d))
    rk = np.zeros((1, T, 1, d))
    rv = np.zeros((1, T, 1, d))
    for i0 in range(0, T, 512):
        i1 = i0 + 512
        a, b, c = ref.attn_bwd(q[:, i0:i1, hs], k[:, :i1, g:g + 1], v[:, :i1, g:g + 1],
                               dout[:, i0:i1, hs], True)
        rq[:, i0:i1] = a
        rk[:, :i1] += b
        rv[:, :i1] += c
    assert rel_err(dq[:, :, hs], rq) <= 2e-2
    assert rel_err(dk[:, :, g:g + 1], rk) <= 2e-2
    assert rel_err(dv[:, :, g:g + 1], rv) <= 2e-2


def test_backward_graph_capture_and_streams(gqa_lib):
    # The dK/dV kernel runs on the library's second stream, forked from and
    # joined back into the caller's stream.  A CUDA graph captured on a side
    # stream must hold both kernels, and its replays, as well as calls on the
    # default stream, must give exactly the eager result (no atomics: the sums
    # run in a fixed order).
    B, T, Hq, Hkv, d = 2, 384, 8, 2, 128
    q, k, v = workloads.prefill_inputs(B, T, Hq, Hkv, d, seeds=(11, 12, 13))
    qc, kc, vc = q.cuda(), k.cuda(), v.cuda()
    o, lse = gqa.attn(qc, kc, vc, causal=True, return_lse=True)
    douts = [workloads.randn((B, T, Hq, d), 40 + i).cuda() for i in range(3)]
    want = [gqa.attn_bwd(qc, kc, vc, o, lse, dd) for dd in douts]
    torch.cuda.synchronize()
    gqa.device_status()
    dout = douts[0].clone()
    ws = torch.empty(gqa.attn_bwd_workspace_size(B, T, Hq), dtype=torch.uint8, device="cuda")
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        gqa.attn_bwd(qc, kc, vc, o, lse, dout, workspace=ws)    # warm-up outside capture
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=s):
            got = gqa.attn_bwd(qc, kc, vc, o, lse, dout, workspace=ws)
    for rep in (2, 1, 0):
        dout.copy_(douts[rep])
        for t in got:
            t.fill_(float("nan"))
        g.replay()
        torch.cuda.synchronize()
        for a, b in zip(got, want[rep]):
            assert torch.equal(a, b), rep
    with torch.cuda.stream(torch.cuda.default_stream()):
        again = gqa.attn_bwd(qc, kc, vc, o, lse, douts[1])
    torch.cuda.synchronize()
    gqa.device_status()
    for a, b in zip(again, want[1]):
        assert torch.equal(a, b)


@pytest.mark.parametrize("B,T,Hq,Hkv,d", [
    (3, 1000, 16, 2, 128),    # G = 8: 16 positions per M tile, 378 tiles (> SMs)
    (1, 64, 4, 4, 64),        # one M tile: one CTA takes it, the others find the queue empty
])
def test_backward_dq_tile_queue(gqa_lib, B, T, Hq, Hkv, d):
    # The dQ kernel takes its M tiles from a counter in the workspace that the
    # rowdot launch resets: a workspace full of stale bytes, and a second call
    # on the same workspace, give the same gradients as the oracle.
    q, k, v = workloads.prefill_inputs(B, T, Hq, Hkv, d, seeds=(B + 3, T, Hq))
    dout = workloads.randn((B, T, Hq, d), 91)
    qc, kc, vc = q.cuda(), k.cuda(), v.cuda()
    o, lse = gqa.attn(qc, kc, vc, causal=True, return_lse=True)
    ws = torch.full((gqa.attn_bwd_workspace_size(B, T, Hq),), 0xFF, dtype=torch.uint8,
                    device="cuda")
    first = gqa.attn_bwd(qc, kc, vc, o, lse, dout.cuda(), workspace=ws)
    second = gqa.attn_bwd(qc, kc, vc, o, lse, dout.cuda(), workspace=ws)
    torch.cuda.synchronize()
    gqa.device_status()
    for a, b in zip(first, second):
        assert torch.equal(a, b)
    if B * T <= 1000:
        rq, rk, rv = ref.attn_bwd(q, k, v, dout, True)
    else:   # batch 0 only (batches are independent problems)
        rq, rk, rv = ref.attn_bwd(q[:1], k[:1], v[:1], dout[:1], True)
        first = tuple(t[:1] for t in first)
    assert rel_err(first[0], rq) <= 2e-2
    assert rel_err(first[1], rk) <= 2e-2
    assert rel_err(first[2], rv) <= 2e-2


def test_backward_from_two_host_threads(gqa_lib):
    # The fork / join events and the second stream are shared per context and
    # used under a lock: two host threads calling the backward at once, each on
    # its own stream with its own workspace, get exactly the eager results.
    import threading
    B, T, Hq, Hkv, d = 1, 512, 8, 2, 128
    q, k, v = workloads.prefill_inputs(B, T, Hq, Hkv, d, seeds=(21, 22, 23))
    qc, kc, vc = q.cuda(), k.cuda(), v.cuda()
    o, lse = gqa.attn(qc, kc, vc, causal=True, return_lse=True)
    douts = [workloads.randn((B, T, Hq, d), 60 + i).cuda() for i in range(2)]
    want = [gqa.attn_bwd(qc, kc, vc, o, lse, dd) for dd in douts]
    torch.cuda.synchronize()
    got = [None, None]
    errors = []

    def run(i):
        try:
            s = torch.cuda.Stream()
            ws = torch.empty(gqa.attn_bwd_workspace_size(B, T, Hq), dtype=torch.uint8,
                             device="cuda")
            with torch.cuda.stream(s):
                for _ in range(20):
                    got[i] = gqa.attn_bwd(qc, kc, vc, o, lse, douts[i], workspace=ws)
            s.synchronize()
        except Exception as e:   # surfaced below
            errors.append(e)

    threads = [threading.Thread(target=run, args=(i,)) for i in range(2)]
    for t in threads:
        t.start()
    for t in threads:
        t.join(timeout=120)
    assert not errors, errors
    torch.cuda.synchronize()
    gqa.device_status()
    for i in range(2):
        for a, b in zip(got[i], want[i]):
            assert torch.equal(a, b), i
