"""Forward on host tensors (gqa_attn_fwd_host): copies up, chunked attention,
copies down, overlapped in the library; checked against the oracle."""

import numpy as np
import pytest
import torch

import grouped_query_attention_attn_b200 as gqa
from grouped_query_attention_attn_b200 import workloads
from oracle import ref
from parity import BF16_TOL, gather_rows, max_abs, sample_rows

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("B,Tq,Tkv,Hq,Hkv,d,causal", [
    (1, 3000, 3000, 8, 2, 128, True),      # 4 chunks of 750 rows, last rows first
    (2, 700, 700, 8, 2, 128, True),        # B = 2: strided copies
    (1, 1000, 300, 8, 2, 128, True),       # Tq > Tkv: leading chunks see no key
    (2, 300, 1000, 4, 1, 64, True),        # Tq < Tkv
    (1, 900, 600, 8, 8, 128, False),       # non-causal: all keys with the first chunk
    (1, 100, 100, 4, 2, 128, True),        # one chunk
])
def test_host_forward_matches_oracle(gqa_lib, B, Tq, Tkv, Hq, Hkv, d, causal):
    q, k, v = workloads.prefill_inputs(B, Tq, Hq, Hkv, d, Tkv=Tkv, seeds=(Tq + 3, Tkv + 4, B))
    qp, kp, vp = q.pin_memory(), k.pin_memory(), v.pin_memory()
    o = gqa.attn_host(qp, kp, vp, causal=causal)
    torch.cuda.synchronize()
    o_ref, _ = ref.attn_fwd(q, k, v, causal)
    assert max_abs(o, o_ref) <= BF16_TOL
    # the device path on the same inputs agrees to rounding
    o_dev = gqa.attn(q.cuda(), k.cuda(), v.cuda(), causal=causal).cpu()
    assert max_abs(o, o_dev.float().numpy().astype(np.float64)) <= BF16_TOL


def test_host_forward_reuses_staging(gqa_lib):
    shapes = [workloads.prefill_inputs(1, 1200, 8, 2, 128, seeds=(s, s + 1, s + 2)) for s in (5, 9)]
    st = gqa.host_staging(shapes[0][0], shapes[0][1])
    out = torch.empty(shapes[0][0].shape, dtype=torch.bfloat16).pin_memory()
    for q, k, v in shapes + shapes[:1]:
        qp, kp, vp = q.pin_memory(), k.pin_memory(), v.pin_memory()
        gqa.attn_host(qp, kp, vp, out=out, staging=st)
        torch.cuda.synchronize()
        o_ref, _ = ref.attn_fwd(q, k, v, True)
        assert max_abs(out, o_ref) <= BF16_TOL


def test_host_forward_pageable_memory(gqa_lib):
    q, k, v = workloads.prefill_inputs(1, 600, 4, 1, 128, seeds=(21, 22, 23))
    o = gqa.attn_host(q, k, v)            # not pinned: the copies are staged, still correct
    torch.cuda.synchronize()
    o_ref, _ = ref.attn_fwd(q, k, v, True)
    assert max_abs(o, o_ref) <= BF16_TOL


def test_host_forward_with_completion_event(gqa_lib):
    # consecutive calls on shared staging, each signalling its own completion
    inputs = [workloads.prefill_inputs(2, 800, 8, 2, 128, seeds=(s, s + 1, s + 2)) for s in (31, 35, 39)]
    # the host buffers must live, unchanged, until their call completes
    pinned = [tuple(t.pin_memory() for t in x) for x in inputs]
    st = gqa.host_staging(inputs[0][0], inputs[0][1])
    outs = [torch.empty(inputs[0][0].shape, dtype=torch.bfloat16).pin_memory() for _ in inputs]
    events = [torch.cuda.Event() for _ in inputs]
    for (q, k, v), o, ev in zip(pinned, outs, events):
        gqa.attn_host(q, k, v, out=o, staging=st, done=ev)
    for (q, k, v), o, ev in zip(inputs, outs, events):
        ev.synchronize()
        o_ref, _ = ref.attn_fwd(q, k, v, True)
        assert max_abs(o, o_ref) <= BF16_TOL


def test_host_forward_alternating_staging(gqa_lib):
    # consecutive overlapped calls alternating two staging sets, then a third,
    # larger set, then a set that is a view into it, with the shapes changing in
    # between: every output against the oracle
    specs = [(2, 800, 8, 2, 128), (2, 800, 8, 2, 128), (2, 800, 8, 2, 128),
             (1, 1700, 8, 2, 128), (2, 800, 8, 2, 128)]
    inputs = [workloads.prefill_inputs(B, T, Hq, Hkv, d, seeds=(41 + 3 * i, 42 + 3 * i, 43 + 3 * i))
              for i, (B, T, Hq, Hkv, d) in enumerate(specs)]
    pinned = [tuple(t.pin_memory() for t in x) for x in inputs]
    big = gqa.host_staging(inputs[3][0], inputs[3][1])
    sets = [gqa.host_staging(inputs[0][0], inputs[0][1]) for _ in range(2)]
    # a set that is a view into the big one overlaps it
    view = tuple(t.view(-1)[: s.numel()].view(s.shape) for t, s in zip(big, sets[0]))
    order = [sets[0], sets[1], sets[0], big, view]
    outs = [torch.empty(x[0].shape, dtype=torch.bfloat16).pin_memory() for x in inputs]
    events = [torch.cuda.Event() for _ in inputs]
    for (q, k, v), o, st, ev in zip(pinned, outs, order, events):
        gqa.attn_host(q, k, v, out=o, staging=st, done=ev)
    for (q, k, v), o, ev in zip(inputs, outs, events):
        ev.synchronize()
        o_ref, _ = ref.attn_fwd(q, k, v, True)
        assert max_abs(o, o_ref) <= BF16_TOL


def test_host_forward_headline_shape(gqa_lib):
    # the end-to-end path the bench times: causal B=1, T=4096, 32 / 8 heads from
    # pinned host tensors (4 chunks of 1024 rows), sampled rows against the oracle
    q, k, v = workloads.prefill_inputs(1, 4096, 32, 8, 128)
    qp, kp, vp = q.pin_memory(), k.pin_memory(), v.pin_memory()
    o = gqa.attn_host(qp, kp, vp, causal=True)
    torch.cuda.synchronize()
    gqa.device_status()
    rows = sample_rows(1, 4096, 32, 512, 3)
    o_ref, _ = ref.attn_fwd_rows(q, k, v, rows, True)
    assert max_abs(gather_rows(o, rows, 4096, 32), o_ref) <= BF16_TOL
