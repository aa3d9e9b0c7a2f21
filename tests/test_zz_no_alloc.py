"""gqa_decode_static: decode for callers that cannot allocate device memory.

Such callers (a runtime whose pool owns all device memory, a plugin that may
not allocate on its hot path, code that must not risk the synchronisation an
allocation can cause) get the same decode with scratch built into the library
instead of a caller workspace.  These tests call it through the C ABI and
check it against gqa_decode, the entry point with a caller workspace.

This file is named to be collected last, so a run that stops at the first
failure has run every other test before it.
"""

import pytest
import torch

from grouped_query_attention_attn_b200 import _binding, workloads
from parity import BF16_TOL, max_abs

STATIC_SCRATCH_BYTES = 32 << 20


def decode_with_workspace(q, kc, vc, sl, o, B, Hq, Hkv, d, Lmax, scale, stream):
    need = _binding.gqa_decode_workspace_size(B, Hq, Hkv, d, Lmax)
    ws = torch.empty(need, dtype=torch.uint8, device="cuda")
    rc = _binding.gqa_decode(q.data_ptr(), kc.data_ptr(), vc.data_ptr(), sl.data_ptr(),
                             o.data_ptr(), B, Hq, Hkv, d, Lmax, scale, ws.data_ptr(), need, stream)
    assert rc == _binding.GQA_OK, _binding.gqa_last_error()


def decode_static(q, kc, vc, sl, o, B, Hq, Hkv, d, Lmax, scale, stream):
    rc = _binding.gqa_decode_static(q.data_ptr(), kc.data_ptr(), vc.data_ptr(), sl.data_ptr(),
                                    o.data_ptr(), B, Hq, Hkv, d, Lmax, scale, stream)
    assert rc == _binding.GQA_OK, _binding.gqa_last_error()


@pytest.mark.gpu
def test_static_scratch_decode_matches_workspace_decode_twice(gqa_lib):
    B, Hq, Hkv, d, Lmax = 16, 32, 8, 128, 3000
    scale = d ** -0.5
    stream = torch.cuda.current_stream().cuda_stream
    # two calls in a row with different lengths: the second must not see the
    # first call's leftovers in the shared scratch
    for call, lengths in enumerate(([3000, 1, 700, 1024, 513, 0, 2999, 64] * 2,
                                    [5, 3000, 1500, 0, 1, 2048, 777, 1025] * 2)):
        q, kc, vc, sl = workloads.decode_inputs(B, Hq, Hkv, d, 1, Lmax, lengths=lengths,
                                                seeds=(10 + call, 20 + call, 30 + call, 0))
        q, kc, vc, sl = q.cuda(), kc.cuda(), vc.cuda(), sl.cuda()
        o_ref = torch.empty_like(q)
        decode_with_workspace(q, kc, vc, sl, o_ref, B, Hq, Hkv, d, Lmax, scale, stream)
        o = torch.full_like(q, float("nan"))
        decode_static(q, kc, vc, sl, o, B, Hq, Hkv, d, Lmax, scale, stream)
        torch.cuda.synchronize()
        assert max_abs(o, o_ref.float().cpu().numpy()) <= BF16_TOL
    assert _binding.gqa_device_status(1) == _binding.GQA_OK


def test_static_scratch_rejects_sizes_beyond_its_capacity(gqa_lib):
    # checked on the host before anything touches the GPU
    B, Hq, Hkv, d, Lmax = 512, 32, 8, 128, 8192
    assert _binding.gqa_decode_workspace_size(B, Hq, Hkv, d, Lmax) > STATIC_SCRATCH_BYTES
    rc = _binding.gqa_decode_static(0x10000, 0x10000, 0x10000, 0x10000, 0x10000, B, Hq, Hkv, d,
                                    Lmax, 0.088, None)
    assert rc == _binding.GQA_ERR_WORKSPACE
    assert "scratch" in _binding.gqa_last_error()
    # the benchmark's decode sizes fit
    assert _binding.gqa_decode_workspace_size(64, 32, 8, 128, 8192) <= STATIC_SCRATCH_BYTES
