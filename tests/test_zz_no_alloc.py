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


# The near-capacity shape: 252 splits of 1024 keys x 16 sequences x 32 query
# heads at d = 64 need 33,546,240 bytes of scratch, 8 KB short of the 32 MiB;
# one more split would not fit.  Its group of 32 heads takes the two-tile
# (G > 16) split kernel.
NEAR_FULL = (16, 32, 1, 64, 258048)

STATIC_CASES = [
    # B, Hq, Hkv, d, Lmax, lengths of the first call, lengths of the second call
    (16, 32, 8, 128, 3000, [3000, 1, 700, 1024, 513, 0, 2999, 64] * 2,
     [5, 3000, 1500, 0, 1, 2048, 777, 1025] * 2),
    (4, 32, 1, 64, 5000, [5000, 1, 1023, 1025], [0, 4999, 64, 3072]),
    NEAR_FULL + ([258048, 1, 258047, 0, 131072, 1024, 5, 258048] * 2,
                 [2, 258048, 0, 100000, 258048, 1025, 77, 257025] * 2),
]


def test_near_full_shape_fits_the_scratch_exactly(gqa_lib):
    B, Hq, Hkv, d, Lmax = NEAR_FULL
    need = _binding.gqa_decode_workspace_size(B, Hq, Hkv, d, Lmax)
    assert STATIC_SCRATCH_BYTES - 8192 <= need <= STATIC_SCRATCH_BYTES
    assert _binding.gqa_decode_workspace_size(B, Hq, Hkv, d, Lmax + 1024) > STATIC_SCRATCH_BYTES


FAKE = 0x10000


@pytest.mark.parametrize("args,code", [
    (dict(q=0), _binding.GQA_ERR_INVALID_ARG),            # NULL q
    (dict(o=FAKE + 4), _binding.GQA_ERR_INVALID_ARG),     # misaligned o
    (dict(sl=0), _binding.GQA_ERR_INVALID_ARG),
    (dict(d=96), _binding.GQA_ERR_UNSUPPORTED),
    (dict(Hq=64, Hkv=1), _binding.GQA_ERR_UNSUPPORTED),   # group of 64 heads
    (dict(Hkv=3), _binding.GQA_ERR_INVALID_ARG),
    (dict(scale=0.0), _binding.GQA_ERR_INVALID_ARG),
])
def test_static_scratch_validates_like_gqa_decode(gqa_lib, args, code):
    # the argument checks run before the scratch is looked up, so they answer
    # without a GPU and with gqa_decode's codes
    a = dict(q=FAKE, kc=FAKE, vc=FAKE, sl=FAKE, o=FAKE, B=4, Hq=8, Hkv=2, d=128, Lmax=1000,
             scale=0.088)
    a.update(args)
    pos = (a["q"], a["kc"], a["vc"], a["sl"], a["o"], a["B"], a["Hq"], a["Hkv"], a["d"],
           a["Lmax"], a["scale"])
    rc = _binding.gqa_decode_static(*pos, None)
    assert rc == code, _binding.gqa_last_error()
    need = max(_binding.gqa_decode_workspace_size(*pos[5:10]), 256)
    assert _binding.gqa_decode(*pos, FAKE, need, None) == code


@pytest.mark.gpu
@pytest.mark.parametrize("B,Hq,Hkv,d,Lmax,len0,len1", STATIC_CASES)
def test_static_scratch_decode_matches_workspace_decode_twice(gqa_lib, B, Hq, Hkv, d, Lmax, len0,
                                                              len1):
    scale = d ** -0.5
    stream = torch.cuda.current_stream().cuda_stream
    # two calls in a row with different lengths: the second must not see the
    # first call's leftovers in the shared scratch
    for call, lengths in enumerate((len0, len1)):
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
