"""GPU fold_kv (bit-exact against the oracle fold) and the bounded-wait failure path."""

import pytest
import torch

import grouped_query_attention_attn_b200 as gqa
from grouped_query_attention_attn_b200 import _binding, workloads
from oracle import ref

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("H,g,d", [(32, 8, 128), (32, 1, 128), (8, 8, 64), (12, 3, 16), (6, 2, 8)])
def test_fold_bit_exact(gqa_lib, H, g, d):
    kv = workloads.randn((2, 37, H, d), H * g + d)
    out = gqa.fold_kv(kv.cuda(), g)
    assert torch.equal(out.cpu(), ref.fold_kv_tensor(kv, g))


def test_bounded_wait_times_out_and_context_survives(gqa_lib):
    # a barrier nothing arrives at: the wait gives up after 2 ms and reports it
    assert _binding.gqa_selftest_wait_timeout(2000) == _binding.GQA_ERR_TIMEOUT
    assert _binding.gqa_device_status(0) == _binding.GQA_OK
    # the context is still usable
    kv = workloads.randn((1, 4, 8, 16), 3)
    assert torch.equal(gqa.fold_kv(kv.cuda(), 2).cpu(), ref.fold_kv_tensor(kv, 2))
