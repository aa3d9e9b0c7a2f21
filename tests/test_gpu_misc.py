"""GPU fold_kv (bit-exact against the oracle fold), the bounded-wait failure path and
the error bound of the exp2 polynomial the prefill softmax uses."""

import numpy as np
import pytest
import torch

import grouped_query_attention_attn_b200 as gqa
from grouped_query_attention_attn_b200 import _binding, workloads
from oracle import ref

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("H,g,d", [(32, 8, 128), (32, 1, 128), (8, 8, 64), (12, 3, 16), (6, 2, 8),
                                   (12, 2, 128), (10, 2, 64)])   # group sizes 6, 5: rounded division
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


def test_exp2_polynomial_error_bound(gqa_lib):
    # The prefill softmax computes a quarter of its exponentials with an FMA-pipe
    # polynomial.  Over a dense grid of the arguments it can see (s*scale*log2e -
    # m_ref lies in [-inf, 8]; masked scores never reach it) its relative error
    # against 2^x in double stays within the fit's 7.5e-5, and below -125 it is
    # clamped to 2^-125.  Points around -126 are included: there the exponent
    # add would leave a denormal if the clamp let them through.
    xs = np.concatenate([np.linspace(-130.0, 8.0, 1 << 21),
                         np.arange(-126, 9, dtype=np.float64),          # integers
                         np.arange(-126, 8, dtype=np.float64) + 0.5,    # reduction edges
                         np.nextafter(np.arange(-125, 8, dtype=np.float32) + 0.5, -np.inf),
                         [-126.0, -125.99999, -125.0, -124.99999, -127.0, -1000.0, 0.0, -0.0, 8.0]])
    x = torch.tensor(xs, dtype=torch.float32)
    if x.numel() % 2:
        x = torch.cat([x, x[:1]])
    y = torch.empty_like(x).cuda()
    xd = x.cuda()
    rc = _binding.gqa_selftest_exp2_poly(xd.data_ptr(), y.data_ptr(), x.numel(),
                                         torch.cuda.current_stream().cuda_stream)
    assert rc == _binding.GQA_OK, _binding.gqa_last_error()
    got = y.cpu().double().numpy()
    xx = x.double().numpy()
    assert np.all(np.isfinite(got)) and np.all(got > 0)
    normal = xx >= -125.0
    rel = np.abs(got[normal] / np.exp2(xx[normal]) - 1.0)
    assert rel.max() <= 7.5e-5, (rel.max(), xx[normal][np.argmax(rel)])
    assert np.all(got >= 2.0 ** -126)                   # never a denormal
    # the clamp: anything below -125 gives the value at -125
    at_clamp = got[xx == -125.0][0]
    assert np.all(got[~normal] == at_clamp)
    assert abs(at_clamp / 2.0 ** -125 - 1.0) <= 7.5e-5


def test_exp2_selftest_rejects_odd_counts(gqa_lib):
    assert _binding.gqa_selftest_exp2_poly(0x1000, 0x1000, 3, None) == _binding.GQA_ERR_INVALID_ARG
