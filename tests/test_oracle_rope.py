"""Pins of the RoPE oracle (course "Неделя 7. Внимание", step 3 and the test names
it lists: the rotation preserves the norm, is the identity at position zero,
and makes attention scores depend only on the position difference)."""

import math

import numpy as np
import pytest
import torch

from oracle import lab, ref


def rand(shape, seed):
    g = torch.Generator().manual_seed(seed)
    return torch.randn(shape, generator=g, dtype=torch.float32)


def test_rope_preserves_norm():
    x = rand((2, 30, 3, 16), 1)
    y = ref.rope_tensor(x, pos0=5)
    assert np.allclose(np.linalg.norm(y, axis=-1), np.linalg.norm(x.double().numpy(), axis=-1),
                       rtol=1e-12, atol=0)


def test_rope_identity_at_position_zero():
    x = rand((1, 1, 4, 32), 2)
    assert np.array_equal(ref.rope_tensor(x, pos0=0), x.double().numpy())


@pytest.mark.parametrize("shift", [1, 7, 1000])
def test_rope_makes_scores_relative(shift):
    # <R_m q, R_n k> depends on m - n only
    q, k = rand((1, 1, 1, 64), 3), rand((1, 1, 1, 64), 4)
    for m, n in [(3, 9), (40, 2), (0, 0)]:
        s1 = float(np.sum(ref.rope_tensor(q, m) * ref.rope_tensor(k, n)))
        s2 = float(np.sum(ref.rope_tensor(q, m + shift) * ref.rope_tensor(k, n + shift)))
        assert abs(s1 - s2) < 1e-9


def test_rope_two_dims_is_a_plain_rotation():
    # d = 2: theta_0 = 1, so position m rotates the pair by m radians
    x = torch.tensor([[[[1.0, 0.0]]]])
    for m in (0, 1, 2, 5):
        y = ref.rope_tensor(x, m)[0, 0, 0]
        assert np.allclose(y, [math.cos(m), math.sin(m)], rtol=0, atol=1e-15)


def test_rope_tensor_matches_lab_rows():
    x = rand((1, 6, 1, 8), 5)
    rows = x[0, :, 0].double().tolist()
    want = np.array(lab.rope(rows, [11 + t for t in range(6)], theta=500.0))
    got = ref.rope_tensor(x, 11, theta=500.0)[0, :, 0]
    assert np.allclose(got, want, rtol=0, atol=1e-13)


def test_rope_decode_q_positions():
    q = rand((4, 2, 16), 6)
    sl = torch.tensor([1, 10, 300, 0], dtype=torch.int32)
    got = ref.rope_decode_q(q, sl)
    for b in range(3):
        want = ref.rope_tensor(q[b][None, None], int(sl[b]) - 1)[0, 0]
        assert np.array_equal(got[b], want)
    assert np.array_equal(got[0], q[0].double().numpy())      # position 0: identity
    assert np.array_equal(got[3], q[3].double().numpy())      # empty cache: position 0


def test_rope_odd_dim_rejected():
    with pytest.raises(ValueError):
        ref.rope_tensor(rand((1, 2, 1, 5), 7), 0)
