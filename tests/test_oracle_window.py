"""Pins of the sliding-window + attention-sink oracle.

Course "Неделя 7. Внимание", step 3: a sliding window limits what a token sees
to the most recent keys, and the first tokens (attention sinks) stay visible.
Reading: with causal bottom-right alignment, row i at key position
p = i + Tkv - Tq sees key j iff j <= p and (j > p - window or j < sinks).
"""

import numpy as np
import pytest
import torch
import torch.nn.functional as F

from oracle import lab, ref


def rand(shape, seed):
    g = torch.Generator().manual_seed(seed)
    return torch.randn(shape, generator=g, dtype=torch.float32)


def mask_of(Tq, Tkv, window, sinks):
    m = torch.zeros(Tq, Tkv, dtype=torch.bool)
    for i in range(Tq):
        for j in range(Tkv):
            m[i, j] = lab.visible(i, j, Tq, Tkv, causal=True, window=window, sinks=sinks)
    return m


@pytest.mark.parametrize("Tq,Tkv,window,sinks", [(20, 20, 5, 0), (20, 20, 5, 2), (9, 30, 4, 3),
                                                 (30, 30, 1, 1), (17, 17, 40, 0), (12, 25, 7, 10)])
def test_window_oracle_equals_lab_brute_force(Tq, Tkv, window, sinks):
    B, Hq, Hkv, d = 2, 4, 2, 6
    q, k, v = rand((B, Tq, Hq, d), 1), rand((B, Tkv, Hkv, d), 2), rand((B, Tkv, Hkv, d), 3)
    o, _ = ref.attn_fwd_window(q, k, v, window, sinks)
    for b in range(B):
        for hq in range(Hq):
            kvh = lab.group_of(hq, Hq, Hkv)
            want = lab.attend(q[b, :, hq].double().tolist(), k[b, :, kvh].double().tolist(),
                              v[b, :, kvh].double().tolist(), causal=True, window=window,
                              sinks=sinks)
            assert np.allclose(o[b, :, hq], np.array(want), rtol=0, atol=1e-12)


@pytest.mark.parametrize("window,sinks", [(8, 0), (8, 4), (3, 1), (64, 0)])
def test_window_oracle_equals_sdpa_with_mask(window, sinks):
    B, T, Hq, Hkv, d = 1, 50, 8, 2, 16
    q, k, v = rand((B, T, Hq, d), 4), rand((B, T, Hkv, d), 5), rand((B, T, Hkv, d), 6)
    o, lse = ref.attn_fwd_window(q, k, v, window, sinks)
    m = mask_of(T, T, window, sinks)
    r = F.scaled_dot_product_attention(q.double().transpose(1, 2), k.double().transpose(1, 2),
                                       v.double().transpose(1, 2), attn_mask=m,
                                       enable_gqa=True).transpose(1, 2)
    assert np.allclose(o, r.numpy(), rtol=0, atol=1e-12)


def test_wide_window_is_plain_causal():
    B, T, Hq, Hkv, d = 2, 40, 4, 1, 8
    q, k, v = rand((B, T, Hq, d), 7), rand((B, T, Hkv, d), 8), rand((B, T, Hkv, d), 9)
    o_w, l_w = ref.attn_fwd_window(q, k, v, window=T, sinks=0)
    o_c, l_c = ref.attn_fwd(q, k, v, causal=True)
    assert np.array_equal(o_w, o_c) and np.array_equal(l_w, l_c)


def test_window_one_sees_only_itself():
    # window 1, no sinks: each row's only visible key is its own position
    B, T, Hq, Hkv, d = 1, 12, 2, 2, 4
    q, k, v = rand((B, T, Hq, d), 10), rand((B, T, Hkv, d), 11), rand((B, T, Hkv, d), 12)
    o, _ = ref.attn_fwd_window(q, k, v, window=1, sinks=0)
    assert np.array_equal(o, v.double().numpy())


def test_keys_outside_window_and_sinks_do_not_matter():
    B, T, Hq, Hkv, d = 1, 60, 4, 2, 8
    window, sinks = 10, 3
    q, k, v = rand((B, T, Hq, d), 13), rand((B, T, Hkv, d), 14), rand((B, T, Hkv, d), 15)
    o, _ = ref.attn_fwd_window(q, k, v, window, sinks)
    k2, v2 = k.clone(), v.clone()
    k2[:, sinks:30] += 5.0                  # hidden from rows >= 39 (p - 10 >= 29)
    v2[:, sinks:30] -= 3.0
    o2, _ = ref.attn_fwd_window(q, k2, v2, window, sinks)
    assert np.array_equal(o[:, 39:], o2[:, 39:])
    assert not np.allclose(o[:, :39], o2[:, :39])
    # the sink keys do matter everywhere
    k3 = k.clone()
    k3[:, :sinks] += 5.0
    o3, _ = ref.attn_fwd_window(q, k3, v, window, sinks)
    assert not np.allclose(o[:, 39:], o3[:, 39:])


def test_decode_window_is_last_row_of_forward():
    B, Hq, Hkv, d, Lmax = 3, 8, 2, 16, 70
    from grouped_query_attention_attn_b200 import workloads
    q, kc, vc, sl = workloads.decode_inputs(B, Hq, Hkv, d, 1, Lmax, dtype=torch.float32,
                                            lengths=[70, 5, 33])
    for window, sinks in [(8, 0), (8, 2), (100, 0), (1, 1)]:
        o, _ = ref.decode_window(q, kc, vc, sl, window, sinks)
        for b in range(B):
            L = int(sl[b])
            of, _ = ref.attn_fwd_window(q[b:b + 1, None], kc[b:b + 1, :L], vc[b:b + 1, :L],
                                        window, sinks)
            assert np.array_equal(o[b], of[0, 0])


def test_window_rejects_bad_arguments():
    q, k, v = rand((1, 4, 2, 4), 1), rand((1, 4, 2, 4), 2), rand((1, 4, 2, 4), 3)
    with pytest.raises(ValueError):
        ref.attn_fwd_window(q, k, v, window=0)
    with pytest.raises(ValueError):
        ref.attn_fwd_window(q, k, v, window=4, sinks=-1)


def test_query_block_against_keys_up_to_its_end_equals_the_full_rows():
    # The full-size GPU window test checks blocks of query rows [i0, i1) against
    # the oracle run on keys [0, i1) only: with bottom-right alignment those rows
    # keep their positions, so window and sinks select the same keys.
    T, W, S = 300, 70, 3
    q, k, v = rand((1, T, 4, 8), 21), rand((1, T, 2, 8), 22), rand((1, T, 2, 8), 23)
    o, lse = ref.attn_fwd_window(q, k, v, W, S)
    for i0, i1 in ((0, 40), (60, 130), (250, 300)):
        ob, lb = ref.attn_fwd_window(q[:, i0:i1], k[:, :i1], v[:, :i1], W, S)
        assert np.array_equal(ob, o[:, i0:i1])
        assert np.array_equal(lb, lse[:, :, i0:i1])
