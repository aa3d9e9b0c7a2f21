"""Pins of the backward oracle: finite differences, the page's sum rule for
shared heads (K3 notes, "Backward: view + sum"), and closed forms."""

import numpy as np
import pytest
import torch

from oracle import ref


def rand(shape, seed):
    g = torch.Generator().manual_seed(seed)
    return torch.randn(shape, generator=g, dtype=torch.float32)


def loss(q, k, v, do, causal, window=0, sinks=0):
    if window:
        o, _ = ref.attn_fwd_window(q, k, v, window, sinks)
    else:
        o, _ = ref.attn_fwd(q, k, v, causal)
    return float(np.sum(o * do.double().numpy()))


@pytest.mark.parametrize("causal,window,sinks", [(False, 0, 0), (True, 0, 0), (True, 3, 1)])
def test_backward_oracle_matches_finite_differences(causal, window, sinks):
    # central differences of <o, do> computed with the independent C forward oracle
    B, Tq, Tkv, Hq, Hkv, d = 1, 5, 7, 4, 2, 3
    q, k, v = rand((B, Tq, Hq, d), 1), rand((B, Tkv, Hkv, d), 2), rand((B, Tkv, Hkv, d), 3)
    do = rand((B, Tq, Hq, d), 4)
    dq, dk, dv = ref.attn_bwd(q, k, v, do, causal, window=window, sinks=sinks)
    h = 1e-3
    for name, t, g in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        flat = t.view(-1)
        for idx in range(0, flat.numel(), 3):
            old = float(flat[idx])
            flat[idx] = old + h
            up = float(flat[idx])              # the float32 value actually stored
            lp = loss(q, k, v, do, causal, window, sinks)
            flat[idx] = old - h
            dn = float(flat[idx])
            lm = loss(q, k, v, do, causal, window, sinks)
            flat[idx] = old
            fd = (lp - lm) / (up - dn)
            assert abs(fd - g.reshape(-1)[idx]) < 1e-5 * max(1.0, abs(fd)), (name, idx)


def test_shared_head_gradient_is_the_sum_over_its_query_heads():
    # run MHA on repeat_interleave'd K/V; the GQA gradient of K/V head h is the
    # SUM over the G expanded heads (view(..., Hkv, G, d).sum), not the mean
    B, T, Hq, Hkv, d = 2, 9, 8, 2, 4
    G = Hq // Hkv
    q, k, v = rand((B, T, Hq, d), 5), rand((B, T, Hkv, d), 6), rand((B, T, Hkv, d), 7)
    do = rand((B, T, Hq, d), 8)
    dq, dk, dv = ref.attn_bwd(q, k, v, do, True)
    dq_e, dk_e, dv_e = ref.attn_bwd(q, k.repeat_interleave(G, 2), v.repeat_interleave(G, 2), do,
                                    True)
    assert np.allclose(dq, dq_e, rtol=0, atol=1e-12)
    assert np.allclose(dk, dk_e.reshape(B, T, Hkv, G, d).sum(3), rtol=0, atol=1e-12)
    assert np.allclose(dv, dv_e.reshape(B, T, Hkv, G, d).sum(3), rtol=0, atol=1e-12)
    assert not np.allclose(dk, dk_e.reshape(B, T, Hkv, G, d).mean(3))


def test_dv_closed_form():
    # dV_j = sum_i P_ij dO_i with P the softmax weights of the forward
    B, T, H, d = 1, 6, 1, 3
    q, k, v = rand((B, T, H, d), 9), rand((B, T, H, d), 10), rand((B, T, H, d), 11)
    do = rand((B, T, H, d), 12)
    _, _, dv = ref.attn_bwd(q, k, v, do, True)
    from oracle import lab
    P = np.array(lab.attention_probs(q[0, :, 0].double().tolist(), k[0, :, 0].double().tolist(),
                                     causal=True))
    assert np.allclose(dv[0, :, 0], P.T @ do[0, :, 0].double().numpy(), rtol=0, atol=1e-12)


def test_backward_over_query_blocks_and_groups_sums_to_the_whole():
    # The full-size GPU test takes one KV group and blocks of query rows
    # against keys [0, i1): groups are independent problems and each query
    # row's output depends on that row and K/V only, so dq of a block is exact
    # and dk / dv are the sums of the blocks' contributions.
    B, T, Hq, Hkv, d, G, blk = 1, 96, 8, 2, 16, 4, 32
    q, k, v = rand((B, T, Hq, d), 11), rand((B, T, Hkv, d), 12), rand((B, T, Hkv, d), 13)
    do = rand((B, T, Hq, d), 14)
    fq, fk, fv = ref.attn_bwd(q, k, v, do, True)
    for g in range(Hkv):
        hs = slice(g * G, (g + 1) * G)
        rq, rk, rv = np.zeros((B, T, G, d)), np.zeros((B, T, 1, d)), np.zeros((B, T, 1, d))
        for i0 in range(0, T, blk):
            i1 = i0 + blk
            a, b, c = ref.attn_bwd(q[:, i0:i1, hs], k[:, :i1, g:g + 1], v[:, :i1, g:g + 1],
                                   do[:, i0:i1, hs], True)
            rq[:, i0:i1] = a
            rk[:, :i1] += b
            rv[:, :i1] += c
        assert np.allclose(rq, fq[:, :, hs], atol=1e-12)
        assert np.allclose(rk, fk[:, :, g:g + 1], atol=1e-12)
        assert np.allclose(rv, fv[:, :, g:g + 1], atol=1e-12)
