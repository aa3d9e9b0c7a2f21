"""Pins of the pure-Python lab oracle against what the pages and mathematics fix.

Pages: TT Lab "キー・バリューヘッドだけ減らしてみる" (tf-gqa-lab, steps 1-8),
course "Неделя 7. Внимание" (steps 1-2, "Типичные ошибки"), and the K3 notes
section "GVA（分组值注意力）" (subsections "Forward: repeat_interleave" and
"Backward: view + sum").
"""

import inspect
import json
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

from oracle import lab
from grouped_query_attention_attn_b200 import workloads

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def to_t(heads):
    return torch.tensor(heads, dtype=torch.float64)


# ---------------------------------------------------------------- grouping --

def test_group_of_contiguous_h8_g2():
    # lab step 1: with h=8, g=2 the heads 0, 1, 2, 3 form group 0.
    assert [lab.group_of(i, 8, 2) for i in range(8)] == [0, 0, 0, 0, 1, 1, 1, 1]
    # the interleaved rule head % g is the wrong one the page warns about
    assert [i % 2 for i in range(8)] != [lab.group_of(i, 8, 2) for i in range(8)]


def test_group_members_built_from_group_of():
    assert lab.group_members(8, 2) == [[0, 1, 2, 3], [4, 5, 6, 7]]
    assert lab.group_members(8, 8) == [[i] for i in range(8)]
    assert lab.group_members(8, 1) == [list(range(8))]


@pytest.mark.parametrize("h,g", [(8, 3), (6, 4), (4, 0), (32, 5)])
def test_uneven_groups_raise(h, g):
    # lab steps 1, 2, 3, 6, 7: uneven division is a ValueError
    with pytest.raises(ValueError):
        lab.group_of(0, h, g)
    with pytest.raises(ValueError):
        lab.group_members(h, g)
    with pytest.raises(ValueError):
        lab.mults(16, 32, h, g, 4)
    with pytest.raises(ValueError):
        lab.kv_table(1, h, [g], 4, 4)
    heads = lab.make_heads(h, 2, 3, 7)
    if g > 0:
        with pytest.raises(ValueError):
            lab.fold_kv(heads, g)


def test_expand_ab_to_aabb():
    # lab step 3: [A, B] expanded to 4 heads is [A, A, B, B], not [A, B, A, B]
    A = [[1.0, 2.0]]
    B = [[3.0, 4.0]]
    out = lab.expand_kv([A, B], 4)
    assert out == [A, A, B, B]
    assert out != [A, B, A, B]
    with pytest.raises(ValueError):
        lab.expand_kv([A, B], 3)


def test_expand_returns_copies():
    A = [[1.0, 2.0]]
    out = lab.expand_kv([A], 2)
    out[0][0][0] = 99.0
    assert out[1][0][0] == 1.0 and A[0][0] == 1.0


@pytest.mark.parametrize("h,g", [(8, 1), (8, 2), (8, 4), (8, 8), (12, 3), (32, 8)])
def test_expand_matches_group_of(h, g):
    # lab step 3: what query head i sees is folded[group_of(i, h, g)]
    folded = lab.make_heads(g, 3, 2, 11)
    out = lab.expand_kv(folded, h)
    for i in range(h):
        assert out[i] == folded[lab.group_of(i, h, g)]


def test_expand_is_repeat_interleave():
    # K3 notes "Forward: repeat_interleave": H=4, G=2 -> head 0 feeds heads 0 and 1,
    # head 1 feeds 2 and 3; the library routine gives the same order.
    heads = lab.make_heads(4, 2, 3, 5)
    out = to_t(lab.expand_kv(heads, 8))
    ref = to_t(heads).repeat_interleave(2, dim=0)
    assert torch.equal(out, ref)
    assert torch.equal(out[0], to_t(heads)[0]) and torch.equal(out[1], to_t(heads)[0])
    assert torch.equal(out[2], to_t(heads)[1]) and torch.equal(out[3], to_t(heads)[1])


def test_repeat_interleave_backward_is_sum():
    # K3 notes "Backward: view + sum": the gradient of a copied head is the SUM
    # of the copies' gradients (not the mean).  Checked on the library routine
    # so the GQA expansion the oracle mirrors has the backward the page states.
    x = torch.randn(2, 3, 4, 5, dtype=torch.float64, requires_grad=True)
    y = x.repeat_interleave(3, dim=2)
    gy = torch.randn_like(y)
    y.backward(gy)
    assert torch.allclose(x.grad, gy.view(2, 3, 4, 3, 5).sum(3), rtol=0, atol=1e-14)


# -------------------------------------------------------------------- fold --

def test_fold_identity_when_g_equals_heads():
    heads = lab.make_heads(4, 3, 5, 9)
    assert lab.fold_kv(heads, 4) == heads


@pytest.mark.parametrize("n,g", [(8, 4), (8, 2), (8, 1), (6, 3), (32, 8)])
def test_fold_is_mean_of_contiguous_slices(n, g):
    heads = lab.make_heads(n, 3, 4, 13)
    out = np.array(lab.fold_kv(heads, g))
    ref = np.array(heads).reshape(g, n // g, 3, 4).mean(axis=1)
    assert np.allclose(out, ref, rtol=0, atol=1e-15)
    if g < n:
        # the two mistakes the lab names: keeping only the first head of each
        # group, and averaging every head regardless of the group
        first_only = np.array(heads)[:: n // g]
        all_mean = np.broadcast_to(np.array(heads).mean(axis=0), out.shape)
        assert not np.allclose(out, first_only)
        if g > 1:
            assert not np.allclose(out, all_mean)


# ------------------------------------------------------------- make_heads --

def test_make_heads_deterministic_and_bounded():
    a = lab.make_heads(8, 6, 4, 101)
    b = lab.make_heads(8, 6, 4, 101)
    c = lab.make_heads(8, 6, 4, 202)
    assert a == b and a != c
    flat = np.array(a).ravel()
    assert flat.shape == (8 * 6 * 4,)
    assert np.all(np.abs(flat) <= 4.0)                 # lab step 1: |x| <= 4
    assert np.all(flat >= -0.5) and np.all(flat < 0.5)  # state/m - 0.5
    assert len(set(flat.tolist())) == flat.size


def test_make_heads_matches_workload_sampler():
    # the shared input sampler and the lab function implement the same LCG
    assert np.array_equal(np.array(lab.make_heads(8, 16, 16, 101)),
                          workloads.lcg_heads(8, 16, 16, 101))


def test_lcg_first_values_from_definition():
    # state_1 = (a*seed + c) mod m computed with Python integers
    s1 = (1664525 * 101 + 1013904223) % 2 ** 32
    s2 = (1664525 * s1 + 1013904223) % 2 ** 32
    h = lab.make_heads(1, 1, 2, 101)
    assert h[0][0] == [s1 / 2 ** 32 - 0.5, s2 / 2 ** 32 - 0.5]


# ------------------------------------------------------------------ attend --

def sdpa64(q, k, v, causal=False, scale=None):
    """torch SDPA in float64 on [T, d] tables."""
    q, k, v = to_t(q)[None, None], to_t(k)[None, None], to_t(v)[None, None]
    mask = None
    if causal:
        tq, tk = q.shape[2], k.shape[2]
        i = torch.arange(tq)[:, None]
        j = torch.arange(tk)[None, :]
        mask = j <= i + (tk - tq)           # bottom-right alignment
    return F.scaled_dot_product_attention(q, k, v, attn_mask=mask, scale=scale)[0, 0]


@pytest.mark.parametrize("tq,tk,d", [(6, 6, 4), (1, 9, 8), (7, 3, 5), (16, 16, 16)])
@pytest.mark.parametrize("causal", [False, True])
def test_attend_matches_sdpa_float64(tq, tk, d, causal):
    q = lab.make_heads(1, tq, d, 1)[0]
    k = lab.make_heads(1, tk, d, 2)[0]
    v = lab.make_heads(1, tk, d, 3)[0]
    out = to_t(lab.attend(q, k, v, causal=causal))
    ref = sdpa64(q, k, v, causal=causal)
    if causal and tq > tk:
        # rows with no visible key: the oracle returns zeros (SDPA gives NaN)
        n_empty = tq - tk
        assert torch.equal(out[:n_empty], torch.zeros_like(out[:n_empty]))
        out, ref = out[n_empty:], ref[n_empty:]
    assert torch.allclose(out, ref, rtol=0, atol=1e-12)


def test_scale_is_one_over_sqrt_head_dim():
    # lab step 4 and the course's step 1: scores are divided by sqrt(head dim)
    q = lab.make_heads(1, 5, 16, 21)[0]
    k = lab.make_heads(1, 7, 16, 22)[0]
    v = lab.make_heads(1, 7, 16, 23)[0]
    out = to_t(lab.attend(q, k, v))
    assert torch.allclose(out, sdpa64(q, k, v, scale=0.25), rtol=0, atol=1e-12)
    assert not torch.allclose(out, sdpa64(q, k, v, scale=1.0), rtol=0, atol=1e-6)


@pytest.mark.parametrize("causal", [False, True])
def test_softmax_rows_sum_to_one(causal):
    q = lab.make_heads(1, 9, 4, 31)[0]
    k = lab.make_heads(1, 9, 4, 32)[0]
    for row in lab.attention_probs(q, k, causal=causal):
        assert abs(sum(row) - 1.0) < 1e-12
        assert all(p >= 0.0 for p in row)


def test_huge_logits_no_overflow():
    # lab step 4: the grader feeds large values; without subtracting the max
    # math.exp overflows.  The limit is a one-hot pick of the top key.
    q = (np.array(lab.make_heads(1, 6, 4, 41)[0]) * 1e4).tolist()
    k = (np.array(lab.make_heads(1, 6, 4, 42)[0]) * 1e4).tolist()
    v = lab.make_heads(1, 6, 4, 43)[0]
    with pytest.raises(OverflowError):
        [math.exp(sum(a * b for a, b in zip(q[0], kk)) / 2.0) for kk in k]
    out = lab.attend(q, k, v)
    s = np.array(q) @ np.array(k).T / 2.0
    for i in range(6):
        top2 = np.sort(s[i])[-2:]
        assert top2[1] - top2[0] > 50          # gap huge for these seeds
        assert out[i] == v[int(np.argmax(s[i]))]


def test_causal_first_row_is_first_value():
    q = lab.make_heads(1, 5, 4, 51)[0]
    k = lab.make_heads(1, 5, 4, 52)[0]
    v = lab.make_heads(1, 5, 4, 53)[0]
    assert lab.attend(q, k, v, causal=True)[0] == v[0]


def test_causal_no_future_leakage():
    # course "Типичные ошибки": the future must not leak into a row
    q = lab.make_heads(1, 8, 4, 61)[0]
    k = lab.make_heads(1, 8, 4, 62)[0]
    v = lab.make_heads(1, 8, 4, 63)[0]
    base = lab.attend(q, k, v, causal=True)
    for i in range(8):
        k2 = [row[:] for row in k]
        v2 = [row[:] for row in v]
        for j in range(i + 1, 8):
            k2[j] = [x + 5.0 for x in k2[j]]
            v2[j] = [x - 3.0 for x in v2[j]]
        assert lab.attend(q, k2, v2, causal=True)[i] == base[i]


def test_mask_after_softmax_breaks_row_sum():
    # course step 1: zeroing weights after the softmax leaves rows that no
    # longer sum to one; the oracle masks before the softmax.
    q = lab.make_heads(1, 6, 4, 71)[0]
    k = lab.make_heads(1, 6, 4, 72)[0]
    full = lab.attention_probs(q, k, causal=False)
    after = [[p if j <= i else 0.0 for j, p in enumerate(row)] for i, row in enumerate(full)]
    assert any(abs(sum(r) - 1.0) > 1e-3 for r in after)
    before = lab.attention_probs(q, k, causal=True)
    assert all(abs(sum(r) - 1.0) < 1e-12 for r in before)


def test_identical_keys_give_mean_of_visible_values():
    q = lab.make_heads(1, 5, 4, 81)[0]
    k = [lab.make_heads(1, 1, 4, 82)[0][0]] * 5
    v = lab.make_heads(1, 5, 4, 83)[0]
    out = lab.attend(q, k, v, causal=True)
    for i in range(5):
        mean = np.array(v[: i + 1]).mean(axis=0)
        assert np.allclose(out[i], mean, rtol=0, atol=1e-15)


# --------------------------------------------------------------- heads_out --

def lab_sample():
    # lab step 8: Q, K, V = make_heads(8, 6, 4, 101 / 202 / 303)
    return (lab.make_heads(8, 6, 4, 101), lab.make_heads(8, 6, 4, 202),
            lab.make_heads(8, 6, 4, 303))


def test_heads_out_g_equals_h_is_mha_exactly():
    q, k, v = lab_sample()
    mha = [lab.attend(q[i], k[i], v[i]) for i in range(8)]
    assert lab.max_gap(lab.heads_out(q, k, v, 8), mha) == 0.0


def test_smaller_g_changes_output():
    q, k, v = lab_sample()
    ref = lab.heads_out(q, k, v, 8)
    gaps = [lab.max_gap(lab.heads_out(q, k, v, g), ref) for g in (8, 4, 2, 1)]
    assert gaps[0] == 0.0
    assert all(gp > 0.0 for gp in gaps[1:])


def test_heads_out_matches_sdpa_gqa():
    # fold+expand then attend == SDPA with enable_gqa on the folded K/V
    q, k, v = lab_sample()
    for g in (4, 2, 1):
        out = to_t(lab.heads_out(q, k, v, g))
        kf, vf = to_t(lab.fold_kv(k, g)), to_t(lab.fold_kv(v, g))
        ref = F.scaled_dot_product_attention(to_t(q)[None], kf[None], vf[None],
                                             enable_gqa=True)[0]
        assert torch.allclose(out, ref, rtol=0, atol=1e-12)


def test_max_gap():
    a = [[[0.0, 1.0], [2.0, 3.0]]]
    b = [[[0.0, 1.5], [1.0, 3.0]]]
    assert lab.max_gap(a, b) == 1.0
    assert lab.max_gap(a, a) == 0.0


# ------------------------------------------------------------------ counts --

def test_kv_cache_elems_has_no_query_head_term():
    params = list(inspect.signature(lab.kv_cache_elems).parameters)
    assert params == ["layers", "kv_heads", "seq_len", "head_dim"]
    assert lab.kv_cache_elems(1, 1, 1, 1) == 2          # K and V


def test_kv_cache_reductions_printed_on_pages():
    # course step 2: Llama-3-8B 32 -> 8 KV heads shrinks the cache 4x; MQA 32x
    full = lab.kv_cache_elems(32, 32, 4096, 128)
    assert full // lab.kv_cache_elems(32, 8, 4096, 128) == 4
    assert full // lab.kv_cache_elems(32, 1, 4096, 128) == 32
    # lab step 8: with h=8 the cache shrinks by up to 8x
    t = dict(lab.kv_table(32, 8, [8, 4, 2, 1], 4096, 128))
    assert t[8] // t[1] == 8


def count_mults_brute(n, d_model, h, g, head_dim):
    """Count multiplications by running a naive loop implementation of one layer."""
    count = {"proj_q": 0, "proj_k": 0, "proj_v": 0, "scores": 0, "weighted": 0,
             "proj_out": 0}
    x = lab.make_heads(1, n, d_model, 3)[0]

    def proj(name, out_dim):
        out = []
        for t in range(n):
            row = []
            for o in range(out_dim):
                acc = 0.0
                for c in range(d_model):
                    acc += x[t][c] * 0.5
                    count[name] += 1
                row.append(acc)
            out.append(row)
        return out

    q = proj("proj_q", h * head_dim)
    k = proj("proj_k", g * head_dim)
    proj("proj_v", g * head_dim)
    ctx = [[0.0] * (h * head_dim) for _ in range(n)]
    for head in range(h):
        kvh = lab.group_of(head, h, g)
        for i in range(n):
            for j in range(n):
                for c in range(head_dim):
                    _ = q[i][head * head_dim + c] * k[j][kvh * head_dim + c]
                    count["scores"] += 1
            for j in range(n):
                for c in range(head_dim):
                    ctx[i][head * head_dim + c] += 0.1 * 0.2
                    count["weighted"] += 1
    for t in range(n):
        for o in range(d_model):
            for c in range(h * head_dim):
                _ = ctx[t][c] * 0.3
                count["proj_out"] += 1
    count["total"] = sum(count.values())
    return count


@pytest.mark.parametrize("n,d_model,h,g,hd", [(3, 4, 4, 2, 2), (2, 6, 6, 3, 2), (4, 2, 2, 1, 3)])
def test_mults_equal_brute_force_count(n, d_model, h, g, hd):
    assert lab.mults(n, d_model, h, g, hd) == count_mults_brute(n, d_model, h, g, hd)


def test_core_mults_do_not_depend_on_g():
    core = {g: lab.mults(4096, 1024, 8, g, 128)["scores"] + lab.mults(4096, 1024, 8, g, 128)["weighted"]
            for g in (8, 4, 2, 1)}
    assert len(set(core.values())) == 1                 # core_same_for_all_g
    m8, m1 = lab.mults(4096, 1024, 8, 8, 128), lab.mults(4096, 1024, 8, 1, 128)
    changed = {key for key in m8 if m8[key] != m1[key]}
    assert changed == {"proj_k", "proj_v", "total"}
    # lab conclusion: cache shrinks 8x while multiplies barely change
    assert m8["total"] / m1["total"] < 1.2


def test_lab_counts_golden():
    with open(os.path.join(GOLDEN, "lab_counts.json")) as f:
        gold = json.load(f)
    s = gold["sizes"]
    assert [list(x) for x in lab.kv_table(s["layers"], s["h"], s["groups"], s["seq_len"],
                                          s["head_dim"])] == gold["kv_table"]
    for g in s["groups"]:
        assert lab.mults(s["n_tokens"], s["d_model"], s["h"], g, s["head_dim"]) == \
            gold["mult_table"][str(g)]
