"""Pins of the C/OpenMP double oracle.

It is checked against the independent pure-Python brute force of the lab
functions, against torch's scaled_dot_product_attention in float64 (a library
routine), and against closed forms and invariants the pages fix.
"""

import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F

from oracle import lab, ref
from grouped_query_attention_attn_b200 import workloads


def rand(shape, seed, std=1.0):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(shape, generator=g, dtype=torch.float32) * std)


def sdpa_ref(q, k, v, causal, scale=None):
    """float64 SDPA on [B,T,H,d] tensors with bottom-right causal alignment."""
    q64, k64, v64 = (x.double().transpose(1, 2) for x in (q, k, v))
    Tq, Tkv = q.shape[1], k.shape[1]
    mask = None
    if causal:
        i = torch.arange(Tq)[:, None]
        j = torch.arange(Tkv)[None, :]
        mask = j <= i + (Tkv - Tq)
    o = F.scaled_dot_product_attention(q64, k64, v64, attn_mask=mask, scale=scale,
                                       enable_gqa=True)
    return o.transpose(1, 2)


def brute(q, k, v, causal):
    """Lab brute force: per batch, fold (identity at g = Hkv), expand, attend."""
    B, Tq, Hq, d = q.shape
    Hkv = k.shape[2]
    out = np.zeros((B, Tq, Hq, d))
    for b in range(B):
        qh = q[b].double().transpose(0, 1).tolist()
        kh = k[b].double().transpose(0, 1).tolist()
        vh = v[b].double().transpose(0, 1).tolist()
        res = lab.heads_out(qh, kh, vh, Hkv, causal=causal)
        out[b] = np.array(res).transpose(1, 0, 2)
    return out


SHAPES = []
for hq in (1, 2, 4, 8):
    for hkv in [x for x in range(1, hq + 1) if hq % x == 0]:
        SHAPES.append((hq, hkv))


@pytest.mark.parametrize("hq,hkv", SHAPES)
@pytest.mark.parametrize("causal", [False, True])
def test_c_oracle_equals_lab_brute_force(hq, hkv, causal):
    B, T, d = 2, 9 + hq, 5
    q, k, v = rand((B, T, hq, d), 1), rand((B, T, hkv, d), 2), rand((B, T, hkv, d), 3)
    o, _ = ref.attn_fwd(q, k, v, causal)
    assert np.allclose(o, brute(q, k, v, causal), rtol=0, atol=1e-12)


@pytest.mark.parametrize("B,Tq,Tkv,Hq,Hkv,d", [(2, 33, 33, 8, 2, 16), (1, 17, 40, 4, 1, 8),
                                              (2, 31, 31, 6, 3, 12), (1, 33, 20, 4, 4, 4)])
@pytest.mark.parametrize("causal", [False, True])
def test_c_oracle_equals_sdpa_float64(B, Tq, Tkv, Hq, Hkv, d, causal):
    q, k, v = rand((B, Tq, Hq, d), 4), rand((B, Tkv, Hkv, d), 5), rand((B, Tkv, Hkv, d), 6)
    o, lse = ref.attn_fwd(q, k, v, causal)
    r = sdpa_ref(q, k, v, causal).numpy()
    n_empty = max(0, Tq - Tkv) if causal else 0
    # rows that see no key: zeros and lse = -inf (SDPA returns NaN there)
    assert np.all(o[:, :n_empty] == 0.0) and np.all(np.isneginf(lse[:, :, :n_empty]))
    assert np.allclose(o[:, n_empty:], r[:, n_empty:], rtol=0, atol=1e-12)
    # lse against logsumexp of the masked scaled scores, computed by torch
    kvh = torch.arange(Hq) // (Hq // Hkv)
    s = torch.einsum("bihc,bjhc->bhij", q.double(), k.double()[:, :, kvh]) / math.sqrt(d)
    if causal:
        i = torch.arange(Tq)[:, None]
        j = torch.arange(Tkv)[None, :]
        s = s.masked_fill(~(j <= i + (Tkv - Tq)), -math.inf)
    ls = torch.logsumexp(s, dim=-1).numpy()
    assert np.allclose(lse[:, :, n_empty:], ls[:, :, n_empty:], rtol=0, atol=1e-12)


def test_mha_special_case_runs_each_head_alone():
    # Hkv = Hq reproduces multi-head attention exactly: every head alone
    B, T, H, d = 1, 20, 4, 8
    q, k, v = rand((B, T, H, d), 7), rand((B, T, H, d), 8), rand((B, T, H, d), 9)
    o, _ = ref.attn_fwd(q, k, v, True)
    for h in range(H):
        oh, _ = ref.attn_fwd(q[:, :, h:h + 1], k[:, :, h:h + 1], v[:, :, h:h + 1], True)
        assert np.array_equal(o[:, :, h], oh[:, :, 0])


def test_gqa_equals_explicit_expansion():
    # reading K/V head hq // G equals running MHA on repeat_interleave'd K/V
    B, T, Hq, Hkv, d = 2, 15, 8, 2, 8
    q, k, v = rand((B, T, Hq, d), 10), rand((B, T, Hkv, d), 11), rand((B, T, Hkv, d), 12)
    o, _ = ref.attn_fwd(q, k, v, True)
    oe, _ = ref.attn_fwd(q, k.repeat_interleave(4, 2), v.repeat_interleave(4, 2), True)
    assert np.array_equal(o, oe)
    # the interleaved expansion [A,B,A,B] is a different (wrong) answer
    ow, _ = ref.attn_fwd(q, k.repeat(1, 1, 4, 1), v.repeat(1, 1, 4, 1), True)
    assert not np.allclose(o, ow)


def test_rows_variant_equals_full():
    B, T, Hq, Hkv, d = 2, 40, 4, 2, 8
    q, k, v = rand((B, T, Hq, d), 13), rand((B, T, Hkv, d), 14), rand((B, T, Hkv, d), 15)
    o, lse = ref.attn_fwd(q, k, v, True)
    rows = np.array([0, 5, 39, 40, 79, 200, B * Hq * T - 1])
    orow, lrow = ref.attn_fwd_rows(q, k, v, rows, True)
    for n, idx in enumerate(rows):
        i, bh = idx % T, idx // T
        hq, b = bh % Hq, bh // Hq
        assert np.array_equal(orow[n], o[b, i, hq])
        assert lrow[n] == lse[b, hq, i]


def test_causal_row0_and_no_leak():
    B, T, Hq, Hkv, d = 1, 12, 4, 2, 8
    q, k, v = rand((B, T, Hq, d), 16), rand((B, T, Hkv, d), 17), rand((B, T, Hkv, d), 18)
    o, _ = ref.attn_fwd(q, k, v, True)
    for hq in range(Hq):
        assert np.array_equal(o[0, 0, hq], v[0, 0, hq // 2].double().numpy())
    k2, v2 = k.clone(), v.clone()
    k2[:, 6:] += 3.0
    v2[:, 6:] -= 2.0
    o2, _ = ref.attn_fwd(q, k2, v2, True)
    assert np.array_equal(o[:, :6], o2[:, :6])
    assert not np.allclose(o[:, 6:], o2[:, 6:])


def test_identical_keys_closed_form():
    B, T, Hq, Hkv, d = 1, 10, 4, 1, 6
    q = rand((B, T, Hq, d), 19)
    k = rand((1, 1, 1, d), 20).expand(B, T, Hkv, d).contiguous()
    v = rand((B, T, Hkv, d), 21)
    o, _ = ref.attn_fwd(q, k, v, True)
    for i in range(T):
        mean = v[0, : i + 1, 0].double().mean(0).numpy()
        for hq in range(Hq):
            assert np.allclose(o[0, i, hq], mean, rtol=0, atol=1e-14)


def test_tiny_config_huge_logits():
    # the tiny fp32 workload rerun with q, k x 1000: the max-subtracted softmax
    # stays finite and picks the top key's value row when the top gap is large
    q, k, v = workloads.tiny_f32_inputs(qk_factor=1000.0)
    o, lse = ref.attn_fwd(q, k, v, False)
    assert np.all(np.isfinite(o)) and np.all(np.isfinite(lse))
    q64, k64 = q.double(), k.double()
    checked = 0
    for hq in range(8):
        s = (q64[0, :, hq] @ k64[0, :, hq // 4].T / 4.0).numpy()
        for i in range(16):
            top = np.sort(s[i])
            if top[-1] - top[-2] > 40.0:
                j = int(np.argmax(s[i]))
                assert np.allclose(o[0, i, hq], v[0, j, hq // 4].double().numpy(),
                                   rtol=0, atol=1e-12)
                checked += 1
    assert checked > 64


def test_tiny_config_against_lab_brute_force():
    for factor in (1.0, 1000.0):
        q, k, v = workloads.tiny_f32_inputs(qk_factor=factor)
        o, _ = ref.attn_fwd(q, k, v, False)
        assert np.allclose(o, brute(q, k, v, False), rtol=0, atol=1e-12)


def test_invalid_head_split_raises():
    q, k, v = rand((1, 4, 6, 4), 1), rand((1, 4, 4, 4), 2), rand((1, 4, 4, 4), 3)
    with pytest.raises(ValueError):
        ref.attn_fwd(q, k, v, False)


# ------------------------------------------------------------------ decode --

def decode_case(B=5, Hq=8, Hkv=2, d=16, Lmax=70, lengths=(70, 1, 33, 0, 64)):
    q, kc, vc, sl = workloads.decode_inputs(B, Hq, Hkv, d, 1, Lmax, dtype=torch.float32,
                                            lengths=lengths)
    return q, kc, vc, sl


def test_decode_is_last_row_of_forward():
    q, kc, vc, sl = decode_case()
    o, lse = ref.decode(q, kc, vc, sl)
    for b in range(q.shape[0]):
        L = int(sl[b])
        if L == 0:
            assert np.all(o[b] == 0.0) and np.all(np.isneginf(lse[b]))
            continue
        of, lf = ref.attn_fwd(q[b:b + 1, None], kc[b:b + 1, :L], vc[b:b + 1, :L], True)
        assert np.array_equal(o[b], of[0, 0])
        assert np.array_equal(lse[b], lf[0, :, 0])


def test_decode_never_reads_padding():
    q, kc, vc, sl = decode_case()
    # the cache tail past each length is NaN; a single read of it would poison o
    for b in range(q.shape[0]):
        L = int(sl[b])
        assert torch.isnan(kc[b, L:]).all() and torch.isnan(vc[b, L:]).all()
        assert not torch.isnan(kc[b, :L]).any()
    o, lse = ref.decode(q, kc, vc, sl)
    assert np.all(np.isfinite(o))


@pytest.mark.parametrize("chunk", [1, 7, 16, 64, 1000])
def test_split_lse_merge_equals_unsplit(chunk):
    q, kc, vc, sl = decode_case()
    o, lse = ref.decode(q, kc, vc, sl)
    os_, ls = ref.decode(q, kc, vc, sl, chunk=chunk)
    assert np.allclose(os_, o, rtol=0, atol=1e-12)
    fin = np.isfinite(lse)
    assert np.array_equal(np.isneginf(ls), ~fin)
    assert np.allclose(ls[fin], lse[fin], rtol=0, atol=1e-12)


def test_decode_against_sdpa():
    q, kc, vc, sl = decode_case()
    o, _ = ref.decode(q, kc, vc, sl)
    for b in range(q.shape[0]):
        L = int(sl[b])
        if L == 0:
            continue
        r = sdpa_ref(q[b:b + 1, None], kc[b:b + 1, :L], vc[b:b + 1, :L], False)
        assert np.allclose(o[b], r[0, 0].numpy(), rtol=0, atol=1e-12)


# -------------------------------------------------------------------- fold --

def test_fold_tensor_matches_lab_fold():
    # bf16 heads folded in float32 then rounded equal the lab's double mean rounded
    kv = workloads.randn((2, 5, 8, 16), 33)
    for g in (8, 4, 2, 1):
        out = ref.fold_kv_tensor(kv, g)
        assert out.dtype == torch.bfloat16 and out.shape == (2, 5, g, 16)
        for b in range(2):
            for t in range(5):
                heads = [[kv[b, t, h].double().tolist()] for h in range(8)]
                want = torch.tensor([f[0] for f in lab.fold_kv(heads, g)],
                                    dtype=torch.float64).to(torch.bfloat16)
                assert torch.equal(out[b, t], want)


@pytest.mark.parametrize("g", [8, 1])
def test_fold_tensor_matches_lab_mean_at_the_sweep_folds(g):
    # The head-sharing sweep folds its 32-head K and V to 8 and to 1 heads.  On
    # positions of those very tensors, the oracle's float32 fold (head order,
    # then one rounding to bf16) equals the lab's double mean rounded to bf16,
    # element for element (TT Lab step 2).
    _, k32, v32 = workloads.prefill_inputs(4, 2048, 32, 32, 128)
    pos = np.random.default_rng(g).choice(2048, size=16, replace=False)
    for kv in (k32, v32):
        block = kv[:, pos]                                   # [4, 16, 32, 128]
        out = ref.fold_kv_tensor(block, g)
        rows = block.double().reshape(64, 32, 128)          # (b, t) pairs as rows
        heads = [rows[:, h].tolist() for h in range(32)]     # [head][row][col]
        want = torch.tensor(lab.fold_kv(heads, g), dtype=torch.float64)   # [g][row][col]
        want = want.permute(1, 0, 2).reshape(4, 16, g, 128).to(torch.bfloat16)
        assert torch.equal(out, want)


def test_fold_tensor_identity_and_errors():
    kv = workloads.randn((1, 3, 4, 8), 34)
    assert torch.equal(ref.fold_kv_tensor(kv, 4), kv)
    with pytest.raises(ValueError):
        ref.fold_kv_tensor(kv, 3)
