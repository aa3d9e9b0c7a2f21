"""The C-ABI library: it loads, exports every entry point include/gqa.h
declares, and rejects invalid arguments on the host before any CUDA call (so
these run without a GPU)."""

import os
import re

import pytest

from grouped_query_attention_attn_b200 import _binding as b

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "gqa.h")

NULL = None
FAKE = 0x10000          # a 16-byte aligned address that is never dereferenced


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(gqa_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for must in ("gqa_attn_fwd", "gqa_attn_fwd_lse", "gqa_attn_fwd_f32", "gqa_decode",
                 "gqa_decode_workspace_size", "gqa_last_error"):
        assert must in names


def test_library_exports_every_declared_symbol(gqa_lib):
    for name in declared_functions():
        assert hasattr(gqa_lib, name), name
        assert name in b._SIGNATURES, f"{name} has no binding"


def test_binding_names_match_the_c_names():
    for name in b._SIGNATURES:
        assert callable(getattr(b, name)), name


def test_status_codes_match_header():
    text = open(HEADER).read()
    for name, val in (("GQA_OK", 0), ("GQA_ERR_INVALID_ARG", 1), ("GQA_ERR_UNSUPPORTED", 2),
                      ("GQA_ERR_CUDA", 3), ("GQA_ERR_WORKSPACE", 4), ("GQA_ERR_TIMEOUT", 5)):
        assert re.search(rf"{name}\s*=\s*{val}\b", text)
        assert getattr(b, name) == val


def fwd(**kw):
    a = dict(q=FAKE, k=FAKE, v=FAKE, o=FAKE, lse=NULL, B=1, Tq=16, Tkv=16, Hq=8, Hkv=2, d=128,
             causal=1, scale=0.088, stream=NULL)
    a.update(kw)
    return b.gqa_attn_fwd_lse(a["q"], a["k"], a["v"], a["o"], a["lse"], a["B"], a["Tq"], a["Tkv"],
                              a["Hq"], a["Hkv"], a["d"], a["causal"], a["scale"], a["stream"])


@pytest.mark.parametrize("kw,code", [
    (dict(Hq=8, Hkv=3), b.GQA_ERR_INVALID_ARG),        # the lab's ValueError: uneven groups
    (dict(Hq=6, Hkv=4), b.GQA_ERR_INVALID_ARG),
    (dict(Hkv=0), b.GQA_ERR_INVALID_ARG),
    (dict(B=-1), b.GQA_ERR_INVALID_ARG),
    (dict(Tq=-2), b.GQA_ERR_INVALID_ARG),
    (dict(scale=0.0), b.GQA_ERR_INVALID_ARG),
    (dict(scale=-1.0), b.GQA_ERR_INVALID_ARG),
    (dict(scale=float("nan")), b.GQA_ERR_INVALID_ARG),
    (dict(scale=float("inf")), b.GQA_ERR_INVALID_ARG),
    (dict(causal=2), b.GQA_ERR_INVALID_ARG),
    (dict(d=96), b.GQA_ERR_UNSUPPORTED),
    (dict(d=0), b.GQA_ERR_INVALID_ARG),
    (dict(Hq=256, Hkv=1), b.GQA_ERR_UNSUPPORTED),
    (dict(q=NULL), b.GQA_ERR_INVALID_ARG),
    (dict(o=FAKE + 8), b.GQA_ERR_INVALID_ARG),         # not 16-byte aligned
    (dict(lse=FAKE + 2), b.GQA_ERR_INVALID_ARG),
])
def test_fwd_rejects_invalid_arguments(gqa_lib, kw, code):
    assert fwd(**kw) == code
    assert b.gqa_last_error() != ""


def test_empty_problems_are_ok_without_a_gpu(gqa_lib):
    assert fwd(B=0, q=NULL, o=NULL) == b.GQA_OK
    assert fwd(Tq=0, q=NULL, o=NULL) == b.GQA_OK
    assert b.gqa_attn_fwd_f32(NULL, NULL, NULL, NULL, NULL, 0, 4, 4, 2, 1, 16, 0, 0.25, NULL) == 0
    assert b.gqa_fold_kv(NULL, NULL, 0, 4, 8, 2, 16, NULL) == b.GQA_OK


def test_f32_rejects(gqa_lib):
    assert b.gqa_attn_fwd_f32(FAKE, FAKE, FAKE, FAKE, NULL, 1, 4, 4, 8, 3, 16, 0, 0.25,
                              NULL) == b.GQA_ERR_INVALID_ARG
    assert b.gqa_attn_fwd_f32(FAKE, FAKE, FAKE, FAKE, NULL, 1, 4, 4, 8, 2, 300, 0, 0.25,
                              NULL) == b.GQA_ERR_UNSUPPORTED
    assert b.gqa_attn_fwd_f32(FAKE + 2, FAKE, FAKE, FAKE, NULL, 1, 4, 4, 8, 2, 16, 0, 0.25,
                              NULL) == b.GQA_ERR_INVALID_ARG


def test_decode_workspace_size(gqa_lib):
    n = b.gqa_decode_workspace_size(64, 32, 8, 128, 8192)
    assert n > 0 and n % 256 == 0
    # one partial row of d floats plus one lse per (split, sequence, query head)
    assert n >= 64 * 32 * (128 + 1) * 4
    assert b.gqa_decode_workspace_size(64, 32, 8, 128, 2 * 8192) > n
    assert b.gqa_decode_workspace_size(64, 32, 3, 128, 8192) == 0   # uneven groups
    assert b.gqa_decode_workspace_size(-1, 32, 8, 128, 8192) == 0


def dec(**kw):
    a = dict(q=FAKE, kc=FAKE, vc=FAKE, sl=FAKE, o=FAKE, B=4, Hq=8, Hkv=2, d=128, Lmax=1000,
             scale=0.088, ws=FAKE, ws_bytes=1 << 30, stream=NULL)
    a.update(kw)
    return b.gqa_decode(a["q"], a["kc"], a["vc"], a["sl"], a["o"], a["B"], a["Hq"], a["Hkv"],
                        a["d"], a["Lmax"], a["scale"], a["ws"], a["ws_bytes"], a["stream"])


@pytest.mark.parametrize("kw,code", [
    (dict(Hkv=3), b.GQA_ERR_INVALID_ARG),
    (dict(d=80), b.GQA_ERR_UNSUPPORTED),
    (dict(Hq=64, Hkv=1), b.GQA_ERR_UNSUPPORTED),
    (dict(Lmax=-1), b.GQA_ERR_INVALID_ARG),
    (dict(sl=NULL), b.GQA_ERR_INVALID_ARG),
    (dict(kc=FAKE + 4), b.GQA_ERR_INVALID_ARG),
    (dict(ws=NULL), b.GQA_ERR_WORKSPACE),
    (dict(ws=FAKE + 16), b.GQA_ERR_WORKSPACE),          # not 256-byte aligned
    (dict(ws_bytes=1000), b.GQA_ERR_WORKSPACE),
    (dict(scale=0.0), b.GQA_ERR_INVALID_ARG),
])
def test_decode_rejects_invalid_arguments(gqa_lib, kw, code):
    assert dec(**kw) == code
    assert b.gqa_last_error() != ""


def test_fold_rejects(gqa_lib):
    assert b.gqa_fold_kv(FAKE, FAKE, 1, 4, 8, 3, 16, NULL) == b.GQA_ERR_INVALID_ARG
    assert b.gqa_fold_kv(FAKE, FAKE, 1, 4, 8, 2, 12, NULL) == b.GQA_ERR_INVALID_ARG
    assert b.gqa_fold_kv(FAKE + 8, FAKE, 1, 4, 8, 2, 16, NULL) == b.GQA_ERR_INVALID_ARG


def test_selftest_rejects_bad_timeout(gqa_lib):
    assert b.gqa_selftest_wait_timeout(0) == b.GQA_ERR_INVALID_ARG


def test_product_package_never_imports_the_oracle():
    pkg = os.path.join(ROOT, "grouped_query_attention_attn_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                text = open(os.path.join(dirpath, f)).read()
                assert not re.search(r"^\s*(from|import)\s+oracle\b", text, re.M), f
                assert "gqa_oracle" not in text and "liboracle" not in text, f


def test_window_entry_points_reject_bad_window(gqa_lib):
    for window, sinks in ((0, 0), (-3, 0), (4, -1)):
        assert b.gqa_attn_fwd_window(FAKE, FAKE, FAKE, FAKE, NULL, 1, 8, 8, 4, 2, 128, window,
                                     sinks, 0.088, NULL) == b.GQA_ERR_INVALID_ARG
        assert b.gqa_decode_window(FAKE, FAKE, FAKE, FAKE, FAKE, 2, 4, 2, 128, 64, window, sinks,
                                   0.088, FAKE, 1 << 20, NULL) == b.GQA_ERR_INVALID_ARG
    # the usual shape checks still apply
    assert b.gqa_attn_fwd_window(FAKE, FAKE, FAKE, FAKE, NULL, 1, 8, 8, 6, 4, 128, 4, 0, 0.088,
                                 NULL) == b.GQA_ERR_INVALID_ARG


def test_host_forward_rejects(gqa_lib):
    args = (1, 64, 64, 4, 2, 128, 1, 0.088, NULL, NULL)
    assert b.gqa_attn_fwd_host(NULL, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, *args) == \
        b.GQA_ERR_INVALID_ARG                                                   # q_host
    assert b.gqa_attn_fwd_host(FAKE, FAKE, FAKE, FAKE, FAKE + 8, FAKE, FAKE, FAKE, *args) == \
        b.GQA_ERR_INVALID_ARG                                                   # q_dev alignment
    assert b.gqa_attn_fwd_host(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE,
                               1, 64, 64, 4, 3, 128, 1, 0.088, NULL, NULL) == b.GQA_ERR_INVALID_ARG
    assert b.gqa_attn_fwd_host(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE,
                               1, 64, 64, 4, 2, 96, 1, 0.088, NULL, NULL) == b.GQA_ERR_UNSUPPORTED
    assert b.gqa_attn_fwd_host(NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL,
                               1, 0, 64, 4, 2, 128, 1, 0.088, NULL, NULL) == b.GQA_OK  # empty


def test_rope_rejects(gqa_lib):
    assert b.gqa_rope(FAKE, 1, 4, 2, 12, 0, 10000.0, NULL) == b.GQA_ERR_INVALID_ARG   # d % 8
    assert b.gqa_rope(FAKE, 1, 4, 2, 128, 0, 0.0, NULL) == b.GQA_ERR_INVALID_ARG      # theta
    assert b.gqa_rope(FAKE + 8, 1, 4, 2, 128, 0, 10000.0, NULL) == b.GQA_ERR_INVALID_ARG
    assert b.gqa_rope(NULL, 0, 4, 2, 128, 0, 10000.0, NULL) == b.GQA_OK              # empty
    assert b.gqa_rope_decode_q(FAKE, NULL, 2, 2, 128, 10000.0, NULL) == b.GQA_ERR_INVALID_ARG
    assert b.gqa_rope_qk(FAKE, FAKE, 1, 4, 4, 2, 128, 0, 10000.0, NULL) == b.GQA_ERR_INVALID_ARG
    assert b.gqa_rope_qk(FAKE, NULL, 1, 4, 4, 2, 128, 0, 10000.0, NULL) == b.GQA_ERR_INVALID_ARG
    assert b.gqa_rope_qk(FAKE, FAKE + 16, 1, 4, 4, 0, 128, 0, 10000.0, NULL) == \
        b.GQA_ERR_INVALID_ARG                                                           # Hkv
    assert b.gqa_rope_qk(NULL, NULL, 1, 0, 4, 2, 128, 0, 10000.0, NULL) == b.GQA_OK    # empty


def test_backward_rejects(gqa_lib):
    def bwd(**kw):
        a = dict(B=1, Tq=8, Tkv=8, Hq=4, Hkv=2, d=128, causal=1, window=0, sinks=0, ws=FAKE,
                 ws_bytes=1 << 20, lse=FAKE)
        a.update(kw)
        return b.gqa_attn_bwd(FAKE, FAKE, FAKE, FAKE, FAKE, a["lse"], FAKE, FAKE, FAKE, a["B"],
                              a["Tq"], a["Tkv"], a["Hq"], a["Hkv"], a["d"], a["causal"],
                              a["window"], a["sinks"], 0.088, a["ws"], a["ws_bytes"], NULL)
    assert bwd(Hkv=3) == b.GQA_ERR_INVALID_ARG
    assert bwd(d=96) == b.GQA_ERR_UNSUPPORTED
    assert bwd(window=4, causal=0) == b.GQA_ERR_INVALID_ARG
    assert bwd(lse=NULL) == b.GQA_ERR_INVALID_ARG
    assert bwd(ws=NULL) == b.GQA_ERR_WORKSPACE
    assert bwd(ws_bytes=16) == b.GQA_ERR_WORKSPACE
    assert bwd(B=0) == b.GQA_OK
    # D per query row rounded up to 256 bytes, then 256 bytes for the dQ work counter
    assert b.gqa_attn_bwd_workspace_size(2, 100, 8) == (2 * 100 * 8 * 4 + 255) // 256 * 256 + 256
    assert b.gqa_attn_bwd_workspace_size(1, 64, 4) == 1024 + 256


def test_fused_rope_entry_points_reject(gqa_lib):
    # the fused-RoPE forward and decode check theta and the position offset first
    fwd = dict(q=FAKE, k=FAKE, v=FAKE, o=FAKE, lse=NULL, B=1, Tq=8, Tkv=8, Hq=4, Hkv=2, d=128,
               causal=1, scale=0.088, q_pos0=0, theta=10000.0)

    def call(**kw):
        a = dict(fwd)
        a.update(kw)
        return b.gqa_attn_fwd_rope(*a.values(), NULL)

    assert call(theta=0.0) == b.GQA_ERR_INVALID_ARG
    assert call(theta=float("inf")) == b.GQA_ERR_INVALID_ARG
    assert call(q_pos0=-1) == b.GQA_ERR_INVALID_ARG
    assert call(Hkv=3) == b.GQA_ERR_INVALID_ARG
    assert call(d=96) == b.GQA_ERR_UNSUPPORTED
    assert call(B=0) == b.GQA_OK
    assert b.gqa_decode_rope(FAKE, FAKE, FAKE, FAKE, FAKE, 4, 8, 2, 128, 100, 0.088, -1.0,
                             FAKE, 1 << 20, NULL) == b.GQA_ERR_INVALID_ARG
    assert b.gqa_decode_rope(NULL, FAKE, FAKE, FAKE, FAKE, 4, 8, 2, 128, 100, 0.088, 1e4,
                             FAKE, 1 << 20, NULL) == b.GQA_ERR_INVALID_ARG
