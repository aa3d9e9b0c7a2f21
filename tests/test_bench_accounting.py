"""The bench's accounting (CPU): visible (query, key) pairs, algorithmic FLOPs
and bytes, and the lookup of recorded DRAM traffic by kernel source hash."""

import itertools

import pytest
import torch

import bench


def brute_pairs(Tq, Tkv, causal, window, sinks):
    # one (i, j) at a time: bottom-right causal mask, window of the last W keys
    # up to the query's position, plus the first `sinks` keys
    n = 0
    for i in range(Tq):
        p = i + (Tkv - Tq)
        for j in range(Tkv):
            if not causal:
                n += 1
            elif j <= p and (window == 0 or j > p - window or j < sinks):
                n += 1
    return n


@pytest.mark.parametrize("Tq,Tkv", [(1, 1), (7, 7), (5, 12), (12, 5), (33, 33), (0, 4)])
def test_visible_pairs_match_brute_force(Tq, Tkv):
    for causal, window, sinks in itertools.product((False, True), (0, 1, 3, 8), (0, 2, 40)):
        if not causal and window:
            continue
        got = bench.visible_pairs(Tq, Tkv, causal, window, sinks)
        assert got == brute_pairs(Tq, Tkv, causal, window, sinks), (causal, window, sinks)


def test_prefill_flops_are_four_d_per_visible_pair_and_head():
    c = bench.PREFILL
    assert bench.prefill_flops(c) == 4 * c["B"] * c["Hq"] * c["d"] * bench.visible_pairs(
        c["T"], c["T"], c["causal"])
    assert bench.prefill_flops(dict(c, causal=False)) == 4 * c["B"] * c["Hq"] * c["d"] * c["T"] ** 2


def test_decode_bytes_count_every_cached_row_once_per_group():
    c = dict(B=3, Hq=8, Hkv=2, d=128)
    sl = torch.tensor([5, 0, 17], dtype=torch.int32)
    kv = (5 + 0 + 17) * 2 * 128 * 2 * 2          # rows x Hkv x d x (K, V) x bf16
    qo = 2 * 3 * 8 * 128 * 2                      # q in, o out
    assert bench.decode_bytes(sl, c) == kv + qo


def test_recorded_traffic_needs_the_matching_source_hash(tmp_path, monkeypatch):
    f = tmp_path / "traffic.txt"
    f.write_text("# comment\nprefill_kernel abcdef0123456789 1000\nother 1 2 3\n")
    monkeypatch.setattr(bench, "TRAFFIC_FILE", str(f))
    assert bench.recorded_traffic("prefill_kernel", "abcdef0123456789") == 1000
    assert bench.recorded_traffic("prefill_kernel", "0000000000000000") is None
    assert bench.recorded_traffic("decode_split_kernel", "abcdef0123456789") is None
    monkeypatch.setattr(bench, "TRAFFIC_FILE", str(tmp_path / "missing.txt"))
    assert bench.recorded_traffic("prefill_kernel", "abcdef0123456789") is None


def test_source_hash_is_stable_and_order_sensitive():
    a = bench.kernel_source_hash(["prefill.cu", "device.cuh"])
    assert a == bench.kernel_source_hash(["prefill.cu", "device.cuh"])
    assert len(a) == 16 and int(a, 16) >= 0
    assert a != bench.kernel_source_hash(["device.cuh", "prefill.cu"])
