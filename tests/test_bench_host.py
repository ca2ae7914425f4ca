"""Host logic of bench.py that needs no GPU: the FLOP count behind every TFLOP/s figure, the
algorithmic bytes behind the HBM fractions, and the gating of the measured DRAM traffic on the
hash of the device sources it was taken on."""
import json
import os
import shutil

import pytest

import bench
from mla_prefill_attention_varlen_b200 import workloads as W


def causal_pairs(lq, lk):
    """Closed form of the visible (query, key) pairs of one sequence and head, bottom-right causal:
    row i sees min(i + lk - lq + 1, lk) keys (none while that is <= 0)."""
    off = lk - lq
    total = 0
    for i in range(lq):
        total += max(0, min(i + off + 1, lk))
    return total


def test_visible_triples_match_closed_forms():
    # uniform: L (L + 1) / 2 per sequence and head
    w = W.get("uniform")
    assert bench.visible_triples(w) == 4 * 16 * (1024 * 1025 // 2)
    # long: one sequence of 16384 over 128 heads (the 21.5 GFLOP / 11.0 TFLOP figures of the docs)
    w = W.get("long")
    assert bench.visible_triples(w) == 128 * (16384 * 16385 // 2) == 17180917760
    # chunked: 512 new rows over a 4096-key prefix, row i sees 3584 + i + 1 keys
    w = W.get("chunked")
    assert bench.visible_triples(w) == 8 * 128 * (512 * 3585 + 511 * 512 // 2) == 2013528064
    # varlen_gqa and tiny: the per-sequence closed form summed (query heads, not kv heads)
    for name in ("varlen_gqa", "tiny"):
        w = W.get(name)
        expect = sum(causal_pairs(lq, lk) for lq, lk in zip(w.q_seqlens, w.kv_seqlens)) * w.head_num
        assert bench.visible_triples(w) == expect


def test_visible_triples_without_mask_and_with_short_prefix():
    w = W.Workload("probe", [3, 5], [7, 2], 2, 1, seed=0)
    w.causal = False
    assert bench.visible_triples(w) == (3 * 7 + 5 * 2) * 2
    w.causal = True
    # lq > lk: the first lq - lk rows see nothing
    assert bench.visible_triples(w) == (causal_pairs(3, 7) + causal_pairs(5, 2)) * 2
    assert causal_pairs(5, 2) == 0 + 0 + 0 + 1 + 2


def test_algorithmic_bytes_of_long():
    # Q, Q_rope, K, K_rope, V read once, O written once: 2 B x 16384 x 128 x (192 + 320 + 128)
    w = W.get("long")
    assert bench.algorithmic_bytes(w) == 2 * 16384 * 128 * (192 + 320 + 128) == 2684354560


def test_traffic_is_reported_only_for_the_sources_it_was_taken_on(tmp_path, monkeypatch):
    # a copy of the device sources and a traffic record in a scratch tree
    for rel in set(bench.KERNEL_SOURCES + bench.PROLOG_Q_SOURCES):
        dst = tmp_path / rel
        dst.parent.mkdir(parents=True, exist_ok=True)
        shutil.copy(os.path.join(bench.ROOT, rel), dst)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    good = bench.kernel_sources_hash()
    good_q = bench.kernel_sources_hash(bench.PROLOG_Q_SOURCES)
    assert good != good_q
    (tmp_path / "profiles").mkdir()
    record = {"launches": {
        "a": {"traffic_bytes_per_launch": 123, "kernel_sources_sha256": good},
        "b": {"traffic_bytes_per_launch": 456, "kernel_sources_sha256": "0" * 64},
        "q": {"traffic_bytes_per_launch": 789, "kernel_sources_sha256": good_q},
        "c": {"kernel_sources_sha256": good},
    }}
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps(record))
    assert bench.measured_traffic("a") == 123
    assert bench.measured_traffic("b") is None       # taken on other sources
    assert bench.measured_traffic("c") is None       # no figure
    assert bench.measured_traffic("missing") is None
    assert bench.measured_traffic("q") is None       # keyed on the q kernel's sources, not these
    assert bench.measured_traffic("q", bench.PROLOG_Q_SOURCES) == 789
    # any edit of a device source invalidates the figure
    src = tmp_path / bench.KERNEL_SOURCES[0]
    src.write_text(src.read_text() + "\n// edited\n")
    assert bench.measured_traffic("a") is None
