"""Host-side pins of bench.py's algorithmic byte and flop counts against the
figures the design states for each workload (closed forms of the shapes)."""
from __future__ import annotations

import bench
from indexed_sparse_attention_kv_b200 import inputs as I


def test_decode_128k_bytes():
    kt, kv, small = bench.algorithmic_bytes(I.workload("decode_128k"))
    assert kt == 4 * 131072 * 8 * 64 * 2 == 536_870_912
    assert kv == 4 * 8 * 2048 * 128 * 2 * 2 == 33_554_432
    assert kt + kv + small == 570_507_264


def test_resident_workload_bytes():
    assert bench.resident_bytes(I.workload("llama8b_32k")) == 35_672_064
    assert bench.resident_bytes(I.workload("hier_1m")) == 29_380_608


def test_prefill_flop():
    # sum over p = T-4096 .. T-1 of (p + 1) keys, 8 KV heads, 2 r flops each
    w = I.workload("prefill_128k")
    pairs = sum(range(w.T - w.nq + 1, w.T + 1))
    assert pairs == 528_484_352
    assert bench.prefill_scoring_flop(w) == 2 * pairs * 8 * 64 == 541_167_976_448


def test_prepare_bytes():
    assert bench.prepare_bytes(bench.PREPARE_SHAPE) == 1_073_741_824 + 536_870_912 + 131_072
