"""Host-side checks of bench.py: its algorithmic byte and flop counts against
the closed forms of each workload's shapes, the secondary-workload summary and
line collection, and the reference arm's JSON line (the oracle on the host)."""
from __future__ import annotations

import json

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


def test_secondary_summary_keeps_the_figures():
    line = {"metric": "m", "value": 2.0, "unit": "steps/s", "steps": 8, "ms_per_step": 0.5, "higher_is_better": True,
            "config": {"workload": "hier_1m", "T": 1 << 20},
            "roofline": {"bound": "hbm", "kernel": "k", "achieved": 1.0, "peak": 2.0, "unit": "GB/s", "frac": 0.5,
                         "traffic": None},
            "e2e": {"value": 1.5, "unit": "steps/s", "h2d_bytes_per_step": 4},
            "clocks": {"sm_mhz": 1965, "sm_max_mhz": 1965, "reasons": []}, "device_status": 0}
    s = bench.secondary_summary(line)
    assert s["workload"] == "hier_1m" and s["value"] == 2.0 and s["ms_per_step"] == 0.5
    assert s["roofline"]["frac"] == 0.5 and s["e2e"] == {"value": 1.5, "unit": "steps/s"}
    assert s["clocks"]["sm_mhz"] == 1965 and s["device_status"] == 0


def test_emit_collects_while_a_sink_is_set(capsys):
    bench._SINK = []
    try:
        bench.emit({"a": 1})
        assert bench._SINK == [{"a": 1}]
    finally:
        bench._SINK = None
    bench.emit({"b": 2})
    assert capsys.readouterr().out.strip() == '{"b": 2}'


def _reference_line(capsys, *argv):
    assert bench.main(["--impl", "reference", *argv]) == 0
    out = capsys.readouterr().out.strip().splitlines()
    assert len(out) == 1
    return json.loads(out[0])


def test_reference_arm_line(capsys):
    """The reference arm (the oracle on the host cores) prints one line with
    the contract's keys; steps x ms_per_step is its timed region."""
    d = _reference_line(capsys, "--workload", "llama8b_32k", "--steps", "1", "--warmup", "1")
    assert d["impl"] == "reference" and d["value"] > 0 and d["steps"] == 1
    assert d["unit"] == "steps/s" and d["higher_is_better"] is True
    assert abs(d["value"] - 1e3 / d["ms_per_step"]) <= 1e-6 * d["value"]
    assert d["config"]["workload"] == "llama8b_32k" and "parallelism" in d["config"]
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"] == {"value": d["value"], "unit": d["unit"], "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}


def test_reference_arm_comparators_unavailable(capsys):
    d = _reference_line(capsys, "--workload", "full_kv_128k")
    assert d["impl"] == "reference" and "unavailable" in d


def test_secondary_workloads_are_collected_into_the_headline(capsys, monkeypatch):
    """run_with_secondaries: the headline line is printed once, with every other
    workload's summary under "secondary"; a workload that raises is recorded
    as an error instead of hiding the others (host logic only: the GPU runs
    are replaced by stubs that emit lines)."""
    import argparse
    import sys
    import types

    fake_torch = types.SimpleNamespace(cuda=types.SimpleNamespace(empty_cache=lambda: None))
    monkeypatch.setitem(sys.modules, "torch", fake_torch)

    def fake_ours(args, rank, world, local_rank):
        bench.emit({"metric": "m", "value": 1.0, "unit": "steps/s", "config": {"workload": "decode_128k"}})
        return 0

    def fake_workload(args, rank, world, local_rank):
        if args.workload == "hier_1m":
            raise RuntimeError("boom")
        assert args.no_cpu_baseline
        bench.emit({"metric": args.workload, "value": 2.0, "unit": "u", "steps": 3, "ms_per_step": 0.5,
                    "config": {"workload": args.workload}, "roofline": {"frac": 0.5}})
        return 0

    monkeypatch.setattr(bench, "run_ours", fake_ours)
    monkeypatch.setattr(bench, "run_workload", fake_workload)
    args = argparse.Namespace(workload="decode_128k", no_cpu_baseline=False, steps=3, warmup=3)
    assert bench.run_with_secondaries(args, 0, 1, 0) == 0
    lines = capsys.readouterr().out.strip().splitlines()
    assert len(lines) == 1
    head = json.loads(lines[0])
    assert head["metric"] == "m" and set(head["secondary"]) == set(bench.SECONDARY)
    assert head["secondary"]["hier_1m"] == {"error": "RuntimeError: boom"}
    assert head["secondary"]["llama8b_32k"]["value"] == 2.0
    assert head["secondary"]["llama8b_32k"]["workload"] == "llama8b_32k"
    assert bench._SINK is None
