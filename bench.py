"""Benchmark: sparse decode steps/s per layer at 128K, B=2048 (one decode step =
group-mean scoring of the projected-key cache, top-B selection and indexed
attention for every query head; batch 4, 32 query heads, 8 KV heads, d=128,
T=131072, r=64).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Prints one JSON line (rank 0). Timing: CUDA events on the launching stream,
W untimed warm-up steps, then K timed steps bracketed by a barrier and
torch.cuda.synchronize() on both sides; max over ranks. Inputs (2.5 GiB per
GPU) exceed the 126 MB L2 and every step streams the 512 MiB projected-key
cache, so no separate L2 flush is needed.

On one GPU the default line also measures, in the same run, every other
workload (the FP8 and paged steps, the L2-resident llama8b_32k and hier_1m
steps, the 128K prefill, the scoring preparation and the two comparisons) and
reports each one's figures under "secondary"; --no-secondary skips them.

Multi-GPU: the decode step shards by sequence and KV head with no exchange, so
each rank runs its own full workload (weak scaling, no data-path collective);
`value` is the steps of all ranks divided by the slowest rank's time.

--impl reference times the CPU oracle (fp64 NumPy) on this host's cores: whole
oracle decode steps for the decode lines (about 1.4 s each at 128K), bounded
samples scaled to whole steps for the prefill and the projection.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "sparse decode steps/s per layer at 128K, B=2048; achieved HBM GB/s vs peak"
METRIC_FP8 = "sparse decode steps/s per layer at 128K, B=2048, FP8 (E4M3) projected-key cache; HBM GB/s vs peak"
METRIC_PAGED = ("sparse decode steps/s per layer at 128K, B=2048, paged KV cache (page size 1, slots in random "
                "order); HBM GB/s vs peak")
UNIT = "steps/s"
WORKLOAD = "decode_128k"
FALLBACK_HBM_GBS = 6650.0
KERNELS_PER_STEP = 3      # scorer, top-B, indexed attention (split combine fused into it)
QUERY_SETS = 8            # decode steps cycle through this many query sets (8 x 32 MiB of rows > L2)
PROFILE_TRAFFIC = os.path.join(ROOT, "profiles", "traffic.json")
SCORER_SOURCES = ["indexed_sparse_attention_kv_b200/csrc/score.cu",
                  "indexed_sparse_attention_kv_b200/csrc/lsa_common.cuh"]


def rank_seed(w, rank):
    """Each rank decodes its own sequences: a distinct seed per rank."""
    return w.seed + 7919 * rank


def max_over_ranks(values, world, device=None):
    """Elementwise max of a list of floats over all ranks (identity at world 1)."""
    import torch

    t = torch.tensor(values, dtype=torch.float64, device=device)
    if world > 1:
        import torch.distributed as dist

        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t.tolist()]


def weak_value(world, steps, ms):
    """Steps of all ranks divided by the slowest rank's time (steps/s)."""
    return world * steps / (ms / 1e3)


def _env_int(name, default):
    try:
        return int(os.environ.get(name, default))
    except ValueError:
        return default


def config_dict(w, extra=None):
    d = {"workload": w.name, "batch": w.batch, "hq": w.hq, "hkv": w.hkv, "d": w.d, "T": w.T, "r": w.r,
         "B": w.B, "heavy_hitters": w.heavy_frac, "kv_layout": "[batch, T, hkv, d] bf16",
         "l2": f"inputs exceed L2 (each step streams the 512 MiB projected-key cache; steps cycle through "
               f"{QUERY_SETS} query sets, so each selects its own 32 MiB of K/V rows)"}
    if extra:
        d.update(extra)
    return d


def algorithmic_bytes(w):
    """Bytes the method must move per decode step: projected-key cache, the
    selected K and V rows, q, the projected queries and out."""
    kt = w.batch * w.T * w.hkv * w.r * 2
    kv = w.batch * w.hkv * w.B * w.d * 2 * 2
    small = w.batch * w.hq * (w.d * 2 + w.r * 2 + w.d * 2)
    return kt, kv, small


def measured_peak():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def source_hash(paths):
    h = hashlib.sha256()
    for p in paths:
        with open(os.path.join(ROOT, p), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


PROJECT_SOURCES = ["indexed_sparse_attention_kv_b200/csrc/project.cu", "indexed_sparse_attention_kv_b200/csrc/tcgen05.cuh",
                   "indexed_sparse_attention_kv_b200/csrc/lsa_common.cuh"]


def project_traffic():
    """DRAM bytes per projection launch (prepare_128k) from the committed ncu
    summary, or None if the kernel's sources changed since it was captured."""
    try:
        with open(os.path.join(ROOT, "profiles", "traffic_project.json")) as f:
            t = json.load(f)
        if t.get("source_hash") != source_hash(PROJECT_SOURCES):
            return None
        return float(t["dram_bytes_per_launch"])
    except Exception:
        return None


def scorer_traffic(w):
    """DRAM bytes per scorer launch from the committed ncu summary, or None if
    the scorer's sources changed since it was captured."""
    try:
        with open(PROFILE_TRAFFIC) as f:
            t = json.load(f)
        if t.get("source_hash") != source_hash(SCORER_SOURCES) or t.get("workload") != w.name:
            return None
        return float(t["dram_bytes_per_launch"])
    except Exception:
        return None


class ClockSampler:
    """SM clock, power and clock-event (throttle) reasons sampled through NVML
    (the library nvidia-smi reads) every ~2 ms in a thread while the timed
    region runs; read-only."""

    REASONS = {0x8: "hw_slowdown", 0x40: "hw_thermal_slowdown", 0x20: "sw_thermal_slowdown",
               0x4: "sw_power_cap", 0x80: "hw_power_brake_slowdown"}

    def __init__(self, torch_device):
        self.dev = torch_device
        self.rows = []
        self.err = None
        self._stop = None
        self._thr = None

    def _handle(self, nv):
        import torch

        try:
            p = torch.cuda.get_device_properties(self.dev)
            bus = f"{p.pci_domain_id:08x}:{p.pci_bus_id:02x}:{p.pci_device_id:02x}.0"
            return nv.nvmlDeviceGetHandleByPciBusId(bus.encode())
        except Exception:
            return nv.nvmlDeviceGetHandleByIndex(self.dev.index or 0)

    def __enter__(self):
        import threading

        try:
            import pynvml as nv

            nv.nvmlInit()
            h = self._handle(nv)
            get_reasons = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                nv.nvmlDeviceGetCurrentClocksThrottleReasons
            self.max_mhz = nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM)
        except Exception as e:  # no NVML: report it, do not guess
            self.err = f"nvml unavailable: {type(e).__name__}"
            return self
        self._stop = threading.Event()

        def loop():
            while True:
                try:
                    self.rows.append((nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM), int(get_reasons(h)),
                                      nv.nvmlDeviceGetPowerUsage(h) / 1e3))
                except Exception as e:
                    self.err = f"nvml sample failed: {type(e).__name__}"
                    return
                if self._stop.wait(0.002):
                    return

        self._thr = threading.Thread(target=loop, daemon=True)
        self._thr.start()
        return self

    def __exit__(self, *exc):
        if self._thr is not None:
            self._stop.set()
            self._thr.join(timeout=5)

    def summary(self):
        if not self.rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [self.err or "no samples"], "samples": 0}
        reasons = sorted({name for _, r, _ in self.rows for bit, name in self.REASONS.items() if r & bit})
        return {"sm_mhz": statistics.median(m for m, _, _ in self.rows), "sm_max_mhz": self.max_mhz,
                "reasons": reasons, "samples": len(self.rows),
                "power_w_max": max(p for _, _, p in self.rows), "source": "nvml"}


def blas_threads():
    try:
        import numpy as np
        import threadpoolctl
        np.ones((64, 64)) @ np.ones((64, 64))
        info = threadpoolctl.threadpool_info()
        n = max((i.get("num_threads", 1) for i in info), default=1)
        return int(n)
    except Exception:
        return 1


def cpu_oracle_sample(w, x, budget_s=12.0, max_units=None):
    """Time the oracle on (sequence, KV head) units of the workload until about
    budget_s seconds of CPU work; returns (steps/s, units, seconds)."""
    import numpy as np
    import torch

    import oracle.lsa_oracle as O

    units_per_step = w.batch * w.hkv
    done, t0 = 0, time.perf_counter()
    elapsed = 0.0
    G = w.G
    while True:
        b = (done // w.hkv) % w.batch
        h = done % w.hkv
        # one unit: the oracle's steps for one KV head of one sequence
        qt = x["qt"][b, h * G:(h + 1) * G].to(torch.float32).numpy()
        kt = x["kt"][b, :, h:h + 1].to(torch.float32).numpy()
        q = x["q"][b, h * G:(h + 1) * G].to(torch.float32).numpy()
        ts = time.perf_counter()
        q_bar = O.group_mean_query(qt, 1)
        s = O.candidate_scores(q_bar, kt)
        idx = O.select_top_b(s[0], w.B)[None]
        sel = idx[0][idx[0] >= 0]
        k_rows = x["k"][b, sel, h:h + 1].to(torch.float32).numpy()
        v_rows = x["v"][b, sel, h:h + 1].to(torch.float32).numpy()
        O.indexed_attention(q, k_rows, v_rows, np.arange(len(sel))[None], w.scale)
        elapsed += time.perf_counter() - ts
        done += 1
        if elapsed >= budget_s or (max_units and done >= max_units):
            break
        if time.perf_counter() - t0 > 3 * budget_s:
            break
    return done / units_per_step / elapsed, done, elapsed


def parallelism(world):
    return f"replicas{world}" if world > 1 else "single"


def decode_config(w, world, fp8=False, paged=False):
    """The `config` of a decode_128k line (either arm)."""
    return config_dict(w, {"parallelism": parallelism(world),
                           **({"workload": "decode_128k_fp8", "kt_dtype": "fp8_e4m3"} if fp8 else {}),
                           **({"workload": "decode_128k_paged",
                               "kv_layout": "pools [batch*T, hkv, d] bf16, page size 1, page table "
                                            "[batch, T] int32 (a random permutation of the slots)"}
                              if paged else {})})


def resident_config(w, world):
    return {"workload": w.name, "batch": w.batch, "hq": w.hq, "hkv": w.hkv, "d": w.d, "T": w.T,
            "r": w.r, "B": w.B, "blk": w.blk, "keep": w.keep,
            "l2": "256 MiB L2 flush after every step, timed alone and subtracted",
            "parallelism": parallelism(world)}


def prefill_config(w, world):
    return {"workload": w.name, "nq": w.nq, "q_start": w.T - w.nq, "T": w.T, "hq": w.hq, "hkv": w.hkv,
            "d": w.d, "r": w.r, "B": w.B, "l2": "inputs exceed L2 (128 MiB projected keys, 512 MiB K/V)",
            "parallelism": parallelism(world)}


def prepare_config(world):
    return {"workload": "prepare_128k", **PREPARE_SHAPE, "nbases": PREPARE_SHAPE["H"],
            "l2": "inputs exceed L2 (1 GiB of keys per step)", "parallelism": parallelism(world)}


def run_reference(args, rank, world):
    """Reference arm: the CPU oracle as it stands, on this host's cores.

    Each timed step is one whole oracle decode step (all (sequence, KV head)
    units) for the decode lines, which take about a second; for the prefill
    and the projection, whose whole step takes hours on the host, each timed
    step is a bounded sample of the workload and `value` is scaled from it.
    Either way `ms_per_step` is the measured time of one timed step, so
    steps x ms_per_step is the timed region."""
    if rank != 0:
        return 0
    from indexed_sparse_attention_kv_b200 import inputs as I

    if args.workload in COMPARE_METRICS:
        print(json.dumps({"impl": "reference", "unavailable": "comparison line: the oracle defines the method, not "
                                                             "the comparison systems"}), flush=True)
        return 0
    cores = blas_threads()
    K, W = max(1, args.steps), max(1, args.warmup)

    def line(metric, value, unit, ms_step, config, sample):
        return {"impl": "reference", "metric": metric, "value": value, "unit": unit, "n_gpus": args.gpus,
                "steps": K, "warmup": W, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
                "vs_baseline": None, "dtype": "f64", "data": "synthetic", "config": config,
                "cpu_baseline": {"value": value, "unit": unit, "cores": cores, "kind": "oracle", "sample": sample},
                "e2e": {"value": value, "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}

    if args.workload in RESIDENT_METRICS:
        w = I.workload(args.workload)
        x = I.make_decode_inputs(w)
        units = w.batch * w.hkv
        for _ in range(W):
            cpu_unit_sample(w, x, budget_s=math.inf, max_units=units)
        el = sum(cpu_unit_sample(w, x, budget_s=math.inf, max_units=units)[2] for _ in range(K))
        out = line(RESIDENT_METRICS[w.name], K / el, UNIT, el / K * 1e3, resident_config(w, world),
                   f"{K} whole decode steps ({units} (sequence, KV head) units each)")
    elif args.workload == "prepare_128k":
        sh = PREPARE_SHAPE
        hx = I.make_projection_inputs(PREPARE_SEED, 1, 4096, sh["H"], sh["d"], sh["r"], sh["H"], None, None)
        per = 4096
        cpu_prepare_sample(hx["x"], hx["P"], budget_s=math.inf, max_tokens=per * W)
        v, n, el = cpu_prepare_sample(hx["x"], hx["P"], budget_s=math.inf, max_tokens=per * K)
        out = line(PREPARE_METRIC, v, PREPARE_UNIT, el / K * 1e3, prepare_config(world),
                   f"each timed step projects {per} token rows x {sh['H']} KV heads ({n} rows in all); "
                   f"GB/s of the same algorithmic bytes per row")
    elif args.workload == "prefill_128k":
        w = I.workload("prefill_128k")
        x = I.make_prefill_inputs(w)
        per = 2
        cpu_prefill_sample(w, x, budget_s=math.inf, max_rows=per * W)
        v, n, el = cpu_prefill_sample(w, x, budget_s=math.inf, max_rows=per * K)
        out = line(PREFILL_METRIC, v, PREFILL_UNIT, el / K * 1e3, prefill_config(w, world),
                   f"each timed step runs {per} of the {w.nq} query rows (index + attention; {n} rows in all), "
                   f"scaled to whole prefills")
    else:
        w = I.workload(WORKLOAD)
        x = I.make_decode_inputs(w)
        units = w.batch * w.hkv
        for _ in range(W):
            cpu_oracle_sample(w, x, budget_s=math.inf, max_units=units)
        el = sum(cpu_oracle_sample(w, x, budget_s=math.inf, max_units=units)[2] for _ in range(K))
        metric = {"decode_128k_fp8": METRIC_FP8, "decode_128k_paged": METRIC_PAGED}.get(args.workload, METRIC)
        out = line(metric, K / el, UNIT, el / K * 1e3,
                   decode_config(w, world, fp8=args.workload == "decode_128k_fp8",
                                 paged=args.workload == "decode_128k_paged"),
                   f"{K} whole decode steps ({units} (sequence, KV head) units each)")
    print(json.dumps(out), flush=True)
    return 0


_SINK = None        # a list while lines are collected for the headline's "secondary" object
_DECODE_INPUTS = {}


def emit(line):
    """Print one JSON line, or collect it while secondary workloads run."""
    if _SINK is not None:
        _SINK.append(line)
    else:
        print(json.dumps(line), flush=True)


def decode_inputs(w, seed):
    """Seeded decode inputs (host tensors, read only), generated once per
    (workload, seed) in this process."""
    from indexed_sparse_attention_kv_b200 import inputs as I

    key = (w.name, seed)
    if key not in _DECODE_INPUTS:
        _DECODE_INPUTS[key] = I.make_decode_inputs(w, seed=seed)
    return _DECODE_INPUTS[key]


def run_ours(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist

    import indexed_sparse_attention_kv_b200 as lsa
    from indexed_sparse_attention_kv_b200 import _lib
    from indexed_sparse_attention_kv_b200 import inputs as I

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    lsa.lib()
    fp8 = args.workload == "decode_128k_fp8"
    paged = args.workload == "decode_128k_paged"
    w = I.workload(WORKLOAD)
    x = decode_inputs(w, rank_seed(w, rank))
    d = {k: x[k].to(dev) for k in ("q", "qt", "k", "v", "kt")}
    if fp8:   # the same integer values, stored as E4M3 (exact)
        d["kt8"] = d["kt"].to(torch.float8_e4m3fn)
    if paged:   # the same K/V rows in pools, token (b, t) at a random slot
        nslots = w.batch * w.T
        perm = torch.randperm(nslots, generator=torch.Generator().manual_seed(w.seed + 17)).to(dev)
        d["page_table"] = perm.to(torch.int32).view(w.batch, w.T)
        for name in ("k", "v"):
            pool = torch.empty((nslots, w.hkv, w.d), dtype=torch.bfloat16, device=dev)
            pool[perm] = d[name].view(nslots, w.hkv, w.d)
            d[name + "_pool"] = pool
    dims = _lib.decode_dims(d["q"], d["qt"], d["k"])
    ws = lsa.workspace(dims, w.B, device=dev)
    idx = torch.empty((w.batch, w.hkv, w.B), dtype=torch.int32, device=dev)
    out = torch.empty_like(d["q"])
    stream = torch.cuda.current_stream(dev)
    # Successive steps use different query sets: each step selects its own K/V
    # rows, as consecutive decode steps of one layer do (with other layers in
    # between), instead of re-reading the previous step's rows from L2.
    qs = I.make_query_sets(w, QUERY_SETS, seed=rank_seed(w, rank) + 100)
    dq, dqt = qs["q"].to(dev), qs["qt"].to(dev)

    def call(q, qt, o, ix):
        if fp8:
            lsa.lsa_decode_step_fp8(q, qt, d["k"], d["v"], d["kt8"], w.B, idx_out=ix, out=o, ws=ws)
        elif paged:
            lsa.lsa_decode_step_paged(q, qt, d["k_pool"], d["v_pool"], d["page_table"], d["kt"], w.B,
                                      idx_out=ix, out=o, ws=ws)
        else:
            lsa.lsa_decode_step(q, qt, d["k"], d["v"], d["kt"], w.B, idx_out=ix, out=o, ws=ws)

    def step(i=None):
        call(d["q"] if i is None else dq[i], d["qt"] if i is None else dqt[i], out, idx)

    def barrier():
        if world > 1:
            dist.barrier()

    for i in range(max(3, args.warmup)):
        step(i % QUERY_SETS)
    torch.cuda.synchronize()
    status = lsa.lsa_read_device_status(ws)

    def graph_of(fn, reps=1):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for _ in range(reps):
                fn()
        g.replay()
        torch.cuda.synchronize()
        return g

    # one graph holds QUERY_SETS whole decode steps (one per query set), as a
    # model's graph holds many layers' steps; single-step graphs cover a remainder
    g_steps = [graph_of(lambda i=i: step(i)) for i in range(QUERY_SETS)]

    def all_sets():
        for i in range(QUERY_SETS):
            step(i)

    g_round = graph_of(all_sets)

    def run_steps(k):
        for _ in range(k // QUERY_SETS):
            g_round.replay()
        for i in range(k % QUERY_SETS):
            g_steps[i].replay()

    run_steps(max(3, args.warmup))
    torch.cuda.synchronize()

    # ---- timed region: K whole decode steps
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    with ClockSampler(dev) as clk:
        barrier()
        torch.cuda.synchronize()
        e0.record(stream)
        run_steps(args.steps)
        e1.record(stream)
        torch.cuda.synchronize()
        barrier()
    ms = e0.elapsed_time(e1)
    clocks = clk.summary()

    # ---- component split (Fig. 9-style): each public call replayed back to back
    # in its own graph; attention is timed after an L2 flush (as in a real step,
    # where the scorer's 512 MiB stream has evicted the K/V rows), the flush
    # alone timed the same way and subtracted.
    scores = torch.empty((w.batch, w.hkv, w.T), dtype=torch.float32, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    lsa.lsa_score(d["qt"], d["kt"], scores)
    lsa.lsa_topk(scores, w.B, idx)
    reps = 8

    def attn_call():
        if paged:
            lsa.lsa_indexed_attn_paged(d["q"], d["k_pool"], d["v_pool"], d["page_table"], idx, out=out, ws=ws)
        else:
            lsa.lsa_indexed_attn(d["q"], d["k"], d["v"], idx, out=out, ws=ws)

    attn_call()

    def attn_after_flush():
        flush.zero_()
        attn_call()

    score_call = (lambda: lsa.lsa_score_fp8(d["qt"], d["kt8"], scores)) if fp8 else \
        (lambda: lsa.lsa_score(d["qt"], d["kt"], scores))
    graphs = {
        "scoring": graph_of(score_call, reps),
        "top_b": graph_of(lambda: lsa.lsa_topk(scores, w.B, idx), reps),
        "attention+flush": graph_of(attn_after_flush, reps),
        "flush": graph_of(lambda: flush.zero_(), reps),
    }
    comp_ms = {}
    n_rep = 5
    for name, g in graphs.items():
        e0.record(stream)
        for _ in range(n_rep):
            g.replay()
        e1.record(stream)
        torch.cuda.synchronize()
        comp_ms[name] = e0.elapsed_time(e1) / (n_rep * reps)
    comp = [comp_ms["scoring"], comp_ms["top_b"], max(0.0, comp_ms["attention+flush"] - comp_ms["flush"])]
    del graphs, flush

    # ---- end to end through the public API: every step copies its q, qt H2D from pinned host
    # memory, runs lsa_decode_step and copies out and idx D2H. The copies run on a second stream
    # with double-buffered device tensors, so step i's outputs and step i+1's inputs move while
    # the GPU computes (as a serving loop overlaps them); the compute stream waits for each
    # step's inputs, and the timed region ends after the last step's outputs reach the host.
    hq = qs["q"].pin_memory()
    hqt = qs["qt"].pin_memory()
    hout = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    hidx = torch.empty(idx.shape, dtype=idx.dtype).pin_memory()
    copy_stream = torch.cuda.Stream(dev)
    bq = [torch.empty_like(d["q"]) for _ in range(2)]
    bqt = [torch.empty_like(d["qt"]) for _ in range(2)]
    bout = [torch.empty_like(out) for _ in range(2)]
    bidx = [torch.empty_like(idx) for _ in range(2)]

    def run_e2e(n):
        h2d = [torch.cuda.Event() for _ in range(n)]
        comp = [torch.cuda.Event() for _ in range(n)]
        d2h = [torch.cuda.Event() for _ in range(n)]

        def load(i):   # H2D of step i's queries into buffer i % 2 (after step i-2 has read it)
            with torch.cuda.stream(copy_stream):
                if i >= 2:
                    copy_stream.wait_event(comp[i - 2])
                bq[i % 2].copy_(hq[i % QUERY_SETS], non_blocking=True)
                bqt[i % 2].copy_(hqt[i % QUERY_SETS], non_blocking=True)
                h2d[i].record(copy_stream)

        copy_stream.wait_stream(stream)
        load(0)
        for i in range(n):
            b = i % 2
            if i + 1 < n:
                load(i + 1)
            stream.wait_event(h2d[i])
            if i >= 2:
                stream.wait_event(d2h[i - 2])   # buffer b's previous outputs have left
            call(bq[b], bqt[b], bout[b], bidx[b])
            comp[i].record(stream)
            with torch.cuda.stream(copy_stream):
                copy_stream.wait_event(comp[i])
                hout.copy_(bout[b], non_blocking=True)
                hidx.copy_(bidx[b], non_blocking=True)
                d2h[i].record(copy_stream)
        stream.wait_event(d2h[n - 1])

    run_e2e(4)
    torch.cuda.synchronize()
    barrier()
    torch.cuda.synchronize()
    e0.record(stream)
    run_e2e(args.steps)
    e1.record(stream)
    torch.cuda.synchronize()
    barrier()
    ms_e2e = e0.elapsed_time(e1)
    # the last step's results, copied back in the timed loop, equal the device-side step's
    if not (torch.equal(hout.to(dev), bout[(args.steps - 1) % 2]) and torch.equal(hidx.to(dev),
                                                                                 bidx[(args.steps - 1) % 2])):
        raise RuntimeError("end-to-end loop: host copies differ from the device results")

    # ---- max over ranks
    ms, ms_e2e = max_over_ranks([ms, ms_e2e], world, dev)

    if rank == 0:
        value = weak_value(world, args.steps, ms)
        e2e = weak_value(world, args.steps, ms_e2e)
        kt_b, kv_b, small_b = algorithmic_bytes(w)
        if fp8:
            kt_b //= 2   # one byte per projected-key value
        peak, peak_kind = measured_peak()
        score_ms = comp[0]
        scorer_bytes = kt_b + w.batch * w.hq * w.r * 2
        achieved = scorer_bytes / (score_ms / 1e3) / 1e9
        traffic = None if fp8 else scorer_traffic(w)
        step_bytes = kt_b + kv_b + small_b
        step_gbs = step_bytes / (ms / args.steps / 1e3) / 1e9
        cpu = None
        if world == 1 and not args.no_cpu_baseline:
            v, n, el = cpu_oracle_sample(w, x, budget_s=args.cpu_budget)
            cpu = {"value": v, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
                   "sample": f"{n} (sequence, KV head) units of the 128K workload ({el:.1f} s), scaled to steps"}
        line = {
            "metric": METRIC_FP8 if fp8 else (METRIC_PAGED if paged else METRIC), "value": value, "unit": UNIT,
            "n_gpus": world, "steps": args.steps,
            "warmup": max(3, args.warmup), "ms_per_step": ms / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": decode_config(w, world, fp8=fp8, paged=paged),
            "roofline": {"bound": "hbm", "kernel": "score_q64_kernel (lsa_score_fp8)" if fp8 else
                         "score_q64_kernel (lsa_score)", "achieved": achieved, "peak": peak,
                         "unit": "GB/s", "frac": achieved / peak, "traffic": traffic,
                         "peak_kind": peak_kind, "algorithmic_bytes_per_launch": scorer_bytes,
                         "avg_launch_ms": score_ms},
            "step_roofline": {"achieved": step_gbs, "peak": peak, "unit": "GB/s", "frac": step_gbs / peak,
                              "algorithmic_bytes_per_step": step_bytes},
            "components_ms": {"scoring": comp[0], "top_b": comp[1], "attention": comp[2]},
            "cpu_baseline": cpu,
            "e2e": {"value": e2e, "unit": UNIT,
                    "h2d_bytes_per_step": (hq.numel() + hqt.numel()) * 2 // QUERY_SETS,
                    "d2h_bytes_per_step": hout.numel() * 2 + hidx.numel() * 4},
            "gpu_launches": KERNELS_PER_STEP * args.steps,
            "clocks": clocks,
            "device_status": status,
        }
        emit(line)
    return 0


COMPARE_METRICS = {
    "full_kv_128k": "full-KV decode attention steps/s at 128K (comparison: dense attention over every cached "
                    "position, the same attention kernel with index sets covering the whole cache)",
    "gather_attend_128k": "gather-then-attend decode steps/s at 128K, B=2048 (comparison: the selected K/V rows "
                          "copied to a dense buffer before attention)",
}


def run_compare(args, rank, world, local_rank):
    """Comparison systems of the pages, measured with this library's kernels
    (JSSA, Fig. 4: sparse decode against full-KV attention; Fig. 2b and Fig. 6:
    gather-free attention against gather-then-attend). Each line also reports
    the gather-free sparse path measured the same way in the same run."""
    import torch
    import torch.distributed as dist

    import indexed_sparse_attention_kv_b200 as lsa
    from indexed_sparse_attention_kv_b200 import _lib
    from indexed_sparse_attention_kv_b200 import inputs as I

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    lsa.lib()
    w = I.workload(WORKLOAD)
    x = decode_inputs(w, rank_seed(w, rank))
    d = {k: x[k].to(dev) for k in ("q", "qt", "k", "v", "kt")}
    qs = I.make_query_sets(w, QUERY_SETS, seed=rank_seed(w, rank) + 100)
    dq, dqt = qs["q"].to(dev), qs["qt"].to(dev)
    dims = _lib.decode_dims(d["q"], d["qt"], d["k"])
    out = torch.empty_like(d["q"])
    stream = torch.cuda.current_stream(dev)
    full = args.workload == "full_kv_128k"
    ws_step = lsa.workspace(dims, w.B, device=dev)
    idx_out = torch.empty((w.batch, w.hkv, w.B), dtype=torch.int32, device=dev)

    def sparse_step(i):   # the gather-free step (the product path)
        lsa.lsa_decode_step(dq[i], dqt[i], d["k"], d["v"], d["kt"], w.B, idx_out=idx_out, out=out, ws=ws_step)

    if full:
        idx_all = torch.arange(w.T, dtype=torch.int32, device=dev).view(1, 1, w.T).expand(
            w.batch, w.hkv, w.T).contiguous()
        ws_full = lsa.workspace(dims, w.T, device=dev)

        def cmp_step(i):
            lsa.lsa_indexed_attn(dq[i], d["k"], d["v"], idx_all, out=out, ws=ws_full)

        cmp_bytes = w.batch * w.T * w.hkv * w.d * 2 * 2 + w.batch * w.hq * w.d * 2 * 2
    else:
        scores = torch.empty((w.batch, w.hkv, w.T), dtype=torch.float32, device=dev)
        idx = torch.empty((w.batch, w.hkv, w.B), dtype=torch.int32, device=dev)
        kg = torch.empty((w.batch, w.B, w.hkv, w.d), dtype=torch.bfloat16, device=dev)
        vg = torch.empty_like(kg)
        bi = torch.arange(w.batch, device=dev).view(-1, 1, 1)
        hi = torch.arange(w.hkv, device=dev).view(1, 1, -1)
        idx_dense = torch.arange(w.B, dtype=torch.int32, device=dev).view(1, 1, w.B).expand(
            w.batch, w.hkv, w.B).contiguous()
        gdims = lsa.lsa_dims(w.batch, w.hq, w.hkv, w.d, w.r, w.B)
        ws_g = lsa.workspace(gdims, w.B, device=dev)

        def cmp_step(i):
            lsa.lsa_score(dqt[i], d["kt"], scores)
            lsa.lsa_topk(scores, w.B, idx)
            it = idx.transpose(1, 2).long()           # [batch, B, hkv]
            kg.copy_(d["k"][bi, it, hi])
            vg.copy_(d["v"][bi, it, hi])
            lsa.lsa_indexed_attn(dq[i], kg, vg, idx_dense, out=out, ws=ws_g)

        cmp_bytes = algorithmic_bytes(w)[0] + 2 * algorithmic_bytes(w)[1] + algorithmic_bytes(w)[2]

    def graph_of(fn):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for i in range(QUERY_SETS):
                fn(i)
        g.replay()
        torch.cuda.synchronize()
        return g

    for i in range(QUERY_SETS):
        cmp_step(i)
        sparse_step(i)
    torch.cuda.synchronize()
    g_cmp, g_sparse = graph_of(cmp_step), graph_of(sparse_step)
    rounds = max(1, args.steps // QUERY_SETS)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    res = {}
    with ClockSampler(dev) as clk:
        for name, g in (("cmp", g_cmp), ("sparse", g_sparse)):
            for _ in range(max(1, args.warmup // QUERY_SETS)):
                g.replay()
            if world > 1:
                dist.barrier()
            torch.cuda.synchronize()
            e0.record(stream)
            for _ in range(rounds):
                g.replay()
            e1.record(stream)
            torch.cuda.synchronize()
            res[name] = e0.elapsed_time(e1) / (rounds * QUERY_SETS)
    clocks = clk.summary()
    ms_cmp, ms_sparse = max_over_ranks([res["cmp"], res["sparse"]], world, dev)
    if rank == 0:
        peak, peak_kind = measured_peak()
        steps = rounds * QUERY_SETS
        line = {
            "metric": COMPARE_METRICS[args.workload], "value": world * 1e3 / ms_cmp, "unit": UNIT, "n_gpus": world,
            "steps": steps, "warmup": max(1, args.warmup // QUERY_SETS) * QUERY_SETS, "ms_per_step": ms_cmp,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {**decode_config(w, world), "workload": args.workload},
            "roofline": {"bound": "hbm", "kernel": "attn_kernel over every position" if full else
                         "scorer + top-B + gather copy + attention", "achieved": cmp_bytes / (ms_cmp / 1e3) / 1e9,
                         "peak": peak, "unit": "GB/s", "frac": cmp_bytes / (ms_cmp / 1e3) / 1e9 / peak,
                         "traffic": None, "peak_kind": peak_kind, "algorithmic_bytes_per_launch": cmp_bytes,
                         "avg_launch_ms": ms_cmp},
            "gather_free_sparse_step_ms": ms_sparse,
            "sparse_speedup": ms_cmp / ms_sparse,
            "cpu_baseline": None,
            "e2e": None,
            "gpu_launches": (1 if full else 5) * steps,
            "clocks": clocks,
        }
        emit(line)
    return 0


RESIDENT_METRICS = {
    "llama8b_32k": "sparse decode steps/s per layer at 32K, B=512 (LLaMA-3.1-8B layer shape)",
    "hier_1m": "coarse-to-fine sparse decode steps/s per layer at 1M tokens (64-token blocks, keep 64, B=2048)",
}


def resident_bytes(w):
    """Algorithmic bytes of one decode step: flat mode streams the projected-key
    cache; coarse-to-fine mode reads the centroids and the kept blocks' projected
    keys; both read the selected K/V rows and q, q~, out."""
    small = w.batch * w.hq * (w.d * 2 + w.r * 2 + w.d * 2)
    kv = w.batch * w.hkv * w.B * w.d * 2 * 2
    if w.blk:
        nblk = -(-w.T // w.blk)
        score = w.batch * nblk * w.hkv * w.r * 2 + w.batch * w.keep * w.blk * w.hkv * w.r * 2
    else:
        score = w.batch * w.T * w.hkv * w.r * 2
    return score + kv + small


def cpu_unit_sample(w, x, budget_s=12.0, max_units=None):
    """The oracle on (sequence, KV head) units of a decode step (flat or
    coarse-to-fine) until about budget_s seconds; returns (steps/s, units, s)."""
    import numpy as np
    import torch

    import oracle.lsa_oracle as O

    units_per_step = w.batch * w.hkv
    done, elapsed = 0, 0.0
    while True:
        b = (done // w.hkv) % w.batch
        h = done % w.hkv
        qt = x["qt"][b, h * w.G:(h + 1) * w.G].to(torch.float32).numpy()
        kt = x["kt"][b, :, h:h + 1].to(torch.float32).numpy()
        q = x["q"][b, h * w.G:(h + 1) * w.G].to(torch.float32).numpy()
        ts = time.perf_counter()
        q_bar = O.group_mean_query(qt, 1)
        if w.blk:
            idx = O.hierarchical_select(q_bar, kt, w.blk, w.keep, w.B)
        else:
            idx = O.select_top_b(O.candidate_scores(q_bar, kt)[0], w.B)[None]
        sel = idx[0][idx[0] >= 0]
        k_rows = x["k"][b, sel, h:h + 1].to(torch.float32).numpy()
        v_rows = x["v"][b, sel, h:h + 1].to(torch.float32).numpy()
        O.indexed_attention(q, k_rows, v_rows, np.arange(len(sel))[None], w.scale)
        elapsed += time.perf_counter() - ts
        done += 1
        if elapsed >= budget_s or (max_units and done >= max_units):
            break
    return done / units_per_step / elapsed, done, elapsed


def run_resident(args, rank, world, local_rank):
    """Decode workloads whose per-step data fits in L2 (32K flat, 1M
    coarse-to-fine): every timed step is followed by a 256 MiB L2 flush, and
    the flush, timed alone the same way, is subtracted."""
    import torch
    import torch.distributed as dist

    import indexed_sparse_attention_kv_b200 as lsa
    from indexed_sparse_attention_kv_b200 import _lib
    from indexed_sparse_attention_kv_b200 import inputs as I

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    lsa.lib()
    w = I.workload(args.workload)
    x = decode_inputs(w, rank_seed(w, rank))
    d = {k: x[k].to(dev) for k in ("q", "qt", "k", "v", "kt")}
    dims = _lib.decode_dims(d["q"], d["qt"], d["k"])
    cen = lsa.lsa_block_centroids(d["kt"], w.blk) if w.blk else None   # maintained offline, outside the step
    ws = lsa.workspace(dims, w.B, w.blk, w.keep if w.blk else 0, device=dev)
    idx = torch.empty((w.batch, w.hkv, w.B), dtype=torch.int32, device=dev)
    out = torch.empty_like(d["q"])
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        lsa.lsa_decode_step(d["q"], d["qt"], d["k"], d["v"], d["kt"], w.B, centroids=cen, blk=w.blk,
                            keep=w.keep, idx_out=idx, out=out, ws=ws)

    def barrier():
        if world > 1:
            dist.barrier()

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize()
    status = lsa.lsa_read_device_status(ws)

    def graph_of(fn):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            fn()
        g.replay()
        torch.cuda.synchronize()
        return g

    def step_flush():
        step()
        flush.zero_()

    g_sf = graph_of(step_flush)
    g_f = graph_of(lambda: flush.zero_())
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)

    def timed(g):
        barrier()
        torch.cuda.synchronize()
        e0.record(stream)
        for _ in range(args.steps):
            g.replay()
        e1.record(stream)
        torch.cuda.synchronize()
        barrier()
        return e0.elapsed_time(e1)

    for _ in range(max(3, args.warmup)):
        g_sf.replay()
    with ClockSampler(dev) as clk:
        ms_sf = timed(g_sf)
    ms_f = timed(g_f)
    clocks = clk.summary()
    ms = max(1e-6, ms_sf - ms_f)
    # end to end through the public API: H2D q, qt; step; D2H out, idx (flush after each, subtracted)
    hq, hqt = x["q"].pin_memory(), x["qt"].pin_memory()
    hout = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    hidx = torch.empty(idx.shape, dtype=idx.dtype).pin_memory()
    torch.cuda.synchronize()
    barrier()
    e0.record(stream)
    for _ in range(args.steps):
        d["q"].copy_(hq, non_blocking=True)
        d["qt"].copy_(hqt, non_blocking=True)
        step()
        hout.copy_(out, non_blocking=True)
        hidx.copy_(idx, non_blocking=True)
        flush.zero_()
    e1.record(stream)
    torch.cuda.synchronize()
    barrier()
    ms_e2e = max(1e-6, e0.elapsed_time(e1) - ms_f)
    ms, ms_e2e = max_over_ranks([ms, ms_e2e], world, dev)
    if rank == 0:
        peak, peak_kind = measured_peak()
        step_bytes = resident_bytes(w)
        achieved = step_bytes / (ms / args.steps / 1e3) / 1e9
        cpu = None
        if world == 1 and not args.no_cpu_baseline:
            v, n, el = cpu_unit_sample(w, x, budget_s=args.cpu_budget)
            cpu = {"value": v, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
                   "sample": f"{n} (sequence, KV head) units of {w.batch * w.hkv} per step ({el:.1f} s), scaled"}
        line = {
            "metric": RESIDENT_METRICS[w.name], "value": weak_value(world, args.steps, ms), "unit": UNIT,
            "n_gpus": world, "steps": args.steps, "warmup": max(3, args.warmup), "ms_per_step": ms / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic",
            "config": resident_config(w, world),
            "roofline": {"bound": "hbm", "kernel": "lsa_decode_step (whole step)", "achieved": achieved,
                         "peak": peak, "unit": "GB/s", "frac": achieved / peak, "traffic": None,
                         "peak_kind": peak_kind, "algorithmic_bytes_per_launch": step_bytes,
                         "avg_launch_ms": ms / args.steps},
            "cpu_baseline": cpu,
            "e2e": {"value": weak_value(world, args.steps, ms_e2e), "unit": UNIT,
                    "h2d_bytes_per_step": hq.numel() * 2 + hqt.numel() * 2,
                    "d2h_bytes_per_step": hout.numel() * 2 + hidx.numel() * 4},
            "gpu_launches": (5 if w.blk else 3) * args.steps,
            "clocks": clocks,
            "device_status": status,
        }
        emit(line)
    return 0


PREFILL_METRIC = "prefill steps/s at 128K (4096 causal queries, B=2048): indexer + indexed attention"
PREFILL_UNIT = "prefills/s"
PREFILL_KERNELS = 6       # group mean, sampled GEMM, thresholds, filter GEMM, selection, attention


def prefill_scoring_flop(w):
    """Useful scoring FLOPs of one prefill: 2 r per causal (query, key, KV head)."""
    q0 = w.T - w.nq
    pairs = sum(q0 + i + 1 for i in range(w.nq)) * w.hkv
    return 2 * pairs * w.r


def measured_tflops():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            return float(json.load(f)["bf16_tflops"]), "measured"
    except Exception:
        return 1590.0, "fallback"


def cpu_prefill_sample(w, x, budget_s=12.0, max_rows=None):
    """Oracle prefill (index + attention) on query rows until about budget_s
    seconds; returns (prefills/s, rows, seconds)."""
    import torch

    import oracle.lsa_oracle as O

    q0 = int(x["q_start"])
    kt = x["kt"].to(torch.float32).numpy()
    done, elapsed = 0, 0.0
    while True:
        i = (done * 577) % w.nq
        qt = x["qt"][i:i + 1].to(torch.float32).numpy()
        q = x["q"][i].to(torch.float32).numpy()
        ts = time.perf_counter()
        idx = O.prefill_index(qt, [q0 + i], kt, w.B)[0]
        sel = [idx[h][idx[h] >= 0] for h in range(w.hkv)]
        for h in range(w.hkv):
            k_rows = x["k"][sel[h], h:h + 1].to(torch.float32).numpy()
            v_rows = x["v"][sel[h], h:h + 1].to(torch.float32).numpy()
            import numpy as np
            O.indexed_attention(q[h * w.G:(h + 1) * w.G], k_rows, v_rows, np.arange(len(sel[h]))[None], w.scale)
        elapsed += time.perf_counter() - ts
        done += 1
        if elapsed >= budget_s or (max_rows and done >= max_rows):
            break
    return done / w.nq / elapsed, done, elapsed


def run_prefill(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist

    import indexed_sparse_attention_kv_b200 as lsa
    from indexed_sparse_attention_kv_b200 import inputs as I

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    lsa.lib()
    w = I.workload("prefill_128k")
    x = I.make_prefill_inputs(w, seed=rank_seed(w, rank))
    q0 = int(x["q_start"])
    d = {k: x[k].to(dev) for k in ("q", "qt", "k", "v", "kt")}
    dims = lsa.lsa_dims(1, w.hq, w.hkv, w.d, w.r, w.T)
    ws = lsa.prefill_workspace(dims, w.nq, w.B, device=dev)
    idx = torch.empty((w.nq, w.hkv, w.B), dtype=torch.int32, device=dev)
    out = torch.empty_like(d["q"])
    stream = torch.cuda.current_stream(dev)

    def index():
        lsa.lsa_prefill_index(d["qt"], d["kt"], q0, w.B, idx=idx, ws=ws)

    def attn():
        lsa.lsa_prefill_attn(d["q"], d["k"], d["v"], idx, out=out, ws=ws)

    def step():
        index()
        attn()

    def barrier():
        if world > 1:
            dist.barrier()

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize()
    status = lsa.lsa_read_device_status(ws)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    with ClockSampler(dev) as clk:
        barrier()
        torch.cuda.synchronize()
        e0.record(stream)
        for _ in range(args.steps):
            step()
        e1.record(stream)
        torch.cuda.synchronize()
        barrier()
    ms = e0.elapsed_time(e1)
    clocks = clk.summary()
    comp = {}
    for name, fn in (("indexer", index), ("attention", attn)):
        e0.record(stream)
        for _ in range(args.steps):
            fn()
        e1.record(stream)
        torch.cuda.synchronize()
        comp[name] = e0.elapsed_time(e1) / args.steps
    # end to end: H2D of the step's queries, D2H of index sets and outputs
    hq, hqt = x["q"].pin_memory(), x["qt"].pin_memory()
    hout = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    hidx = torch.empty(idx.shape, dtype=idx.dtype).pin_memory()
    torch.cuda.synchronize()
    barrier()
    e0.record(stream)
    for _ in range(args.steps):
        d["q"].copy_(hq, non_blocking=True)
        d["qt"].copy_(hqt, non_blocking=True)
        step()
        hout.copy_(out, non_blocking=True)
        hidx.copy_(idx, non_blocking=True)
    e1.record(stream)
    torch.cuda.synchronize()
    barrier()
    ms_e2e = e0.elapsed_time(e1)
    ms, ms_e2e = max_over_ranks([ms, ms_e2e], world, dev)
    if rank == 0:
        peak, peak_kind = measured_tflops()
        flop = prefill_scoring_flop(w)
        achieved = flop / (comp["indexer"] / 1e3) / 1e12
        cpu = None
        if world == 1 and not args.no_cpu_baseline:
            v, n, el = cpu_prefill_sample(w, x, budget_s=args.cpu_budget)
            cpu = {"value": v, "unit": PREFILL_UNIT, "cores": blas_threads(), "kind": "oracle",
                   "sample": f"{n} query rows of 4096 ({el:.1f} s), scaled to whole prefills"}
        line = {
            "metric": PREFILL_METRIC, "value": weak_value(world, args.steps, ms), "unit": PREFILL_UNIT,
            "n_gpus": world, "steps": args.steps, "warmup": max(3, args.warmup),
            "ms_per_step": ms / args.steps, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16", "data": "synthetic",
            "config": prefill_config(w, world),
            "roofline": {"bound": "tensor", "kernel": "lsa_prefill_index (score GEMMs + selection)",
                         "achieved": achieved, "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak,
                         "traffic": None, "peak_kind": peak_kind, "algorithmic_flop_per_launch": flop,
                         "avg_launch_ms": comp["indexer"]},
            "components_ms": comp,
            "cpu_baseline": cpu,
            "e2e": {"value": weak_value(world, args.steps, ms_e2e), "unit": PREFILL_UNIT,
                    "h2d_bytes_per_step": hq.numel() * 2 + hqt.numel() * 2,
                    "d2h_bytes_per_step": hout.numel() * 2 + hidx.numel() * 4},
            "gpu_launches": PREFILL_KERNELS * args.steps,
            "clocks": clocks,
            "device_status": status,
        }
        emit(line)
    return 0


PREPARE_METRIC = ("scoring preparation at 128K: projected-key cache build (batch 4 x 131072 tokens x 8 KV heads, "
                  "d 128 -> r 64, bf16), HBM GB/s")
PREPARE_UNIT = "GB/s"
PREPARE_SHAPE = dict(batch=4, T=131072, H=8, d=128, r=64, hq=32)
PREPARE_SEED = 1006


def prepare_bytes(sh):
    """Algorithmic bytes of one full projection: read x, write y, read the bases."""
    rows = sh["batch"] * sh["T"] * sh["H"]
    return rows * sh["d"] * 2 + rows * sh["r"] * 2 + sh["H"] * sh["r"] * sh["d"] * 2


def cpu_prepare_sample(x, P, budget_s=12.0, max_tokens=None):
    """Oracle projection of whole token rows (all heads) of sequence 0 until the
    budget (or max_tokens) is spent; returns (GB/s of the algorithmic bytes, tokens, seconds)."""
    import torch

    import oracle.lsa_oracle as O

    Pn = P.to(torch.float32).numpy()
    t0 = time.perf_counter()
    n = 0
    chunk = 256
    T = x.shape[1]
    while True:
        s0 = n % T
        xs = x[0, s0:min(T, s0 + chunk)].to(torch.float32).numpy()
        O.project_bf16(xs, Pn, 1)
        n += xs.shape[0]
        el = time.perf_counter() - t0
        if (max_tokens is not None and n >= max_tokens) or (max_tokens is None and el >= budget_s):
            break
    sh = PREPARE_SHAPE
    byt = n * sh["H"] * (sh["d"] * 2 + sh["r"] * 2)
    return byt / el / 1e9, n, el


def run_prepare(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist

    import indexed_sparse_attention_kv_b200 as lsa
    from indexed_sparse_attention_kv_b200 import inputs as I

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    lsa.lib()
    sh = PREPARE_SHAPE
    hx = I.make_projection_inputs(PREPARE_SEED + 7919 * rank, sh["batch"], sh["T"], sh["H"], sh["d"], sh["r"],
                                  sh["H"], None, None)
    x, P = hx["x"].to(dev), hx["P"].to(dev)
    y = torch.empty((sh["batch"], sh["T"], sh["H"], sh["r"]), dtype=torch.bfloat16, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        lsa.lsa_project(x, P, y=y, dev_status=status)

    def barrier():
        if world > 1:
            dist.barrier()

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    with ClockSampler(dev) as clk:
        barrier()
        torch.cuda.synchronize()
        e0.record(stream)
        for _ in range(args.steps):
            step()
        e1.record(stream)
        torch.cuda.synchronize()
        barrier()
    ms = e0.elapsed_time(e1)
    clocks = clk.summary()
    # decode-time append: one new key row per (sequence, KV head), the step's
    # 32 query rows, and the new key's block centroid
    q = torch.randn((sh["batch"], 1, sh["hq"], sh["d"]), device=dev).to(torch.bfloat16)
    qt = torch.empty((sh["batch"], 1, sh["hq"], sh["r"]), dtype=torch.bfloat16, device=dev)
    cen = torch.zeros((sh["batch"], sh["T"] // 64, sh["H"], sh["r"]), dtype=torch.bfloat16, device=dev)

    def append():
        lsa.lsa_project(x, P, sh["T"] - 1, 1, y=y)
        lsa.lsa_project(q, P, y=qt)
        lsa.lsa_update_centroids(y, cen, 64, sh["T"] - 1, 1)

    for _ in range(5):
        append()
    g = torch.cuda.CUDAGraph()
    s2 = torch.cuda.Stream(dev)
    s2.wait_stream(stream)
    with torch.cuda.stream(s2):
        append()
    torch.cuda.synchronize()
    with torch.cuda.graph(g):
        append()
    reps = 200
    torch.cuda.synchronize()
    e0.record(stream)
    for _ in range(reps):
        g.replay()
    e1.record(stream)
    torch.cuda.synchronize()
    append_us = e0.elapsed_time(e1) / reps * 1e3
    del g
    # end to end: the cache rows from pinned host memory, the projections back
    hxp = hx["x"].pin_memory()
    hy = torch.empty(y.shape, dtype=y.dtype).pin_memory()
    e2e_steps = max(1, min(args.steps, 10))
    barrier()
    torch.cuda.synchronize()
    e0.record(stream)
    for _ in range(e2e_steps):
        x.copy_(hxp, non_blocking=True)
        step()
        hy.copy_(y, non_blocking=True)
    e1.record(stream)
    torch.cuda.synchronize()
    barrier()
    ms_e2e = e0.elapsed_time(e1)
    ms, ms_e2e = max_over_ranks([ms, ms_e2e], world, dev)
    st = int(status.item())
    if rank == 0:
        peak, peak_kind = measured_peak()
        byt = prepare_bytes(sh)
        per_ms = ms / args.steps
        achieved = byt / (per_ms / 1e3) / 1e9
        cpu = None
        if world == 1 and not args.no_cpu_baseline:
            v, n, el = cpu_prepare_sample(hx["x"], hx["P"], budget_s=args.cpu_budget)
            cpu = {"value": v, "unit": PREPARE_UNIT, "cores": blas_threads(), "kind": "oracle",
                   "sample": f"{n} token rows x 8 KV heads of sequence 0 ({el:.1f} s), same algorithmic bytes per row"}
        line = {
            "metric": PREPARE_METRIC, "value": achieved * world, "unit": PREPARE_UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": max(3, args.warmup), "ms_per_step": per_ms, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": prepare_config(world),
            "roofline": {"bound": "hbm", "kernel": "project_kernel (lsa_project)", "achieved": achieved,
                         "peak": peak, "unit": "GB/s", "frac": achieved / peak, "traffic": project_traffic(),
                         "peak_kind": peak_kind, "algorithmic_bytes_per_launch": byt, "avg_launch_ms": per_ms},
            "append_us": append_us,
            "cpu_baseline": cpu,
            "e2e": {"value": prepare_bytes(sh) * e2e_steps / (ms_e2e / 1e3) / 1e9 * world, "unit": PREPARE_UNIT,
                    "h2d_bytes_per_step": hxp.numel() * 2, "d2h_bytes_per_step": hy.numel() * 2},
            "gpu_launches": args.steps,
            "clocks": clocks,
            "device_status": st,
        }
        emit(line)
    return 0


def run_ncu_case(args):
    """A small, self-contained launch sequence for ncu captures: batch 2 of the
    128K workload (kt 256 MiB > L2, 1.3 GiB on the device), `--steps` launches
    of the chosen component after `--warmup` untimed ones."""
    import torch

    import indexed_sparse_attention_kv_b200 as lsa
    from indexed_sparse_attention_kv_b200 import _lib
    from indexed_sparse_attention_kv_b200 import inputs as I

    if args.ncu_case == "project":   # one sequence of the 128K projection (256 MiB of keys in)
        sh = PREPARE_SHAPE
        hx = I.make_projection_inputs(PREPARE_SEED, 1, sh["T"], sh["H"], sh["d"], sh["r"], sh["H"], None, None)
        xd, Pd = hx["x"].cuda(), hx["P"].cuda()
        y = torch.empty((1, sh["T"], sh["H"], sh["r"]), dtype=torch.bfloat16, device="cuda")
        for _ in range(args.warmup + args.steps):
            lsa.lsa_project(xd, Pd, y=y)
        torch.cuda.synchronize()
        print(f"ncu case project: {args.warmup}+{args.steps} launches")
        return 0
    if args.ncu_case in ("prefill_mid", "prefill_attn_mid"):
        # mid-size prefill: T = 65536 keys, 1024 causal queries at T-1024..T-1, 32 / 8 heads, r 64,
        # B 2048, integer-valued bf16 scoring inputs (80 MiB of K/V, 8 MiB of projected keys)
        w = I.Workload("prefill_mid", 77, batch=1, hq=32, hkv=8, d=128, T=65536, r=64, B=2048, nq=1024)
        x = I.make_prefill_inputs(w)
        qt, kt = x["qt"].cuda(), x["kt"].cuda()
        q0 = int(x["q_start"])
        dims = _lib.prefill_dims(w.hq, kt)
        ws = lsa.prefill_workspace(dims, w.nq, w.B)
        idx = lsa.lsa_prefill_index(qt, kt, q0, w.B, ws=ws)
        if args.ncu_case == "prefill_attn_mid":
            q, k, v = x["q"].cuda(), x["k"].cuda(), x["v"].cuda()
            out = torch.empty_like(q)
            fn = lambda: lsa.lsa_prefill_attn(q, k, v, idx, out=out, ws=ws)  # noqa: E731
        else:
            fn = lambda: lsa.lsa_prefill_index(qt, kt, q0, w.B, idx=idx, ws=ws)  # noqa: E731
        for _ in range(args.warmup + args.steps):
            fn()
        torch.cuda.synchronize()
        print(f"ncu case {args.ncu_case}: {args.warmup}+{args.steps} calls, status {lsa.lsa_read_device_status(ws)}")
        return 0
    w = I.workload(WORKLOAD).with_(batch=2, name="decode_128k_b2")
    x = I.make_decode_inputs(w)
    d = {k: x[k].cuda() for k in ("q", "qt", "k", "v", "kt")}
    dims = _lib.decode_dims(d["q"], d["qt"], d["k"])
    ws = lsa.workspace(dims, w.B)
    scores = lsa.lsa_score(d["qt"], d["kt"])
    idx = lsa.lsa_topk(scores, w.B)
    out = torch.empty_like(d["q"])
    kt8 = d["kt"].to(torch.float8_e4m3fn) if args.ncu_case == "score8" else None
    fn = {
        "score": lambda: lsa.lsa_score(d["qt"], d["kt"], scores),
        "score8": lambda: lsa.lsa_score_fp8(d["qt"], kt8, scores),
        "topk": lambda: lsa.lsa_topk(scores, w.B, idx),
        "attn": lambda: lsa.lsa_indexed_attn(d["q"], d["k"], d["v"], idx, out=out, ws=ws),
        "step": lambda: lsa.lsa_decode_step(d["q"], d["qt"], d["k"], d["v"], d["kt"], w.B, idx_out=idx, out=out,
                                            ws=ws),
    }[args.ncu_case]
    for _ in range(args.warmup + args.steps):
        fn()
    torch.cuda.synchronize()
    print(f"ncu case {args.ncu_case}: {args.warmup}+{args.steps} launches, status {lsa.lsa_read_device_status(ws)}")
    return 0


def run_workload(args, rank, world, local_rank):
    if args.workload == "prefill_128k":
        return run_prefill(args, rank, world, local_rank)
    if args.workload == "prepare_128k":
        return run_prepare(args, rank, world, local_rank)
    if args.workload in RESIDENT_METRICS:
        return run_resident(args, rank, world, local_rank)
    if args.workload in COMPARE_METRICS:
        return run_compare(args, rank, world, local_rank)
    return run_ours(args, rank, world, local_rank)


SECONDARY = ("decode_128k_fp8", "decode_128k_paged", "llama8b_32k", "hier_1m", "prefill_128k", "prepare_128k",
             "full_kv_128k", "gather_attend_128k")


def secondary_summary(line):
    """The figures of one workload's line kept under the headline's
    "secondary" object."""
    keep = ("metric", "value", "unit", "steps", "ms_per_step", "higher_is_better", "components_ms",
            "gather_free_sparse_step_ms", "sparse_speedup", "device_status", "gpu_launches")
    out = {k: line[k] for k in keep if k in line}
    out["workload"] = line.get("config", {}).get("workload")
    roof = line.get("roofline") or {}
    out["roofline"] = {k: roof.get(k) for k in ("bound", "kernel", "achieved", "peak", "unit", "frac")}
    if line.get("step_roofline"):
        out["step_roofline_frac"] = line["step_roofline"].get("frac")
    e2e = line.get("e2e")
    out["e2e"] = None if e2e is None else {"value": e2e.get("value"), "unit": e2e.get("unit")}
    clk = line.get("clocks") or {}
    out["clocks"] = {"sm_mhz": clk.get("sm_mhz"), "reasons": clk.get("reasons")}
    return out


def run_with_secondaries(args, rank, world, local_rank):
    """The headline decode_128k line, then every other workload measured in
    the same process (each with its own warm-up, CUDA-event timing and clock
    samples; no CPU baseline), summarised under the headline's "secondary"
    object so that one run records them all."""
    global _SINK
    import gc

    import torch

    _SINK = []
    try:
        rc = run_ours(args, rank, world, local_rank)
        head = _SINK.pop() if _SINK else None
        secondary = {}
        for name in SECONDARY:
            sub = argparse.Namespace(**{**vars(args), "workload": name, "no_cpu_baseline": True})
            try:
                run_workload(sub, rank, world, local_rank)
                secondary[name] = secondary_summary(_SINK.pop()) if _SINK else {"error": "no line"}
            except Exception as e:   # one failing workload must not hide the others
                secondary[name] = {"error": f"{type(e).__name__}: {e}"[:300]}
            gc.collect()
            torch.cuda.empty_cache()
    finally:
        _SINK = None
    _DECODE_INPUTS.clear()
    if head is not None:
        head["secondary"] = secondary
        emit(head)
    return rc


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--cpu-budget", type=float, default=12.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-secondary", action="store_true",
                    help="the default decode_128k line on one GPU also measures every other workload in the same "
                         "run and reports them under \"secondary\"; this skips them")
    ap.add_argument("--workload", choices=["decode_128k", "decode_128k_fp8", "decode_128k_paged", "prefill_128k",
                                           "llama8b_32k", "hier_1m", "prepare_128k", "full_kv_128k",
                                           "gather_attend_128k"],
                    default="decode_128k",
                    help="decode_128k (the headline), decode_128k_fp8 (the same step over an FP8 projected-key "
                         "cache), decode_128k_paged (the same step with K/V in page-size-1 pools), prefill_128k "
                         "(indexer + indexed attention), the L2-resident decode steps "
                         "llama8b_32k and hier_1m, prepare_128k (scoring preparation: projecting the 128K "
                         "key cache, and the decode-time append), or the comparisons full_kv_128k (dense "
                         "attention over the whole cache) and gather_attend_128k (selected rows copied first)")
    ap.add_argument("--ncu-case", choices=["score", "score8", "topk", "attn", "step", "project", "prefill_mid",
                                           "prefill_attn_mid"], default=None,
                    help="run one component on a reduced case for an ncu capture (batch 2 of the 128K decode; "
                         "one 128K sequence for project; a 64K-key, 1024-query prefill for prefill_mid and "
                         "prefill_attn_mid); no JSON")
    args = ap.parse_args(argv)
    if args.ncu_case:
        return run_ncu_case(args)
    rank = _env_int("RANK", 0)
    world = _env_int("WORLD_SIZE", 1)
    local_rank = _env_int("LOCAL_RANK", 0)
    if args.impl == "reference":
        return run_reference(args, rank, world)
    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist

        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    try:
        if args.workload == "decode_128k" and world == 1 and not args.no_secondary:
            return run_with_secondaries(args, rank, world, local_rank)
        return run_workload(args, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist

            dist.destroy_process_group()


if __name__ == "__main__":
    sys.exit(main())
