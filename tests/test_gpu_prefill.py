"""GPU parity of the prefill indexer and prefill indexed attention against the
CPU oracle, through the C ABI.

Index sets are compared bit-exactly (integer-valued projected queries and
keys make every score exact in fp32 and the bf16 group mean exact); attention
outputs within 1e-2 absolute and relative. Small cases cover every supported
r, group sizes 1 to 16, ragged query counts, full causal prefills from
position 0 (rows shorter than B, rows that keep every key), queries that stop
short of the cache end, heavy ties (the exact re-selection path) and B == 1;
the 128K workload runs at full size with sampled rows checked against the
oracle and every row checked for the properties of an index set.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import indexed_sparse_attention_kv_b200 as lsa
import oracle.lsa_oracle as O
from indexed_sparse_attention_kv_b200 import inputs as I

from _util import LazyRows, assert_out_close, np32

pytestmark = pytest.mark.gpu

SMALL = [
    # hq, hkv, r, T, nq, B, int_range
    (8, 2, 64, 4096, 256, 256, 8),
    (4, 1, 64, 1000, 1000, 64, 8),
    (16, 1, 128, 3000, 200, 512, 8),
    (8, 4, 32, 2000, 130, 128, 8),
    (4, 2, 16, 1500, 300, 100, 8),
    (8, 2, 64, 5000, 128, 512, 1),
    (4, 1, 64, 2048, 64, 1, 8),
    (4, 1, 64, 300, 300, 512, 8),
    (32, 8, 64, 8192, 384, 2048, 8),
    (8, 2, 64, 6000, 200, 2048, 8),
]


def _inputs(case, seed=11):
    hq, hkv, r, T, nq, B, R = case
    w = I.Workload(f"prefill_{case}", seed, batch=1, hq=hq, hkv=hkv, d=128, T=T, r=r, B=B, int_range=R, nq=nq)
    return w, I.make_prefill_inputs(w)


def _oracle_idx(x, rows, q_start, B):
    qt = np32(x["qt"][rows])
    kt = np32(x["kt"])
    pos = q_start + np.asarray(rows)
    return O.prefill_index(qt, pos, kt, B)


@pytest.mark.parametrize("case", SMALL, ids=[str(c) for c in SMALL])
def test_prefill_index_small(case):
    w, x = _inputs(case)
    q_start = int(x["q_start"])
    idx = lsa.lsa_prefill_index(x["qt"].cuda(), x["kt"].cuda(), q_start, w.B)
    torch.cuda.synchronize()
    ref = _oracle_idx(x, np.arange(w.nq), q_start, w.B)
    got = idx.cpu().numpy()
    bad = np.argwhere((got != ref).any(axis=-1))
    assert bad.size == 0, f"{len(bad)} rows differ, first (query, head) {bad[:4].tolist()}"


def test_prefill_index_stops_short_of_cache_end():
    """Keys after the last query's position are in the cache but never selected."""
    w, x = _inputs((8, 2, 64, 4096, 256, 256, 8), seed=12)
    q_start = 3000
    idx = lsa.lsa_prefill_index(x["qt"].cuda(), x["kt"].cuda(), q_start, w.B)
    ref = _oracle_idx(x, np.arange(w.nq), q_start, w.B)
    assert np.array_equal(idx.cpu().numpy(), ref)


def test_prefill_index_all_equal_scores():
    """Every score equal: the B lowest positions of each row."""
    w, x = _inputs((4, 1, 64, 3000, 128, 256, 8), seed=13)
    kt = torch.zeros_like(x["kt"])
    q_start = int(x["q_start"])
    idx = lsa.lsa_prefill_index(x["qt"].cuda(), kt.cuda(), q_start, w.B).cpu().numpy()
    assert np.array_equal(idx, np.broadcast_to(np.arange(w.B, dtype=np.int32), idx.shape))


def test_prefill_index_repeatable_and_workspace_reuse():
    w, x = _inputs((8, 2, 64, 4096, 256, 256, 8), seed=14)
    qt, kt = x["qt"].cuda(), x["kt"].cuda()
    dims = lsa.lsa_dims(1, w.hq, w.hkv, 128, w.r, w.T)
    ws = lsa.prefill_workspace(dims, w.nq, w.B)
    a = lsa.lsa_prefill_index(qt, kt, int(x["q_start"]), w.B, ws=ws).clone()
    b = lsa.lsa_prefill_index(qt, kt, int(x["q_start"]), w.B, ws=ws)
    assert torch.equal(a, b)


@pytest.mark.parametrize("case", [SMALL[0], SMALL[2], SMALL[7]], ids=str)
def test_prefill_attention_small(case):
    w, x = _inputs(case, seed=21)
    q_start = int(x["q_start"])
    ref_idx = _oracle_idx(x, np.arange(w.nq), q_start, w.B)
    idx = torch.from_numpy(ref_idx.astype(np.int32)).cuda()
    out = lsa.lsa_prefill_attn(x["q"].cuda(), x["k"].cuda(), x["v"].cuda(), idx)
    torch.cuda.synchronize()
    ref = O.prefill_attention(np32(x["q"]), np32(x["k"]), np32(x["v"]), ref_idx, w.scale)
    assert_out_close(out, ref)


def _check_index_sets(idx: torch.Tensor, q_start: int, B: int):
    """Every row: ascending, unique, within [0, p], min(B, p + 1) entries then -1."""
    nq = idx.shape[0]
    p = (q_start + torch.arange(nq, device=idx.device)).view(nq, 1, 1)
    n_valid = torch.clamp(p + 1, max=B)
    j = torch.arange(B, device=idx.device).view(1, 1, B)
    valid = j < n_valid
    assert bool(((idx >= 0) == valid).all()), "padding in the wrong place"
    assert bool((idx[valid.expand_as(idx)] <= p.expand_as(idx)[valid.expand_as(idx)]).all()), "non-causal index"
    d = idx[..., 1:] - idx[..., :-1]
    both = valid[..., 1:].expand_as(d)
    assert bool((d[both] > 0).all()), "not strictly ascending"


@pytest.mark.slow
def test_prefill_128k_full_size():
    w = I.workload("prefill_128k")
    x = I.make_prefill_inputs(w)
    q_start = int(x["q_start"])
    qt, kt = x["qt"].cuda(), x["kt"].cuda()
    idx = lsa.lsa_prefill_index(qt, kt, q_start, w.B)
    torch.cuda.synchronize()
    _check_index_sets(idx, q_start, w.B)
    rng = np.random.default_rng(5)
    rows = np.unique(np.concatenate([[0, 1, 127, 128, w.nq - 1], rng.choice(w.nq, 11, replace=False)]))
    ref = _oracle_idx(x, rows, q_start, w.B)
    got = idx[torch.from_numpy(rows).cuda()].cpu().numpy()
    assert np.array_equal(got, ref)
    # prefill attention on the full problem, sampled rows against the oracle
    out = lsa.lsa_prefill_attn(x["q"].cuda(), x["k"].cuda(), x["v"].cuda(), idx)
    torch.cuda.synchronize()
    sel = rows[:6]
    ref_out = O.prefill_attention(np32(x["q"][sel]), LazyRows(x["k"]), LazyRows(x["v"]), ref[:6], w.scale)
    assert_out_close(out[torch.from_numpy(sel).cuda()], ref_out)
