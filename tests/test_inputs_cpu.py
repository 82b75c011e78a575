"""The seeded input recipe: determinism, value ranges and the heavy-hitter
rule (chosen positions have both their K row and their projected-key row
scaled, so the projection stays linear)."""
from __future__ import annotations

import torch

from indexed_sparse_attention_kv_b200 import inputs as I


def _small(heavy):
    return I.Workload("t", 77, batch=2, hq=8, hkv=2, d=16, T=300, r=8, B=20, heavy_frac=heavy)


def test_seeded_and_deterministic():
    a, b = I.make_decode_inputs(_small(0.05)), I.make_decode_inputs(_small(0.05))
    for k in ("q", "qt", "k", "v", "kt", "heavy"):
        assert torch.equal(a[k], b[k]), k
    c = I.make_decode_inputs(_small(0.05), seed=78)
    assert not torch.equal(a["kt"], c["kt"])


def test_integer_projected_values_in_range():
    w = _small(0.0)
    x = I.make_decode_inputs(w)
    for k in ("qt", "kt"):
        v = x[k].float()
        assert torch.equal(v, v.round()) and v.abs().max() <= w.int_range, k


def test_heavy_hitters_scale_k_and_kt_together():
    w0, w1 = _small(0.0), _small(0.05)
    x0, x1 = I.make_decode_inputs(w0), I.make_decode_inputs(w1)
    heavy = x1["heavy"]
    assert heavy.shape == (2, 2, round(0.05 * 300))
    for b in range(2):
        for h in range(2):
            p = heavy[b, h]
            assert len(set(p.tolist())) == len(p)                 # without replacement
            s = float(w1.heavy_scale)
            assert torch.equal(x1["kt"][b, p, h].float(), x0["kt"][b, p, h].float() * s)
            assert torch.equal(x1["k"][b, p, h], (x0["k"][b, p, h].float() * s).to(torch.bfloat16))
            rest = torch.ones(300, dtype=torch.bool)
            rest[p] = False
            assert torch.equal(x1["kt"][b, rest, h], x0["kt"][b, rest, h])


def test_projection_inputs():
    a = I.make_projection_inputs(5, 1, 10, 4, 16, 8, 2)
    b = I.make_projection_inputs(5, 1, 10, 4, 16, 8, 2)
    assert torch.equal(a["x"], b["x"]) and torch.equal(a["P"], b["P"])
    assert a["x"].shape == (1, 10, 4, 16) and a["P"].shape == (2, 8, 16)
    assert a["x"].float().abs().max() <= 3 and a["P"].float().abs().max() <= 2


def test_query_sets_seeded_distinct_and_in_range():
    """Rotating query sets: deterministic per seed, set i from seed + i (so the
    sets differ), projected queries integers in [-R, R], queries bf16."""
    w = _small(0.0)
    a, b = I.make_query_sets(w, 3, seed=500), I.make_query_sets(w, 3, seed=500)
    assert torch.equal(a["q"], b["q"]) and torch.equal(a["qt"], b["qt"])
    assert a["q"].shape == (3, 2, 8, 16) and a["qt"].shape == (3, 2, 8, 8)
    assert not torch.equal(a["qt"][0], a["qt"][1]) and not torch.equal(a["q"][1], a["q"][2])
    c = I.make_query_sets(w, 1, seed=501)   # set 1 of seed 500 is set 0 of seed 501
    assert torch.equal(c["qt"][0], a["qt"][1]) and torch.equal(c["q"][0], a["q"][1])
    v = a["qt"].float()
    assert torch.equal(v, v.round()) and v.abs().max() <= w.int_range
    assert a["q"].dtype == torch.bfloat16
