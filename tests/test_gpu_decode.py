"""GPU parity of the decode path against the CPU oracle, through the C ABI.

Index sets are compared bit-exactly; attention outputs within 1e-2 absolute
and 1e-2 relative (to the largest reference magnitude). Small cases span
several tiles with ragged tails, every supported group size, B > T, B == T,
T == 1, B == 1, KV-head counts that do and do not divide the scorer's warp
count; the named workloads run at full size.
"""
from __future__ import annotations

import math

import numpy as np
import pytest
import torch

import indexed_sparse_attention_kv_b200 as lsa
import oracle.lsa_oracle as O
from indexed_sparse_attention_kv_b200 import inputs as I

from _util import assert_out_close, decode_inputs, np32, oracle_decode, to_dev

pytestmark = pytest.mark.gpu

SMALL = [
    # batch, hq, hkv, d, r, T, B
    (1, 4, 1, 128, 64, 4096, 256),
    (2, 8, 2, 128, 64, 1000, 100),
    (1, 8, 8, 64, 32, 777, 777),
    (3, 12, 3, 128, 64, 2500, 300),
    (1, 16, 1, 256, 128, 300, 64),
    (2, 4, 2, 64, 16, 129, 200),
    (1, 2, 1, 128, 64, 1, 4),
    (1, 32, 8, 128, 64, 5000, 1),
    (1, 16, 16, 128, 64, 3000, 512),
    (2, 64, 4, 128, 64, 700, 96),
]


def _small(case, seed=7, int_range=8, heavy=0.0):
    batch, hq, hkv, d, r, T, B = case
    w = I.Workload(f"small_{case}", seed, batch=batch, hq=hq, hkv=hkv, d=d, T=T, r=r, B=B,
                   int_range=int_range, heavy_frac=heavy)
    return w, I.make_decode_inputs(w)


@pytest.mark.parametrize("case", SMALL, ids=[str(c) for c in SMALL])
def test_decode_step_small(case):
    w, x = _small(case, heavy=0.05 if case[5] >= 1000 else 0.0)
    dx = to_dev(x)
    idx, out = lsa.lsa_decode_step(dx["q"], dx["qt"], dx["k"], dx["v"], dx["kt"], w.B)
    torch.cuda.synchronize()
    ref_idx, ref_out = oracle_decode(x, w)
    assert np.array_equal(idx.cpu().numpy(), ref_idx)
    assert_out_close(out, ref_out)


@pytest.mark.parametrize("case", SMALL[:6], ids=[str(c) for c in SMALL[:6]])
def test_components_small(case):
    """lsa_score exact, lsa_topk bit-exact, lsa_indexed_attn within tolerance."""
    w, x = _small(case, seed=11)
    dx = to_dev(x)
    s = lsa.lsa_score(dx["qt"], dx["kt"])
    idx = lsa.lsa_topk(s, w.B)
    out = lsa.lsa_indexed_attn(dx["q"], dx["k"], dx["v"], idx)
    torch.cuda.synchronize()
    for b in range(w.batch):
        q_bar = O.group_mean_query(np32(x["qt"][b]), w.hkv)
        ref_s = O.candidate_scores(q_bar, np32(x["kt"][b]))
        assert np.array_equal(s[b].cpu().numpy().astype(np.float64), ref_s)
        ref_idx = np.stack([O.select_top_b(ref_s[h], w.B) for h in range(w.hkv)])
        assert np.array_equal(idx[b].cpu().numpy(), ref_idx)
        ref_out = O.indexed_attention(np32(x["q"][b]), np32(x["k"][b]), np32(x["v"][b]), ref_idx, w.scale)
        assert_out_close(out[b], ref_out)


def _topk_rows(rng, n, kind):
    if kind == "ties":
        return rng.integers(-3, 4, size=n).astype(np.float32)
    if kind == "nan":
        v = rng.integers(-50, 50, size=n).astype(np.float32)
        v[rng.random(n) < 0.3] = np.nan
        return v
    if kind == "signed_zero":
        v = rng.integers(-1, 2, size=n).astype(np.float32)
        v[v == 0] = np.where(rng.random(int((v == 0).sum())) < 0.5, -0.0, 0.0)
        return v
    if kind == "float":
        v = rng.standard_normal(n).astype(np.float32) * 100
        v[rng.random(n) < 0.01] = np.inf
        v[rng.random(n) < 0.01] = -np.inf
        return v
    if kind == "equal":
        return np.full(n, 2.5, dtype=np.float32)
    if kind == "allnan":
        return np.full(n, np.nan, dtype=np.float32)
    raise ValueError(kind)


@pytest.mark.parametrize("n", [1, 31, 1000, 4097, 40000, 65537, 131072, 131077, 200003])
@pytest.mark.parametrize("kind", ["ties", "nan", "signed_zero", "float", "equal", "allnan"])
def test_topk_rows(n, kind):
    rng = np.random.default_rng(n * 7 + len(kind))
    rows = 3
    S = np.stack([_topk_rows(rng, n, kind) for _ in range(rows)])
    for B in sorted({1, 2, max(1, n // 64), max(1, n // 2), n, n + 5, 2048} - {0}):
        if B > 65536:
            continue
        idx = lsa.lsa_topk(torch.from_numpy(S).cuda(), B)
        got = idx.cpu().numpy()
        for r in range(rows):
            want = O.select_top_b(S[r].astype(np.float64), B)
            assert np.array_equal(got[r], want), (n, kind, B, r)


def test_determinism_and_components_equal_step():
    w, x = decode_inputs("tiny_4k")
    dx = to_dev(x)
    i1, o1 = lsa.lsa_decode_step(dx["q"], dx["qt"], dx["k"], dx["v"], dx["kt"], w.B)
    i2, o2 = lsa.lsa_decode_step(dx["q"], dx["qt"], dx["k"], dx["v"], dx["kt"], w.B)
    s = lsa.lsa_score(dx["qt"], dx["kt"])
    i3 = lsa.lsa_topk(s, w.B)
    o3 = lsa.lsa_indexed_attn(dx["q"], dx["k"], dx["v"], i3)
    torch.cuda.synchronize()
    assert torch.equal(i1, i2) and torch.equal(o1, o2)
    assert torch.equal(i1, i3) and torch.equal(o1, o3)


def test_bad_index_is_skipped_and_flagged():
    w, x = _small((1, 8, 2, 128, 64, 500, 40), seed=3)
    dx = to_dev(x)
    idx = torch.stack([torch.randperm(w.T, generator=torch.Generator().manual_seed(h))[: w.B].sort().values
                       for h in range(w.hkv)]).to(torch.int32)[None]
    bad = idx.clone()
    bad[0, 0, 3] = w.T          # out of range
    bad[0, 1, 7] = -5           # below -1
    bad[0, 1, 9] = 1 << 30
    ws = lsa.workspace(lsa._lib.decode_dims(dx["q"], dx["qt"], dx["k"]), w.B)
    out = lsa.lsa_indexed_attn(dx["q"], dx["k"], dx["v"], bad.cuda(), ws=ws)
    assert lsa.lsa_read_device_status(ws) & lsa._lib.DEV_BAD_INDEX
    ref_idx = bad[0].numpy().copy()
    ref_idx[(ref_idx < -1) | (ref_idx >= w.T)] = -1
    ref = O.indexed_attention(np32(x["q"][0]), np32(x["k"][0]), np32(x["v"][0]), ref_idx, w.scale)
    assert_out_close(out[0], ref)
    lsa.lsa_clear_device_status(ws)
    lsa.lsa_indexed_attn(dx["q"], dx["k"], dx["v"], idx.cuda(), ws=ws)
    assert lsa.lsa_read_device_status(ws) == 0


def test_bounded_wait_reports_timeout():
    """A zero poll budget makes the scorer's pipeline waits run out: the step
    sets LSA_DEV_TIMEOUT and returns; the context stays usable."""
    w, x = decode_inputs("tiny_4k")
    dx = to_dev(x)
    dims = lsa._lib.decode_dims(dx["q"], dx["qt"], dx["k"])
    ws = lsa.workspace(dims, w.B)
    try:
        lsa.lsa_debug_set_wait_limit(0)
        lsa.lsa_decode_step(dx["q"], dx["qt"], dx["k"], dx["v"], dx["kt"], w.B, ws=ws)
        status = lsa.lsa_read_device_status(ws)
    finally:
        lsa.lsa_debug_set_wait_limit(-1)
    assert status & lsa._lib.DEV_TIMEOUT
    lsa.lsa_clear_device_status(ws)
    idx, out = lsa.lsa_decode_step(dx["q"], dx["qt"], dx["k"], dx["v"], dx["kt"], w.B, ws=ws)
    assert lsa.lsa_read_device_status(ws) == 0
    ref_idx, ref_out = oracle_decode(x, w)
    assert np.array_equal(idx.cpu().numpy(), ref_idx)
    assert_out_close(out, ref_out)


HIER = [
    # batch, hq, hkv, d, r, T, B, blk, keep
    (1, 8, 2, 128, 64, 5000, 300, 64, 8),
    (2, 4, 1, 128, 64, 1000, 100, 16, 100),     # keep >= blocks: equals flat selection
    (1, 32, 8, 128, 64, 8192, 2048, 64, 64),
    (1, 6, 3, 64, 32, 999, 50, 32, 3),
]


@pytest.mark.parametrize("case", HIER, ids=[str(c) for c in HIER])
def test_hierarchical_small(case):
    batch, hq, hkv, d, r, T, B, blk, keep = case
    w = I.Workload(f"hier_{case}", 5, batch=batch, hq=hq, hkv=hkv, d=d, T=T, r=r, B=B, int_range=4,
                   blk=blk, keep=keep)
    x = I.make_decode_inputs(w)
    dx = to_dev(x)
    cen = lsa.lsa_block_centroids(dx["kt"], blk)
    idx, out = lsa.lsa_decode_step(dx["q"], dx["qt"], dx["k"], dx["v"], dx["kt"], B, centroids=cen, blk=blk,
                                   keep=keep)
    torch.cuda.synchronize()
    for b in range(batch):
        ref_c = O.block_centroids(np32(x["kt"][b]), blk)
        assert np.array_equal(np32(cen[b]).astype(np.float64), ref_c)   # |sum| <= 4 * 64: exact in bf16
    ref_idx, ref_out = oracle_decode(x, w, blk=blk, keep=keep)
    assert np.array_equal(idx.cpu().numpy(), ref_idx)
    assert_out_close(out, ref_out)
    if keep * blk >= T:
        flat_idx, _ = oracle_decode(x, w)
        assert np.array_equal(idx.cpu().numpy(), flat_idx)


def test_centroids_round_to_bf16():
    """Sums too large for bf16 are rounded to nearest even (8 significant bits)."""
    w = I.Workload("cen_round", 9, batch=2, hq=8, hkv=2, d=128, T=1000, r=64, B=16, int_range=8)
    x = I.make_decode_inputs(w)
    cen = lsa.lsa_block_centroids(x["kt"].cuda(), 64)
    for b in range(2):
        ref = torch.from_numpy(O.block_centroids(np32(x["kt"][b]), 64)).to(torch.bfloat16)
        assert torch.equal(cen[b].cpu(), ref)


# ------------------------------------------------------------------- full sizes

@pytest.mark.slow
@pytest.mark.parametrize("name", ["tiny_4k", "llama8b_32k", "decode_128k"])
def test_named_workload_flat(name):
    w, x = decode_inputs(name)
    dx = to_dev(x)
    idx, out = lsa.lsa_decode_step(dx["q"], dx["qt"], dx["k"], dx["v"], dx["kt"], w.B)
    torch.cuda.synchronize()
    ref_idx, ref_out = oracle_decode(x, w)
    assert np.array_equal(idx.cpu().numpy(), ref_idx)
    assert_out_close(out, ref_out)
    del dx
    torch.cuda.empty_cache()


@pytest.mark.slow
def test_named_workload_hier_1m():
    w, x = decode_inputs("hier_1m")
    dx = to_dev(x)
    cen = lsa.lsa_block_centroids(dx["kt"], w.blk)
    idx, out = lsa.lsa_decode_step(dx["q"], dx["qt"], dx["k"], dx["v"], dx["kt"], w.B, centroids=cen,
                                   blk=w.blk, keep=w.keep)
    torch.cuda.synchronize()
    kt0 = np32(x["kt"][0])
    ref_c = O.block_centroids(kt0, w.blk)
    assert np.array_equal(np32(cen[0]).astype(np.float64), ref_c)
    ref_idx, ref_out = oracle_decode(x, w, blk=w.blk, keep=w.keep)
    assert np.array_equal(idx.cpu().numpy(), ref_idx)
    assert_out_close(out, ref_out)
    del dx, cen
    torch.cuda.empty_cache()


def test_attention_over_a_whole_cache():
    """An index set may cover every cached position (B = T > 65536): the
    dense full-KV attention, equal to the oracle over all positions."""
    w = I.Workload("whole_cache", 109, batch=1, hq=4, hkv=1, d=128, T=70000, r=64, B=70000)
    x = I.make_decode_inputs(w)
    dx = to_dev(x, ("q", "k", "v"))
    idx = torch.arange(w.T, dtype=torch.int32, device="cuda").view(1, 1, w.T)
    out = lsa.lsa_indexed_attn(dx["q"], dx["k"], dx["v"], idx)
    torch.cuda.synchronize()
    ref = O.indexed_attention(np32(x["q"][0]), np32(x["k"][0]), np32(x["v"][0]), np.arange(w.T)[None], w.scale)
    assert_out_close(out[0], ref)


# Shapes whose attention runs in cluster mode (every unit has 8 .. 64 tiles of
# 64 entries and all units' 8-CTA clusters fit in one wave): ragged last tiles,
# every head dimension and group size, empty rows (NaN keys), and the paged
# cache; the whole step is compared with the oracle.
CLUSTER = [
    # batch, hq, hkv, d, r, T, B
    (1, 4, 1, 128, 64, 6000, 1000),
    (2, 16, 2, 64, 32, 5000, 600),
    (1, 16, 1, 256, 128, 5000, 4096),
    (3, 6, 6, 128, 64, 3000, 513),
    (1, 4, 2, 128, 64, 2000, 1100),
    (2, 32, 8, 128, 64, 9000, 2048),
]


@pytest.mark.parametrize("case", CLUSTER, ids=[str(c) for c in CLUSTER])
def test_decode_step_cluster_mode(case):
    w, x = _small(case, heavy=0.05)
    dx = to_dev(x)
    idx, out = lsa.lsa_decode_step(dx["q"], dx["qt"], dx["k"], dx["v"], dx["kt"], w.B)
    torch.cuda.synchronize()
    ref_idx, ref_out = oracle_decode(x, w)
    assert np.array_equal(idx.cpu().numpy(), ref_idx)
    assert_out_close(out, ref_out)


def test_cluster_mode_empty_rows_bad_index_and_paged():
    """Cluster mode: a head whose set is all -1 gives zeros, out-of-range
    entries are skipped and flagged, and the paged cache gives the same bits
    as the contiguous one."""
    w, x = _small((2, 8, 2, 128, 64, 3000, 700), seed=11)
    dx = to_dev(x)
    g = torch.Generator().manual_seed(12)
    idx = torch.stack([torch.stack([torch.randperm(w.T, generator=g)[: w.B].sort().values for _ in range(w.hkv)])
                       for _ in range(w.batch)]).to(torch.int32)
    idx[1, 0, :] = -1                 # an empty set
    idx[0, 1, 5] = w.T                # out of range: skipped, flagged
    ws = lsa.workspace(lsa._lib.decode_dims(dx["q"], dx["qt"], dx["k"]), w.B)
    out = lsa.lsa_indexed_attn(dx["q"], dx["k"], dx["v"], idx.cuda(), ws=ws)
    torch.cuda.synchronize()
    assert lsa.lsa_read_device_status(ws) & lsa._lib.DEV_BAD_INDEX
    ref_idx = idx.numpy().copy()
    ref_idx[ref_idx >= w.T] = -1
    for b in range(w.batch):
        ref = O.indexed_attention(np32(x["q"][b]), np32(x["k"][b]), np32(x["v"][b]), ref_idx[b], w.scale)
        assert_out_close(out[b], ref)
    assert torch.all(out[1, :4] == 0)
    # paged: the same rows in a shuffled pool
    n = w.batch * w.T
    perm = torch.randperm(n, generator=torch.Generator().manual_seed(13)).cuda()
    kp = torch.empty((n, w.hkv, w.d), dtype=torch.bfloat16, device="cuda")
    vp = torch.empty_like(kp)
    kp[perm] = dx["k"].reshape(n, w.hkv, w.d)
    vp[perm] = dx["v"].reshape(n, w.hkv, w.d)
    idx_ok = idx.clone()
    idx_ok[idx_ok >= w.T] = -1
    out_c = lsa.lsa_indexed_attn(dx["q"], dx["k"], dx["v"], idx_ok.cuda())
    out_p = lsa.lsa_indexed_attn_paged(dx["q"], kp, vp, perm.to(torch.int32).view(w.batch, w.T), idx_ok.cuda())
    torch.cuda.synchronize()
    assert torch.equal(out_c, out_p)
