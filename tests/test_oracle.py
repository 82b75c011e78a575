"""Pins for the CPU oracle: each check fixes the oracle by something other than itself.

* brute force on tiny inputs (exhaustive lexicographic sort for top-B, integer
  loops for group-mean scores),
* special cases that reduce to a library routine (indexed attention over every
  position == torch's scaled_dot_product_attention with GQA; over a subset ==
  SDPA on the gathered rows; top-1 == numpy argmax),
* closed forms (one-hot projected keys, ramp centroids, zero query == mean of
  the selected values, single key == its value row),
* invariants (weights sum to 1, unselected rows never matter, keeping every
  block reduces coarse-to-fine to flat selection, block score == sum of token
  scores, a prefill row == decode selection over the row's causal prefix),
* hand-derived worked examples under tests/golden/ (the pages print none),
* for scoring preparation: torch's fp32 -> bf16 / float8_e4m3fn casts on
  values where one rounding is the whole story, hand-derived ties and
  saturation, permuted unit bases (closed form), orthonormal bases
  (Pythagoras), integer brute force, and incremental centroids that must
  rebuild the (separately pinned) block sums.

``test_planted_mistakes_are_caught`` plants typical mistakes in copies of the
oracle's functions and checks that at least one pin fails for every mistake.
"""
from __future__ import annotations

import json
import math
import os
import types

import numpy as np
import pytest
import torch

import oracle.lsa_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _load(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


# ----------------------------------------------------------------------------- checks
# Each check takes a namespace with the oracle's functions, so that the same
# check can be run against planted-mistake variants.

def check_select_bruteforce(o):
    rng = np.random.default_rng(7)
    for trial in range(300):
        n = int(rng.integers(1, 40))
        vals = rng.integers(-3, 4, size=n).astype(np.float64)   # many ties
        if trial % 5 == 0:
            vals[rng.random(n) < 0.2] = np.nan                     # non-candidates
        if trial % 7 == 0:
            vals[vals == 0] = -0.0                                 # -0 ties +0
        B = int(rng.integers(1, n + 4))
        got = o.select_top_b(vals, B)
        valid = np.nonzero(~np.isnan(vals))[0]
        order = np.lexsort((valid, -vals[valid]))                  # score desc, position asc
        want = np.full(B, -1)
        pick = np.sort(valid[order[:B]])
        want[: len(pick)] = pick
        assert np.array_equal(got, want), (vals, B, got, want)


def check_select_special(o):
    rng = np.random.default_rng(8)
    for _ in range(50):
        n = int(rng.integers(1, 200))
        vals = rng.integers(-5, 6, size=n).astype(np.float64)
        assert o.select_top_b(vals, 1)[0] == int(np.argmax(vals))     # first maximum
        assert np.array_equal(o.select_top_b(vals, n), np.arange(n))
    flat = np.zeros(10)
    assert np.array_equal(o.select_top_b(flat, 4), np.arange(4))


def check_scores_bruteforce(o):
    """Integer loops over every query head of the group (exact with Python ints)."""
    rng = np.random.default_rng(9)
    for hq, hkv in [(4, 1), (8, 2), (6, 3), (8, 8), (32, 8)]:
        T, r = 11, 5
        qt = rng.integers(-8, 9, size=(hq, r))
        kt = rng.integers(-8, 9, size=(T, hkv, r))
        G = hq // hkv
        s = o.candidate_scores(o.group_mean_query(qt, hkv), kt)
        for h in range(hkv):
            for t in range(T):
                tot = 0
                for i in range(hq):
                    if i * hkv // hq == h:            # the G query heads of KV head h
                        tot += sum(int(qt[i, j]) * int(kt[t, h, j]) for j in range(r))
                assert s[h, t] == tot / G, (hq, hkv, h, t)


def check_scores_onehot(o):
    """kt[t, h] = c_t * e_{j(t)} gives s[h, t] = c_t * q_bar[h, j(t)]."""
    hq, hkv, r, T = 8, 2, 6, 12
    qt = np.arange(hq * r, dtype=np.float64).reshape(hq, r) - 20
    kt = np.zeros((T, hkv, r))
    for t in range(T):
        for h in range(hkv):
            kt[t, h, (t + h) % r] = t - 5
    q_bar = np.stack([qt[h * 4:(h + 1) * 4].mean(0) for h in range(hkv)])
    s = o.candidate_scores(o.group_mean_query(qt, hkv), kt)
    for t in range(T):
        for h in range(hkv):
            assert s[h, t] == (t - 5) * q_bar[h, (t + h) % r]


def _sdpa(q, k, v, scale):
    """torch SDPA in float64 with GQA: q [hq, L, d], k/v [hkv, S, d]."""
    return torch.nn.functional.scaled_dot_product_attention(
        torch.as_tensor(q)[None], torch.as_tensor(k)[None], torch.as_tensor(v)[None],
        scale=scale, enable_gqa=True)[0]


def check_attention_full_budget_sdpa(o):
    rng = np.random.default_rng(10)
    for hq, hkv, T, d in [(4, 1, 37, 16), (8, 2, 64, 8), (32, 8, 19, 32), (6, 3, 5, 4)]:
        q = rng.standard_normal((hq, d))
        k = rng.standard_normal((T, hkv, d)) * 2
        v = rng.standard_normal((T, hkv, d))
        scale = 1.0 / math.sqrt(d)
        idx = np.tile(np.arange(T), (hkv, 1))
        got = o.indexed_attention(q, k, v, idx, scale)
        want = _sdpa(q[:, None, :], k.transpose(1, 0, 2), v.transpose(1, 0, 2), scale)[:, 0, :].numpy()
        assert np.allclose(got, want, rtol=1e-12, atol=1e-12)


def check_attention_subset_sdpa(o):
    rng = np.random.default_rng(11)
    for hq, hkv, T, d, B in [(4, 1, 50, 16, 7), (8, 2, 40, 8, 13), (32, 8, 30, 16, 3)]:
        q = rng.standard_normal((hq, d))
        k = rng.standard_normal((T, hkv, d))
        v = rng.standard_normal((T, hkv, d))
        idx = np.stack([np.sort(rng.choice(T, B, replace=False)) for _ in range(hkv)])
        idx[0, -1] = -1                                   # a padded slot is ignored
        scale = 1.0 / math.sqrt(d)
        got = o.indexed_attention(q, k, v, idx, scale)
        G = hq // hkv
        for h in range(hkv):
            sel = torch.as_tensor(idx[h][idx[h] >= 0])
            kh = torch.as_tensor(k[:, h, :]).index_select(0, sel)
            vh = torch.as_tensor(v[:, h, :]).index_select(0, sel)
            qh = torch.as_tensor(q[h * G:(h + 1) * G])
            want = _sdpa(qh[:, None, :], kh[None], vh[None], scale)[:, 0, :].numpy()
            assert np.allclose(got[h * G:(h + 1) * G], want, rtol=1e-12, atol=1e-12)


def check_attention_closed_forms(o):
    rng = np.random.default_rng(12)
    T, hkv, d, hq = 20, 2, 8, 4
    k = rng.standard_normal((T, hkv, d))
    v = rng.standard_normal((T, hkv, d))
    # single selected key: output is exactly that value row
    idx = np.array([[5, -1, -1], [17, -1, -1]])
    out = o.indexed_attention(rng.standard_normal((hq, d)), k, v, idx, 0.3)
    assert np.allclose(out[0], v[5, 0]) and np.allclose(out[3], v[17, 1])
    # zero query: uniform weights, the mean of the selected values
    idx = np.array([[1, 4, 9], [0, 2, 3]])
    out = o.indexed_attention(np.zeros((hq, d)), k, v, idx, 0.3)
    assert np.allclose(out[1], v[[1, 4, 9], 0].mean(0)) and np.allclose(out[2], v[[0, 2, 3], 1].mean(0))
    # weights form a distribution and scale the logit differences by `scale`
    w = o.attention_weights(np.array([1.0, 0.0]), np.array([[1.0, 0.0], [0.0, 0.0]]), 2.0)
    assert abs(w.sum() - 1) < 1e-15 and abs(w[0] / w[1] - math.exp(2.0)) < 1e-12
    # empty selection gives zeros
    out = o.indexed_attention(np.ones((hq, d)), k, v, np.full((hkv, 2), -1), 0.3)
    assert not out.any()


def check_attention_unselected_irrelevant(o):
    rng = np.random.default_rng(13)
    T, hkv, d, hq, B = 64, 2, 16, 8, 10
    q = rng.standard_normal((hq, d))
    k = rng.standard_normal((T, hkv, d))
    v = rng.standard_normal((T, hkv, d))
    idx = np.stack([np.sort(rng.choice(T, B, replace=False)) for _ in range(hkv)])
    base = o.indexed_attention(q, k, v, idx, 0.25)
    k2, v2 = k.copy(), v.copy()
    for h in range(hkv):
        rest = np.setdiff1d(np.arange(T), idx[h])
        k2[rest, h] = rng.permutation(k2[rest, h]) * 1e3
        v2[rest, h] = 1e6
    assert np.array_equal(o.indexed_attention(q, k2, v2, idx, 0.25), base)


def check_centroids_closed_form(o):
    T, blk = 200, 64                                   # last block partial (8 tokens)
    kt = np.zeros((T, 2, 3))
    kt[:, 0, 0] = np.arange(T)
    kt[:, 1, 2] = 1
    c = o.block_centroids(kt, blk)
    assert c.shape == (4, 2, 3)
    for j in range(4):
        lo, hi = j * blk, min(T, (j + 1) * blk)
        assert c[j, 0, 0] == (lo + hi - 1) * (hi - lo) / 2    # arithmetic series
        assert c[j, 1, 2] == hi - lo
        assert c[j, 0, 1] == 0 and c[j, 1, 0] == 0


def check_hier_reductions(o):
    rng = np.random.default_rng(14)
    for T, blk, hkv, hq, B in [(256, 16, 2, 8, 20), (300, 32, 1, 4, 50), (64, 8, 3, 3, 64)]:
        kt = rng.integers(-2, 3, size=(T, hkv, 4)).astype(np.float64)
        qt = rng.integers(-2, 3, size=(hq, 4)).astype(np.float64)
        q_bar = o.group_mean_query(qt, hkv)
        nblk = -(-T // blk)
        hier = o.hierarchical_select(q_bar, kt, blk, nblk, B)            # keep every block
        s = o.candidate_scores(q_bar, kt)
        flat = np.stack([o.select_top_b(s[h], B) for h in range(hkv)])
        assert np.array_equal(hier, flat)
        # block score == sum of its token scores (linearity)
        c = o.block_centroids(kt, blk)
        for h in range(hkv):
            cs = c[:, h, :] @ q_bar[h]
            for j in range(nblk):
                assert abs(cs[j] - s[h, j * blk:(j + 1) * blk].sum()) < 1e-9
        # brute force: blocks by (score desc, index asc), then tokens by (score desc, position asc)
        for keep in (1, 2, 3):
            hier = o.hierarchical_select(q_bar, kt, blk, keep, B)
            for h in range(hkv):
                cs = c[:, h, :] @ q_bar[h]
                blocks = np.lexsort((np.arange(nblk), -cs))[:keep]
                cand = np.concatenate([np.arange(j * blk, min(T, (j + 1) * blk)) for j in blocks])
                order = np.lexsort((cand, -s[h, cand]))[:B]
                want = np.full(B, -1)
                want[: len(order)] = np.sort(cand[order])
                assert np.array_equal(hier[h], want), (T, blk, keep, h)
    # tied block scores: the lower block index wins
    kt = np.zeros((32, 1, 1))
    kt[[0, 9, 17, 25], 0, 0] = [1, 1, 1, 2]          # blocks of 8: scores [1, 1, 1, 2]
    got = o.hierarchical_select(np.ones((1, 1)), kt, 8, 2, 1)
    assert np.array_equal(got, [[25]])
    got = o.hierarchical_select(np.ones((1, 1)), kt, 8, 3, 3)
    assert np.array_equal(got, [[0, 9, 25]])


def check_prefill_vs_decode_prefix(o):
    rng = np.random.default_rng(15)
    T, hkv, hq, r, B = 90, 2, 4, 6, 12
    kt = rng.integers(-8, 9, size=(T, hkv, r)).astype(np.float64)
    positions = np.array([0, 5, 11, 12, 47, 89])
    qt_rows = rng.integers(-8, 9, size=(len(positions), hq, r)).astype(np.float64)
    idx = o.prefill_index(qt_rows, positions, kt, B)
    for n, p in enumerate(positions):
        q_bar = o.group_mean_query(qt_rows[n], hkv)
        s = o.candidate_scores(q_bar, kt[: p + 1])
        for h in range(hkv):
            assert np.array_equal(idx[n, h], o.select_top_b(s[h], B))
            assert idx[n, h].max() <= p


def check_golden(o):
    g = _load("select_ties_group2.json")
    q_bar = o.group_mean_query(np.array(g["qt"]), g["hkv"])
    s = o.candidate_scores(q_bar, np.array(g["kt"], dtype=np.float64))
    assert np.array_equal(s, np.array(g["scores"], dtype=np.float64))
    for B, want in g["expected"].items():
        got = np.stack([o.select_top_b(s[h], int(B)) for h in range(g["hkv"])])
        assert np.array_equal(got, np.array(want)), (B, got)

    g = _load("select_two_heads.json")
    q_bar = o.group_mean_query(np.array(g["qt"]), g["hkv"])
    s = o.candidate_scores(q_bar, np.array(g["kt"], dtype=np.float64))
    assert np.array_equal(s, np.array(g["scores"], dtype=np.float64))
    got = np.stack([o.select_top_b(s[h], 2) for h in range(g["hkv"])])
    assert np.array_equal(got, np.array(g["expected"]["2"]))

    g = _load("attention_closed_form.json")
    q, k, v = (np.array(g[x], dtype=np.float64) for x in ("q", "k", "v"))
    w = o.attention_weights(q[0], k[np.array(g["idx"][0]), 0, :], g["scale"])
    assert np.allclose(w, g["weights"], rtol=0, atol=1e-14)
    out = o.indexed_attention(q, k, v, np.array(g["idx"]), g["scale"])
    assert np.allclose(out, g["out"], rtol=0, atol=1e-14)

    g = _load("scoring_preparation.json")
    x, P = np.array(g["x"], dtype=np.float64), np.array(g["P"], dtype=np.float64)
    assert np.array_equal(o.project_rows(x, P, g["G"]), np.array(g["exact"], dtype=np.float64))
    assert np.array_equal(o.round_to_bf16(o.project_rows(x, P, g["G"])), np.array(g["bf16"], dtype=np.float64))
    assert np.array_equal(o.round_to_e4m3(o.project_rows(x, P, g["G"])), np.array(g["e4m3"], dtype=np.float64))
    assert np.array_equal(o.project_bf16(x, P, g["G"]), np.array(g["bf16"], dtype=np.float64))
    assert np.array_equal(o.project_e4m3(x, P, g["G"]), np.array(g["e4m3"], dtype=np.float64))
    c = o.update_centroids(np.array(g["centroid_start"], dtype=np.float64), np.array(g["kt"], dtype=np.float64),
                           g["t0"], g["n"], g["blk"])
    assert np.array_equal(c, np.array(g["centroid_end"], dtype=np.float64))

    g = _load("hierarchical_blocks.json")
    kt = np.array(g["kt"], dtype=np.float64)
    assert np.array_equal(o.block_centroids(kt, g["blk"]), np.array(g["centroids"], dtype=np.float64))
    q_bar = o.group_mean_query(np.array(g["qt"]), g["hkv"])
    for case in g["cases"]:
        got = o.hierarchical_select(q_bar, kt, g["blk"], case["keep"], case["B"])
        assert np.array_equal(got, np.array(case["idx"])), case

    g = _load("prefill_causal.json")
    got = o.prefill_index(np.array(g["qt"], dtype=np.float64), np.array(g["positions"]),
                          np.array(g["kt"], dtype=np.float64), g["B"])
    assert np.array_equal(got, np.array(g["idx"]))


# ------------------------------------------------------------------ scoring preparation

def check_paged_attention(o):
    """Identity page table == the contiguous cache; a permuted pool read
    through the matching table == the contiguous cache; unfilled slots of
    positions outside the index sets do not matter."""
    rng = np.random.default_rng(27)
    T, hkv, hq, d, B = 40, 2, 4, 8, 6
    q = rng.standard_normal((hq, d))
    k = rng.standard_normal((T, hkv, d))
    v = rng.standard_normal((T, hkv, d))
    idx = np.stack([np.sort(rng.choice(T, B, replace=False)) for _ in range(hkv)])
    ref = o.indexed_attention(q, k, v, idx, 0.3)
    assert np.array_equal(o.indexed_attention_paged(q, k, v, np.arange(T), idx, 0.3), ref)
    perm = rng.permutation(T + 5)                     # pool with 5 spare slots
    pool_k = rng.standard_normal((T + 5, hkv, d))
    pool_v = rng.standard_normal((T + 5, hkv, d))
    slots = perm[:T]
    pool_k[slots] = k
    pool_v[slots] = v
    assert np.allclose(o.indexed_attention_paged(q, pool_k, pool_v, slots, idx, 0.3), ref, rtol=0, atol=1e-12)
    holes = slots.copy()
    unused = np.setdiff1d(np.arange(T), idx.ravel())
    holes[unused[:3]] = -1
    assert np.allclose(o.indexed_attention_paged(q, pool_k, pool_v, holes, idx, 0.3), ref, rtol=0, atol=1e-12)


def check_round_bf16(o):
    """fp32-representable values: one rounding, so torch's fp32 -> bf16 cast
    (round to nearest even) is the reference; plus hand-derived ties."""
    rng = np.random.default_rng(21)
    x32 = np.concatenate([rng.standard_normal(4000) * 10.0 ** rng.integers(-40, 38, 4000),
                          rng.standard_normal(200) * 1e-39]).astype(np.float32)
    x32 = x32[np.isfinite(x32)]
    want = torch.from_numpy(x32).to(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(o.round_to_bf16(x32.astype(np.float64)), want)
    # ulp 2 above 256: 257 and 259 are ties -> even mantissa; ulp 2^-7 at 1
    hand = {257.0: 256.0, 259.0: 260.0, 1 + 2 ** -8: 1.0, 1 + 3 * 2 ** -8: 1 + 2 ** -6,
            -(1 + 3 * 2 ** -8): -(1 + 2 ** -6), 1 + 2 ** -8 + 2 ** -30: 1 + 2 ** -7}
    got = o.round_to_bf16(np.array(list(hand)))
    assert np.array_equal(got, np.array(list(hand.values()))), got


def check_round_e4m3(o):
    """In-range fp32 values against torch's float8_e4m3fn cast; hand ties and
    saturation at 448."""
    rng = np.random.default_rng(22)
    x32 = (rng.standard_normal(4000) * 2.0 ** rng.integers(-12, 8, 4000)).astype(np.float32)
    x32 = x32[np.abs(x32) <= 448]
    want = torch.from_numpy(x32).to(torch.float8_e4m3fn).to(torch.float64).numpy()
    assert np.array_equal(o.round_to_e4m3(x32.astype(np.float64)), want)
    # ulp 2 at 16: 17, 19 are ties; subnormal ulp 2^-9: 1.5 * 2^-9 is a tie -> 2^-8
    hand = {17.0: 16.0, 19.0: 20.0, 1.5 * 2 ** -9: 2 ** -8, 1000.0: 448.0, -500.0: -448.0, 450.0: 448.0}
    got = o.round_to_e4m3(np.array(list(hand)))
    assert np.array_equal(got, np.array(list(hand.values()))), got


def check_project_shifted_unit_basis(o):
    """P[h, j] = unit vector e_{(j + 3h) mod d}: y[..., i, j] = x[..., i, (j + 3 (i // G)) mod d]
    (closed form; fixes the group of head i and the orientation of the basis)."""
    rng = np.random.default_rng(23)
    for nb, G, d, r in [(2, 4, 16, 5), (3, 1, 6, 6), (4, 2, 8, 8)]:
        H = nb * G
        P = np.zeros((nb, r, d))
        for h in range(nb):
            for j in range(r):
                P[h, j, (j + 3 * h) % d] = 1.0
        x = rng.standard_normal((2, 3, H, d))
        y = o.project_rows(x, P, G)
        for i in range(H):
            for j in range(r):
                assert np.array_equal(y[..., i, j], x[..., i, (j + 3 * (i // G)) % d])


def check_project_orthonormal(o):
    """Orthonormal basis rows: ||P x||^2 + ||P' x||^2 = ||x||^2 for the complement P'."""
    rng = np.random.default_rng(24)
    d, r = 12, 5
    Q, _ = np.linalg.qr(rng.standard_normal((d, d)))
    x = rng.standard_normal((7, 1, d))
    y = o.project_rows(x, Q[:r][None], 1)
    z = o.project_rows(x, Q[r:][None], 1)
    assert np.allclose((y ** 2).sum(-1) + (z ** 2).sum(-1), (x ** 2).sum(-1), rtol=1e-12)


def check_project_integer_exact(o):
    """Small integers: the bf16 cache rows equal exact integer dot products
    (|y| <= 32 is exact in bf16), brute force with Python ints."""
    rng = np.random.default_rng(25)
    nb, G, d, r = 2, 2, 16, 4
    x = rng.integers(-2, 3, size=(3, nb * G, d))
    P = rng.integers(-1, 2, size=(nb, r, d))
    y = o.project_bf16(x, P, G)
    for a in range(3):
        for i in range(nb * G):
            for j in range(r):
                assert y[a, i, j] == sum(int(P[i // G, j, c]) * int(x[a, i, c]) for c in range(d))


def check_update_centroids(o):
    """Appending every token (in chunks) to zero centroids rebuilds the block
    sums when they are exact; and a hand-derived rounding sequence: 256 + 1 +
    1 + 3 in bf16 is 256, 256, 260 (each sum rounded: 257 and 259 are ties)."""
    rng = np.random.default_rng(26)
    T, hkv, r, blk = 37, 2, 3, 4
    kt = rng.integers(-3, 4, size=(T, hkv, r)).astype(np.float64)
    c = np.zeros(((T + blk - 1) // blk, hkv, r))
    t = 0
    for n in [5, 1, 0, 13, 18]:
        c = o.update_centroids(c, kt, t, n, blk)
        t += n
    assert np.array_equal(c, o.block_centroids(kt, blk))
    kt2 = np.array([[[0.0]], [[1.0]], [[1.0]], [[3.0]]])
    c2 = o.update_centroids(np.array([[[256.0]]]), kt2, 1, 3, 4)
    assert c2[0, 0, 0] == 260.0, c2
    c3 = o.update_centroids(np.array([[[256.0]]]), kt2, 1, 2, 4)
    assert c3[0, 0, 0] == 256.0, c3


def check_prefill_attention_rows(o):
    """Every prefill row attends over its own index sets: row n equals torch
    SDPA (fp64) on the K/V rows gathered by idx[n], with a different set for
    every row and some rows padded with -1."""
    rng = np.random.default_rng(28)
    n, T, hkv, hq, d, B = 6, 30, 2, 8, 8, 7
    G = hq // hkv
    q = rng.standard_normal((n, hq, d))
    k = rng.standard_normal((T, hkv, d)) * 2
    v = rng.standard_normal((T, hkv, d))
    idx = np.full((n, hkv, B), -1)
    for i in range(n):
        for h in range(hkv):
            m = B - (i % 3)
            idx[i, h, :m] = np.sort(rng.choice(T, m, replace=False))
    assert len({idx[i].tobytes() for i in range(n)}) == n
    got = o.prefill_attention(q, k, v, idx, 0.3)
    assert got.shape == (n, hq, d)
    for i in range(n):
        for h in range(hkv):
            sel = torch.as_tensor(idx[i, h][idx[i, h] >= 0])
            kh = torch.as_tensor(k[:, h, :]).index_select(0, sel)
            vh = torch.as_tensor(v[:, h, :]).index_select(0, sel)
            qh = torch.as_tensor(q[i, h * G:(h + 1) * G])
            want = _sdpa(qh[:, None, :], kh[None], vh[None], 0.3)[:, 0, :].numpy()
            assert np.allclose(got[i, h * G:(h + 1) * G], want, rtol=1e-12, atol=1e-12), (i, h)


def _int_dot_bruteforce(x, P, G):
    """Projections from integer numerators with Python ints: x = X / 16 and
    P = Q / 4 give y = (X . Q) / 64 exactly."""
    X = np.rint(np.asarray(x) * 16).astype(np.int64)
    Q = np.rint(np.asarray(P) * 4).astype(np.int64)
    y = np.zeros(X.shape[:-1] + (Q.shape[1],))
    for idx in np.ndindex(*X.shape[:-1]):
        i = idx[-1]
        for j in range(Q.shape[1]):
            y[idx + (j,)] = sum(int(a) * int(b) for a, b in zip(X[idx], Q[i // G, j])) / 64
    return y


def check_project_casts(o):
    """The cached projection rows are the exact dot products rounded once:
    on inputs whose exact projections are fp32 values (multiples of 1/64
    below 2^10), torch's fp32 -> float8_e4m3fn and -> bfloat16 casts are the
    reference for project_e4m3 and project_bf16 (JSSA, Fig. 10: the
    projected-key cache held in FP8); plus hand-derived E4M3 ties (17 -> 16,
    19 -> 20) and saturation (+-1000 -> +-448) through a unit basis."""
    rng = np.random.default_rng(29)
    nb, G, d, r = 2, 2, 16, 8
    x = rng.integers(-40, 41, size=(5, nb * G, d)) / 16.0
    P = rng.integers(-3, 4, size=(nb, r, d)) / 4.0
    exact = _int_dot_bruteforce(x, P, G)
    assert np.abs(exact).max() < 448
    e32 = torch.from_numpy(exact.astype(np.float32))
    assert np.array_equal(e32.double().numpy(), exact)                # exact in fp32
    want8 = e32.to(torch.float8_e4m3fn).double().numpy()
    want16 = e32.to(torch.bfloat16).double().numpy()
    assert (want8 != exact).sum() > 20 and (want16 != exact).sum() > 5   # rounding is exercised
    assert np.array_equal(o.project_e4m3(x, P, G), want8)
    assert np.array_equal(o.project_bf16(x, P, G), want16)
    unit = np.zeros((1, 2, 4))
    unit[0, 0, 0] = unit[0, 1, 3] = 1.0
    xs = np.array([[[17.0, 0, 0, 19.0]], [[1000.0, 0, 0, -1000.0]], [[-17.0, 5, 5, 0.4375]]])
    got = o.project_e4m3(xs, unit, 1)
    assert np.array_equal(got[:, 0, :], [[16.0, 20.0], [448.0, -448.0], [-16.0, 0.4375]]), got


def check_decode_step_bruteforce(o):
    """A whole decode step against brute force: integer group scores with
    Python ints, selection by lexicographic sort (score desc, position asc),
    the set ascending, and SDPA (fp64) over the gathered rows; in the
    coarse-to-fine mode, blocks by (block score desc, block index asc) first."""
    rng = np.random.default_rng(30)
    cases = [(8, 2, 60, 4, 16, 9, 0, 0), (4, 1, 33, 3, 8, 33, 0, 0), (6, 3, 20, 2, 8, 40, 0, 0),
             (8, 2, 64, 3, 8, 10, 8, 3), (4, 1, 45, 2, 8, 12, 8, 2)]
    for hq, hkv, T, r, d, B, blk, keep in cases:
        G = hq // hkv
        qt = rng.integers(-2, 3, size=(hq, r)).astype(np.float64)
        kt = rng.integers(-2, 3, size=(T, hkv, r)).astype(np.float64)
        q = rng.standard_normal((hq, d))
        k = rng.standard_normal((T, hkv, d))
        v = rng.standard_normal((T, hkv, d))
        scale = 1.0 / math.sqrt(d)
        idx, out = o.decode_step(q, qt, k, v, kt, B, scale, blk=blk, keep=keep)
        assert idx.shape == (hkv, B) and out.shape == (hq, d)
        for h in range(hkv):
            s = np.array([sum(int(qt[i, j]) * int(kt[t, h, j]) for i in range(h * G, (h + 1) * G)
                              for j in range(r)) for t in range(T)])
            cand = np.arange(T)
            if blk:
                nblk = -(-T // blk)
                bs = np.array([s[j * blk:(j + 1) * blk].sum() for j in range(nblk)])
                blocks = np.lexsort((np.arange(nblk), -bs))[:keep]
                cand = np.concatenate([np.arange(j * blk, min(T, (j + 1) * blk)) for j in blocks])
            order = np.lexsort((cand, -s[cand]))[:B]
            want = np.full(B, -1)
            want[:len(order)] = np.sort(cand[order])
            assert np.array_equal(idx[h], want), (hq, hkv, T, blk, h)
            sel = torch.as_tensor(want[want >= 0])
            kh = torch.as_tensor(k[:, h, :]).index_select(0, sel)
            vh = torch.as_tensor(v[:, h, :]).index_select(0, sel)
            ref = _sdpa(torch.as_tensor(q[h * G:(h + 1) * G])[:, None, :], kh[None], vh[None], scale)
            assert np.allclose(out[h * G:(h + 1) * G], ref[:, 0, :].numpy(), rtol=1e-12, atol=1e-12)


CHECKS = [
    check_select_bruteforce, check_select_special, check_scores_bruteforce, check_scores_onehot,
    check_attention_full_budget_sdpa, check_attention_subset_sdpa, check_attention_closed_forms,
    check_attention_unselected_irrelevant, check_centroids_closed_form, check_hier_reductions,
    check_prefill_vs_decode_prefix, check_golden,
    check_round_bf16, check_round_e4m3, check_project_shifted_unit_basis, check_project_orthonormal,
    check_project_integer_exact, check_update_centroids, check_paged_attention,
    check_prefill_attention_rows, check_project_casts, check_decode_step_bruteforce,
]


@pytest.mark.parametrize("check", CHECKS, ids=[c.__name__ for c in CHECKS])
def test_oracle_pin(check):
    check(O)


def test_decode_step_composes():
    """decode_step == group mean -> scores -> top-B -> indexed attention."""
    rng = np.random.default_rng(16)
    T, hkv, hq, r, d, B = 100, 2, 8, 8, 16, 9
    q = rng.standard_normal((hq, d))
    qt = rng.integers(-8, 9, size=(hq, r)).astype(np.float64)
    k = rng.standard_normal((T, hkv, d))
    v = rng.standard_normal((T, hkv, d))
    kt = rng.integers(-8, 9, size=(T, hkv, r)).astype(np.float64)
    idx, out = O.decode_step(q, qt, k, v, kt, B, 0.25)
    s = O.candidate_scores(O.group_mean_query(qt, hkv), kt)
    idx2 = np.stack([O.select_top_b(s[h], B) for h in range(hkv)])
    assert np.array_equal(idx, idx2)
    assert np.array_equal(out, O.indexed_attention(q, k, v, idx2, 0.25))


# ------------------------------------------------------------------ planted mistakes

def _mutant(**overrides):
    ns = types.SimpleNamespace(**{name: getattr(O, name) for name in O.__all__})
    for k, fn in overrides.items():
        setattr(ns, k, fn)
    # functions that call helpers must see the mutated helpers: rebind via closures
    return ns


def _gm_wrong_group(qt, hkv):            # query head i -> KV head i % hkv
    qt = np.asarray(qt, dtype=np.float64)
    hq, r = qt.shape
    return np.stack([qt[h::hkv].mean(0) for h in range(hkv)])


def _gm_sum(qt, hkv):                    # dropped the 1/G of the mean
    return O.group_mean_query(qt, hkv) * (np.asarray(qt).shape[0] // hkv)


def _sel_upper_ties(s, B):               # ties go to the higher position
    s = np.asarray(s, dtype=np.float64)
    pos = np.nonzero(~np.isnan(s))[0]
    out = np.full(B, -1)
    if len(pos) <= B:
        out[: len(pos)] = pos
        return out
    vals = s[pos]
    th = np.partition(vals, len(vals) - B)[len(vals) - B]
    above, ties = pos[vals > th], pos[vals == th]
    out[:] = np.sort(np.concatenate([above, ties[len(ties) - (B - len(above)):]]))
    return out


def _sel_strict(s, B):                   # forgot the tie fill
    s = np.asarray(s, dtype=np.float64)
    pos = np.nonzero(~np.isnan(s))[0]
    out = np.full(B, -1)
    if len(pos) <= B:
        out[: len(pos)] = pos
        return out
    vals = s[pos]
    th = np.partition(vals, len(vals) - B)[len(vals) - B]
    keep = np.sort(pos[vals > th])
    out[: len(keep)] = keep
    return out


def _attn_scale_d(q, k, v, idx, scale):  # 1/d instead of 1/sqrt(d)
    return O.indexed_attention(q, k, v, idx, scale * scale)


def _attn_wrong_head(q, k, v, idx, scale):   # query head i reads KV head i % hkv
    q = np.asarray(q, dtype=np.float64)
    hq, d = q.shape
    hkv = k.shape[1]
    out = np.zeros((hq, d))
    for i in range(hq):
        h = i % hkv
        sel = np.asarray(idx[h]); sel = sel[sel >= 0]
        if len(sel):
            out[i] = O.attention_weights(q[i], k[sel, h], scale) @ np.asarray(v[sel, h], dtype=np.float64)
    return out


def _attn_no_norm(q, k, v, idx, scale):  # softmax without the denominator
    q = np.asarray(q, dtype=np.float64)
    hq, d = q.shape
    hkv = k.shape[1]
    G = hq // hkv
    out = np.zeros((hq, d))
    for i in range(hq):
        h = i // G
        sel = np.asarray(idx[h]); sel = sel[sel >= 0]
        if len(sel):
            lg = scale * (np.asarray(k[sel, h], dtype=np.float64) @ q[i])
            out[i] = np.exp(lg - lg.max()) @ np.asarray(v[sel, h], dtype=np.float64)
    return out


def _cent_drop_last(kt, blk):            # each block misses its last token
    T, hkv, r = kt.shape
    nblk = -(-T // blk)
    return np.stack([np.asarray(kt[j * blk: min(T, (j + 1) * blk) - 1], dtype=np.float64).sum(0)
                     for j in range(nblk)])


def _scores_transposed(q_bar, kt):       # reads kt as [hkv, T, r] (wrong layout)
    T, hkv, r = kt.shape
    kk = np.asarray(kt, dtype=np.float64).reshape(hkv, T, r)
    return np.stack([kk[h] @ np.asarray(q_bar, dtype=np.float64)[h] for h in range(hkv)])


def _prefill_off_by_one(qt_rows, positions, kt, B):   # query does not see its own key
    return O.prefill_index(qt_rows, np.asarray(positions) - 1, kt, B)


def _hier_wrapped(select=None, centroids=None):
    def hs(q_bar, kt, blk, keep, B):
        q_bar = np.asarray(q_bar, dtype=np.float64)
        T, hkv, r = kt.shape
        cent = (centroids or O.block_centroids)(kt, blk)
        sel = select or O.select_top_b
        idx = np.full((hkv, B), -1)
        for h in range(hkv):
            blocks = sel(cent[:, h, :] @ q_bar[h], keep)
            blocks = blocks[blocks >= 0]
            cand = np.concatenate([np.arange(j * blk, min(T, (j + 1) * blk)) for j in blocks])
            pick = sel(np.asarray(kt[cand, h, :], dtype=np.float64) @ q_bar[h], B)
            idx[h] = np.where(pick >= 0, cand[np.maximum(pick, 0)], -1)
        return idx
    return hs


def _hier_block_upper_ties(q_bar, kt, blk, keep, B):
    return _hier_wrapped(select=lambda s, n: _sel_upper_ties(s, n) if n == keep else O.select_top_b(s, n))(
        q_bar, kt, blk, keep, B)


def _bf16_truncate(x):                    # rounds toward zero
    x = np.asarray(x, dtype=np.float64)
    m, e = np.frexp(np.abs(x))
    ulp = np.ldexp(1.0, np.maximum(e - 1, -126) - 7)
    return np.sign(x) * np.floor(np.abs(x) / ulp) * ulp


def _bf16_ties_away(x):                   # ties away from zero instead of to even
    x = np.asarray(x, dtype=np.float64)
    m, e = np.frexp(np.abs(x))
    ulp = np.ldexp(1.0, np.maximum(e - 1, -126) - 7)
    return np.sign(x) * np.floor(np.abs(x) / ulp + 0.5) * ulp


def _e4m3_no_saturation(x):               # forgot the clamp to +-448
    x = np.asarray(x, dtype=np.float64)
    m, e = np.frexp(np.abs(x))
    ulp = np.ldexp(1.0, np.maximum(e - 1, -6) - 3)
    return np.sign(x) * np.rint(np.abs(x) / ulp) * ulp


def _proj_i_mod_nb(x, P, G):              # head i uses basis i % nbases
    x = np.asarray(x, dtype=np.float64)
    P = np.asarray(P, dtype=np.float64)
    H = x.shape[-2]
    return np.stack([x[..., i, :] @ P[i % P.shape[0]].T for i in range(H)], axis=-2)


def _proj_transposed(x, P, G):            # basis used as columns (P^T) instead of rows
    x = np.asarray(x, dtype=np.float64)
    P = np.asarray(P, dtype=np.float64)
    H = x.shape[-2]
    return np.stack([x[..., i, :] @ P[i // G] for i in range(H)], axis=-2)


def _cent_round_once(c, kt, t0, n, blk):  # sums exactly, rounds once per block
    c = np.asarray(c, dtype=np.float64).copy()
    acc = c.copy()
    for t in range(t0, t0 + n):
        acc[t // blk] += np.asarray(kt[t], dtype=np.float64)
    return O.round_to_bf16(acc)


def _cent_wrong_block(c, kt, t0, n, blk):  # token t lands in block (t + 1) // blk
    c = np.asarray(c, dtype=np.float64).copy()
    for t in range(t0, t0 + n):
        j = min((t + 1) // blk, c.shape[0] - 1)
        c[j] = O.round_to_bf16(c[j] + np.asarray(kt[t], dtype=np.float64))
    return c


def _paged_inverse(q, k_pool, v_pool, slots, idx, scale):   # reads the table backwards (slot -> position)
    slots = np.asarray(slots)
    inv = np.argsort(np.where(slots >= 0, slots, np.iinfo(np.int64).max))[: len(slots)]
    return O.indexed_attention(q, O.paged_rows(k_pool, inv), O.paged_rows(v_pool, inv), idx, scale)


def _prefill_attn_row0(q_rows, k, v, idx, scale):   # every row uses row 0's index sets
    return O.prefill_attention(q_rows, k, v, np.broadcast_to(np.asarray(idx)[:1], np.shape(idx)), scale)


def _prefill_attn_shifted(q_rows, k, v, idx, scale):   # row n uses row n-1's index sets
    idx = np.asarray(idx)
    return O.prefill_attention(q_rows, k, v, np.concatenate([idx[:1], idx[:-1]]), scale)


def _e4m3_proj_as_bf16(x, P, G):           # the FP8 cache rounded to bf16 instead
    return O.round_to_bf16(O.project_rows(x, P, G))


def _e4m3_proj_truncates(x, P, G):         # E4M3 rounding toward zero
    y = O.project_rows(x, P, G)
    m, e = np.frexp(np.abs(y))
    ulp = np.ldexp(1.0, np.maximum(e - 1, -6) - 3)
    return np.clip(np.sign(y) * np.floor(np.abs(y) / ulp) * ulp, -448, 448)


def _step_unsorted(q, qt, k, v, kt, B, scale, blk=0, keep=0):   # the set left in score order
    idx, out = O.decode_step(q, qt, k, v, kt, B, scale, blk=blk, keep=keep)
    s = O.candidate_scores(O.group_mean_query(qt, kt.shape[1]), kt)
    idx = idx.copy()
    for h in range(idx.shape[0]):
        sel = idx[h][idx[h] >= 0]
        idx[h, :len(sel)] = sel[np.argsort(-s[h, sel], kind="stable")]
    return idx, out


def _step_ignores_hierarchy(q, qt, k, v, kt, B, scale, blk=0, keep=0):   # always flat
    return O.decode_step(q, qt, k, v, kt, B, scale)


def _step_other_group_query(q, qt, k, v, kt, B, scale, blk=0, keep=0):   # attention with head i's query shifted by one
    idx, _ = O.decode_step(q, qt, k, v, kt, B, scale, blk=blk, keep=keep)
    return idx, O.indexed_attention(np.roll(np.asarray(q), 1, axis=0), k, v, idx, scale)


MUTANTS = {
    "prefill_rows_use_row0_idx": dict(prefill_attention=_prefill_attn_row0),
    "prefill_rows_shifted_idx": dict(prefill_attention=_prefill_attn_shifted),
    "project_e4m3_rounds_to_bf16": dict(project_e4m3=_e4m3_proj_as_bf16),
    "project_e4m3_truncates": dict(project_e4m3=_e4m3_proj_truncates),
    "decode_step_set_unsorted": dict(decode_step=_step_unsorted),
    "decode_step_ignores_hierarchy": dict(decode_step=_step_ignores_hierarchy),
    "decode_step_rolled_queries": dict(decode_step=_step_other_group_query),
    "paged_table_inverted": dict(indexed_attention_paged=_paged_inverse),
    "bf16_truncates": dict(round_to_bf16=_bf16_truncate),
    "bf16_ties_away": dict(round_to_bf16=_bf16_ties_away),
    "e4m3_not_saturated": dict(round_to_e4m3=_e4m3_no_saturation),
    "projection_basis_i_mod_nbases": dict(project_rows=_proj_i_mod_nb),
    "projection_basis_transposed": dict(project_rows=_proj_transposed),
    "centroid_update_rounds_once": dict(update_centroids=_cent_round_once),
    "centroid_update_wrong_block": dict(update_centroids=_cent_wrong_block),
    "group_i_mod_hkv": dict(group_mean_query=_gm_wrong_group),
    "group_sum_not_mean": dict(group_mean_query=_gm_sum),
    "ties_to_higher_position": dict(select_top_b=_sel_upper_ties),
    "ties_dropped": dict(select_top_b=_sel_strict),
    "scale_1_over_d": dict(indexed_attention=_attn_scale_d),
    "attn_head_i_mod_hkv": dict(indexed_attention=_attn_wrong_head),
    "softmax_unnormalised": dict(indexed_attention=_attn_no_norm),
    "centroid_drops_last_token": dict(block_centroids=_cent_drop_last,
                                      hierarchical_select=_hier_wrapped(centroids=_cent_drop_last)),
    "scores_wrong_layout": dict(candidate_scores=_scores_transposed),
    "prefill_excludes_own_key": dict(prefill_index=_prefill_off_by_one),
    "block_ties_to_higher_index": dict(hierarchical_select=_hier_block_upper_ties),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_mistakes_are_caught(name):
    o = _mutant(**MUTANTS[name])
    failed = []
    for check in CHECKS:
        try:
            check(o)
        except AssertionError:
            failed.append(check.__name__)
        except Exception as e:  # a crash also counts as caught
            failed.append(f"{check.__name__}:{type(e).__name__}")
    assert failed, f"planted mistake {name!r} passed every pin"
