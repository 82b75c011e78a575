"""CPU oracle for indexed sparse attention over a GQA KV cache (fp64, NumPy).

TEST INFRASTRUCTURE. This module is the plain, slow, obviously-correct
definition of what the CUDA path computes. Only the test suite, the smoke
check in ``__graft_entry__`` and the benchmark's CPU-baseline leg may import
it. It shares no code with the CUDA path and imports nothing from it.

Sources (page title, then the passage):
  * Joint Subspace Sparse Attention for Efficient Long-Context Decoding
    (JSSA), Fig. 1: per KV head, the mean of the head's query group scores a
    projected-key cache in a shared low-dimensional subspace; the top-B token
    positions are selected; the group's query heads share that index set and
    attend over it.  Key contributions: the attention reads the selected rows
    in place from the standard GQA KV-cache layout (no gather copy).
  * LongCat Sparse Attention: Taming the Lightning via Streaming-aware
    Hierarchical Cross-Layer Indexing, Abstract, strategy (3) Hierarchical
    Indexing: coarse-to-fine scoring narrows the candidate set; and the
    Lightning-Indexer prefill whose dense scoring is O(L^2).
  * Latent Sparse Attention: Towards Subquadratic Ultra-Long Context
    Attention, summary: queries score clusters instead of every key.

Readings where the pages are silent:
  * query head i belongs to KV head i // G (contiguous GQA groups);
  * the B-th largest score is the threshold; every position above it is kept,
    and ties at the threshold go to the lower position (lower block index in
    the coarse stage); the index set is returned in ascending order and padded
    with -1 when fewer than B candidates exist; NaN marks a non-candidate;
  * attention uses scale = 1/sqrt(d), a max-subtracted softmax over the
    selected positions, no RoPE/softcap/bias, and no forced sink/local tokens;
  * a block centroid is the sum of the projected keys of its (up to) ``blk``
    tokens, blocks starting at t = 0;
  * prefill query at absolute position p sees keys 0 .. p inclusive;
  * scoring preparation (JSSA, Fig. 9 and Fig. 1, "a shared low-dimensional
    subspace"): every KV head h has a basis P[h] of r vectors of length d; a
    key of head h and the queries of h's group are both projected onto it,
    y_j = <P[h, j], x> (one basis per layer is the case of equal P[h]). The
    projected cache holds bf16 (round to nearest even, from the exact value)
    or FP8 E4M3 (round to nearest even, saturated to +-448) values;
  * a centroid maintained incrementally adds each new projected key to its
    block in position order and rounds the sum to bf16 after every add.

All parity statements in the tests hold against these functions. Parity pins
(what fixes each function independently of itself) live in tests/test_oracle.py.
"""
from __future__ import annotations

import math

import numpy as np

__all__ = [
    "group_mean_query",
    "candidate_scores",
    "select_top_b",
    "block_centroids",
    "hierarchical_select",
    "attention_weights",
    "indexed_attention",
    "decode_step",
    "prefill_scores",
    "prefill_index",
    "prefill_attention",
    "paged_rows",
    "indexed_attention_paged",
    "round_to_bf16",
    "round_to_e4m3",
    "project_rows",
    "project_bf16",
    "project_e4m3",
    "update_centroids",
]


def _f64(x) -> np.ndarray:
    return np.asarray(x, dtype=np.float64)


def group_mean_query(qt, hkv: int) -> np.ndarray:
    """Scoring query of every KV head: the mean of its GQA query group.

    JSSA, Fig. 1 ("the mean of its associated query heads"). ``qt`` is
    [hq, r]; query head i belongs to KV head i // G with G = hq / hkv.
    Returns q_bar [hkv, r] in fp64.
    """
    qt = _f64(qt)
    hq, r = qt.shape
    assert hq % hkv == 0, "hq must be a multiple of hkv"
    G = hq // hkv
    q_bar = np.zeros((hkv, r), dtype=np.float64)
    for h in range(hkv):
        for g in range(G):
            q_bar[h] += qt[h * G + g]
        q_bar[h] /= G
    return q_bar


def candidate_scores(q_bar, kt) -> np.ndarray:
    """s[h, t] = q_bar[h] . kt[t, h] for every cached position t.

    JSSA, Fig. 1 (one dot product per cached position against the projected-key
    cache) and Fig. 2a (the channel budget r of the scoring subspace).
    ``q_bar`` is [hkv, r]; ``kt`` is [T, hkv, r]. Returns [hkv, T] fp64.
    """
    q_bar = _f64(q_bar)
    T, hkv, r = kt.shape
    s = np.empty((hkv, T), dtype=np.float64)
    for h in range(hkv):
        s[h] = _f64(kt[:, h, :]) @ q_bar[h]
    return s


def select_top_b(s, B: int) -> np.ndarray:
    """The top-B positions of one score vector, ascending, padded with -1.

    JSSA, Fig. 1 ("select the top-B token positions"). The threshold theta is
    the B-th largest score among the candidates (NaN = not a candidate). Every
    position with s > theta is taken, then positions with s == theta in
    ascending order until B are taken. Fewer than B candidates: all of them,
    then -1 padding. Returns int64 [B].
    """
    s = _f64(s)
    assert B >= 1
    pos = np.nonzero(~np.isnan(s))[0]
    vals = s[pos]
    out = np.full(B, -1, dtype=np.int64)
    if len(pos) <= B:
        out[: len(pos)] = pos
        return out
    theta = np.partition(vals, len(vals) - B)[len(vals) - B]
    above = pos[vals > theta]
    ties = pos[vals == theta]                 # ascending, since pos is ascending
    need = B - len(above)
    chosen = np.sort(np.concatenate([above, ties[:need]]))
    out[:] = chosen
    return out


def block_centroids(kt, blk: int) -> np.ndarray:
    """Coarse keys: c[j, h] = sum of kt[t, h] over the tokens t of block j.

    LongCat Sparse Attention, Abstract, strategy (3) Hierarchical Indexing, and
    Latent Sparse Attention, summary (queries score clusters of keys). Blocks
    are the contiguous token ranges [j*blk, (j+1)*blk) starting at 0; the last
    block may be partial. ``kt`` is [T, hkv, r]; returns [ceil(T/blk), hkv, r].
    """
    T, hkv, r = kt.shape
    nblk = (T + blk - 1) // blk
    c = np.zeros((nblk, hkv, r), dtype=np.float64)
    for j in range(nblk):
        c[j] = _f64(kt[j * blk: min(T, (j + 1) * blk)]).sum(axis=0)
    return c


def hierarchical_select(q_bar, kt, blk: int, keep: int, B: int) -> np.ndarray:
    """Coarse-to-fine top-B for every KV head: blocks first, then tokens.

    LongCat Sparse Attention, Abstract, strategy (3): score the block
    centroids with q_bar, keep the top ``keep`` blocks (ties to the lower block
    index), then score only the tokens of the kept blocks and select the top-B
    of those (ties to the lower position). Returns idx [hkv, B] (ascending,
    -1 padded).
    """
    q_bar = _f64(q_bar)
    T, hkv, r = kt.shape
    cent = block_centroids(kt, blk)
    idx = np.full((hkv, B), -1, dtype=np.int64)
    for h in range(hkv):
        coarse = cent[:, h, :] @ q_bar[h]
        blocks = select_top_b(coarse, keep)
        blocks = blocks[blocks >= 0]
        cand = np.concatenate([np.arange(j * blk, min(T, (j + 1) * blk)) for j in blocks]) \
            if len(blocks) else np.zeros(0, dtype=np.int64)
        fine = _f64(kt[cand, h, :]) @ q_bar[h]
        pick = select_top_b(fine, B)
        idx[h] = np.where(pick >= 0, cand[np.maximum(pick, 0)] if len(cand) else -1, -1)
    return idx


def attention_weights(q_i, k_rows, scale: float) -> np.ndarray:
    """Softmax over the selected keys of one query head (max-subtracted)."""
    logits = scale * (_f64(k_rows) @ _f64(q_i))
    m = logits.max()
    e = np.exp(logits - m)
    return e / e.sum()


def indexed_attention(q, k, v, idx, scale: float) -> np.ndarray:
    """o[i] = sum over t in S(h) of softmax_t(scale * q[i].k[t,h]) v[t,h], h = i // G.

    JSSA, Fig. 1 and Key contributions: every query head of KV head h attends
    over the index set S(h) of that head only, reading K/V rows in place from
    the [T, hkv, d] cache. ``q`` is [hq, d]; ``idx`` is [hkv, B] with -1
    padding (ignored). An empty set gives a zero output row. Returns [hq, d].
    """
    q = _f64(q)
    hq, d = q.shape
    T, hkv, _ = k.shape
    G = hq // hkv
    out = np.zeros((hq, d), dtype=np.float64)
    for i in range(hq):
        h = i // G
        sel = np.asarray(idx[h])
        sel = sel[sel >= 0]
        if len(sel) == 0:
            continue
        p = attention_weights(q[i], k[sel, h, :], scale)
        out[i] = p @ _f64(v[sel, h, :])
    return out


def decode_step(q, qt, k, v, kt, B: int, scale: float, blk: int = 0, keep: int = 0):
    """One decode step for one sequence: (idx [hkv, B], out [hq, d]).

    Flat mode (blk == 0): group-mean scoring of every cached position, then
    top-B. Hierarchical mode: ``hierarchical_select``. Then indexed attention.
    """
    T, hkv, r = kt.shape
    q_bar = group_mean_query(qt, hkv)
    if blk:
        idx = hierarchical_select(q_bar, kt, blk, keep, B)
    else:
        s = candidate_scores(q_bar, kt)
        idx = np.stack([select_top_b(s[h], B) for h in range(hkv)])
    out = indexed_attention(q, k, v, idx, scale)
    return idx, out


def prefill_scores(qt_rows, positions, kt) -> np.ndarray:
    """Dense causal indexer scores S[n, h, t] = q_bar[n, h] . kt[t, h], NaN for t > p_n.

    LongCat Sparse Attention, Abstract (the Lightning Indexer's dense
    O(L^2) scoring); JSSA, Fig. 1 for the group-mean query of each row.
    ``qt_rows`` is [n, hq, r]; ``positions`` the absolute positions p_n.
    """
    qt_rows = _f64(qt_rows)
    n, hq, r = qt_rows.shape
    T, hkv, _ = kt.shape
    S = np.empty((n, hkv, T), dtype=np.float64)
    t = np.arange(T)
    q_bars = [group_mean_query(qt_rows[i], hkv) for i in range(n)]
    for h in range(hkv):
        kh = _f64(kt[:, h, :])
        for i in range(n):
            row = kh @ q_bars[i][h]
            row[t > positions[i]] = np.nan
            S[i, h] = row
    return S


def prefill_index(qt_rows, positions, kt, B: int) -> np.ndarray:
    """Per-query causal top-B: idx [n, hkv, B] (ascending, -1 padded)."""
    S = prefill_scores(qt_rows, positions, kt)
    n, hkv, _ = S.shape
    idx = np.empty((n, hkv, B), dtype=np.int64)
    for i in range(n):
        for h in range(hkv):
            idx[i, h] = select_top_b(S[i, h], B)
    return idx


def prefill_attention(q_rows, k, v, idx, scale: float) -> np.ndarray:
    """Indexed attention for every prefill query row: out [n, hq, d]."""
    q_rows = _f64(q_rows)
    return np.stack([indexed_attention(q_rows[i], k, v, idx[i], scale) for i in range(q_rows.shape[0])])


def paged_rows(pool, slots) -> np.ndarray:
    """The logical [T, hkv, d] cache of one sequence held in a pool of slots
    (page size 1: "Their 42x decode speedup never compiled on my GPU", What
    their numbers claim): row t is pool[slots[t]]; a slot outside the pool
    (e.g. -1, an unfilled position) gives a NaN row, which a correct index set
    never selects."""
    pool = _f64(pool)
    slots = np.asarray(slots)
    out = np.full((len(slots),) + pool.shape[1:], np.nan)
    ok = (slots >= 0) & (slots < pool.shape[0])
    out[ok] = pool[slots[ok]]
    return out


def indexed_attention_paged(q, k_pool, v_pool, slots, idx, scale: float) -> np.ndarray:
    """indexed_attention over the K/V rows of a paged cache: the index sets
    hold logical positions, mapped through ``slots`` [T] to pool rows."""
    return indexed_attention(q, paged_rows(k_pool, slots), paged_rows(v_pool, slots), idx, scale)


def default_scale(d: int) -> float:
    return 1.0 / math.sqrt(d)


# ---------------------------------------------------------------- scoring preparation
def _round_to_grid(x, mant_bits: int, min_exp: int) -> np.ndarray:
    """Round fp64 values to a binary format with `mant_bits` stored mantissa
    bits and smallest normal exponent `min_exp`, ties to even; no overflow
    handling (the callers clamp). Works on the exact fp64 value: one rounding."""
    x = _f64(x)
    out = np.zeros_like(x)
    nz = (x != 0) & np.isfinite(x)
    m, e = np.frexp(np.abs(x[nz]))         # |x| = m * 2**e, m in [0.5, 1)
    e = np.maximum(e - 1, min_exp)         # exponent of the leading bit, or the subnormal floor
    ulp = np.ldexp(1.0, e - mant_bits)
    out[nz] = np.sign(x[nz]) * np.rint(np.abs(x[nz]) / ulp) * ulp   # np.rint: ties to even
    out[~np.isfinite(x)] = x[~np.isfinite(x)]
    return out


def round_to_bf16(x) -> np.ndarray:
    """Nearest bfloat16 value (8 exponent bits, 7 stored mantissa bits; ties
    to even), as fp64. Values past the largest finite bf16 by half an ulp or
    more become +-inf."""
    y = _round_to_grid(x, 7, -126)
    big = np.ldexp(2.0 - 2.0 ** -7, 127)
    y[np.isfinite(y) & (np.abs(y) > big)] = np.sign(y[np.isfinite(y) & (np.abs(y) > big)]) * np.inf
    return y


def round_to_e4m3(x) -> np.ndarray:
    """Nearest FP8 E4M3 value (4 exponent bits with bias 7, 3 stored mantissa
    bits, largest finite 448, no infinities; ties to even), saturated to
    +-448, as fp64."""
    y = _round_to_grid(x, 3, -6)
    return np.clip(y, -448.0, 448.0)


def project_rows(x, P, G: int) -> np.ndarray:
    """Exact projections y[..., i, j] = <P[i // G, j, :], x[..., i, :]> in fp64.

    JSSA, Fig. 1 (a projected-key cache in a subspace shared with the scoring
    query) and Fig. 9 (scoring preparation: the key projection). ``x`` is
    [..., H, d] (keys: H = hkv, G = 1; queries: H = hq, G = hq / hkv), ``P`` is
    [nbases, r, d] with H = nbases * G. Returns [..., H, r].
    """
    x = _f64(x)
    P = _f64(P)
    H, d = x.shape[-2:]
    nb, r, dp = P.shape
    assert dp == d and H == nb * G, "basis shape"
    y = np.zeros(x.shape[:-1] + (r,), dtype=np.float64)
    for i in range(H):
        y[..., i, :] = x[..., i, :] @ P[i // G].T
    return y


def project_bf16(x, P, G: int) -> np.ndarray:
    """The bf16 projected cache rows: round_to_bf16(project_rows(x, P, G))."""
    return round_to_bf16(project_rows(x, P, G))


def project_e4m3(x, P, G: int) -> np.ndarray:
    """The FP8 E4M3 projected cache rows (JSSA, Fig. 10: the projected-key
    cache held in FP8): round_to_e4m3(project_rows(x, P, G))."""
    return round_to_e4m3(project_rows(x, P, G))


def update_centroids(c, kt, t0: int, n: int, blk: int) -> np.ndarray:
    """Incremental block centroids: for t = t0 .. t0+n-1 in order,
    c[t // blk, h] <- round_to_bf16(c[t // blk, h] + kt[t, h]).

    LongCat Sparse Attention, Abstract, strategy (3) Hierarchical Indexing (the
    block-level keys of the coarse stage), kept current as tokens are appended
    (JSSA, Fig. 9, scoring preparation). ``c`` is [nblk, hkv, r] (bf16 values),
    ``kt`` is [T, hkv, r]. Returns the updated copy of ``c`` in fp64.
    """
    c = _f64(c).copy()
    kt = _f64(kt)
    for t in range(t0, t0 + n):
        j = t // blk
        c[j] = round_to_bf16(c[j] + kt[t])
    return c
