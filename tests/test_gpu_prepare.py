"""GPU parity of scoring preparation (JSSA, Fig. 9 and Fig. 1): lsa_project /
lsa_project_fp8 (tcgen05 projection onto per-KV-head bases) and
lsa_update_centroids against the CPU oracle.

Integer-valued inputs make every fp32 projection exact, so both sides round
the same exact value once: bf16 and E4M3 outputs must be bit-identical. For
real-valued inputs the fp32 sum may differ from the exact one, so each output
must be the oracle's rounding or a neighbouring value (one unit in the last
place). Rows outside [t0, t0 + n) must keep what they held."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import indexed_sparse_attention_kv_b200 as lsa
import oracle.lsa_oracle as O
from indexed_sparse_attention_kv_b200 import inputs as I

from _util import assert_out_close, np32

pytestmark = pytest.mark.gpu

SENTINEL = -12288.0   # -3 * 2^12, exact in bf16

CASES = [
    # batch, T, H, d, r, nbases, t0, n
    (2, 1000, 8, 128, 64, 8, 37, 700),     # ragged range inside each sequence
    (1, 300, 4, 64, 32, 4, 0, 300),        # whole sequences: one flattened range
    (2, 129, 2, 32, 16, 1, 0, 129),        # d 32 (64-byte swizzle), one basis per layer
    (1, 200, 2, 16, 16, 2, 5, 150),        # d 16 (32-byte swizzle)
    (1, 500, 2, 96, 48, 2, 100, 400),      # d 96: a partial 64-element atom
    (1, 260, 2, 256, 64, 2, 0, 260),       # largest d
    (2, 257, 2, 128, 128, 2, 1, 256),      # largest r
    (3, 5, 8, 128, 64, 8, 4, 1),           # decode append: one row per sequence
]


def _run(case, fp8=False, x_range=3, p_range=2, seed=61):
    batch, T, H, d, r, nb, t0, n = case
    x = I.make_projection_inputs(seed, batch, T, H, d, r, nb, x_range, p_range)
    dt = torch.float8_e4m3fn if fp8 else torch.bfloat16
    y0 = torch.full((batch, T, H, r), SENTINEL if not fp8 else -448.0, dtype=torch.float32).to(dt).cuda()
    fn = lsa.lsa_project_fp8 if fp8 else lsa.lsa_project
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    y = fn(x["x"].cuda(), x["P"].cuda(), t0, n, y=y0, dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    got = y.float().double().cpu().numpy()
    rnd = O.project_e4m3 if fp8 else O.project_bf16
    want = rnd(np32(x["x"][:, t0:t0 + n]), np32(x["P"]), H // nb)
    fill = -448.0 if fp8 else SENTINEL
    outside = np.ones(T, dtype=bool)
    outside[t0:t0 + n] = False
    assert np.all(got[:, outside] == fill), "rows outside [t0, t0+n) were written"
    return got[:, t0:t0 + n], want, x


@pytest.mark.parametrize("case", CASES, ids=[str(c) for c in CASES])
def test_project_integer_bit_exact(case):
    got, want, _ = _run(case)
    assert np.array_equal(got, want), np.argwhere(got != want)[:5]


@pytest.mark.parametrize("case", CASES[:4] + CASES[6:7], ids=[str(c) for c in CASES[:4] + CASES[6:7]])
def test_project_fp8_bit_exact(case):
    # x in [-3, 3], P in [-2, 2]: E4M3 keeps 3 mantissa bits, so most
    # projections round
    got, want, _ = _run(case, fp8=True)
    assert np.array_equal(got, want), np.argwhere(got != want)[:5]


def test_project_fp8_saturates():
    # x, P in [-8, 8]: projections with a standard deviation near 270, so
    # many pass 448 and saturate
    got, want, _ = _run(CASES[0], fp8=True, x_range=8, p_range=8, seed=70)
    assert np.array_equal(got, want), np.argwhere(got != want)[:5]
    assert (np.abs(want) == 448.0).mean() > 0.05


def _within_bound(got, want, absdot, d):
    """|got - want| <= one bf16 ulp of the oracle's value + the fp32 summation
    error bound 2 d 2^-24 sum_e |P_e x_e| (any order of d - 1 fp32 adds; the
    factor 2 leaves room for the tensor core's internal accumulation)."""
    a = np.abs(want)
    e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    ulp = np.ldexp(1.0, (np.maximum(e, -126) - 7).astype(np.int64))
    return np.abs(got - want) <= ulp + 2.0 * d * 2.0 ** -24 * absdot


@pytest.mark.parametrize("case", [CASES[0], CASES[4], CASES[6]], ids=[str(c) for c in (CASES[0], CASES[4], CASES[6])])
def test_project_real_valued_within_fp32_bound(case):
    got, want, x = _run(case, x_range=None, p_range=None, seed=62)
    batch, T, H, d, r, nb, t0, n = case
    absdot = O.project_rows(np.abs(np32(x["x"][:, t0:t0 + n])), np.abs(np32(x["P"])), H // nb)
    ok = _within_bound(got, want, absdot, d)
    assert ok.all(), np.argwhere(~ok)[:5]
    assert (got == want).mean() > 0.98


def test_project_queries_share_group_basis():
    """Queries [batch, 1, hq, d] with nbases = hkv: query head i uses basis i // G."""
    batch, hq, hkv, d, r = 4, 32, 8, 128, 64
    x = I.make_projection_inputs(63, batch, 1, hq, d, r, hkv)
    qt = lsa.lsa_project(x["x"].cuda(), x["P"].cuda())
    torch.cuda.synchronize()
    want = O.project_bf16(np32(x["x"]), np32(x["P"]), hq // hkv)
    assert np.array_equal(qt.to(torch.float64).cpu().numpy(), want)


def test_update_centroids_bit_exact():
    """Integer kt and centroids above 256 in magnitude: every add rounds."""
    batch, T, hkv, r, blk, t0, n = 2, 1000, 8, 64, 64, 50, 300
    gen = torch.Generator().manual_seed(64)
    kt = torch.randint(-3, 4, (batch, T, hkv, r), generator=gen).to(torch.bfloat16)
    nblk = (T + blk - 1) // blk
    c0 = torch.randint(-600, 601, (batch, nblk, hkv, r), generator=gen).to(torch.bfloat16)
    c = c0.cuda()
    lsa.lsa_update_centroids(kt.cuda(), c, blk, t0, n)
    torch.cuda.synchronize()
    got = c.to(torch.float64).cpu().numpy()
    for b in range(batch):
        want = O.update_centroids(np32(c0[b]), np32(kt[b]), t0, n, blk)
        assert np.array_equal(got[b], want), b


def test_append_rebuilds_centroids():
    """Appending every token one at a time from zero centroids gives
    lsa_block_centroids' result when the sums are exact."""
    batch, T, hkv, r, blk = 1, 200, 2, 32, 16
    gen = torch.Generator().manual_seed(65)
    kt = torch.randint(-2, 3, (batch, T, hkv, r), generator=gen).to(torch.bfloat16).cuda()
    c = torch.zeros((batch, (T + blk - 1) // blk, hkv, r), dtype=torch.bfloat16, device="cuda")
    for t in range(0, T, 7):
        lsa.lsa_update_centroids(kt, c, blk, t, min(7, T - t))
    ref = lsa.lsa_block_centroids(kt, blk)
    torch.cuda.synchronize()
    assert torch.equal(c, ref)


def test_prepared_inputs_drive_the_decode_step():
    """k and q projected by lsa_project feed lsa_decode_step; the result equals
    the oracle's decode step on the oracle's projections (integer inputs)."""
    batch, hq, hkv, d, r, T, B = 2, 32, 8, 128, 64, 3000, 256
    gen = torch.Generator().manual_seed(66)
    xk = I.make_projection_inputs(67, batch, T, hkv, d, r, hkv, 2, 1)
    q = torch.randint(-2, 3, (batch, hq, d), generator=gen).to(torch.bfloat16)
    v = torch.randn((batch, T, hkv, d), generator=gen).to(torch.bfloat16)
    k, P = xk["x"], xk["P"]
    kt = lsa.lsa_project(k.cuda(), P.cuda())
    qt = lsa.lsa_project(q.view(batch, 1, hq, d).cuda(), P.cuda()).view(batch, hq, r)
    kd, vd, qd = k.cuda(), v.cuda(), q.cuda()
    scale = 1.0 / np.sqrt(d)
    idx, out = lsa.lsa_decode_step(qd, qt, kd, vd, kt, B, scale=scale)
    torch.cuda.synchronize()
    for b in range(batch):
        kt_o = O.project_bf16(np32(k[b]), np32(P), 1)
        qt_o = O.project_bf16(np32(q[b]), np32(P), hq // hkv)
        ref_idx, ref_out = O.decode_step(np32(q[b]), qt_o, np32(k[b]), np32(v[b]), kt_o, B, scale)
        assert np.array_equal(idx[b].cpu().numpy(), ref_idx), b
        assert_out_close(out[b], ref_out)


@pytest.mark.slow
def test_project_128k_sampled_rows():
    """The 128K key cache of the decode workload (batch 4, 8 KV heads, d 128,
    r 64), projected in one call; 4096 sampled rows checked one by one."""
    batch, T, H, d, r = 4, 131072, 8, 128, 64
    g = torch.Generator(device="cuda").manual_seed(68)
    x = torch.randint(-3, 4, (batch, T, H, d), generator=g, device="cuda", dtype=torch.int32).to(torch.bfloat16)
    P = torch.randint(-2, 3, (H, r, d), generator=g, device="cuda", dtype=torch.int32).to(torch.bfloat16)
    y = lsa.lsa_project(x, P)
    torch.cuda.synchronize()
    rs = np.random.default_rng(69)
    bs, ts = rs.integers(0, batch, 4096), rs.integers(0, T, 4096)
    ts[:8] = [0, 1, 127, 128, T - 129, T - 128, T - 2, T - 1]
    xs = x[torch.as_tensor(bs), torch.as_tensor(ts)].cpu()       # [4096, H, d]
    got = y[torch.as_tensor(bs), torch.as_tensor(ts)].to(torch.float64).cpu().numpy()
    want = O.project_bf16(np32(xs), np32(P.cpu()), 1)
    assert np.array_equal(got, want)
