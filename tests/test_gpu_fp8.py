"""GPU parity of the FP8 (E4M3) projected-key cache path (JSSA, Fig. 10):
lsa_score_fp8 and lsa_decode_step_fp8 against the bf16 path on the same values
and against the CPU oracle. The integer scoring inputs convert to E4M3 exactly,
so scores must be identical to the bf16 path's and index sets bit-exact."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import indexed_sparse_attention_kv_b200 as lsa
from indexed_sparse_attention_kv_b200 import inputs as I

from _util import assert_out_close, oracle_decode, to_dev

pytestmark = pytest.mark.gpu

CASES = [
    # batch, hq, hkv, d, r, T, B
    (1, 16, 4, 128, 64, 4096, 256),
    (2, 32, 8, 128, 64, 3001, 300),
    (1, 64, 16, 64, 64, 1500, 100),
    (2, 8, 8, 128, 64, 777, 800),
    (1, 32, 32, 128, 64, 1000, 64),
]


def _case(case, seed=31, heavy=0.05):
    batch, hq, hkv, d, r, T, B = case
    w = I.Workload(f"fp8_{case}", seed, batch=batch, hq=hq, hkv=hkv, d=d, T=T, r=r, B=B, heavy_frac=heavy)
    return w, I.make_decode_inputs(w)


@pytest.mark.parametrize("case", CASES, ids=[str(c) for c in CASES])
def test_fp8_matches_bf16_and_oracle(case):
    w, x = _case(case)
    kt8 = x["kt"].to(torch.float8_e4m3fn)
    assert torch.equal(kt8.to(torch.bfloat16), x["kt"]), "inputs not exact in E4M3"
    d = to_dev(x)
    kt8 = kt8.cuda()
    s16 = lsa.lsa_score(d["qt"], d["kt"])
    s8 = lsa.lsa_score_fp8(d["qt"], kt8)
    assert torch.equal(s8, s16)
    idx8, out8 = lsa.lsa_decode_step_fp8(d["q"], d["qt"], d["k"], d["v"], kt8, w.B)
    idx16, out16 = lsa.lsa_decode_step(d["q"], d["qt"], d["k"], d["v"], d["kt"], w.B)
    torch.cuda.synchronize()
    assert torch.equal(idx8, idx16)
    assert torch.equal(out8, out16)
    ref_idx, ref_out = oracle_decode(x, w)
    assert np.array_equal(idx8.cpu().numpy(), ref_idx)
    assert_out_close(out8, ref_out)


def test_fp8_workspace_reuse_and_repeat():
    w, x = _case((2, 32, 8, 128, 64, 5000, 512), seed=32)
    d = to_dev(x)
    kt8 = x["kt"].to(torch.float8_e4m3fn).cuda()
    dims = lsa.lsa_dims(w.batch, w.hq, w.hkv, w.d, w.r, w.T)
    ws = lsa.workspace(dims, w.B)
    a = lsa.lsa_decode_step_fp8(d["q"], d["qt"], d["k"], d["v"], kt8, w.B, ws=ws)
    b = lsa.lsa_decode_step_fp8(d["q"], d["qt"], d["k"], d["v"], kt8, w.B, ws=ws)
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])
    assert lsa.lsa_read_device_status(ws) == 0


@pytest.mark.slow
def test_fp8_decode_128k_full_size():
    from _util import decode_inputs

    w, x = decode_inputs("decode_128k")
    kt8 = x["kt"].to(torch.float8_e4m3fn)
    assert torch.equal(kt8.to(torch.bfloat16), x["kt"])
    d = to_dev(x)
    kt8 = kt8.cuda()
    idx8, out8 = lsa.lsa_decode_step_fp8(d["q"], d["qt"], d["k"], d["v"], kt8, w.B)
    idx16, out16 = lsa.lsa_decode_step(d["q"], d["qt"], d["k"], d["v"], d["kt"], w.B)
    torch.cuda.synchronize()
    assert torch.equal(idx8, idx16)
    assert torch.equal(out8, out16)


def test_fp8_nan_keys_are_never_selected():
    """E4M3 NaN keys (in any channel) give NaN scores, as in the bf16 path, and
    are never selected; every other score is identical."""
    w, x = _case((2, 32, 8, 128, 64, 3000, 400), seed=33)
    g = torch.Generator().manual_seed(34)
    n_nan = 300
    b = torch.randint(0, w.batch, (n_nan,), generator=g)
    t = torch.randint(0, w.T, (n_nan,), generator=g)
    h = torch.randint(0, w.hkv, (n_nan,), generator=g)
    c = torch.randint(0, w.r, (n_nan,), generator=g)
    x["kt"][b, t, h, c] = float("nan")
    d = to_dev(x)
    kt8 = x["kt"].to(torch.float8_e4m3fn).cuda()
    s16 = lsa.lsa_score(d["qt"], d["kt"])
    s8 = lsa.lsa_score_fp8(d["qt"], kt8)
    torch.cuda.synchronize()
    assert torch.equal(torch.isnan(s8), torch.isnan(s16))
    assert int(torch.isnan(s8).sum()) > 0
    ok = ~torch.isnan(s16)
    assert torch.equal(s8[ok], s16[ok])
    idx8, out8 = lsa.lsa_decode_step_fp8(d["q"], d["qt"], d["k"], d["v"], kt8, w.B)
    idx16, out16 = lsa.lsa_decode_step(d["q"], d["qt"], d["k"], d["v"], d["kt"], w.B)
    torch.cuda.synchronize()
    assert torch.equal(idx8, idx16) and torch.equal(out8, out16)
    ref_idx, ref_out = oracle_decode(x, w)
    assert np.array_equal(idx8.cpu().numpy(), ref_idx)
