"""GPU parity of decode steps whose rows take the thread-block-cluster top-B
(more than 16K keys per row) at sizes between the small cases and 128K:
group sizes 1, 2, 4 and 8, slices of up to and past 1024 index entries per
CTA, B > T; index sets bit-exact against the oracle, outputs within the
attention tolerance of the oracle and equal to lsa_indexed_attn on the same
index sets; the FP8 and paged steps equal the bf16 step."""
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
    (2, 32, 8, 128, 64, 40000, 2048),   # G 4
    (1, 16, 8, 128, 64, 20000, 300),    # G 2
    (2, 8, 8, 128, 64, 30001, 1000),    # G 1, ragged T
    (1, 32, 8, 128, 64, 17000, 8192),   # B about half of T
    (1, 32, 8, 128, 64, 20000, 9000),
    (1, 64, 8, 128, 64, 20000, 512),    # G 8
]


def _case(case, seed=91, heavy=0.02):
    batch, hq, hkv, d, r, T, B = case
    w = I.Workload(f"cluster_{case}", seed, batch=batch, hq=hq, hkv=hkv, d=d, T=T, r=r, B=B, heavy_frac=heavy)
    return w, I.make_decode_inputs(w)


@pytest.mark.parametrize("case", CASES, ids=[str(c) for c in CASES])
def test_cluster_step_matches_oracle_and_attention_call(case):
    w, x = _case(case)
    d = to_dev(x)
    dims = lsa.lsa_dims(w.batch, w.hq, w.hkv, w.d, w.r, w.T)
    ws = lsa.workspace(dims, w.B)
    idx, out = lsa.lsa_decode_step(d["q"], d["qt"], d["k"], d["v"], d["kt"], w.B, ws=ws)
    sep = lsa.lsa_indexed_attn(d["q"], d["k"], d["v"], idx)
    torch.cuda.synchronize()
    assert lsa.lsa_read_device_status(ws) == 0
    ref_idx, ref_out = oracle_decode(x, w)
    assert np.array_equal(idx.cpu().numpy(), ref_idx)
    assert_out_close(out, ref_out)
    assert_out_close(sep, ref_out)
    assert torch.equal(out, sep)


def test_cluster_fp8_and_paged_equal_bf16_step():
    w, x = _case((2, 32, 8, 128, 64, 24000, 2048), seed=92)
    d = to_dev(x)
    idx0, out0 = lsa.lsa_decode_step(d["q"], d["qt"], d["k"], d["v"], d["kt"], w.B)
    kt8 = d["kt"].to(torch.float8_e4m3fn)
    idx1, out1 = lsa.lsa_decode_step_fp8(d["q"], d["qt"], d["k"], d["v"], kt8, w.B)
    n = w.batch * w.T
    perm = torch.randperm(n, generator=torch.Generator().manual_seed(93)).cuda()
    kp = torch.empty((n, w.hkv, w.d), dtype=torch.bfloat16, device="cuda")
    vp = torch.empty_like(kp)
    kp[perm] = d["k"].reshape(n, w.hkv, w.d)
    vp[perm] = d["v"].reshape(n, w.hkv, w.d)
    table = perm.to(torch.int32).view(w.batch, w.T)
    idx2, out2 = lsa.lsa_decode_step_paged(d["q"], d["qt"], kp, vp, table, d["kt"], w.B)
    torch.cuda.synchronize()
    assert torch.equal(idx1, idx0) and torch.equal(out1, out0)
    assert torch.equal(idx2, idx0) and torch.equal(out2, out0)


def test_cluster_padded_sets():
    """B > T: every position is selected and the sets are padded with -1."""
    w, x = _case((1, 32, 8, 128, 64, 16500, 20000), seed=94, heavy=0.0)
    d = to_dev(x)
    idx, out = lsa.lsa_decode_step(d["q"], d["qt"], d["k"], d["v"], d["kt"], w.B)
    torch.cuda.synchronize()
    ref_idx, ref_out = oracle_decode(x, w)
    assert np.array_equal(idx.cpu().numpy(), ref_idx)
    assert_out_close(out, ref_out)
