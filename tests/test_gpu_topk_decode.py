"""GPU parity of the decode step's top-B on rows of more than 16K keys (the
scorer's key histogram feeding the cluster selection) in its special cases,
against the oracle: every score equal (the whole row in the threshold bin,
the cluster's exact fallback), rows with fewer valid keys than B (NaN
projected keys are not candidates; the sets are padded with -1), many ties at
the boundary (small integer ranges), KV-head count 4 with the FP8 and paged
steps, and repeated calls on one workspace (its histograms and counters left
at zero)."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import indexed_sparse_attention_kv_b200 as lsa
from indexed_sparse_attention_kv_b200 import inputs as I

from _util import assert_out_close, oracle_decode, to_dev

pytestmark = pytest.mark.gpu


def _run(w, x, calls=2):
    d = to_dev(x)
    dims = lsa.lsa_dims(w.batch, w.hq, w.hkv, w.d, w.r, w.T)
    ws = lsa.workspace(dims, w.B)
    outs = []
    for _ in range(calls):
        outs.append(lsa.lsa_decode_step(d["q"], d["qt"], d["k"], d["v"], d["kt"], w.B, ws=ws))
    torch.cuda.synchronize()
    assert lsa.lsa_read_device_status(ws) == 0
    for idx, out in outs[1:]:
        assert torch.equal(idx, outs[0][0]) and torch.equal(out, outs[0][1])
    return outs[0]


def test_equal_scores():
    """Every projected key equal: all scores of a row tie, and the selection
    keeps positions 0 .. B-1."""
    w = I.Workload("equal_scores", 101, batch=2, hq=32, hkv=8, d=128, T=40000, r=64, B=2048)
    x = I.make_decode_inputs(w)
    x["kt"].fill_(1.0)
    idx, out = _run(w, x)
    ref_idx, ref_out = oracle_decode(x, w)
    assert np.array_equal(idx.cpu().numpy(), ref_idx)
    assert_out_close(out, ref_out)


def test_fewer_valid_keys_than_budget():
    """NaN projected keys give NaN scores, which are never candidates: rows
    with fewer valid keys than B keep all of them and pad with -1."""
    w = I.Workload("nan_keys", 102, batch=1, hq=32, hkv=8, d=128, T=24000, r=64, B=3000)
    x = I.make_decode_inputs(w)
    g = torch.Generator().manual_seed(103)
    for h in range(w.hkv):
        n_valid = [1000, 2999, 3000, 3001, 5000, 24000, 0, 2500][h]
        drop = torch.randperm(w.T, generator=g)[: w.T - n_valid]
        x["kt"][0, drop, h, :] = float("nan")
    idx, out = _run(w, x)
    ref_idx, ref_out = oracle_decode(x, w)
    assert np.array_equal(idx.cpu().numpy(), ref_idx)
    got = out.float().cpu().numpy()
    # a head with no valid key has an empty set and a zero output
    assert np.all(got[0, 6 * 4:7 * 4] == 0)
    assert_out_close(out, ref_out)


@pytest.mark.parametrize("int_range,T,B", [(1, 40000, 2048), (2, 65536, 512), (3, 131072, 7000)])
def test_boundary_ties(int_range, T, B):
    w = I.Workload(f"ties_{int_range}", 104 + int_range, batch=1, hq=32, hkv=8, d=128, T=T, r=64, B=B,
                   int_range=int_range)
    x = I.make_decode_inputs(w)
    idx, out = _run(w, x)
    ref_idx, ref_out = oracle_decode(x, w)
    assert np.array_equal(idx.cpu().numpy(), ref_idx)
    assert_out_close(out, ref_out)


def test_hkv4_fp8_and_paged_steps():
    """hkv 4 (the scorer's histogram for 4 KV heads) and the FP8 / paged steps,
    which reach the same selection: all equal to the bf16 step and the oracle."""
    w = I.Workload("hkv4", 107, batch=3, hq=16, hkv=4, d=128, T=50000, r=64, B=1500, heavy_frac=0.01)
    x = I.make_decode_inputs(w)
    d = to_dev(x)
    idx0, out0 = lsa.lsa_decode_step(d["q"], d["qt"], d["k"], d["v"], d["kt"], w.B)
    idx1, out1 = lsa.lsa_decode_step_fp8(d["q"], d["qt"], d["k"], d["v"], d["kt"].to(torch.float8_e4m3fn), w.B)
    n = w.batch * w.T
    perm = torch.randperm(n, generator=torch.Generator().manual_seed(108)).cuda()
    kp = torch.empty((n, w.hkv, w.d), dtype=torch.bfloat16, device="cuda")
    vp = torch.empty_like(kp)
    kp[perm] = d["k"].reshape(n, w.hkv, w.d)
    vp[perm] = d["v"].reshape(n, w.hkv, w.d)
    idx2, out2 = lsa.lsa_decode_step_paged(d["q"], d["qt"], kp, vp, perm.to(torch.int32).view(w.batch, w.T),
                                           d["kt"], w.B)
    torch.cuda.synchronize()
    ref_idx, ref_out = oracle_decode(x, w)
    assert np.array_equal(idx0.cpu().numpy(), ref_idx)
    assert_out_close(out0, ref_out)
    assert torch.equal(idx1, idx0) and torch.equal(out1, out0)
    assert torch.equal(idx2, idx0) and torch.equal(out2, out0)
