"""GPU parity of the paged KV cache (page size 1: "Their 42x decode speedup
never compiled on my GPU", What their numbers claim) and of cross-layer index
reuse (LongCat Sparse Attention, Abstract, strategy (2)).

The paged kernels read the same rows as the contiguous ones in the same order,
so their outputs must be bit-identical to the contiguous path's, and within
the attention tolerance of the oracle read through the page table."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import indexed_sparse_attention_kv_b200 as lsa
import oracle.lsa_oracle as O
from indexed_sparse_attention_kv_b200 import inputs as I

from _util import assert_out_close, np32, oracle_decode, to_dev

pytestmark = pytest.mark.gpu

CASES = [
    # batch, hq, hkv, d, r, T, B
    (2, 32, 8, 128, 64, 3001, 300),
    (1, 16, 8, 64, 64, 1500, 100),
    (3, 8, 4, 128, 64, 700, 800),      # B > T: padded index sets
    (1, 32, 2, 256, 64, 2000, 64),
]


def _case(case, seed=81):
    batch, hq, hkv, d, r, T, B = case
    w = I.Workload(f"paged_{case}", seed, batch=batch, hq=hq, hkv=hkv, d=d, T=T, r=r, B=B)
    return w, I.make_decode_inputs(w)


def _pools(x, w, spare=37, seed=82):
    """K/V rows of every (b, t) at a random slot of pools with `spare` unused slots."""
    n = w.batch * w.T
    perm = torch.randperm(n + spare, generator=torch.Generator().manual_seed(seed))[:n]
    table = perm.to(torch.int32).view(w.batch, w.T)
    pools = []
    for name in ("k", "v"):
        pool = torch.randn((n + spare, w.hkv, w.d), generator=torch.Generator().manual_seed(seed + 1))
        pool = pool.to(torch.bfloat16)
        pool[perm] = x[name].reshape(n, w.hkv, w.d)
        pools.append(pool)
    return table, pools[0], pools[1]


@pytest.mark.parametrize("case", CASES, ids=[str(c) for c in CASES])
def test_paged_step_equals_contiguous_and_oracle(case):
    w, x = _case(case)
    table, kp, vp = _pools(x, w)
    d = to_dev(x)
    idx0, out0 = lsa.lsa_decode_step(d["q"], d["qt"], d["k"], d["v"], d["kt"], w.B)
    idx1, out1 = lsa.lsa_decode_step_paged(d["q"], d["qt"], kp.cuda(), vp.cuda(), table.cuda(), d["kt"], w.B)
    out2 = lsa.lsa_indexed_attn_paged(d["q"], kp.cuda(), vp.cuda(), table.cuda(), idx0)
    out3 = lsa.lsa_indexed_attn(d["q"], d["k"], d["v"], idx0)
    torch.cuda.synchronize()
    assert torch.equal(idx1, idx0)
    assert torch.equal(out1, out0)     # the same step over the same rows
    assert torch.equal(out2, out3)     # the same attention kernel over the same rows
    ref_idx, _ = oracle_decode(x, w)
    assert np.array_equal(idx1.cpu().numpy(), ref_idx)
    for b in range(w.batch):
        ref = O.indexed_attention_paged(np32(x["q"][b]), np32(kp), np32(vp), table[b].numpy(), ref_idx[b], w.scale)
        assert_out_close(out1[b], ref)


def test_paged_bad_slot_is_skipped_and_flagged():
    w, x = _case((1, 8, 2, 128, 64, 500, 40), seed=83)
    table, kp, vp = _pools(x, w)
    d = to_dev(x)
    idx, _ = lsa.lsa_decode_step(d["q"], d["qt"], d["k"], d["v"], d["kt"], w.B)
    torch.cuda.synchronize()
    bad_t = int(idx[0, 1, 5])
    table[0, bad_t] = -1
    dims = lsa.lsa_dims(w.batch, w.hq, w.hkv, w.d, w.r, w.T)
    ws = lsa.workspace(dims, w.B)
    out = lsa.lsa_indexed_attn_paged(d["q"], kp.cuda(), vp.cuda(), table.cuda(), idx, ws=ws)
    torch.cuda.synchronize()
    assert lsa.lsa_read_device_status(ws) & lsa._lib.DEV_BAD_INDEX
    kept = idx[0].cpu().numpy().copy()
    kept[1, 5] = -1            # the skipped row
    ref = O.indexed_attention_paged(np32(x["q"][0]), np32(kp), np32(vp), table[0].numpy(), kept, w.scale)
    assert_out_close(out[0], ref)


def test_cross_layer_index_reuse():
    """Layer 2 attends over layer 1's index sets: lsa_indexed_attn with the
    other layer's q, k, v and the idx from layer 1's decode step."""
    w, x1 = _case((2, 32, 8, 128, 64, 2500, 256), seed=84)
    _, x2 = _case((2, 32, 8, 128, 64, 2500, 256), seed=85)
    d1, d2 = to_dev(x1), to_dev(x2)
    idx1, _ = lsa.lsa_decode_step(d1["q"], d1["qt"], d1["k"], d1["v"], d1["kt"], w.B)
    out2 = lsa.lsa_indexed_attn(d2["q"], d2["k"], d2["v"], idx1)
    torch.cuda.synchronize()
    ref_idx, _ = oracle_decode(x1, w)
    assert np.array_equal(idx1.cpu().numpy(), ref_idx)
    for b in range(w.batch):
        ref = O.indexed_attention(np32(x2["q"][b]), np32(x2["k"][b]), np32(x2["v"][b]), ref_idx[b], w.scale)
        assert_out_close(out2[b], ref)
