"""lsa_indexed_attn_noalloc (fixed per-device scratch, no workspace) against
lsa_indexed_attn (caller workspace) on the same inputs: two calls in a row,
each within the attention tolerance of the workspace call. Runs last (file
name) so that it also sees the scratch after every other test in the process.
"""
import ctypes

import pytest
import torch

import indexed_sparse_attention_kv_b200._lib as L
from _util import assert_out_close, np32

pytestmark = pytest.mark.gpu

# (batch, hq, hkv, d, T, B, seed): several 64-row tiles with a ragged tail,
# a split across CTAs, G = 16 with d = 256, and sets shorter than B.
CASES = [
    (1, 4, 1, 128, 4096, 256, 7001),
    (2, 32, 8, 128, 32768, 2048, 7002),
    (1, 16, 1, 256, 3000, 1000, 7003),
    (3, 8, 2, 64, 500, 700, 7004),
]


def _inputs(batch, hq, hkv, d, T, B, seed):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(batch, hq, d, generator=g).to(torch.bfloat16)
    k = torch.randn(batch, T, hkv, d, generator=g).to(torch.bfloat16)
    v = torch.randn(batch, T, hkv, d, generator=g).to(torch.bfloat16)
    n = min(B, T)
    idx = torch.full((batch, hkv, B), -1, dtype=torch.int32)
    for b in range(batch):
        for h in range(hkv):
            idx[b, h, :n] = torch.randperm(T, generator=g)[:n].sort().values.to(torch.int32)
    return [t.cuda() for t in (q, k, v, idx)]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "b{}_hq{}_hkv{}_d{}_T{}_B{}".format(*c[:6]))
def test_noalloc_matches_workspace_call_twice(case):
    q, k, v, idx = _inputs(*case)
    ref = L.lsa_indexed_attn(q, k, v, idx)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    outs = []
    for call in range(2):
        out = torch.full_like(q, float("nan"))
        torch.cuda.synchronize()
        free0 = torch.cuda.mem_get_info()[0]
        L.lsa_indexed_attn_noalloc(q, k, v, idx, out=out, dev_status=status)
        torch.cuda.synchronize()
        if call > 0:   # the first call may load the module image; later calls allocate nothing
            assert torch.cuda.mem_get_info()[0] == free0
        outs.append(out)
    assert int(status.item()) == 0
    r = np32(ref).astype("float64")
    for out in outs:
        assert_out_close(out, r, "noalloc vs workspace call")


def test_noalloc_reports_bad_index_in_caller_status():
    q, k, v, idx = _inputs(1, 8, 2, 128, 2048, 256, 7005)
    idx[0, 1, 3] = 5000          # outside [-1, T): skipped by both entry points
    ref = L.lsa_indexed_attn(q, k, v, idx)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = L.lsa_indexed_attn_noalloc(q, k, v, idx, dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) & L.DEV_BAD_INDEX
    assert_out_close(out, np32(ref).astype("float64"), "noalloc vs workspace call, bad index")
    # a clean call afterwards still matches: the shared counters were left at zero
    q, k, v, idx = _inputs(1, 8, 2, 128, 2048, 256, 7006)
    ref2 = L.lsa_indexed_attn(q, k, v, idx)
    out2 = L.lsa_indexed_attn_noalloc(q, k, v, idx)
    assert_out_close(out2, np32(ref2).astype("float64"), "noalloc after a bad-index call")


def test_noalloc_rejects_sizes_beyond_scratch():
    # 64 x 8 units, G 16, d 256, B 65536 needs well over the fixed scratch.
    T = 1 << 17
    q = torch.zeros(64, 128, 256, dtype=torch.bfloat16, device="cuda")
    k = torch.zeros(1, T, 8, 256, dtype=torch.bfloat16, device="cuda").expand(64, T, 8, 256)
    idx = torch.zeros(1, 8, 65536, dtype=torch.int32, device="cuda").expand(64, 8, 65536)
    dims = L.make_dims(64, 128, 8, 256, 16, T)
    rc = L.lib().lsa_indexed_attn_noalloc(ctypes.byref(dims), L._ptr(q), L._ptr(k), L._ptr(k), L._ptr(idx), 65536,
                                          ctypes.c_float(0.0625), L._ptr(q), None, None)
    assert rc == -8
    assert L.lib().lsa_status_string(rc).decode().startswith("LSA_ERR_SCRATCH")
