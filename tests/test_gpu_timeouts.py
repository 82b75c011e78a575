"""Bounded device waits in the pipelined kernels: with a zero poll budget the
first unfinished barrier probe gives up, the kernel drains the copies and MMAs
it already issued, reports LSA_DEV_TIMEOUT in the status word and returns.
The context stays usable: the next call with the normal budget is exact
against the oracle. No kernel is made to fault, trap or hang; the waits that
run out are ordinary pipeline waits on work that completes moments later.

Covered here: the warp-specialised r = 64 scorer (KV heads in {4, 8, 16, 32};
the one-KV-head case of the flat scorer is in test_gpu_decode.py), the
prefill indexer's tensor-core GEMM, and the tensor-core projection."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import indexed_sparse_attention_kv_b200 as lsa
import oracle.lsa_oracle as O
from indexed_sparse_attention_kv_b200 import inputs as I

from _util import assert_out_close, np32, oracle_decode, to_dev

pytestmark = pytest.mark.gpu


class _zero_wait_budget:
    def __enter__(self):
        lsa.lsa_debug_set_wait_limit(0)

    def __exit__(self, *exc):
        lsa.lsa_debug_set_wait_limit(-1)
        return False


def test_q64_scorer_timeout_then_exact():
    w = I.Workload("timeout_q64", 71, batch=2, hq=32, hkv=8, d=128, T=3000, r=64, B=200)
    x = I.make_decode_inputs(w)
    dx = to_dev(x)
    dims = lsa._lib.decode_dims(dx["q"], dx["qt"], dx["k"])
    ws = lsa.workspace(dims, w.B)
    with _zero_wait_budget():
        lsa.lsa_decode_step(dx["q"], dx["qt"], dx["k"], dx["v"], dx["kt"], w.B, ws=ws)
        status = lsa.lsa_read_device_status(ws)
    assert status & lsa._lib.DEV_TIMEOUT
    lsa.lsa_clear_device_status(ws)
    for _ in range(2):
        idx, out = lsa.lsa_decode_step(dx["q"], dx["qt"], dx["k"], dx["v"], dx["kt"], w.B, ws=ws)
        assert lsa.lsa_read_device_status(ws) == 0
    ref_idx, ref_out = oracle_decode(x, w)
    assert np.array_equal(idx.cpu().numpy(), ref_idx)
    assert_out_close(out, ref_out)


def test_prefill_gemm_timeout_then_exact():
    w = I.Workload("timeout_prefill", 72, batch=1, hq=8, hkv=2, d=128, T=2000, r=64, B=128, nq=256)
    x = I.make_prefill_inputs(w)
    q0 = int(x["q_start"])
    qt, kt = x["qt"].cuda(), x["kt"].cuda()
    dims = lsa._lib.prefill_dims(w.hq, kt)
    ws = lsa._lib.prefill_workspace(dims, w.nq, w.B, device=qt.device)
    with _zero_wait_budget():
        lsa.lsa_prefill_index(qt, kt, q0, w.B, ws=ws)
        status = lsa.lsa_read_device_status(ws)
    assert status & lsa._lib.DEV_TIMEOUT
    lsa.lsa_clear_device_status(ws)
    idx = lsa.lsa_prefill_index(qt, kt, q0, w.B, ws=ws)
    assert lsa.lsa_read_device_status(ws) == 0
    rows = np.arange(0, w.nq, 17)
    want = O.prefill_index(np32(x["qt"][rows]), q0 + rows, np32(x["kt"]), w.B)
    assert np.array_equal(idx.cpu().numpy()[rows], want)


def test_projection_timeout_then_exact():
    batch, T, H, d, r, nb = 2, 700, 8, 128, 64, 8
    x = I.make_projection_inputs(73, batch, T, H, d, r, nb)
    xs, P = x["x"].cuda(), x["P"].cuda()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    with _zero_wait_budget():
        lsa.lsa_project(xs, P, dev_status=status)
        torch.cuda.synchronize()
    assert int(status.item()) & lsa._lib.DEV_TIMEOUT
    status.zero_()
    y = lsa.lsa_project(xs, P, dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    want = O.project_bf16(np32(x["x"]), np32(x["P"]), 1)
    assert np.array_equal(y.float().double().cpu().numpy(), want)
