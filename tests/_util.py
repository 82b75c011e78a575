"""Helpers shared by the GPU parity tests (tolerances, conversions, oracle runs)."""
from __future__ import annotations

import functools

import numpy as np
import torch

import oracle.lsa_oracle as O
from indexed_sparse_attention_kv_b200 import inputs as I

# Attention outputs ("within 1e-2 max-abs and 1e-2 relative of the oracle"),
# checked three ways: every element |gpu - ref| <= ATOL + RTOL * |ref|; the
# largest error <= ATOL; and the largest error relative to the largest
# reference magnitude <= RTOL (binding when outputs are small). A purely
# per-element relative bound is not used: an output element near zero has no
# meaningful relative error after the bf16 store. Index sets: bit-exact.
ATOL = 1e-2
RTOL = 1e-2


def np32(t: torch.Tensor) -> np.ndarray:
    """bf16/fp32 torch tensor (any device) -> float32 numpy (exact for bf16)."""
    return t.detach().to("cpu", torch.float32).numpy()


def assert_out_close(gpu: torch.Tensor, ref: np.ndarray, what: str = "out") -> None:
    g = np32(gpu).astype(np.float64)
    err = np.abs(g - ref)
    mx = float(err.max()) if err.size else 0.0
    scale = float(np.abs(ref).max()) if ref.size else 0.0
    assert np.isfinite(g).all(), f"{what}: non-finite GPU output"
    bad = err > ATOL + RTOL * np.abs(ref)
    assert not bad.any(), f"{what}: {int(bad.sum())} elements outside atol + rtol*|ref|, first at " \
        f"{np.argwhere(bad)[0].tolist()}"
    assert mx <= ATOL, f"{what}: max abs err {mx:.3e} > {ATOL}"
    if scale > 0:
        assert mx / scale <= RTOL, f"{what}: max rel err {mx / scale:.3e} > {RTOL}"


class LazyRows:
    """Read-only view of a host bf16 tensor that converts only the rows the
    oracle indexes to float32 numpy (keeps full-size caches out of fp32/fp64)."""

    def __init__(self, t: torch.Tensor):
        self.t = t
        self.shape = tuple(t.shape)

    def __getitem__(self, key):
        if isinstance(key, tuple):
            key = tuple(torch.from_numpy(np.asarray(k)) if isinstance(k, np.ndarray) else k for k in key)
        elif isinstance(key, np.ndarray):
            key = torch.from_numpy(key)
        return self.t[key].to(torch.float32).numpy()


def oracle_decode(x: dict, w: I.Workload, batches=None, blk: int = 0, keep: int = 0):
    """Oracle idx [nb, hkv, B] (int64) and out [nb, hq, d] for the listed batch rows."""
    batches = range(w.batch) if batches is None else batches
    idx_all, out_all = [], []
    for b in batches:
        q = np32(x["q"][b])
        qt = np32(x["qt"][b])
        k = LazyRows(x["k"][b])
        v = LazyRows(x["v"][b])
        kt = LazyRows(x["kt"][b])
        idx, out = O.decode_step(q, qt, k, v, kt, w.B, w.scale, blk=blk, keep=keep)
        idx_all.append(idx)
        out_all.append(out)
    return np.stack(idx_all), np.stack(out_all)


@functools.lru_cache(maxsize=2)
def decode_inputs(name: str):
    w = I.workload(name)
    return w, I.make_decode_inputs(w)


def to_dev(x: dict, keys=("q", "qt", "k", "v", "kt")) -> dict:
    return {k: x[k].cuda() for k in keys}
