"""Host-only checks of liblsa.so: it loads, exports every function lsa.h
declares, and rejects bad arguments before launching anything (no GPU needed:
every call below fails validation on the host)."""
import ctypes

import pytest

import indexed_sparse_attention_kv_b200._lib as L


@pytest.fixture(scope="module", autouse=True)
def _built_library():
    """The boundary's host-side checks must never vanish from a CPU run: build
    liblsa.so (incremental) when it is missing, and fail if that is impossible."""
    import os
    if not os.path.exists(L.LIB_PATH):
        from indexed_sparse_attention_kv_b200.csrc import build as B
        B.build()
    assert os.path.exists(L.LIB_PATH), "liblsa.so could not be built"


ALIGNED = ctypes.c_void_p(1 << 20)      # never dereferenced: validation fails first
MISALIGNED = ctypes.c_void_p((1 << 20) + 8)


def test_exports_every_declared_symbol():
    names = L.header_functions()
    assert len(names) >= 14
    lib = L.lib()
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(L._SIGS), set(names) ^ set(L._SIGS)


def test_version_and_status_strings():
    lib = L.lib()
    assert lib.lsa_version() == 100
    for code, name in L.STATUS_NAMES.items():
        assert lib.lsa_status_string(code).decode().startswith(name)
    assert lib.lsa_status_string(-99).decode() == "LSA_ERR_UNKNOWN"


def _dims(**kw):
    base = dict(batch=1, hq=4, hkv=1, d=128, r=64, T=4096)
    base.update(kw)
    return L.make_dims(**base)


@pytest.mark.parametrize("kw,code", [
    (dict(batch=0), -1), (dict(hq=0), -1), (dict(T=0), -1), (dict(hq=6, hkv=4), -1),
    (dict(hq=12, hkv=4), -7), (dict(r=48), -7), (dict(d=96), -7), (dict(hq=64, hkv=64, r=128), -7),
])
def test_bad_dims(kw, code):
    lib = L.lib()
    d = _dims(**kw)
    assert lib.lsa_score(ctypes.byref(d), ALIGNED, ALIGNED, ALIGNED, None) == code
    assert lib.lsa_workspace_size(ctypes.byref(d), 256, 0, 0) == 0


def test_null_and_alignment():
    lib = L.lib()
    d = _dims()
    assert lib.lsa_score(None, ALIGNED, ALIGNED, ALIGNED, None) == -1
    assert lib.lsa_score(ctypes.byref(d), None, ALIGNED, ALIGNED, None) == -1
    assert lib.lsa_score(ctypes.byref(d), MISALIGNED, ALIGNED, ALIGNED, None) == -2
    assert lib.lsa_topk(ctypes.byref(d), ALIGNED, 0, ALIGNED, None, 0, None) == -1
    assert lib.lsa_topk(ctypes.byref(d), ALIGNED, 70000, ALIGNED, None, 0, None) == -7
    assert lib.lsa_topk(ctypes.byref(d), MISALIGNED, 16, ALIGNED, None, 0, None) == -2
    f = ctypes.c_float
    assert lib.lsa_indexed_attn(ctypes.byref(d), ALIGNED, ALIGNED, ALIGNED, None, 16, f(0.1), ALIGNED,
                                ALIGNED, 1 << 30, None) == -1
    assert lib.lsa_indexed_attn(ctypes.byref(d), ALIGNED, ALIGNED, ALIGNED, ALIGNED, 16, f(float("nan")),
                                ALIGNED, ALIGNED, 1 << 30, None) == -1
    # index sets longer than 65536 are read by the attention entries (up to 2^24), not selected
    assert lib.lsa_indexed_attn(ctypes.byref(d), ALIGNED, ALIGNED, ALIGNED, ALIGNED, (1 << 24) + 1, f(0.1),
                                ALIGNED, ALIGNED, 1 << 30, None) == -7
    assert lib.lsa_workspace_size(ctypes.byref(d), 131072, 0, 0) > 0
    assert lib.lsa_workspace_size(ctypes.byref(d), (1 << 24) + 1, 0, 0) == 0
    assert lib.lsa_block_centroids(ctypes.byref(d), ALIGNED, 0, ALIGNED, None) == -1
    assert lib.lsa_block_centroids(ctypes.byref(d), ALIGNED, 64, MISALIGNED, None) == -2
    assert lib.lsa_read_device_status(None, ALIGNED, None) == -1
    assert lib.lsa_clear_device_status(None, None) == -1


def test_workspace_checks():
    lib = L.lib()
    d = _dims()
    need = lib.lsa_workspace_size(ctypes.byref(d), 256, 0, 0)
    assert need > 0 and need % 256 == 0
    # coarse-to-fine: block scores + candidate scores + block ids replace the T scores
    hier = lib.lsa_workspace_size(ctypes.byref(d), 256, 64, 16)
    assert hier > 0 and hier % 256 == 0 and hier != need
    assert lib.lsa_workspace_size(ctypes.byref(d), 256, 64, 0) == 0
    f = ctypes.c_float
    args = (ctypes.byref(d), ALIGNED, ALIGNED, ALIGNED, ALIGNED, 256, f(0.1), ALIGNED)
    assert lib.lsa_indexed_attn(*args, None, need, None) == -4
    assert lib.lsa_indexed_attn(*args, ctypes.c_void_p((1 << 20) + 16), need, None) == -4
    assert lib.lsa_indexed_attn(*args, ALIGNED, need - 1, None) == -4
    step = lib.lsa_decode_step
    assert step(ctypes.byref(d), ALIGNED, ALIGNED, ALIGNED, ALIGNED, ALIGNED, None, 0, 0, 256, f(0.1), None,
                ALIGNED, ALIGNED, 16, None) == -4
    assert step(ctypes.byref(d), ALIGNED, ALIGNED, ALIGNED, ALIGNED, ALIGNED, ALIGNED, 0, 16, 256, f(0.1), None,
                ALIGNED, ALIGNED, 1 << 30, None) == -1     # centroids given, blk = 0


def test_binding_refuses_cpu_tensors():
    import torch
    q = torch.zeros(1, 4, 128, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="CUDA"):
        L.lsa_score(q[:, :, :64], torch.zeros(1, 8, 1, 64, dtype=torch.bfloat16))


def test_prefill_validation():
    lib = L.lib()
    d = _dims(T=4096)
    assert lib.lsa_prefill_workspace_size(ctypes.byref(d), 256, 256) > 0
    assert lib.lsa_prefill_workspace_size(ctypes.byref(_dims(batch=2)), 256, 256) == 0
    assert lib.lsa_prefill_workspace_size(ctypes.byref(d), 0, 256) == 0
    args = (ALIGNED, 256, 3840, ALIGNED, 256, ALIGNED, ALIGNED, 1 << 40, None)
    assert lib.lsa_prefill_index(ctypes.byref(_dims(batch=2)), *args) == -3
    assert lib.lsa_prefill_index(ctypes.byref(d), ALIGNED, 256, 3841, ALIGNED, 256, ALIGNED, ALIGNED, 1 << 40,
                                 None) == -3
    assert lib.lsa_prefill_index(ctypes.byref(d), ALIGNED, 0, 0, ALIGNED, 256, ALIGNED, ALIGNED, 1 << 40,
                                 None) == -1
    assert lib.lsa_prefill_index(ctypes.byref(_dims(T=(1 << 18) + 1)), *args) == -7
    assert lib.lsa_prefill_index(ctypes.byref(d), MISALIGNED, 256, 3840, ALIGNED, 256, ALIGNED, ALIGNED, 1 << 40,
                                 None) == -2
    assert lib.lsa_prefill_index(ctypes.byref(d), ALIGNED, 256, 3840, ALIGNED, 256, ALIGNED, ALIGNED, 16,
                                 None) == -4
    f = ctypes.c_float
    assert lib.lsa_prefill_attn(ctypes.byref(d), ALIGNED, 256, ALIGNED, ALIGNED, ALIGNED, 256, f(0.1), ALIGNED,
                                ALIGNED, 16, None) == -4
    assert lib.lsa_prefill_attn(ctypes.byref(d), ALIGNED, 256, ALIGNED, ALIGNED, ALIGNED, 256, f(float("nan")),
                                ALIGNED, ALIGNED, 1 << 40, None) == -1


def test_noalloc_rejects_before_any_device_use():
    lib = L.lib()
    d = L.make_dims(64, 128, 8, 256, 16, 1 << 17)
    f = ctypes.c_float
    assert lib.lsa_indexed_attn_noalloc(ctypes.byref(d), ALIGNED, ALIGNED, ALIGNED, ALIGNED, 65536, f(0.06),
                                        ALIGNED, None, None) == -8
    assert lib.lsa_indexed_attn_noalloc(ctypes.byref(d), MISALIGNED, ALIGNED, ALIGNED, ALIGNED, 16, f(0.06),
                                        ALIGNED, None, None) == -2


def test_fp8_validation():
    lib = L.lib()
    f = ctypes.c_float
    for kw in (dict(r=32), dict(hq=8, hkv=2), dict(r=128, hkv=8, hq=32)):
        d = _dims(**kw)
        assert lib.lsa_score_fp8(ctypes.byref(d), ALIGNED, ALIGNED, ALIGNED, None) == -7
        assert lib.lsa_decode_step_fp8(ctypes.byref(d), ALIGNED, ALIGNED, ALIGNED, ALIGNED, ALIGNED, 16, f(0.1),
                                       None, ALIGNED, ALIGNED, 1 << 40, None) == -7
    d = _dims(hq=32, hkv=8)
    assert lib.lsa_score_fp8(ctypes.byref(d), None, ALIGNED, ALIGNED, None) == -1
    assert lib.lsa_score_fp8(ctypes.byref(d), ALIGNED, MISALIGNED, ALIGNED, None) == -2
    assert lib.lsa_decode_step_fp8(ctypes.byref(d), ALIGNED, ALIGNED, ALIGNED, ALIGNED, ALIGNED, 16, f(0.1),
                                   None, ALIGNED, ALIGNED, 16, None) == -4


def _pd(**kw):
    base = dict(batch=2, T=1000, H=8, d=128, r=64, nbases=8)
    base.update(kw)
    return L.lsa_proj_dims(*(base[k] for k in ("batch", "T", "H", "d", "r", "nbases")))


@pytest.mark.parametrize("fn", ["lsa_project", "lsa_project_fp8"])
def test_project_validation(fn):
    """Every rejection happens on the host, before any device use."""
    f = getattr(L.lib(), fn)
    ok = _pd()
    call = lambda d, x=ALIGNED, P=ALIGNED, t0=0, n=10, y=ALIGNED, st=None: f(  # noqa: E731
        ctypes.byref(d), x, P, t0, n, y, st, None)
    assert call(ok, x=None) == -1
    assert call(ok, y=None) == -1
    assert call(_pd(H=6, nbases=4)) == -1            # H % nbases != 0
    assert call(_pd(T=0)) == -1
    assert call(ok, t0=-1) == -3
    assert call(ok, t0=995, n=6) == -3               # t0 + n > T
    assert call(ok, n=-1) == -3
    assert call(ok, x=MISALIGNED) == -2
    assert call(ok, st=ctypes.c_void_p(ALIGNED.value + 2)) == -2
    for kw in (dict(d=48), dict(d=24), dict(d=320), dict(r=8), dict(r=40), dict(r=144), dict(d=256, r=96)):
        assert call(_pd(**kw)) == -7, kw
    assert call(ok, n=0) == 0                        # nothing to do, nothing launched


def test_update_centroids_validation():
    lib = L.lib()
    d = _dims()
    assert lib.lsa_update_centroids(ctypes.byref(d), None, 64, 0, 1, ALIGNED, None) == -1
    assert lib.lsa_update_centroids(ctypes.byref(d), ALIGNED, 0, 0, 1, ALIGNED, None) == -1
    assert lib.lsa_update_centroids(ctypes.byref(d), ALIGNED, 64, d.T, 1, ALIGNED, None) == -3
    assert lib.lsa_update_centroids(ctypes.byref(d), ALIGNED, 64, 0, 1, MISALIGNED, None) == -2
    assert lib.lsa_update_centroids(ctypes.byref(d), ALIGNED, 64, 5, 0, ALIGNED, None) == 0


def test_paged_validation():
    lib = L.lib()
    f = ctypes.c_float
    d = _dims()
    a = lambda **kw: lib.lsa_indexed_attn_paged(  # noqa: E731
        ctypes.byref(d), kw.get("q", ALIGNED), ALIGNED, ALIGNED, kw.get("nslots", 10), kw.get("pt", ALIGNED),
        ALIGNED, 16, f(0.1), ALIGNED, kw.get("ws", ALIGNED), kw.get("wsb", 1 << 40), None)
    assert a(q=None) == -1
    assert a(pt=None) == -1
    assert a(nslots=0) == -1
    assert a(pt=MISALIGNED) == -2
    assert a(wsb=16) == -4
    s = lambda **kw: lib.lsa_decode_step_paged(  # noqa: E731
        ctypes.byref(d), ALIGNED, ALIGNED, ALIGNED, ALIGNED, kw.get("nslots", 10), kw.get("pt", ALIGNED),
        kw.get("kt", ALIGNED), 16, f(0.1), None, ALIGNED, ALIGNED, kw.get("wsb", 1 << 40), None)
    assert s(kt=None) == -1
    assert s(nslots=-3) == -1
    assert s(pt=MISALIGNED) == -2
    assert s(wsb=16) == -4


def test_prefill_workspace_matches_header_note():
    """lsa.h states about 3.26 GiB of prefill workspace for nq 4096, T 128K, B 2048."""
    d = L.make_dims(1, 32, 8, 128, 64, 131072)
    gib = L.lsa_prefill_workspace_size(d, 4096, 2048) / 2 ** 30
    assert abs(gib - 3.26) < 0.01, gib


def test_binding_argument_counts_match_header():
    """Every ctypes signature has as many arguments as the lsa.h prototype."""
    import re

    text = open(L.HEADER_PATH).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    protos = re.findall(r"LSA_API\s+[\w\s\*]+?\b(lsa_\w+)\s*\(([^)]*)\)\s*;", text, flags=re.S)
    assert len(protos) == len(L._SIGS)
    for name, params in protos:
        params = params.strip()
        n = 0 if params in ("", "void") else params.count(",") + 1
        assert n == len(L._SIGS[name][1]), (name, n, len(L._SIGS[name][1]))
