"""Indexed sparse attention over a GQA KV cache for NVIDIA B200 (sm_100a).

The compute lives in liblsa.so (hand-written CUDA, C ABI in include/lsa.h);
this package is its Python binding (``_lib``) and the seeded synthetic inputs
(``inputs``). Importing the package does not load the library; the first call
does, and raises if liblsa.so has not been built.
"""
from ._lib import (  # noqa: F401
    LsaError,
    lib,
    lsa_block_centroids,
    lsa_clear_device_status,
    lsa_debug_set_wait_limit,
    lsa_decode_step,
    lsa_decode_step_fp8,
    lsa_dims,
    lsa_indexed_attn,
    lsa_indexed_attn_noalloc,
    lsa_indexed_attn_paged,
    lsa_decode_step_paged,
    lsa_prefill_attn,
    lsa_prefill_index,
    lsa_prefill_workspace_size,
    lsa_proj_dims,
    lsa_project,
    lsa_project_fp8,
    lsa_update_centroids,
    prefill_workspace,
    lsa_read_device_status,
    lsa_score,
    lsa_score_fp8,
    lsa_topk,
    lsa_workspace_size,
    workspace,
)

__version__ = "0.1.0"
