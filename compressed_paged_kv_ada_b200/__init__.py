"""Spherical KV angle-domain attention (ADA) decode over a paged,
tier-homogeneous compressed KV cache, for NVIDIA B200 (sm_100a).

The compute lives in libsphkv.so (hand-written CUDA, C ABI in
include/sphkv.h); this package only binds it.  Build it with
`python -m compressed_paged_kv_ada_b200.build`.
"""
from ._lib import (  # noqa: F401
    SphkvError,
    lib,
    make_cache,
    sphkv_build_page_table,
    sphkv_decode_attention,
    sphkv_decode_attention_mq,
    sphkv_decode_attention_noalloc,
    sphkv_decode_mq_workspace_bytes,
    sphkv_decode_workspace_bytes,
    sphkv_encode,
    sphkv_merge_partials,
    sphkv_migrate,
    sphkv_page_bytes,
    sphkv_rdr_assign,
    sphkv_rdr_rerun,
    sphkv_rdr_workspace_bytes,
    sphkv_set_keep,
)
from .cache import PagedCache  # noqa: F401
