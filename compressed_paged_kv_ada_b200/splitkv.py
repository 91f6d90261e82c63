"""Split-KV of one long stream across GPUs: host-side plumbing.

Each rank holds a contiguous, page-aligned range of the stream's tokens in its
own paged cache and decodes the query against it with the library (an
ordinary sphkv_decode_attention call: out normalised over its own keys, lse
their log-sum-exp).  The ranks then all-gather their (out, lse) pairs and
combine them with sphkv_merge_partials, which gives attention over the whole
stream (Spherical KV, Abstract: long-context inference).  The exchange is one
all-gather of B * H_q * (128 + 1) floats per rank, over NCCL on NVLink.

This module only partitions token ranges and moves tensors; the decode and the
merge run in libsphkv.
"""
from __future__ import annotations

from typing import Callable, List, Optional, Tuple

PAGE = 16


def split_stream(n_tokens: int, world: int) -> List[Tuple[int, int]]:
    """Contiguous token ranges [t0, t1), one per rank, cut at page boundaries;
    page counts differ by at most one (the earlier ranks take the extra
    pages).  A rank may get an empty range when the stream has fewer pages
    than ranks."""
    if world < 1 or n_tokens < 0:
        raise ValueError("need world >= 1 and n_tokens >= 0")
    n_pages = (n_tokens + PAGE - 1) // PAGE
    base, extra = divmod(n_pages, world)
    out, p = [], 0
    for r in range(world):
        q = p + base + (1 if r < extra else 0)
        out.append((min(n_tokens, p * PAGE), min(n_tokens, q * PAGE)))
        p = q
    return out


def gather_parts(out, lse, group=None):
    """All-gather every rank's decode result: out [..., 128], lse [...] ->
    out_parts [world, ..., 128], lse_parts [world, ...] (rank order)."""
    import torch
    import torch.distributed as dist

    world = dist.get_world_size(group)
    outs = [torch.empty_like(out) for _ in range(world)]
    lses = [torch.empty_like(lse) for _ in range(world)]
    dist.all_gather(outs, out.contiguous(), group=group)
    dist.all_gather(lses, lse.contiguous(), group=group)
    return torch.stack(outs), torch.stack(lses)


def merge_over_ranks(out, lse, group=None, merge: Optional[Callable] = None):
    """Attention over the whole stream from each rank's result over its own
    range: all-gather, then the log-sum-exp combine (sphkv_merge_partials on
    the GPU, or `merge(out_parts, lse_parts) -> (out, lse)` if given).  Every
    rank of the group must call this, in the same order."""
    out_parts, lse_parts = gather_parts(out, lse, group)
    if merge is not None:
        return merge(out_parts, lse_parts)
    import torch

    from . import _lib

    res_out = torch.empty_like(out)
    res_lse = torch.empty_like(lse)
    _lib.sphkv_merge_partials(out_parts, lse_parts, res_out, res_lse)
    return res_out, res_lse
