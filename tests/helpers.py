"""Shared helpers for the parity tests: build the same seeded workload on the
GPU (through libsphkv) and in the CPU oracle, and compare.

Tolerances (stated once, used by every float comparison):
  max |out_gpu - out_ref| <= 1e-3 * max |out_ref|   (per query-head row)
  |lse_gpu - lse_ref|     <= 1e-4                    (absolute, natural log)
Codes, tiers, page tables and page bytes are compared bit for bit.
"""
from __future__ import annotations

import numpy as np

import oracle
from compressed_paged_kv_ada_b200 import workloads as W

OUT_RTOL = 1e-3
LSE_ATOL = 1e-4


def to_torch(x, dtype=None, device="cuda"):
    import torch

    t = torch.from_numpy(np.ascontiguousarray(x))
    if dtype is not None:
        t = t.to(dtype)
    return t.to(device)


def dense_torch(w: W.Workload, K, V):
    import torch

    dt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    return to_torch(K, dt), to_torch(V, dt)


def gpu_cache(w: W.Workload, lens=None, tiers=None, perms=None, encode=True):
    """PagedCache on cuda:0 for workload w, every present token encoded by the
    library's encode kernel."""
    import torch

    from compressed_paged_kv_ada_b200 import PagedCache

    lens = w.seq_lens if lens is None else np.asarray(lens, np.int32)
    tiers = w.tiers if tiers is None else tiers
    perms = w.pool_perms() if perms is None else perms
    cache = PagedCache(w.page_offsets, lens, tiers, perms)
    if encode:
        for b in range(w.B):
            n = int(lens[b])
            if n == 0:
                continue
            K, V = w.dense_rows(b, 0, n)
            Kt, Vt = dense_torch(w, K, V)
            seq = torch.full((n,), b, dtype=torch.int32, device="cuda")
            pos = torch.arange(n, dtype=torch.int32, device="cuda")
            cache.encode(Kt, Vt, seq, pos)
        cache.check()
    return cache


def oracle_full_cache(w: W.Workload, lens=None, tiers=None, perms=(None, None, None)):
    """The oracle's own cache (its encoder, packer and page table)."""
    lens = w.seq_lens if lens is None else np.asarray(lens, np.int32)
    tiers = w.tiers if tiers is None else tiers
    table = oracle.build_page_table(tiers, perms)
    K, V = w.dense(lens)
    seq, pos = w.token_index(lens)
    counts = [int((tiers == t).sum()) for t in (1, 2, 3)]
    pools = oracle.encode_cache(K, V, seq, pos, w.page_offsets, table, counts)
    return dict(B=w.B, H_q=w.H_q, H_kv=w.H_kv, page_offsets=w.page_offsets, seq_lens=lens,
                page_table=table, pools=pools)


def oracle_unit(w: W.Workload, b: int, g: int, q, lens=None, tiers=None):
    """Oracle attention of the G query heads of kv head g of sequence b, from
    a one-unit cache built with the oracle's own encoder (the storage layout
    does not change the result)."""
    lens = w.seq_lens if lens is None else lens
    tiers = w.tiers if tiers is None else tiers
    n = int(lens[b])
    po = w.page_offsets
    cap = int(po[b + 1] - po[b])
    row = np.ascontiguousarray(tiers[g:g + 1, po[b]:po[b + 1]])
    table = oracle.build_page_table(row)
    K, V = w.dense_rows(b, 0, n)
    G = w.H_q // w.H_kv
    counts = [int((row == t).sum()) for t in (1, 2, 3)]
    pools = oracle.encode_cache(K[:, g:g + 1], V[:, g:g + 1], np.zeros(n, np.int32),
                                np.arange(n), np.array([0, cap]), table, counts)
    c = dict(B=1, H_q=G, H_kv=1, page_offsets=np.array([0, cap], np.int32),
             seq_lens=np.array([n], np.int32), page_table=table, pools=pools)
    qb = np.asarray(q, np.float64)[b, g * G:(g + 1) * G][None]
    out, lse = oracle.cache_attention(c, qb, [(0, 0)])
    return out[0], lse[0]


def oracle_all_units(w: W.Workload, q, lens=None, tiers=None):
    """Oracle attention of every (sequence, kv head) unit of w, over the
    oracle's own encoding of the whole workload (the pool page ids do not
    change the result).  Returns out [B, H_q, 128], lse [B, H_q]."""
    ref = oracle_full_cache(w, lens=lens, tiers=tiers)
    units = [(b, g) for b in range(w.B) for g in range(w.H_kv)]
    ro, rl = oracle.cache_attention(ref, q, units)
    return ro.reshape(w.B, w.H_q, -1), rl.reshape(w.B, w.H_q)


def oracle_unit_dense(w: W.Workload, b: int, g: int, n: int, tiers):
    """Keys and values of the first n tokens of sequence b, kv head g, as the
    oracle encodes and decodes them (fp64), with the mask of kept tokens
    (their page is not dropped).  Returns khat [n, 128], vhat [n, 128], keep."""
    K, V = w.dense_rows(b, 0, n)
    po = w.page_offsets
    tok_tier = np.repeat(np.asarray(tiers)[g, po[b]:po[b] + (n + 15) // 16], 16)[:n]
    khat = np.zeros((n, 128))
    vhat = np.zeros((n, 128))
    for t in (1, 2, 3):
        idx = np.nonzero(tok_tier == t)[0]
        if idx.size == 0:
            continue
        c = oracle.encode(K[idx, g], V[idx, g], t)
        bl, bu, _ = oracle.TIER_BITS[t]
        khat[idx] = oracle.decode_keys(c["leaf"], c["up"], c["r16"], bl, bu)
        vhat[idx] = oracle.decode_values(c["vq"], c["s16"])
    return khat, vhat, tok_tier != 0


def assert_close(out_gpu, lse_gpu, out_ref, lse_ref, what=""):
    out_gpu = np.asarray(out_gpu, np.float64)
    lse_gpu = np.asarray(lse_gpu, np.float64)
    out_ref = np.asarray(out_ref, np.float64)
    lse_ref = np.asarray(lse_ref, np.float64)
    assert out_gpu.shape == out_ref.shape, what
    inf_ref = np.isneginf(lse_ref)
    assert np.array_equal(np.isneginf(lse_gpu), inf_ref), f"{what}: -inf pattern of lse differs"
    assert np.all(np.abs(lse_gpu[~inf_ref] - lse_ref[~inf_ref]) <= LSE_ATOL), \
        f"{what}: lse max err {np.abs(lse_gpu[~inf_ref] - lse_ref[~inf_ref]).max()}"
    rows_g = out_gpu.reshape(-1, out_gpu.shape[-1])
    rows_r = out_ref.reshape(-1, out_ref.shape[-1])
    err = np.abs(rows_g - rows_r).max(axis=1)
    scale = np.abs(rows_r).max(axis=1)
    bad = err > OUT_RTOL * scale
    bad &= ~((scale == 0) & (err == 0))
    assert not bad.any(), f"{what}: out err {err[bad][:4]} vs scale {scale[bad][:4]}"
