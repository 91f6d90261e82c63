"""Python handle on the fp64 CPU oracle (``sphkv_oracle.c``).

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the CPU
baseline leg of ``bench.py`` are the only callers.  The product package never
imports this module and shares no code with it.

The wrapper only marshals numpy arrays; every step of the method runs in the C
file, which states its sources (the Spherical KV abstract, arXiv 2605.18856)
and the readings it takes.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "sphkv_oracle.c")
_SO = os.path.join(_HERE, "libsphkv_oracle.so")

# Tier -> (b_leaf, b_up, v_bits).  Tier 0 is "drop".
TIER_BITS = {1: (8, 8, 8), 2: (4, 6, 4), 3: (3, 4, 4)}
PAGE = 16
D = 128

_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (-O2, no FMA contraction, OpenMP)."""
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-ffp-contract=off", "-fno-fast-math", "-fopenmp", "-fPIC",
               "-shared", "-o", _SO + ".tmp", _SRC, "-lm"]
        subprocess.check_call(cmd)
        os.replace(_SO + ".tmp", _SO)
    return _SO


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_SO)
        c = ctypes
        P = c.c_void_p
        L.orc_f64_to_f16.restype = c.c_uint16
        L.orc_f64_to_f16.argtypes = [c.c_double]
        L.orc_f16_to_f64.restype = c.c_double
        L.orc_f16_to_f64.argtypes = [c.c_uint16]
        L.orc_page_bytes.restype = c.c_int
        L.orc_page_bytes.argtypes = [c.c_int]
        L.orc_encode_tokens.restype = c.c_int64
        L.orc_encode_tokens.argtypes = [c.c_int64, c.c_int, P, P, c.c_int, c.c_int, c.c_int,
                                        P, P, P, P, P]
        L.orc_decode_keys.restype = None
        L.orc_decode_keys.argtypes = [c.c_int64, c.c_int, P, P, P, c.c_int, c.c_int, P]
        L.orc_decode_values.restype = None
        L.orc_decode_values.argtypes = [c.c_int64, c.c_int, P, P, P]
        L.orc_tree_logits.restype = None
        L.orc_tree_logits.argtypes = [c.c_int64, c.c_int, P, P, P, c.c_int, c.c_int, P, P]
        L.orc_attention.restype = None
        L.orc_attention.argtypes = [c.c_int64, c.c_int, P, P, c.c_int, P, P, P]
        L.orc_pack_token.restype = None
        L.orc_pack_token.argtypes = [c.c_int, c.c_int, P, P, c.c_uint16, c.c_uint16, P, P]
        L.orc_unpack_token.restype = None
        L.orc_unpack_token.argtypes = [c.c_int, c.c_int, P, P, P, P, P, P]
        L.orc_pack_tokens.restype = None
        L.orc_pack_tokens.argtypes = [c.c_int64, c.c_int, P, P, P, P, P, P, P, P]
        L.orc_build_page_table.restype = None
        L.orc_build_page_table.argtypes = [c.c_int64, P, P, P, P, P]
        L.orc_cache_attention.restype = c.c_int
        L.orc_cache_attention.argtypes = [c.c_int, c.c_int, c.c_int, c.c_int64, P, P, P, P, P, P,
                                          P, P, c.c_int, P, P, P, P]
        L.orc_rdr_assign.restype = c.c_int
        L.orc_rdr_assign.argtypes = [c.c_int, c.c_int, c.c_int64, P, P, P, P, c.c_int64,
                                     c.c_int, c.c_int, P, P, P]
        L.orc_rdr_rerun.restype = c.c_int
        L.orc_rdr_rerun.argtypes = [c.c_int, c.c_int, c.c_int64, P, P, P, P, c.c_int64,
                                    c.c_int, c.c_int, P, P, P]
        L.orc_transcode_token.restype = None
        L.orc_transcode_token.argtypes = [c.c_int, c.c_int, P, P, c.c_uint16, P, P, P, P, P]
        L.orc_migrate.restype = c.c_int
        L.orc_migrate.argtypes = [c.c_int, c.c_int, c.c_int64, P, P, P, P, P, P, P, P, P, P, P, P]
        L.orc_set_keep.restype = c.c_int
        L.orc_set_keep.argtypes = [c.c_int, c.c_int, c.c_int64, P, P, P, P, P, P, P, P]
        L.orc_merge_partials.restype = None
        L.orc_merge_partials.argtypes = [c.c_int, c.c_int64, c.c_int, P, P, P, P]
        L.orc_num_threads.restype = c.c_int
        L.orc_num_threads.argtypes = []
        _lib = L
    return _lib


def _p(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"], "arrays passed to the oracle must be C-contiguous"
    return a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def num_threads() -> int:
    return int(lib().orc_num_threads())


def page_bytes(tier: int) -> int:
    return int(lib().orc_page_bytes(tier))


def f64_to_f16_bits(x: float) -> int:
    return int(lib().orc_f64_to_f16(float(x)))


def f16_bits_to_f64(h: int) -> float:
    return float(lib().orc_f16_to_f64(int(h)))


def encode(K, V, tier: int = None, bits=None):
    """Encode rows of K and V ([n, d] each, any float dtype, converted exactly
    to fp64).  Returns dict(leaf [n, d/2] u8, up [n, d/2-1] u8, r16 [n] u16,
    s16 [n] u16, vq [n, d] i8, n_overflow)."""
    b_leaf, b_up, v_bits = bits if bits is not None else TIER_BITS[tier]
    K = _c(K, np.float64)
    V = _c(V, np.float64)
    n, d = K.shape
    leaf = np.zeros((n, d // 2), np.uint8)
    up = np.zeros((n, max(d // 2 - 1, 0)), np.uint8)
    r16 = np.zeros(n, np.uint16)
    s16 = np.zeros(n, np.uint16)
    vq = np.zeros((n, d), np.int8)
    bad = lib().orc_encode_tokens(n, d, _p(K), _p(V), b_leaf, b_up, v_bits, _p(leaf), _p(up),
                                  _p(r16), _p(s16), _p(vq))
    return dict(leaf=leaf, up=up, r16=r16, s16=s16, vq=vq, n_overflow=int(bad))


def decode_keys(leaf, up, r16, b_leaf, b_up):
    leaf = _c(leaf, np.uint8)
    up = _c(up, np.uint8)
    r16 = _c(r16, np.uint16)
    n, L = leaf.shape
    d = 2 * L
    out = np.zeros((n, d), np.float64)
    lib().orc_decode_keys(n, d, _p(leaf), _p(up), _p(r16), b_leaf, b_up, _p(out))
    return out


def decode_values(vq, s16):
    vq = _c(vq, np.int8)
    s16 = _c(s16, np.uint16)
    n, d = vq.shape
    out = np.zeros((n, d), np.float64)
    lib().orc_decode_values(n, d, _p(vq), _p(s16), _p(out))
    return out


def tree_logits(leaf, up, r16, b_leaf, b_up, q):
    leaf = _c(leaf, np.uint8)
    up = _c(up, np.uint8)
    r16 = _c(r16, np.uint16)
    q = _c(q, np.float64)
    n, L = leaf.shape
    out = np.zeros(n, np.float64)
    lib().orc_tree_logits(n, 2 * L, _p(leaf), _p(up), _p(r16), b_leaf, b_up, _p(q), _p(out))
    return out


def attention(khat, vhat, q):
    """Dense softmax attention of q [n_q, d] over all rows of khat/vhat."""
    khat = _c(khat, np.float64)
    vhat = _c(vhat, np.float64)
    q = _c(np.atleast_2d(q), np.float64)
    n_q, d = q.shape
    n = khat.shape[0] if khat.size else 0
    if n == 0:
        khat = np.zeros((1, d))
        vhat = np.zeros((1, d))
    out = np.zeros((n_q, d), np.float64)
    lse = np.zeros(n_q, np.float64)
    lib().orc_attention(n, d, _p(khat), _p(vhat), n_q, _p(q), _p(out), _p(lse))
    return out, lse


def set_keep(cache, keep):
    """Per-token keep/drop: keep [H_kv, total_pages * 16] (nonzero = keep), in
    RDR's utility layout.  Sets (drop) or clears (keep) the drop flag, the sign
    bit of the stored radius, of every present token of every kept page of the
    cache dict's pools, in place.  Dropped tokens are then skipped by
    cache_attention exactly as if deleted."""
    po = _c(cache["page_offsets"], np.int32)
    sl = _c(cache["seq_lens"], np.int32)
    pt = _c(cache["page_table"], np.int32)
    H_kv, total_pages = pt.shape
    keep = _c(keep, np.uint8)
    assert keep.shape == (H_kv, total_pages * PAGE)
    pools = cache["pools"]
    flat = []
    for t, p in enumerate(pools):
        assert p.flags["C_CONTIGUOUS"] and p.dtype == np.uint8
        flat.append(p if p.size else np.zeros((1, page_bytes(t + 1)), np.uint8))
    pool_pages = np.array([p.shape[0] if p.size else 0 for p in pools], np.int64)
    st = lib().orc_set_keep(sl.size, H_kv, total_pages, _p(po), _p(sl), _p(pt), _p(flat[0]), _p(flat[1]),
                            _p(flat[2]), _p(pool_pages), _p(keep))
    if st != 0:
        raise ValueError(f"oracle set_keep status {st}")


def merge_partials(out_parts, lse_parts):
    """Log-sum-exp combine of attention results over disjoint key sets:
    out_parts [n_parts, ..., d], lse_parts [n_parts, ...].  Returns (out, lse)
    of attention over the union of the parts' keys."""
    op = _c(out_parts, np.float64)
    lp = _c(lse_parts, np.float64)
    n_parts = op.shape[0]
    d = op.shape[-1]
    n_rows = int(np.prod(lp.shape[1:], dtype=np.int64))
    out = np.zeros(op.shape[1:], np.float64)
    lse = np.zeros(lp.shape[1:], np.float64)
    lib().orc_merge_partials(n_parts, n_rows, d, _p(op), _p(lp), _p(out), _p(lse))
    return out, lse


def pack_token(tier, slot, leaf, up, r16, s16, vq, page):
    lib().orc_pack_token(tier, slot, _p(_c(leaf, np.uint8)), _p(_c(up, np.uint8)), int(r16),
                         int(s16), _p(_c(vq, np.int8)), _p(page))


def unpack_token(tier, slot, page):
    leaf = np.zeros(D // 2, np.uint8)
    up = np.zeros(D // 2 - 1, np.uint8)
    r16 = np.zeros(1, np.uint16)
    s16 = np.zeros(1, np.uint16)
    vq = np.zeros(D, np.int8)
    lib().orc_unpack_token(tier, slot, _p(_c(page, np.uint8)), _p(leaf), _p(up), _p(r16),
                           _p(s16), _p(vq))
    return dict(leaf=leaf, up=up, r16=int(r16[0]), s16=int(s16[0]), vq=vq)


def build_page_table(tiers, perms=(None, None, None)):
    """tiers: [H_kv, total_pages] u8 (0 drop, 1..3) -> int32 entries; the k-th
    page of tier t (in table order) gets pool index perms[t-1][k] (or k)."""
    tiers = _c(tiers, np.uint8)
    table = np.zeros(tiers.shape, np.int32)
    ps = [None if p is None else _c(p, np.int32) for p in perms]
    lib().orc_build_page_table(tiers.size, _p(tiers),
                               *[(None if p is None else _p(p)) for p in ps], _p(table))
    return table


def cache_attention(cache, q, units):
    """Slow decode attention over a packed cache for the (b, g) pairs in
    ``units``.  cache: dict(B, H_q, H_kv, page_offsets, seq_lens, page_table,
    pools=[p1, p2, p3]).  Returns out [n, G, 128], lse [n, G]."""
    B, H_q, H_kv = cache["B"], cache["H_q"], cache["H_kv"]
    G = H_q // H_kv
    po = _c(cache["page_offsets"], np.int32)
    sl = _c(cache["seq_lens"], np.int32)
    pt = _c(cache["page_table"], np.int32)
    total_pages = pt.shape[-1]
    pools = [_c(p, np.uint8).reshape(-1) for p in cache["pools"]]
    pool_pages = np.array([p.size // page_bytes(t + 1) for t, p in enumerate(pools)], np.int64)
    pools = [p if p.size else np.zeros(1, np.uint8) for p in pools]
    q = _c(q, np.float64)
    units = np.asarray(units, np.int32).reshape(-1, 2)
    sb = _c(units[:, 0], np.int32)
    sg = _c(units[:, 1], np.int32)
    n = units.shape[0]
    out = np.zeros((n, G, D), np.float64)
    lse = np.zeros((n, G), np.float64)
    st = lib().orc_cache_attention(B, H_q, H_kv, total_pages, _p(po), _p(sl), _p(pt), _p(pools[0]),
                                   _p(pools[1]), _p(pools[2]), _p(pool_pages), _p(q), n, _p(sb),
                                   _p(sg), _p(out), _p(lse))
    if st != 0:
        raise ValueError(f"oracle cache_attention status {st}")
    return out, lse


def multi_query_attention(cache, q, units, n_q):
    """Decode attention for n_q query tokens per sequence, q [B, n_q, H_q, 128].
    Reading (the pages describe one decode query per step; several query
    tokens per step, as in speculative or chunked decode, are this project's
    extension): query token i is causal and sees the first
    seq_len - (n_q - 1 - i) tokens, so the last one sees them all.  Each token
    is then plain single-query attention (cache_attention) over its prefix.
    Returns out [n_q, n, G, 128], lse [n_q, n, G]."""
    q = np.asarray(q)
    outs, lses = [], []
    for i in range(n_q):
        lens = np.maximum(np.asarray(cache["seq_lens"], np.int64) - (n_q - 1 - i), 0).astype(np.int32)
        o, l = cache_attention(dict(cache, seq_lens=lens), q[:, i], units)
        outs.append(o)
        lses.append(l)
    return np.stack(outs), np.stack(lses)


def rdr_assign(page_offsets, seq_lens, utility, eps, budget, n_sink, n_recent, H_kv,
               tiers_init=None):
    """Lagrangian tier assignment.  utility: [H_kv, total_pages*16] f32.
    Returns (tiers [H_kv, total_pages] u8, lambda, bytes) or raises on an
    infeasible budget."""
    po = _c(page_offsets, np.int32)
    sl = _c(seq_lens, np.int32)
    B = sl.size
    total_pages = int(po[-1])
    util = _c(utility, np.float32)
    eps = _c(eps, np.float64)
    tiers = (np.zeros((H_kv, total_pages), np.uint8) if tiers_init is None
             else _c(tiers_init, np.uint8).copy())
    lam = np.zeros(1, np.float64)
    nbytes = np.zeros(1, np.int64)
    st = lib().orc_rdr_assign(B, H_kv, total_pages, _p(po), _p(sl), _p(util), _p(eps),
                              int(budget), n_sink, n_recent, _p(tiers), _p(lam), _p(nbytes))
    if st == 3:
        raise OverflowError("forced pages alone exceed the budget")
    if st != 0:
        raise ValueError(f"oracle rdr status {st}")
    return tiers, float(lam[0]), int(nbytes[0])


def rdr_rerun(page_offsets, seq_lens, utility, eps, budget, n_sink, n_recent, tiers):
    """RDR again on a cache that already holds codes: each page may only keep
    its tier or become coarser (drop included); forced pages keep the finest
    tier allowed.  tiers: the current [H_kv, total_pages] tiers.  Returns
    (new tiers, lambda, bytes) or raises OverflowError if infeasible."""
    po = _c(page_offsets, np.int32)
    sl = _c(seq_lens, np.int32)
    util = _c(utility, np.float32)
    eps = _c(eps, np.float64)
    t = _c(tiers, np.uint8).copy()
    H_kv, total_pages = t.shape
    lam = np.zeros(1, np.float64)
    nbytes = np.zeros(1, np.int64)
    st = lib().orc_rdr_rerun(sl.size, H_kv, total_pages, _p(po), _p(sl), _p(util), _p(eps), int(budget),
                             n_sink, n_recent, _p(t), _p(lam), _p(nbytes))
    if st == 3:
        raise OverflowError("forced pages alone exceed the budget")
    if st != 0:
        raise ValueError(f"oracle rdr status {st}")
    return t, float(lam[0]), int(nbytes[0])


def transcode_token(t_from, t_to, leaf, up, s16, vq):
    """One token's codes from tier t_from to the coarser (or same) tier t_to.
    Returns dict(leaf, up, s16, vq); the radius does not change."""
    leaf2 = np.zeros(D // 2, np.uint8)
    up2 = np.zeros(D // 2 - 1, np.uint8)
    s2 = np.zeros(1, np.uint16)
    vq2 = np.zeros(D, np.int8)
    lib().orc_transcode_token(t_from, t_to, _p(_c(leaf, np.uint8)), _p(_c(up, np.uint8)), int(s16),
                              _p(_c(vq, np.int8)), _p(leaf2), _p(up2), _p(s2), _p(vq2))
    return dict(leaf=leaf2, up=up2, s16=int(s2[0]), vq=vq2)


def migrate(cache, new_table, new_counts):
    """Rewrite the cache dict's tokens into fresh pools laid out by new_table
    ([H_kv, total_pages] entries; new_counts pages per tier), transcoding the
    pages whose tier became coarser.  Returns the new pools."""
    po = _c(cache["page_offsets"], np.int32)
    sl = _c(cache["seq_lens"], np.int32)
    ot = _c(cache["page_table"], np.int32)
    nt = _c(new_table, np.int32)
    H_kv, total_pages = ot.shape
    old = [p if p.size else np.zeros((1, page_bytes(t + 1)), np.uint8) for t, p in enumerate(cache["pools"])]
    old_pages = np.array([p.shape[0] if p.size else 0 for p in cache["pools"]], np.int64)
    new = [np.zeros((int(new_counts[t]), page_bytes(t + 1)), np.uint8) for t in range(3)]
    newp = [p if p.size else np.zeros((1, page_bytes(t + 1)), np.uint8) for t, p in enumerate(new)]
    new_pages = np.array([int(c) for c in new_counts], np.int64)
    st = lib().orc_migrate(sl.size, H_kv, total_pages, _p(po), _p(sl), _p(ot), _p(old[0]), _p(old[1]), _p(old[2]),
                           _p(old_pages), _p(nt), _p(newp[0]), _p(newp[1]), _p(newp[2]), _p(new_pages))
    if st != 0:
        raise ValueError(f"oracle migrate status {st}")
    return [newp[t] if new[t].size else new[t] for t in range(3)]


def encode_cache(K, V, tok_seq, tok_pos, page_offsets, page_table, pool_pages):
    """Encode dense rows K, V [n_tok, H_kv, 128] into packed pools with the
    oracle's own encoder and packer.  Each token goes to page
    page_offsets[seq] + pos // 16, slot pos % 16, of every kv head; dropped
    pages are skipped.  Returns the three pools as [n_pages_t, page_bytes_t]."""
    K = np.asarray(K)
    V = np.asarray(V)
    n_tok, H_kv, d = K.shape
    assert d == D
    pools = [np.zeros((int(pool_pages[t]), page_bytes(t + 1)), np.uint8) for t in range(3)]
    tok_seq = np.asarray(tok_seq, np.int64)
    tok_pos = np.asarray(tok_pos, np.int64)
    lpage = np.asarray(page_offsets, np.int64)[tok_seq] + tok_pos // PAGE
    slot = tok_pos % PAGE
    for g in range(H_kv):
        ent = np.asarray(page_table)[g, lpage].astype(np.int64) & 0xFFFFFFFF
        tier = (ent >> 30).astype(np.int64)
        phys = ent & 0x3FFFFFFF
        for t in (1, 2, 3):
            idx = np.nonzero(tier == t)[0]
            if idx.size == 0:
                continue
            codes = encode(K[idx, g, :], V[idx, g, :], t)
            if codes["n_overflow"]:
                raise OverflowError("radius or value scale overflows fp16")
            dst = _c(phys[idx], np.int64)
            sl = _c(slot[idx], np.int32)
            lib().orc_pack_tokens(idx.size, t, _p(dst), _p(sl), _p(codes["leaf"]), _p(codes["up"]),
                                  _p(codes["r16"]), _p(codes["s16"]), _p(codes["vq"]),
                                  _p(pools[t - 1]))
    return pools
