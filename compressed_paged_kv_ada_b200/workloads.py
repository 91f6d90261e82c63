"""Seeded synthetic inputs for ADA decode over a paged, tier-homogeneous cache.

This module holds random draws and index bookkeeping only (sequence lengths,
page offsets, token positions, tier draws, pool permutations, utilities).  It
contains none of the method's arithmetic, so both the CUDA path and the CPU
oracle can take their inputs from it.

Every stream is a numpy Generator seeded by SeedSequence([seed, cfg, stream,
...]); dense K/V rows are drawn in blocks of 4096 tokens per sequence so that
any slice can be regenerated on its own.

Workloads (the shapes of the published configurations of the method's decode
path, all synthetic: no dataset or trained weight is involved):
  tiny       B 1, 4 q / 1 kv heads, ctx 2048, every page T1, fp32 K/V
  llama32k   B 8, 32 / 8 heads, ctx 32768, tier mix, bf16 K/V (headline)
  ragged64   B 64, ctx ~ U{1024..16384}, tier mix, permuted pool ids
  long512k   B 1, ctx 524288, tier mix (split-KV over the SMs)
  e2e_rdr    B 16, ctx 32768 prefill, RDR at 25 % of fp16 bytes, 256 appends
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import Optional, Sequence

import numpy as np

D = 128
PAGE = 16
BLOCK = 4096
# Categorical tier draw for the mixed workloads: T1, T2, T3, drop.
TIER_MIX = (0.20, 0.40, 0.25, 0.15)
N_SINK, N_RECENT = 4, 8

_STREAM = dict(sigma=0, outlier=1, k=2, v=3, q=4, tier=5, lens=6, perm=7, util=8)


def _rng(seed: int, cfg: int, stream: str, *extra: int) -> np.random.Generator:
    return np.random.default_rng(np.random.SeedSequence([seed, cfg, _STREAM[stream], *extra]))


def round_to_bf16(x: np.ndarray) -> np.ndarray:
    """Round fp32 values to the nearest bf16 (ties to even); returned as fp32."""
    import torch

    return torch.from_numpy(np.ascontiguousarray(x, np.float32)).to(torch.bfloat16).float().numpy()


@dataclass
class Workload:
    name: str
    cfg: int
    B: int
    H_q: int
    H_kv: int
    dtype: str                      # "bf16" or "fp32": dtype of dense K/V
    seq_lens: np.ndarray            # int32 [B]: tokens present now
    cap_pages: np.ndarray           # int32 [B]: logical pages reserved per sequence
    tiers: np.ndarray               # uint8 [H_kv, total_pages]: 0 drop, 1..3
    permute_pools: bool = False
    n_outlier: int = 4
    seed: int = 0
    extra: dict = field(default_factory=dict)

    d: int = D

    # ------------------------------------------------------------ layout --
    @property
    def page_offsets(self) -> np.ndarray:
        return np.concatenate([[0], np.cumsum(self.cap_pages)]).astype(np.int32)

    @property
    def total_pages(self) -> int:
        return int(self.cap_pages.sum())

    @property
    def n_pages(self) -> np.ndarray:
        """Pages that hold tokens, per sequence."""
        return ((self.seq_lens.astype(np.int64) + PAGE - 1) // PAGE).astype(np.int32)

    def token_index(self, lens: Optional[np.ndarray] = None):
        """(tok_seq, tok_pos) for every present token, sequence-major."""
        lens = self.seq_lens if lens is None else lens
        seq = np.repeat(np.arange(self.B, dtype=np.int32), lens)
        starts = np.concatenate([[0], np.cumsum(lens)[:-1]]).astype(np.int64)
        pos = (np.arange(int(np.sum(lens)), dtype=np.int64) - np.repeat(starts, lens)).astype(np.int32)
        return seq, pos

    def pool_counts(self) -> np.ndarray:
        """Number of pages of each tier (T1, T2, T3) in the page table."""
        return np.array([(self.tiers == t).sum() for t in (1, 2, 3)], np.int64)

    def pool_perms(self):
        """Per tier, the pool index of the k-th page of that tier (table
        order), or None for the identity."""
        if not self.permute_pools:
            return (None, None, None)
        r = _rng(self.seed, self.cfg, "perm")
        return tuple(r.permutation(int(c)).astype(np.int32) for c in self.pool_counts())

    # ------------------------------------------------------------- draws --
    def sigma(self) -> np.ndarray:
        """Per (kv head, channel) std of K: LogNormal(0, 0.5), outliers x8."""
        s = _rng(self.seed, self.cfg, "sigma").lognormal(0.0, 0.5, size=(self.H_kv, D))
        if self.n_outlier:
            r = _rng(self.seed, self.cfg, "outlier")
            for g in range(self.H_kv):
                s[g, r.choice(D, self.n_outlier, replace=False)] *= 8.0
        return s.astype(np.float32)

    def dense_rows(self, b: int, t0: int, t1: int):
        """Dense K, V rows [t1-t0, H_kv, 128] (fp32 holding exact bf16 values
        for bf16 workloads) for positions t0..t1-1 of sequence b."""
        sig = self.sigma()
        ks, vs = [], []
        for blk in range(t0 // BLOCK, (t1 + BLOCK - 1) // BLOCK):
            rk = _rng(self.seed, self.cfg, "k", b, blk)
            rv = _rng(self.seed, self.cfg, "v", b, blk)
            k = rk.standard_normal((BLOCK, self.H_kv, D), dtype=np.float32) * sig[None]
            v = rv.standard_normal((BLOCK, self.H_kv, D), dtype=np.float32)
            lo = max(t0, blk * BLOCK) - blk * BLOCK
            hi = min(t1, (blk + 1) * BLOCK) - blk * BLOCK
            ks.append(k[lo:hi])
            vs.append(v[lo:hi])
        K = np.concatenate(ks) if ks else np.zeros((0, self.H_kv, D), np.float32)
        V = np.concatenate(vs) if vs else np.zeros((0, self.H_kv, D), np.float32)
        if self.dtype == "bf16":
            K, V = round_to_bf16(K), round_to_bf16(V)
        return np.ascontiguousarray(K), np.ascontiguousarray(V)

    def dense(self, lens: Optional[np.ndarray] = None):
        """All present tokens, sequence-major: K, V [sum(lens), H_kv, 128]."""
        lens = self.seq_lens if lens is None else lens
        parts = [self.dense_rows(b, 0, int(lens[b])) for b in range(self.B)]
        K = np.concatenate([p[0] for p in parts])
        V = np.concatenate([p[1] for p in parts])
        return K, V

    def queries(self, step: int = 0) -> np.ndarray:
        """q [B, H_q, 128] fp32 ~ N(0, 1); step > 0 gives later decode steps."""
        return _rng(self.seed, self.cfg, "q", step).standard_normal((self.B, self.H_q, D), dtype=np.float32)

    def utility(self, lens: Optional[np.ndarray] = None) -> np.ndarray:
        """Per token and kv head utility [H_kv, total_pages*16] f32:
        LogNormal(0, 1) / (1 + age/4096), age = len - 1 - position; slots
        without a token are 0.  The LogNormal draw of a slot does not depend
        on len (one draw per reserved slot), so utilities stay consistent as
        a sequence grows; only the age term changes."""
        lens = self.seq_lens if lens is None else np.asarray(lens)
        out = np.zeros((self.H_kv, self.total_pages * PAGE), np.float32)
        po = self.page_offsets
        for b in range(self.B):
            n = int(lens[b])
            r = _rng(self.seed, self.cfg, "util", b)
            u = r.lognormal(0.0, 1.0, size=(self.H_kv, int(self.cap_pages[b]) * PAGE))[:, :n]
            age = (n - 1 - np.arange(n)).astype(np.float64)
            out[:, po[b] * PAGE: po[b] * PAGE + n] = (u / (1.0 + age / 4096.0)).astype(np.float32)
        return out


def draw_tiers(seed: int, cfg: int, H_kv: int, seq_lens, cap_pages, mix=TIER_MIX,
               all_t1: bool = False) -> np.ndarray:
    """Tier per (kv head, logical page): categorical draw with the first
    N_SINK and last N_RECENT token-holding pages forced to T1; reserved pages
    beyond the tokens are T1 (appends land there)."""
    cap_pages = np.asarray(cap_pages, np.int64)
    po = np.concatenate([[0], np.cumsum(cap_pages)])
    tiers = np.ones((H_kv, int(po[-1])), np.uint8)
    if all_t1:
        return tiers
    r = _rng(seed, cfg, "tier")
    choices = np.array([1, 2, 3, 0], np.uint8)
    for b in range(len(cap_pages)):
        n = int((int(seq_lens[b]) + PAGE - 1) // PAGE)
        draw = choices[r.choice(4, size=(H_kv, n), p=np.asarray(mix))]
        draw[:, :min(N_SINK, n)] = 1
        draw[:, max(0, n - N_RECENT):] = 1
        tiers[:, po[b]: po[b] + n] = draw
    return tiers


def make(name: str, seed: int = 0, *, B: Optional[int] = None, ctx: Optional[int] = None,
         H_q: Optional[int] = None, H_kv: Optional[int] = None,
         seq_lens: Optional[Sequence[int]] = None, extra_pages: int = 0,
         mix=TIER_MIX, dtype: Optional[str] = None) -> Workload:
    """Build a named workload; the keyword arguments shrink it for tests."""
    spec = {
        "tiny": dict(cfg=0, B=1, H_q=4, H_kv=1, ctx=2048, dtype="fp32", all_t1=True, n_outlier=0),
        "llama32k": dict(cfg=1, B=8, H_q=32, H_kv=8, ctx=32768, dtype="bf16"),
        "ragged64": dict(cfg=2, B=64, H_q=32, H_kv=8, ctx=None, dtype="bf16", permute=True),
        "long512k": dict(cfg=3, B=1, H_q=32, H_kv=8, ctx=524288, dtype="bf16"),
        "e2e_rdr": dict(cfg=4, B=16, H_q=32, H_kv=8, ctx=32768, dtype="bf16", steps=256),
    }[name]
    cfg = spec["cfg"]
    Bv = B if B is not None else spec["B"]
    Hq = H_q if H_q is not None else spec["H_q"]
    Hkv = H_kv if H_kv is not None else spec["H_kv"]
    if seq_lens is not None:
        lens = np.asarray(seq_lens, np.int32)
        Bv = lens.size
    elif spec["ctx"] is None and ctx is None:
        lens = _rng(seed, cfg, "lens").integers(1024, 16384, size=Bv, endpoint=True).astype(np.int32)
    else:
        lens = np.full(Bv, ctx if ctx is not None else spec["ctx"], np.int32)
    if name == "e2e_rdr" and extra_pages == 0:
        extra_pages = (spec["steps"] + PAGE - 1) // PAGE
    cap = ((lens.astype(np.int64) + PAGE - 1) // PAGE + extra_pages).astype(np.int32)
    tiers = draw_tiers(seed, cfg, Hkv, lens, cap, mix=mix, all_t1=spec.get("all_t1", False))
    w = Workload(name=name, cfg=cfg, B=Bv, H_q=Hq, H_kv=Hkv, dtype=dtype or spec["dtype"],
                 seq_lens=lens, cap_pages=cap, tiers=tiers,
                 permute_pools=spec.get("permute", False),
                 n_outlier=spec.get("n_outlier", 4), seed=seed)
    if name == "e2e_rdr":
        w.extra["steps"] = spec["steps"]
        w.extra["budget"] = int(0.25 * (2 * D * 2) * Hkv * int(lens.sum()))
    return w
