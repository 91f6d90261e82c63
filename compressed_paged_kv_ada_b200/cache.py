"""PagedCache: device buffers of a tier-homogeneous paged KV cache, allocated
with torch, plus calls into libsphkv.  Plumbing only: every step of the
method (page-table construction, encode, RDR, decode attention) runs in the
CUDA library; this class allocates memory and passes pointers and streams.
"""
from __future__ import annotations

from typing import Optional, Sequence

import numpy as np
import torch

from . import _lib as L

PAGE = 16
D = 128


class PagedCache:
    def __init__(self, page_offsets, seq_lens, tiers, perms: Sequence = (None, None, None),
                 device: str = "cuda"):
        """page_offsets: [B+1] int; seq_lens: [B] int; tiers: [H_kv, total_pages]
        uint8 (0 drop, 1..3).  Pools are sized from the tier counts and zeroed;
        the page table is built on the device (k-th page of tier t in table
        order -> perms[t-1][k], or k)."""
        self.device = torch.device(device)
        tiers_np = np.ascontiguousarray(tiers, np.uint8)
        self.H_kv, self.total_pages = tiers_np.shape
        self.page_offsets = torch.as_tensor(np.asarray(page_offsets, np.int32), device=self.device)
        self.seq_lens = torch.as_tensor(np.asarray(seq_lens, np.int32), device=self.device)
        self.B = int(self.seq_lens.numel())
        self.status = torch.zeros(1, dtype=torch.int32, device=self.device)
        counts = [int((tiers_np == t).sum()) for t in (1, 2, 3)]
        self.pools = [torch.zeros((counts[t], L.sphkv_page_bytes(t + 1)), dtype=torch.uint8,
                                  device=self.device) for t in range(3)]
        self.tiers = torch.as_tensor(tiers_np, device=self.device)
        self.page_table = torch.empty((self.H_kv, self.total_pages), dtype=torch.int32, device=self.device)
        self.perms = [None if p is None else torch.as_tensor(np.asarray(p, np.int32), device=self.device)
                      for p in perms]
        self.build_page_table()
        self._ws = None

    # ------------------------------------------------------------------
    def descriptor(self) -> L.sphkv_cache:
        return L.make_cache(self.page_offsets, self.seq_lens, self.page_table, self.pools)

    def build_page_table(self):
        L.sphkv_build_page_table(self.tiers, self.page_table, self.perms, status=self.status)

    def check(self):
        """Synchronise and raise if a kernel reported a device-side error."""
        torch.cuda.synchronize(self.device)
        code = int(self.status.item())
        if code:
            self.status.zero_()
            raise L.SphkvError("device", code)

    def encode(self, K: torch.Tensor, V: torch.Tensor, tok_seq: torch.Tensor, tok_pos: torch.Tensor):
        L.sphkv_encode(self.descriptor(), K, V, tok_seq, tok_pos, status=self.status)

    def set_keep(self, keep: torch.Tensor):
        """Per-token keep/drop flags: keep [H_kv, total_pages * 16] uint8
        (nonzero = keep), in the layout of RDR's utility."""
        L.sphkv_set_keep(self.descriptor(), keep, status=self.status)

    def workspace(self, H_q: int) -> torch.Tensor:
        n = L.sphkv_decode_workspace_bytes(self.B, H_q, self.H_kv, self.total_pages)
        if self._ws is None or self._ws.numel() < n:
            self._ws = torch.empty(n, dtype=torch.uint8, device=self.device)
        return self._ws

    def decode(self, q: torch.Tensor, out: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None):
        B, H_q, d = q.shape
        out = torch.empty((B, H_q, d), dtype=torch.float32, device=self.device) if out is None else out
        lse = torch.empty((B, H_q), dtype=torch.float32, device=self.device) if lse is None else lse
        L.sphkv_decode_attention(self.descriptor(), H_q, q, out, lse, self.workspace(H_q), status=self.status)
        return out, lse

    def decode_mq(self, q: torch.Tensor, out: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None):
        """Decode for n_q causal query tokens per sequence: q [B, n_q, H_q, 128];
        query token i sees the first seq_len - (n_q - 1 - i) tokens."""
        B, n_q, H_q, d = q.shape
        out = torch.empty((B, n_q, H_q, d), dtype=torch.float32, device=self.device) if out is None else out
        lse = torch.empty((B, n_q, H_q), dtype=torch.float32, device=self.device) if lse is None else lse
        n = L.sphkv_decode_mq_workspace_bytes(self.B, H_q, self.H_kv, self.total_pages)
        if self._ws is None or self._ws.numel() < n:
            self._ws = torch.empty(n, dtype=torch.uint8, device=self.device)
        L.sphkv_decode_attention_mq(self.descriptor(), n_q, H_q, q, out, lse, self._ws, status=self.status)
        return out, lse

    def rdr_assign(self, utility: torch.Tensor, eps, budget: int, n_sink: int, n_recent: int):
        """Choose tiers by RDR (on the device) and write them into self.tiers.
        Returns (lambda, bytes) as device tensors."""
        ws = torch.empty(L.sphkv_rdr_workspace_bytes(self.B, self.H_kv, self.total_pages),
                         dtype=torch.uint8, device=self.device)
        lam = torch.zeros(1, dtype=torch.float64, device=self.device)
        nbytes = torch.zeros(1, dtype=torch.int64, device=self.device)
        L.sphkv_rdr_assign(self.descriptor(), utility, eps, budget, n_sink, n_recent, self.tiers, lam,
                           nbytes, ws, status=self.status)
        return lam, nbytes

    def rdr_rerun(self, utility: torch.Tensor, eps, budget: int, n_sink: int, n_recent: int):
        """RDR again on the grown cache, each page capped at its current tier,
        then the tokens transcoded into new, compacted pools (sphkv_rdr_rerun,
        sphkv_build_page_table, sphkv_migrate).  Returns (lambda, bytes) as
        device tensors; self.tiers, page_table and pools are replaced."""
        ws = torch.empty(L.sphkv_rdr_workspace_bytes(self.B, self.H_kv, self.total_pages),
                         dtype=torch.uint8, device=self.device)
        lam = torch.zeros(1, dtype=torch.float64, device=self.device)
        nbytes = torch.zeros(1, dtype=torch.int64, device=self.device)
        new_tiers = self.tiers.clone()
        L.sphkv_rdr_rerun(self.descriptor(), utility, eps, budget, n_sink, n_recent, new_tiers, lam, nbytes, ws,
                          status=self.status)
        self.check()
        old = self.descriptor()
        old_keep = (self.pools, self.page_table)   # alive until the migration has run
        counts = [int((new_tiers == t).sum().item()) for t in (1, 2, 3)]
        self.tiers = new_tiers
        self.pools = [torch.zeros((counts[t], L.sphkv_page_bytes(t + 1)), dtype=torch.uint8,
                                  device=self.device) for t in range(3)]
        self.page_table = torch.empty((self.H_kv, self.total_pages), dtype=torch.int32, device=self.device)
        self.perms = [None, None, None]
        self.build_page_table()
        L.sphkv_migrate(old, self.descriptor(), status=self.status)
        self.check()
        del old_keep
        return lam, nbytes

    def reallocate_pools(self):
        """Size the pools for the current tiers (after RDR) and rebuild the
        page table; pool contents are reset to zero."""
        counts = [int((self.tiers == t).sum().item()) for t in (1, 2, 3)]
        self.pools = [torch.zeros((counts[t], L.sphkv_page_bytes(t + 1)), dtype=torch.uint8,
                                  device=self.device) for t in range(3)]
        self.perms = [None, None, None]
        self.build_page_table()

    def compressed_bytes(self) -> int:
        """Stored page bytes of pages that hold tokens (host view of tiers)."""
        tiers = self.tiers.cpu().numpy()
        po = self.page_offsets.cpu().numpy()
        lens = self.seq_lens.cpu().numpy()
        size = np.array([0] + [L.sphkv_page_bytes(t) for t in (1, 2, 3)], np.int64)
        tot = 0
        for b in range(self.B):
            n = (int(lens[b]) + PAGE - 1) // PAGE
            tot += int(size[tiers[:, po[b]:po[b] + n]].sum())
        return tot
