"""ctypes binding of libsphkv (include/sphkv.h): argument marshalling only.

Every entry point keeps the C name.  Tensors are torch CUDA tensors; their
device pointers and the current CUDA stream are passed straight through.
There is no fallback: if libsphkv.so is missing or a call fails, an exception
is raised.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libsphkv.so")

OK, ERR_ARG, ERR_RANGE, ERR_BUDGET, ERR_DEVICE, ERR_TIMEOUT, ERR_DATA = range(7)
STATUS_NAMES = {0: "OK", 1: "ERR_ARG", 2: "ERR_RANGE", 3: "ERR_BUDGET", 4: "ERR_DEVICE",
                5: "ERR_TIMEOUT", 6: "ERR_DATA"}
DTYPE_F32, DTYPE_BF16 = 0, 1


class SphkvError(RuntimeError):
    def __init__(self, fn: str, code: int, msg: str = ""):
        super().__init__(f"{fn}: {STATUS_NAMES.get(code, code)} {msg}".strip())
        self.code = code


class sphkv_cache(ctypes.Structure):
    _fields_ = [
        ("B", ctypes.c_int32),
        ("H_kv", ctypes.c_int32),
        ("total_pages", ctypes.c_int64),
        ("page_offsets", ctypes.c_void_p),
        ("seq_lens", ctypes.c_void_p),
        ("page_table", ctypes.c_void_p),
        ("pool", ctypes.c_void_p * 3),
        ("pool_pages", ctypes.c_int64 * 3),
    ]


_lib = None
_EXPORTS = ("sphkv_page_bytes", "sphkv_last_error", "sphkv_encode", "sphkv_rdr_workspace_bytes",
            "sphkv_rdr_assign", "sphkv_build_page_table", "sphkv_decode_workspace_bytes",
            "sphkv_decode_attention", "sphkv_decode_attention_noalloc", "sphkv_decode_mq_workspace_bytes",
            "sphkv_decode_attention_mq", "sphkv_merge_partials", "sphkv_set_keep", "sphkv_rdr_rerun",
            "sphkv_migrate")


def lib() -> ctypes.CDLL:
    """Load libsphkv.so (built in-tree by compressed_paged_kv_ada_b200.build)."""
    global _lib
    if _lib is None:
        _lib = load(LIB_PATH)
    return _lib


def load(path: str) -> ctypes.CDLL:
    """Open a build of the library at `path` with the C signatures declared."""
    if not os.path.exists(path):
        raise ImportError(f"{path} is missing: run `python -m compressed_paged_kv_ada_b200.build`")
    L = ctypes.CDLL(path)
    c, P = ctypes, ctypes.c_void_p
    L.sphkv_page_bytes.restype = c.c_int
    L.sphkv_page_bytes.argtypes = [c.c_int]
    L.sphkv_last_error.restype = c.c_char_p
    L.sphkv_last_error.argtypes = []
    L.sphkv_encode.restype = c.c_int
    L.sphkv_encode.argtypes = [c.POINTER(sphkv_cache), P, P, c.c_int, P, P, c.c_int64, P, P]
    L.sphkv_rdr_workspace_bytes.restype = c.c_size_t
    L.sphkv_rdr_workspace_bytes.argtypes = [c.c_int32, c.c_int32, c.c_int64]
    L.sphkv_rdr_assign.restype = c.c_int
    L.sphkv_rdr_assign.argtypes = [c.POINTER(sphkv_cache), P, c.POINTER(c.c_double), c.c_int64,
                                   c.c_int32, c.c_int32, P, P, P, P, c.c_size_t, P, P]
    L.sphkv_build_page_table.restype = c.c_int
    L.sphkv_build_page_table.argtypes = [P, c.c_int64, P, P, P, P, P, P, P]
    L.sphkv_decode_workspace_bytes.restype = c.c_size_t
    L.sphkv_decode_workspace_bytes.argtypes = [c.c_int32, c.c_int32, c.c_int32, c.c_int64, c.c_int32]
    L.sphkv_decode_attention.restype = c.c_int
    L.sphkv_decode_attention.argtypes = [c.POINTER(sphkv_cache), c.c_int32, P, P, P, P, c.c_size_t,
                                         P, P]
    L.sphkv_decode_attention_noalloc.restype = c.c_int
    L.sphkv_decode_attention_noalloc.argtypes = [c.POINTER(sphkv_cache), c.c_int32, P, P, P, P, P]
    L.sphkv_decode_mq_workspace_bytes.restype = c.c_size_t
    L.sphkv_decode_mq_workspace_bytes.argtypes = [c.c_int32, c.c_int32, c.c_int32, c.c_int64, c.c_int32]
    L.sphkv_decode_attention_mq.restype = c.c_int
    L.sphkv_decode_attention_mq.argtypes = [c.POINTER(sphkv_cache), c.c_int32, c.c_int32, P, P, P, P,
                                            c.c_size_t, P, P]
    L.sphkv_rdr_rerun.restype = c.c_int
    L.sphkv_rdr_rerun.argtypes = L.sphkv_rdr_assign.argtypes
    L.sphkv_migrate.restype = c.c_int
    L.sphkv_migrate.argtypes = [c.POINTER(sphkv_cache), c.POINTER(sphkv_cache), P, P]
    L.sphkv_set_keep.restype = c.c_int
    L.sphkv_set_keep.argtypes = [c.POINTER(sphkv_cache), P, P, P]
    L.sphkv_merge_partials.restype = c.c_int
    L.sphkv_merge_partials.argtypes = [P, P, c.c_int32, c.c_int64, P, P, P]
    return L


def _check(fn: str, code: int):
    if code != OK:
        raise SphkvError(fn, code, lib().sphkv_last_error().decode())


def _ptr(t: Optional[torch.Tensor], dtype=None, name: str = "tensor"):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    return ctypes.c_void_p(t.data_ptr()) if t.numel() else None


def _stream(stream) -> ctypes.c_void_p:
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def make_cache(page_offsets: torch.Tensor, seq_lens: torch.Tensor, page_table: torch.Tensor,
               pools: Sequence[torch.Tensor]) -> sphkv_cache:
    """C descriptor of a cache whose buffers are torch CUDA tensors.
    pools[t-1] is a uint8 tensor of shape [n_pages, page_bytes(t)]."""
    c = sphkv_cache()
    c.B = int(seq_lens.numel())
    c.H_kv = int(page_table.shape[0])
    c.total_pages = int(page_table.shape[1])
    c.page_offsets = _ptr(page_offsets, torch.int32, "page_offsets")
    c.seq_lens = _ptr(seq_lens, torch.int32, "seq_lens")
    c.page_table = _ptr(page_table, torch.int32, "page_table")
    for t in range(3):
        pool = pools[t]
        c.pool[t] = _ptr(pool, torch.uint8, f"pool[{t}]")
        c.pool_pages[t] = int(pool.shape[0]) if pool.numel() else 0
    return c


def sphkv_page_bytes(tier: int) -> int:
    return int(lib().sphkv_page_bytes(tier))


def sphkv_encode(cache: sphkv_cache, K: torch.Tensor, V: torch.Tensor, tok_seq: torch.Tensor,
                 tok_pos: torch.Tensor, status: Optional[torch.Tensor] = None, stream=None):
    if K.dtype not in (torch.float32, torch.bfloat16) or V.dtype != K.dtype:
        raise ValueError("K and V must both be float32 or bfloat16")
    dt = DTYPE_BF16 if K.dtype == torch.bfloat16 else DTYPE_F32
    _check("sphkv_encode", lib().sphkv_encode(
        ctypes.byref(cache), _ptr(K, name="K"), _ptr(V, name="V"), dt,
        _ptr(tok_seq, torch.int32, "tok_seq"), _ptr(tok_pos, torch.int32, "tok_pos"),
        int(tok_seq.numel()), _ptr(status, torch.int32, "status"), _stream(stream)))


def sphkv_rdr_workspace_bytes(B: int, H_kv: int, total_pages: int) -> int:
    return int(lib().sphkv_rdr_workspace_bytes(B, H_kv, total_pages))


def sphkv_rdr_assign(cache: sphkv_cache, utility: torch.Tensor, eps: Sequence[float], budget: int,
                     n_sink: int, n_recent: int, tiers_out: torch.Tensor, lambda_out: torch.Tensor,
                     bytes_out: torch.Tensor, workspace: torch.Tensor,
                     status: Optional[torch.Tensor] = None, stream=None):
    e = (ctypes.c_double * 4)(*[float(x) for x in eps])
    _check("sphkv_rdr_assign", lib().sphkv_rdr_assign(
        ctypes.byref(cache), _ptr(utility, torch.float32, "utility"), e, int(budget), int(n_sink),
        int(n_recent), _ptr(tiers_out, torch.uint8, "tiers_out"),
        _ptr(lambda_out, torch.float64, "lambda_out"), _ptr(bytes_out, torch.int64, "bytes_out"),
        _ptr(workspace, torch.uint8, "workspace"), int(workspace.numel()),
        _ptr(status, torch.int32, "status"), _stream(stream)))


def sphkv_rdr_rerun(cache: sphkv_cache, utility: torch.Tensor, eps: Sequence[float], budget: int,
                    n_sink: int, n_recent: int, tiers_io: torch.Tensor, lambda_out: torch.Tensor,
                    bytes_out: torch.Tensor, workspace: torch.Tensor,
                    status: Optional[torch.Tensor] = None, stream=None):
    e = (ctypes.c_double * 4)(*[float(x) for x in eps])
    _check("sphkv_rdr_rerun", lib().sphkv_rdr_rerun(
        ctypes.byref(cache), _ptr(utility, torch.float32, "utility"), e, int(budget), int(n_sink),
        int(n_recent), _ptr(tiers_io, torch.uint8, "tiers_io"),
        _ptr(lambda_out, torch.float64, "lambda_out"), _ptr(bytes_out, torch.int64, "bytes_out"),
        _ptr(workspace, torch.uint8, "workspace"), int(workspace.numel()),
        _ptr(status, torch.int32, "status"), _stream(stream)))


def sphkv_migrate(src: sphkv_cache, dst: sphkv_cache, status: Optional[torch.Tensor] = None, stream=None):
    _check("sphkv_migrate", lib().sphkv_migrate(ctypes.byref(src), ctypes.byref(dst),
                                                _ptr(status, torch.int32, "status"), _stream(stream)))


def sphkv_build_page_table(tiers: torch.Tensor, table: torch.Tensor, perms=(None, None, None),
                           counts: Optional[torch.Tensor] = None, status: Optional[torch.Tensor] = None,
                           stream=None):
    p = [_ptr(x, torch.int32, "perm") for x in perms]
    _check("sphkv_build_page_table", lib().sphkv_build_page_table(
        _ptr(tiers, torch.uint8, "tiers"), int(tiers.numel()), p[0], p[1], p[2],
        _ptr(table, torch.int32, "table"), _ptr(counts, torch.int64, "counts"),
        _ptr(status, torch.int32, "status"), _stream(stream)))


def sphkv_decode_workspace_bytes(B: int, H_q: int, H_kv: int, total_pages: int, n_sm: int = 0) -> int:
    return int(lib().sphkv_decode_workspace_bytes(B, H_q, H_kv, total_pages, n_sm))


def sphkv_decode_attention(cache: sphkv_cache, H_q: int, q: torch.Tensor, out: torch.Tensor,
                           lse: torch.Tensor, workspace: torch.Tensor,
                           status: Optional[torch.Tensor] = None, stream=None):
    _check("sphkv_decode_attention", lib().sphkv_decode_attention(
        ctypes.byref(cache), int(H_q), _ptr(q, torch.float32, "q"), _ptr(out, torch.float32, "out"),
        _ptr(lse, torch.float32, "lse"), _ptr(workspace, torch.uint8, "workspace"),
        int(workspace.numel()), _ptr(status, torch.int32, "status"), _stream(stream)))


def sphkv_decode_attention_noalloc(cache: sphkv_cache, H_q: int, q: torch.Tensor, out: torch.Tensor,
                                   lse: torch.Tensor, status: Optional[torch.Tensor] = None, stream=None):
    """Decode attention with the library's static scratch instead of a
    caller workspace, for callers that cannot allocate device memory."""
    _check("sphkv_decode_attention_noalloc", lib().sphkv_decode_attention_noalloc(
        ctypes.byref(cache), int(H_q), _ptr(q, torch.float32, "q"), _ptr(out, torch.float32, "out"),
        _ptr(lse, torch.float32, "lse"), _ptr(status, torch.int32, "status"), _stream(stream)))


def sphkv_decode_mq_workspace_bytes(B: int, H_q: int, H_kv: int, total_pages: int, n_sm: int = 0) -> int:
    return int(lib().sphkv_decode_mq_workspace_bytes(B, H_q, H_kv, total_pages, n_sm))


def sphkv_decode_attention_mq(cache: sphkv_cache, n_q: int, H_q: int, q: torch.Tensor, out: torch.Tensor,
                              lse: torch.Tensor, workspace: torch.Tensor,
                              status: Optional[torch.Tensor] = None, stream=None):
    """Decode attention for n_q causal query tokens per sequence:
    q, out [B, n_q, H_q, 128], lse [B, n_q, H_q]."""
    _check("sphkv_decode_attention_mq", lib().sphkv_decode_attention_mq(
        ctypes.byref(cache), int(n_q), int(H_q), _ptr(q, torch.float32, "q"), _ptr(out, torch.float32, "out"),
        _ptr(lse, torch.float32, "lse"), _ptr(workspace, torch.uint8, "workspace"),
        int(workspace.numel()), _ptr(status, torch.int32, "status"), _stream(stream)))


def sphkv_merge_partials(out_parts: torch.Tensor, lse_parts: torch.Tensor, out: torch.Tensor, lse: torch.Tensor,
                         stream=None):
    """Log-sum-exp combine of decode results over disjoint parts of the same
    sequences: out_parts [n_parts, ..., 128], lse_parts [n_parts, ...] ->
    out [..., 128], lse [...]."""
    n_parts = int(lse_parts.shape[0])
    n_rows = int(lse.numel())
    if out_parts.shape[0] != n_parts or out_parts[0].numel() != n_rows * 128 or out.numel() != n_rows * 128:
        raise ValueError("sphkv_merge_partials: shapes do not match")
    _check("sphkv_merge_partials", lib().sphkv_merge_partials(
        _ptr(out_parts, torch.float32, "out_parts"), _ptr(lse_parts, torch.float32, "lse_parts"), n_parts, n_rows,
        _ptr(out, torch.float32, "out"), _ptr(lse, torch.float32, "lse"), _stream(stream)))


def sphkv_set_keep(cache: sphkv_cache, keep: torch.Tensor, status: Optional[torch.Tensor] = None, stream=None):
    """Per-token keep/drop: keep [H_kv, total_pages * 16] uint8 (nonzero =
    keep) sets or clears each present token's drop flag."""
    _check("sphkv_set_keep", lib().sphkv_set_keep(
        ctypes.byref(cache), _ptr(keep, torch.uint8, "keep"), _ptr(status, torch.int32, "status"), _stream(stream)))
