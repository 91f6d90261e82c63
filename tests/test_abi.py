"""CPU checks of the boundary: libsphkv.so builds for sm_100a, loads, and
exports every function include/sphkv.h declares; host-only helpers agree with
the format.  No kernel is launched here."""
import ctypes
import os
import re

import numpy as np

import oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    src = open(os.path.join(ROOT, "include", "sphkv.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(sphkv_[a-z_0-9]+)\s*\(", src)))


def test_library_exports_every_declared_symbol():
    from compressed_paged_kv_ada_b200 import build
    from compressed_paged_kv_ada_b200 import _lib

    build.build()
    lib = ctypes.CDLL(_lib.LIB_PATH)
    names = _declared()
    assert len(names) == 15, names
    missing = [n for n in names if not hasattr(lib, n)]
    assert not missing, missing
    # the binding covers the same names
    for n in names:
        assert n in _lib._EXPORTS or n in ("sphkv_last_error",), n
    # the test-hook and checked builds (loaded only by tests) export the same interface
    for path in (build.TEST_LIB, build.DEBUG_LIB):
        T = ctypes.CDLL(path)
        assert not [n for n in names if not hasattr(T, n)], path


def test_host_helpers_agree_with_the_format():
    from compressed_paged_kv_ada_b200 import _lib

    for t in (1, 2, 3):
        assert _lib.sphkv_page_bytes(t) == oracle.page_bytes(t)
    assert _lib.sphkv_page_bytes(0) == 0 and _lib.sphkv_page_bytes(4) == 0
    L = _lib.lib()
    # workspace sizes are pure host arithmetic
    assert L.sphkv_decode_workspace_bytes(8, 32, 8, 8 * 2048, 148) > 0
    assert L.sphkv_rdr_workspace_bytes(16, 8, 16 * 2064) >= 8 * 16 * 2064 * 9
    assert L.sphkv_decode_workspace_bytes(0, 32, 8, 10, 148) == 0
    assert L.sphkv_decode_mq_workspace_bytes(8, 32, 8, 8 * 2048, 148) > \
        L.sphkv_decode_workspace_bytes(8, 32, 8, 8 * 2048, 148)


def test_workloads_are_deterministic_and_shaped():
    from compressed_paged_kv_ada_b200 import workloads as W

    a = W.make("llama32k", B=2, ctx=5000)
    b = W.make("llama32k", B=2, ctx=5000)
    ka, va = a.dense_rows(1, 4000, 4100)
    kb, vb = b.dense_rows(1, 4000, 4100)
    assert np.array_equal(ka, kb) and np.array_equal(va, vb)
    full_k, _ = a.dense_rows(1, 0, 5000)
    assert np.array_equal(full_k[4000:4100], ka)
    assert np.array_equal(a.tiers, b.tiers)
    n = (5000 + 15) // 16
    row = a.tiers[0, :n]
    assert np.all(row[:4] == 1) and np.all(row[-8:] == 1)
    mix = np.bincount(a.tiers[:, :n].ravel(), minlength=4) / a.tiers[:, :n].size
    assert abs(mix[0] - 0.15) < 0.03 and abs(mix[2] - 0.40) < 0.04
    # bf16 inputs are exact bf16 values
    u = ka.view(np.uint32)
    assert np.all((u & 0xFFFF) == 0)
    r = W.make("ragged64")
    assert r.B == 64 and r.seq_lens.min() >= 1024 and r.seq_lens.max() <= 16384
    t = W.make("tiny")
    assert t.dtype == "fp32" and np.all(t.tiers == 1) and t.total_pages == 128
    e = W.make("e2e_rdr")
    assert e.extra["budget"] == int(0.25 * 512 * 8 * 16 * 32768)
    assert np.all(e.cap_pages == 2048 + 16)
