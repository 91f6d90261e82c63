"""A bounded device wait that runs out reports SPHKV_ERR_TIMEOUT, and the
context stays usable afterwards.

The test loads libsphkv_testhooks.so: the same library with decode.cu built
with SPHKV_TEST_HOOKS.  With SPHKV_TEST_SKIP_FIRST_COPY set, warp 0 of CTA 0
skips its first page copy and waits for it with a shortened limit, so that
wait runs out; every other warp and CTA runs as in the product library.
Nothing faults and no wait is unbounded.  The product library is built without
the flag.
"""
import ctypes

import pytest

from compressed_paged_kv_ada_b200 import workloads as W

from helpers import gpu_cache, to_torch

pytestmark = pytest.mark.gpu


def test_page_wait_timeout_reports_and_context_recovers(monkeypatch):
    import torch

    from compressed_paged_kv_ada_b200 import _lib, build

    build.build()   # no-op when both libraries are current
    T = _lib.load(build.TEST_LIB)
    w = W.make("ragged64", seq_lens=[2049, 1500], H_kv=2, H_q=8)
    cache = gpu_cache(w)
    q = to_torch(w.queries(), torch.float32)
    out = torch.empty((w.B, w.H_q, 128), dtype=torch.float32, device="cuda")
    lse = torch.empty((w.B, w.H_q), dtype=torch.float32, device="cuda")
    ws = torch.empty(_lib.sphkv_decode_workspace_bytes(w.B, w.H_q, w.H_kv, w.total_pages), dtype=torch.uint8,
                     device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    desc = cache.descriptor()

    def run():
        code = T.sphkv_decode_attention(ctypes.byref(desc), w.H_q, q.data_ptr(), out.data_ptr(), lse.data_ptr(),
                                        ws.data_ptr(), ws.numel(), status.data_ptr(), None)
        assert code == _lib.OK, T.sphkv_last_error()
        torch.cuda.synchronize()

    ref_out, ref_lse = cache.decode(q)
    cache.check()
    monkeypatch.setenv("SPHKV_TEST_SKIP_FIRST_COPY", "1")
    run()
    assert int(status.item()) == _lib.ERR_TIMEOUT
    # Only CTA 0 stopped.  Its pages all lie in unit (0, 0): that unit holds the
    # first 129 of the 446 pages, and with at least 4 CTAs (min(7, SM count))
    # CTA 0 takes at most 112 of them.  Every other unit is exact.
    for b, g in [(0, 1), (1, 0), (1, 1)]:
        rows = slice(4 * g, 4 * g + 4)
        assert torch.equal(out[b, rows], ref_out[b, rows]) and torch.equal(lse[b, rows], ref_lse[b, rows])
    # the context is still usable: the next call (no skipped copy) is correct
    monkeypatch.delenv("SPHKV_TEST_SKIP_FIRST_COPY")
    status.zero_()
    run()
    assert int(status.item()) == _lib.OK
    assert torch.equal(out, ref_out) and torch.equal(lse, ref_lse)
