"""The checked build (libsphkv_debug.so: decode.cu compiled with SPHKV_DEBUG)
on mixed caches: every shared-memory table address the decode kernels form is
checked against its table and alignment, a canary past each shorter page copy
must survive, and every call synchronises.  On valid inputs none of the checks
may fire (status OK) and the results must be bit-identical to the product
library's, for one query token and for query pairs, on ragged, permuted,
mixed-tier caches with dropped pages, dropped tokens and split units.
"""
import ctypes

import numpy as np
import pytest

from compressed_paged_kv_ada_b200 import workloads as W

from helpers import gpu_cache, to_torch

pytestmark = pytest.mark.gpu


def _debug_lib():
    from compressed_paged_kv_ada_b200 import _lib, build

    build.build()   # no-op when every library is current
    return _lib, _lib.load(build.DEBUG_LIB)


@pytest.mark.parametrize("n_q", [1, 2, 3])
def test_checked_build_is_silent_and_bit_identical(n_q):
    import torch

    _lib, D = _debug_lib()
    w = W.make("ragged64", seq_lens=[2049, 33, 1, 0, 4000, 777], H_kv=2, H_q=8)
    w.permute_pools = True
    cache = gpu_cache(w)
    keep = (np.random.default_rng(3).random((w.H_kv, w.total_pages * 16)) < 0.8).astype(np.uint8)
    cache.set_keep(to_torch(keep))
    cache.check()
    rng = np.random.default_rng(40 + n_q)
    q = to_torch(rng.standard_normal((w.B, n_q, w.H_q, 128)).astype(np.float32), torch.float32)
    ref_out, ref_lse = cache.decode_mq(q)
    cache.check()

    out = torch.full_like(ref_out, float("nan"))
    lse = torch.full_like(ref_lse, float("nan"))
    ws = torch.empty(_lib.sphkv_decode_mq_workspace_bytes(w.B, w.H_q, w.H_kv, w.total_pages), dtype=torch.uint8,
                     device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    desc = cache.descriptor()
    code = D.sphkv_decode_attention_mq(ctypes.byref(desc), n_q, w.H_q, q.data_ptr(), out.data_ptr(), lse.data_ptr(),
                                       ws.data_ptr(), ws.numel(), status.data_ptr(), None)
    assert code == _lib.OK, D.sphkv_last_error()
    torch.cuda.synchronize()
    assert int(status.item()) == _lib.OK
    assert torch.equal(out, ref_out) and torch.equal(lse, ref_lse)


def test_checked_build_full_size_one_query():
    """The 32k workload's shape (every unit split across CTAs) through the
    checked build's single-query entry point."""
    import torch

    _lib, D = _debug_lib()
    w = W.make("llama32k", B=2)
    cache = gpu_cache(w)
    q = to_torch(w.queries(), torch.float32)
    ref_out, ref_lse = cache.decode(q)
    cache.check()
    out = torch.empty_like(ref_out)
    lse = torch.empty_like(ref_lse)
    ws = torch.empty(_lib.sphkv_decode_workspace_bytes(w.B, w.H_q, w.H_kv, w.total_pages), dtype=torch.uint8,
                     device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    desc = cache.descriptor()
    code = D.sphkv_decode_attention(ctypes.byref(desc), w.H_q, q.data_ptr(), out.data_ptr(), lse.data_ptr(),
                                    ws.data_ptr(), ws.numel(), status.data_ptr(), None)
    assert code == _lib.OK, D.sphkv_last_error()
    assert int(status.item()) == _lib.OK
    assert torch.equal(out, ref_out) and torch.equal(lse, ref_lse)
