"""The no-allocation decode entry point (sphkv_decode_attention_noalloc).

Some callers cannot allocate device memory: an engine that owns all of it
and forbids allocation after start-up, or a latency-critical loop that cannot
afford cudaMalloc.  For them the library keeps its decode scratch in a static
device array.  These tests call that entry point through the C ABI and check
its results against the workspace entry point, on two calls in a row (the
array keeps the previous call's contents), and check that an oversized cache
is refused before anything is launched.  This file is collected last.
"""
import numpy as np
import pytest

from compressed_paged_kv_ada_b200 import workloads as W

from helpers import assert_close, gpu_cache, to_torch

pytestmark = pytest.mark.gpu


def test_noalloc_matches_workspace_entry_point_twice():
    import torch

    from compressed_paged_kv_ada_b200 import _lib as L

    # long enough that units are split over several CTAs (partials + merge)
    w = W.make("ragged64", seq_lens=[40000, 1111, 0, 2222], H_kv=2, H_q=8)
    cache = gpu_cache(w)
    q = to_torch(w.queries(), torch.float32)
    ref_out, ref_lse = cache.decode(q)
    cache.check()
    ref_out, ref_lse = ref_out.cpu().numpy(), ref_lse.cpu().numpy()
    for call in range(2):
        out = torch.full((w.B, w.H_q, 128), float("nan"), dtype=torch.float32, device="cuda")
        lse = torch.full((w.B, w.H_q), float("nan"), dtype=torch.float32, device="cuda")
        L.sphkv_decode_attention_noalloc(cache.descriptor(), w.H_q, q, out, lse, status=cache.status)
        cache.check()
        assert_close(out.cpu().numpy(), lse.cpu().numpy(), ref_out, ref_lse, f"noalloc call {call}")


def test_noalloc_refuses_oversized_cache():
    import torch

    from compressed_paged_kv_ada_b200 import _lib as L

    B, H_kv = 2000, 8   # 16000 units: partials far above the 4 MiB static area
    lens = np.full(B, 16, np.int32)
    w = W.make("llama32k", seq_lens=lens, H_kv=H_kv, H_q=4 * H_kv, mix=(1.0, 0.0, 0.0, 0.0))
    cache = gpu_cache(w, encode=False)
    q = torch.zeros((B, 4 * H_kv, 128), dtype=torch.float32, device="cuda")
    out = torch.empty_like(q)
    lse = torch.empty((B, 4 * H_kv), dtype=torch.float32, device="cuda")
    with pytest.raises(L.SphkvError) as e:
        L.sphkv_decode_attention_noalloc(cache.descriptor(), 4 * H_kv, q, out, lse, status=cache.status)
    assert e.value.code == L.ERR_ARG and "4194304" in str(e.value)
