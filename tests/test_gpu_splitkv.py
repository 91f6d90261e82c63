"""Split-KV of one long stream, on the GPU: the stream's pages are cut into
page-aligned ranges (as split_stream gives the ranks of a multi-GPU run), each
range is decoded by the library as its own cache, and sphkv_merge_partials
combines the parts.  The parts run one after another on one GPU (no kernel
waits on another); the result must match the decode of the whole stream and
the oracle.
"""
import numpy as np
import pytest

import oracle
from compressed_paged_kv_ada_b200 import splitkv
from compressed_paged_kv_ada_b200 import workloads as W

from helpers import assert_close, dense_torch, gpu_cache, oracle_all_units, to_torch

pytestmark = pytest.mark.gpu


def _part_cache(w, t0, t1):
    """A one-sequence cache holding tokens [t0, t1) of sequence 0 of w, at
    positions 0 .. t1 - t0 - 1 (attention does not depend on positions)."""
    import torch

    from compressed_paged_kv_ada_b200 import PagedCache

    p0, p1 = t0 // 16, (t1 + 15) // 16
    tiers = np.ascontiguousarray(w.tiers[:, p0:p1])
    cache = PagedCache(np.array([0, p1 - p0], np.int32), np.array([t1 - t0], np.int32), tiers)
    if t1 > t0:
        K, V = w.dense_rows(0, t0, t1)
        Kt, Vt = dense_torch(w, K, V)
        cache.encode(Kt, Vt, torch.zeros(t1 - t0, dtype=torch.int32, device="cuda"),
                     torch.arange(t1 - t0, dtype=torch.int32, device="cuda"))
    cache.check()
    return cache


def _split_decode(w, world, q):
    import torch

    from compressed_paged_kv_ada_b200 import sphkv_merge_partials

    outs, lses = [], []
    for t0, t1 in splitkv.split_stream(int(w.seq_lens[0]), world):
        cache = _part_cache(w, t0, t1)
        o, l = cache.decode(q)
        cache.check()
        outs.append(o)
        lses.append(l)
    out = torch.empty_like(outs[0])
    lse = torch.empty_like(lses[0])
    sphkv_merge_partials(torch.stack(outs), torch.stack(lses), out, lse)
    torch.cuda.synchronize()
    return out.cpu().numpy(), lse.cpu().numpy()


@pytest.mark.parametrize("world", [2, 3, 5])
def test_split_stream_merge_matches_whole_and_oracle(world):
    import torch

    w = W.make("long512k", ctx=40000, H_kv=2, H_q=8)
    q = to_torch(w.queries(), torch.float32)
    out, lse = _split_decode(w, world, q)
    whole = gpu_cache(w)
    wo, wl = whole.decode(q)
    whole.check()
    assert_close(out, lse, wo.cpu().numpy(), wl.cpu().numpy(), f"split x{world} vs whole")
    ro, rl = oracle_all_units(w, w.queries())
    assert_close(out, lse, ro, rl, f"split x{world} vs oracle")


def test_merge_empty_parts_and_single_part():
    """A part with no kept token (lse -inf) contributes nothing; merging one
    part returns it; all parts empty gives out 0, lse -inf."""
    import torch

    from compressed_paged_kv_ada_b200 import sphkv_merge_partials

    rng = np.random.default_rng(3)
    o = rng.standard_normal((6, 128)).astype(np.float32)
    l = rng.standard_normal(6).astype(np.float32)
    empty_o = np.zeros_like(o)
    empty_l = np.full_like(l, -np.inf)
    for parts in ([o], [o, empty_o], [empty_o, o, empty_o]):
        ls = [l if p is o else empty_l for p in parts]
        out = torch.empty((6, 128), dtype=torch.float32, device="cuda")
        lse = torch.empty(6, dtype=torch.float32, device="cuda")
        sphkv_merge_partials(to_torch(np.stack(parts)), to_torch(np.stack(ls)), out, lse)
        torch.cuda.synchronize()
        np.testing.assert_allclose(out.cpu().numpy(), o, rtol=1e-6, atol=1e-6)
        np.testing.assert_allclose(lse.cpu().numpy(), l, rtol=1e-6, atol=1e-6)
    out = torch.empty((6, 128), dtype=torch.float32, device="cuda")
    lse = torch.empty(6, dtype=torch.float32, device="cuda")
    sphkv_merge_partials(to_torch(np.stack([empty_o, empty_o])), to_torch(np.stack([empty_l, empty_l])), out, lse)
    torch.cuda.synchronize()
    assert np.all(out.cpu().numpy() == 0) and np.all(np.isneginf(lse.cpu().numpy()))


def test_full_size_long512k_split_over_8():
    """The 524288-token stream cut as 8 ranks would hold it: every part decoded
    by the library, merged, and every unit checked against the oracle."""
    import torch

    w = W.make("long512k")
    q = to_torch(w.queries(), torch.float32)
    out, lse = _split_decode(w, 8, q)
    ro, rl = oracle_all_units(w, w.queries())
    for g in range(w.H_kv):
        rs = slice(4 * g, 4 * g + 4)
        assert_close(out[0, rs], lse[0, rs], ro[0, rs], rl[0, rs], f"long512k split x8 unit (0, {g})")
