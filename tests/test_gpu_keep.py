"""Per-token keep/drop inside kept pages (sphkv_set_keep) on the GPU, against
the oracle: the flag bytes bit for bit, and decode (one query and query pairs)
within tolerance on ragged, mixed-tier caches with permuted pool pages, whole
pages and whole units dropped token by token.
"""
import numpy as np
import pytest

import oracle
from compressed_paged_kv_ada_b200 import workloads as W

from helpers import assert_close, dense_torch, gpu_cache, oracle_full_cache, to_torch

pytestmark = pytest.mark.gpu


def _keep_mask(w, frac, seed):
    rng = np.random.default_rng(seed)
    keep = (rng.random((w.H_kv, w.total_pages * 16)) < frac).astype(np.uint8)
    po = w.page_offsets
    keep[0, po[0] * 16:po[0] * 16 + 16] = 0     # the first page of unit (0, 0): every token dropped
    if w.B > 2:
        keep[1, po[2] * 16:po[3] * 16] = 0      # unit (2, 1): every token dropped
    return keep


def _oracle_cache_with_keep(w, keep):
    ref = oracle_full_cache(w, perms=w.pool_perms())
    oracle.set_keep(ref, keep)
    return ref


def test_set_keep_bytes_match_oracle():
    import torch

    w = W.make("ragged64", seq_lens=[700, 33, 1200, 17], H_kv=2, H_q=8)
    w.permute_pools = True
    cache = gpu_cache(w)
    keep = _keep_mask(w, 0.7, 1)
    cache.set_keep(to_torch(keep))
    cache.check()
    ref = _oracle_cache_with_keep(w, keep)
    for t in range(3):
        assert np.array_equal(cache.pools[t].cpu().numpy(), ref["pools"][t]), f"tier {t + 1}"
    # keeping every token again restores the encoder's pages
    cache.set_keep(torch.ones_like(to_torch(keep)))
    cache.check()
    fresh = oracle_full_cache(w, perms=w.pool_perms())
    for t in range(3):
        assert np.array_equal(cache.pools[t].cpu().numpy(), fresh["pools"][t])


@pytest.mark.parametrize("frac", [0.9, 0.5, 0.05])
def test_decode_with_dropped_tokens_matches_oracle(frac):
    import torch

    w = W.make("ragged64", seq_lens=[2049, 33, 1500, 1, 4000], H_kv=2, H_q=8)
    w.permute_pools = True
    cache = gpu_cache(w)
    keep = _keep_mask(w, frac, 7)
    cache.set_keep(to_torch(keep))
    q = w.queries()
    out, lse = cache.decode(to_torch(q, torch.float32))
    cache.check()
    out, lse = out.cpu().numpy(), lse.cpu().numpy()
    ref = _oracle_cache_with_keep(w, keep)
    units = [(b, g) for b in range(w.B) for g in range(w.H_kv)]
    ro, rl = oracle.cache_attention(ref, q, units)
    for i, (b, g) in enumerate(units):
        assert_close(out[b, 4 * g:4 * g + 4], lse[b, 4 * g:4 * g + 4], ro[i], rl[i], f"keep {frac} unit {(b, g)}")
    assert np.all(np.isneginf(lse[2, 4:8])) and np.all(out[2, 4:8] == 0)   # unit (2, 1): all dropped


def test_multi_query_decode_with_dropped_tokens():
    import torch

    w = W.make("ragged64", seq_lens=[700, 33, 1, 2049], H_kv=2, H_q=8)
    cache = gpu_cache(w)
    keep = _keep_mask(w, 0.6, 11)
    cache.set_keep(to_torch(keep))
    rng = np.random.default_rng(12)
    n_q = 3
    q = rng.standard_normal((w.B, n_q, w.H_q, 128)).astype(np.float32)
    out, lse = cache.decode_mq(to_torch(q, torch.float32))
    cache.check()
    out, lse = out.cpu().numpy(), lse.cpu().numpy()
    ref = _oracle_cache_with_keep(w, keep)
    units = [(b, g) for b in range(w.B) for g in range(w.H_kv)]
    ro, rl = oracle.multi_query_attention(ref, q, units, n_q)
    for i in range(n_q):
        for k, (b, g) in enumerate(units):
            assert_close(out[b, i, 4 * g:4 * g + 4], lse[b, i, 4 * g:4 * g + 4], ro[i, k], rl[i, k],
                         f"query {i} unit {(b, g)}")


def test_encode_writes_tokens_as_kept():
    """Re-encoding a dropped token (an append into the same slot) keeps it."""
    import torch

    w = W.make("ragged64", seq_lens=[40], H_kv=1, H_q=4)
    cache = gpu_cache(w)
    cache.set_keep(torch.zeros((w.H_kv, w.total_pages * 16), dtype=torch.uint8, device="cuda"))
    K, V = w.dense_rows(0, 0, 40)
    Kt, Vt = dense_torch(w, K, V)
    cache.encode(Kt, Vt, torch.zeros(40, dtype=torch.int32, device="cuda"),
                 torch.arange(40, dtype=torch.int32, device="cuda"))
    cache.check()
    fresh = oracle_full_cache(w, perms=w.pool_perms())
    for t in range(3):
        assert np.array_equal(cache.pools[t].cpu().numpy(), fresh["pools"][t])
