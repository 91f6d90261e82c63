"""RDR run again as the context grows (sphkv_rdr_rerun), with the tokens of
demoted pages transcoded from their codes into new, compacted pools
(sphkv_migrate), on the GPU against the oracle: tiers, lambda and bytes
exact; pools byte for byte; decode within tolerance; and an end-to-end run of
appends with periodic re-runs that keeps the stored bytes within the budget.
"""
import numpy as np
import pytest

import oracle
from compressed_paged_kv_ada_b200 import workloads as W

from helpers import assert_close, dense_torch, gpu_cache, oracle_full_cache, to_torch

pytestmark = pytest.mark.gpu

EPS = (1.1e-4, 2.75e-2, 7.12e-2, 2.0)


def _first_assign(w, budget):
    """RDR at prefill, on the GPU and in the oracle (asserted equal)."""
    cache = gpu_cache(w, encode=False)
    lam, nb = cache.rdr_assign(to_torch(w.utility()), EPS, budget, 4, 8)
    cache.check()
    want = oracle.rdr_assign(w.page_offsets, w.seq_lens, w.utility(), EPS, budget, 4, 8, w.H_kv, tiers_init=w.tiers)
    tiers = cache.tiers.cpu().numpy()
    assert np.array_equal(tiers, want[0]) and float(lam.item()) == want[1] and int(nb.item()) == want[2]
    return cache, tiers


def _encode_tokens(cache, w, lens):
    import torch

    for b in range(w.B):
        n = int(lens[b])
        K, V = w.dense_rows(b, 0, n)
        Kt, Vt = dense_torch(w, K, V)
        cache.encode(Kt, Vt, torch.full((n,), b, dtype=torch.int32, device="cuda"),
                     torch.arange(n, dtype=torch.int32, device="cuda"))
    cache.check()


@pytest.mark.parametrize("frac", [0.30, 0.22])
def test_rerun_tiers_exact_and_migrated_pools_bit_exact(frac):
    import torch

    w = W.make("e2e_rdr", B=3, ctx=1500, H_kv=2, H_q=8)
    budget0 = int(0.35 * 512 * w.H_kv * int(w.seq_lens.sum()))
    cache, tiers0 = _first_assign(w, budget0)
    cache.reallocate_pools()
    lens2 = w.seq_lens + 200   # appended tokens land in the reserved T1 pages
    cache.seq_lens.copy_(to_torch(lens2.astype(np.int32)))
    _encode_tokens(cache, w, lens2)
    util2 = w.utility(lens2)
    budget = int(frac * 512 * w.H_kv * int(lens2.sum()))
    # the re-run alone, on a copy of the tiers
    from compressed_paged_kv_ada_b200 import _lib as L

    ws = torch.empty(L.sphkv_rdr_workspace_bytes(w.B, w.H_kv, w.total_pages), dtype=torch.uint8, device="cuda")
    lam = torch.zeros(1, dtype=torch.float64, device="cuda")
    nb = torch.zeros(1, dtype=torch.int64, device="cuda")
    t_io = cache.tiers.clone()
    L.sphkv_rdr_rerun(cache.descriptor(), to_torch(util2), EPS, budget, 4, 8, t_io, lam, nb, ws, status=cache.status)
    cache.check()
    want_t, want_lam, want_b = oracle.rdr_rerun(w.page_offsets, lens2, util2, EPS, budget, 4, 8, tiers0)
    assert np.array_equal(t_io.cpu().numpy(), want_t)
    assert float(lam.item()) == want_lam and int(nb.item()) == want_b <= budget
    # re-run + page table + migrate through the cache helper
    cache.rdr_rerun(to_torch(util2), EPS, budget, 4, 8)
    assert np.array_equal(cache.tiers.cpu().numpy(), want_t)
    ref = oracle_full_cache(w, lens=lens2, tiers=tiers0)
    counts = [int((want_t == t).sum()) for t in (1, 2, 3)]
    new_pools = oracle.migrate(ref, oracle.build_page_table(want_t), counts)
    for t in range(3):
        assert np.array_equal(cache.pools[t].cpu().numpy(), new_pools[t]), f"tier {t + 1}"
    # decode over the migrated cache
    q = w.queries(3)
    out, lse = cache.decode(to_torch(q, torch.float32))
    cache.check()
    out, lse = out.cpu().numpy(), lse.cpu().numpy()
    mref = dict(ref, page_table=oracle.build_page_table(want_t), pools=new_pools)
    units = [(b, g) for b in range(w.B) for g in range(w.H_kv)]
    ro, rl = oracle.cache_attention(mref, q, units)
    for i, (b, g) in enumerate(units):
        assert_close(out[b, 4 * g:4 * g + 4], lse[b, 4 * g:4 * g + 4], ro[i], rl[i], f"migrated unit {(b, g)}")


def test_appends_with_periodic_reruns_stay_within_budget():
    """Prefill, RDR, then appends; every 16 steps RDR runs again under the
    same budget and the pools are rewritten.  The GPU state is replayed in the
    oracle (its encoder for each appended token, its re-run, its migrate): pools
    byte for byte after every re-run, stored bytes within the budget, and the
    final decode against the oracle."""
    import torch

    w = W.make("e2e_rdr", B=2, ctx=2048, H_kv=2, H_q=8)
    budget = int(0.25 * 512 * w.H_kv * int(w.seq_lens.sum()))
    cache, tiers = _first_assign(w, budget)
    cache.reallocate_pools()
    _encode_tokens(cache, w, w.seq_lens)
    ref = oracle_full_cache(w, tiers=tiers)
    lens = w.seq_lens.copy()
    for step in range(64):
        rows = [w.dense_rows(b, int(lens[b]), int(lens[b]) + 1) for b in range(w.B)]
        Kd, Vd = dense_torch(w, np.concatenate([r[0] for r in rows]), np.concatenate([r[1] for r in rows]))
        cache.encode(Kd, Vd, torch.arange(w.B, dtype=torch.int32, device="cuda"), to_torch(lens.astype(np.int32)))
        for b in range(w.B):   # the oracle: encode the token into its page (always a T1 page)
            for g in range(w.H_kv):
                e = int(ref["page_table"][g, w.page_offsets[b] + lens[b] // 16]) & 0xFFFFFFFF
                t, phys = e >> 30, e & 0x3FFFFFFF
                assert t == 1
                c = oracle.encode(rows[b][0][:, g], rows[b][1][:, g], 1)
                oracle.pack_token(1, int(lens[b]) % 16, c["leaf"][0], c["up"][0], c["r16"][0], c["s16"][0],
                                  c["vq"][0], ref["pools"][0][phys])
        lens += 1
        cache.seq_lens.copy_(to_torch(lens.astype(np.int32)))
        ref["seq_lens"] = lens.copy()
        if step % 16 == 15:
            util = w.utility(lens)
            lam, nb = cache.rdr_rerun(to_torch(util), EPS, budget, 4, 8)
            assert int(nb.item()) <= budget
            new_t, _, want_b = oracle.rdr_rerun(w.page_offsets, lens, util, EPS, budget, 4, 8, tiers)
            assert np.array_equal(cache.tiers.cpu().numpy(), new_t) and int(nb.item()) == want_b
            counts = [int((new_t == t).sum()) for t in (1, 2, 3)]
            table = oracle.build_page_table(new_t)
            ref["pools"] = oracle.migrate(ref, table, counts)
            ref["page_table"] = table
            tiers = new_t
            for t in range(3):
                assert np.array_equal(cache.pools[t].cpu().numpy(), ref["pools"][t]), f"step {step} tier {t + 1}"
            assert cache.compressed_bytes() <= budget
    q = w.queries(99)
    out, lse = cache.decode(to_torch(q, torch.float32))
    cache.check()
    out, lse = out.cpu().numpy(), lse.cpu().numpy()
    units = [(b, g) for b in range(w.B) for g in range(w.H_kv)]
    ro, rl = oracle.cache_attention(ref, q, units)
    for i, (b, g) in enumerate(units):
        assert_close(out[b, 4 * g:4 * g + 4], lse[b, 4 * g:4 * g + 4], ro[i], rl[i], f"final unit {(b, g)}")


def test_migrate_refuses_a_finer_tier():
    """A page the new table makes finer than before cannot be rebuilt from its
    codes: the call reports SPHKV_ERR_DATA and leaves that page unwritten."""
    import torch

    from compressed_paged_kv_ada_b200 import PagedCache, SphkvError
    from compressed_paged_kv_ada_b200 import _lib as L

    w = W.make("ragged64", seq_lens=[64], H_kv=1, H_q=4)
    tiers = np.full((1, w.total_pages), 3, np.uint8)
    cache = gpu_cache(w, tiers=tiers, perms=(None, None, None))
    finer = np.full_like(tiers, 2)
    dst = PagedCache(w.page_offsets, w.seq_lens, finer)
    L.sphkv_migrate(cache.descriptor(), dst.descriptor(), status=dst.status)
    with pytest.raises(SphkvError) as e:
        dst.check()
    assert e.value.code == 6
    assert int(dst.pools[1].to(torch.int64).sum().item()) == 0
