"""GPU parity: libsphkv (through its C ABI) against the fp64 CPU oracle.

Bit for bit: page tables, encoded pages, RDR tiers.  Within the stated float
tolerance (tests/helpers.py): decode out and lse.
"""
import numpy as np
import pytest

import oracle
from compressed_paged_kv_ada_b200 import workloads as W

from helpers import (assert_close, dense_torch, gpu_cache, oracle_all_units, oracle_full_cache, oracle_unit,
                     oracle_unit_dense, to_torch)

pytestmark = pytest.mark.gpu


def _torch():
    import torch

    return torch


def _decode(cache, q_np):
    out, lse = cache.decode(to_torch(q_np, _torch().float32))
    cache.check()
    return out.cpu().numpy(), lse.cpu().numpy()


# ------------------------------------------------------------ page table --
def test_page_table_matches_oracle():
    rng = np.random.default_rng(0)
    torch = _torch()
    from compressed_paged_kv_ada_b200 import sphkv_build_page_table

    for n in (1, 5, 1000, 5000, 70000):
        tiers = rng.integers(0, 4, n).astype(np.uint8)
        counts = [int((tiers == t).sum()) for t in (1, 2, 3)]
        perms = [rng.permutation(c).astype(np.int32) for c in counts]
        for use_perm in (False, True):
            ps = perms if use_perm else [None, None, None]
            want = oracle.build_page_table(tiers[None], ps)[0]
            table = torch.empty(n, dtype=torch.int32, device="cuda")
            cnt = torch.zeros(3, dtype=torch.int64, device="cuda")
            sphkv_build_page_table(to_torch(tiers), table,
                                   [None if p is None else to_torch(p) for p in ps], counts=cnt)
            torch.cuda.synchronize()
            assert np.array_equal(table.cpu().numpy(), want)
            assert cnt.cpu().tolist() == counts


# ---------------------------------------------------------------- encode --
@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
def test_encode_pages_bit_exact(dtype):
    """Every page the library writes equals the oracle's page byte for byte
    (all tiers, partial last pages, permuted pool ids)."""
    w = W.make("ragged64", seq_lens=[1, 16, 17, 300, 1000], H_q=8, H_kv=2, dtype=dtype)
    w.permute_pools = True
    cache = gpu_cache(w)
    ref = oracle_full_cache(w, perms=w.pool_perms())
    assert np.array_equal(cache.page_table.cpu().numpy(), ref["page_table"])
    for t in range(3):
        got = cache.pools[t].cpu().numpy()
        want = ref["pools"][t]
        assert got.shape == want.shape
        if not np.array_equal(got, want):
            bad = np.nonzero((got != want).any(axis=1))[0]
            raise AssertionError(f"tier {t + 1}: {bad.size} pages differ, first {bad[:5]}")


def test_encode_append_matches_bulk():
    """Encoding tokens one position at a time (append) writes the same pages as
    one bulk prefill encode."""
    torch = _torch()
    w = W.make("llama32k", B=3, ctx=70, H_q=8, H_kv=2)
    bulk = gpu_cache(w)
    app = gpu_cache(w, encode=False)
    K = [w.dense_rows(b, 0, 70) for b in range(3)]
    for pos in range(70):
        Kt = np.stack([K[b][0][pos] for b in range(3)])
        Vt = np.stack([K[b][1][pos] for b in range(3)])
        Kd, Vd = dense_torch(w, Kt, Vt)
        app.encode(Kd, Vd, torch.arange(3, dtype=torch.int32, device="cuda"),
                   torch.full((3,), pos, dtype=torch.int32, device="cuda"))
    app.check()
    for t in range(3):
        assert torch.equal(bulk.pools[t], app.pools[t])


# ---------------------------------------------------------------- decode --
def test_decode_tiny_parity():
    """Tiny config: B 1, 4 q heads / 1 kv head, ctx 2048, all T1, fp32 K/V."""
    w = W.make("tiny")
    cache = gpu_cache(w)
    q = w.queries()
    out, lse = _decode(cache, q)
    ref = oracle_full_cache(w)
    ro, rl = oracle.cache_attention(ref, q, [(0, 0)])
    assert_close(out[0], lse[0], ro[0], rl[0], "tiny")


@pytest.mark.parametrize("case", [
    dict(seq_lens=[5], H_kv=1),
    dict(seq_lens=[16, 17, 31, 33], H_kv=2),
    dict(seq_lens=[0, 100, 1, 2049], H_kv=3),
    dict(seq_lens=[4000, 257, 1500], H_kv=8),
])
def test_decode_small_mixed_parity(case):
    """Mixed tiers, drops, ragged tails, empty and one-token sequences."""
    w = W.make("ragged64", seq_lens=case["seq_lens"], H_kv=case["H_kv"], H_q=4 * case["H_kv"])
    w.permute_pools = True
    cache = gpu_cache(w)
    q = w.queries()
    out, lse = _decode(cache, q)
    ref = oracle_full_cache(w)
    units = [(b, g) for b in range(w.B) for g in range(w.H_kv)]
    ro, rl = oracle.cache_attention(ref, q, units)
    for i, (b, g) in enumerate(units):
        assert_close(out[b, 4 * g:4 * g + 4], lse[b, 4 * g:4 * g + 4], ro[i], rl[i], f"unit {(b, g)}")


def test_decode_reads_oracle_pages():
    """The decode kernel on pools packed by the oracle (not by the library's
    encoder) matches the oracle's attention over the same pools."""
    torch = _torch()
    from compressed_paged_kv_ada_b200 import PagedCache

    w = W.make("ragged64", seq_lens=[700, 33, 1200], H_kv=2, H_q=8)
    ref = oracle_full_cache(w)
    cache = PagedCache(w.page_offsets, w.seq_lens, w.tiers)
    for t in range(3):
        cache.pools[t].copy_(to_torch(ref["pools"][t]))
    assert np.array_equal(cache.page_table.cpu().numpy(), ref["page_table"])
    q = w.queries()
    out, lse = _decode(cache, q)
    units = [(b, g) for b in range(w.B) for g in range(w.H_kv)]
    ro, rl = oracle.cache_attention(ref, q, units)
    for i, (b, g) in enumerate(units):
        assert_close(out[b, 4 * g:4 * g + 4], lse[b, 4 * g:4 * g + 4], ro[i], rl[i], f"unit {(b, g)}")


def test_large_value_scales():
    """Tokens whose value scales are far above 16 (|v| up to ~1e5): p * vscale
    * 2^12 would leave the f16 range of the tensor-core weights, so the decode
    lowers its weight scale; the result stays within tolerance of the oracle."""
    from compressed_paged_kv_ada_b200 import PagedCache

    w = W.make("ragged64", seq_lens=[700, 33, 1200], H_kv=2, H_q=8)
    K, V = w.dense(w.seq_lens)
    rng = np.random.default_rng(11)
    big = rng.random(len(V)) < 0.05
    V = V.astype(np.float64) * np.where(big, rng.choice([300.0, 3000.0, 30000.0], len(V)), 1.0)[:, None, None]
    seq, pos = w.token_index(w.seq_lens)
    table = oracle.build_page_table(w.tiers, (None, None, None))
    counts = [int((w.tiers == t).sum()) for t in (1, 2, 3)]
    pools = oracle.encode_cache(K, V, seq, pos, w.page_offsets, table, counts)
    ref = dict(B=w.B, H_q=w.H_q, H_kv=w.H_kv, page_offsets=w.page_offsets, seq_lens=w.seq_lens,
               page_table=table, pools=pools)
    cache = PagedCache(w.page_offsets, w.seq_lens, w.tiers)
    for t in range(3):
        cache.pools[t].copy_(to_torch(pools[t]))
    q = w.queries()
    out, lse = _decode(cache, q)
    assert np.all(np.isfinite(out)) and np.all(np.isfinite(lse))
    units = [(b, g) for b in range(w.B) for g in range(w.H_kv)]
    ro, rl = oracle.cache_attention(ref, q, units)
    for i, (b, g) in enumerate(units):
        assert_close(out[b, 4 * g:4 * g + 4], lse[b, 4 * g:4 * g + 4], ro[i], rl[i], f"unit {(b, g)}")


def test_all_dropped_and_q_zero():
    """A unit whose pages are all dropped gives out 0 and lse -inf; q = 0 gives
    the mean of the kept values and lse = ln(#kept)."""
    w = W.make("ragged64", seq_lens=[300, 300], H_kv=1, H_q=4)
    tiers = w.tiers.copy()
    po = w.page_offsets
    tiers[0, po[0]:po[1]] = 0
    cache = gpu_cache(w, tiers=tiers, perms=(None, None, None))
    q = np.zeros((2, 4, 128), np.float32)
    out, lse = _decode(cache, q)
    assert np.all(out[0] == 0) and np.all(np.isneginf(lse[0]))
    ro, rl = oracle_unit(w, 1, 0, q, tiers=tiers)
    assert_close(out[1], lse[1], ro, rl, "q=0")
    kept = sum(min(16, 300 - 16 * p) for p in range(19) if tiers[0, po[1] + p] != 0)
    assert np.all(np.abs(lse[1] - np.log(kept)) <= 1e-4)


@pytest.mark.parametrize("n_q", [1, 2, 3, 4])
def test_multi_query_decode(n_q):
    """n_q causal query tokens per sequence (query i sees the first
    seq_len - (n_q - 1 - i) tokens), through sphkv_decode_attention_mq, against
    the oracle: ragged lengths, drops, a one-token sequence and an empty one."""
    torch = _torch()
    w = W.make("ragged64", seq_lens=[700, 33, 1, 0, 2049], H_kv=2, H_q=8)
    w.permute_pools = True
    cache = gpu_cache(w)
    rng = np.random.default_rng(17 + n_q)
    q = rng.standard_normal((w.B, n_q, w.H_q, 128)).astype(np.float32)
    out, lse = cache.decode_mq(to_torch(q, torch.float32))
    cache.check()
    out, lse = out.cpu().numpy(), lse.cpu().numpy()
    ref = oracle_full_cache(w)
    units = [(b, g) for b in range(w.B) for g in range(w.H_kv)]
    ro, rl = oracle.multi_query_attention(ref, q, units, n_q)
    for i in range(n_q):
        for k, (b, g) in enumerate(units):
            assert_close(out[b, i, 4 * g:4 * g + 4], lse[b, i, 4 * g:4 * g + 4], ro[i, k], rl[i, k],
                         f"query {i} unit {(b, g)}")
    if n_q == 1:   # the same kernel as sphkv_decode_attention
        o1, l1 = _decode(cache, q[:, 0])
        assert np.array_equal(o1, out[:, 0]) and np.array_equal(l1, lse[:, 0])


def test_multi_query_full_size_every_unit():
    """Two query tokens per sequence at the 32k workload's full size, on the
    launch path bench.py --n-q 2 times (one launch of the pair kernel): every
    (query, sequence, kv head) unit against the oracle."""
    torch = _torch()
    w = W.make("llama32k")
    cache = gpu_cache(w)
    rng = np.random.default_rng(23)
    q = rng.standard_normal((w.B, 2, w.H_q, 128)).astype(np.float32)
    out, lse = cache.decode_mq(to_torch(q, torch.float32))
    cache.check()
    out, lse = out.cpu().numpy(), lse.cpu().numpy()
    ref = oracle_full_cache(w)
    units = [(b, g) for b in range(w.B) for g in range(w.H_kv)]
    ro, rl = oracle.multi_query_attention(ref, q, units, 2)
    for i in range(2):
        for k, (b, g) in enumerate(units):
            assert_close(out[b, i, 4 * g:4 * g + 4], lse[b, i, 4 * g:4 * g + 4], ro[i, k], rl[i, k],
                         f"query {i} unit {(b, g)}")


def test_physical_permutation_is_bit_identical():
    torch = _torch()
    w = W.make("ragged64", seq_lens=[3000, 1111, 2222], H_kv=2, H_q=8)
    a = gpu_cache(w, perms=(None, None, None))
    w.permute_pools = True
    b = gpu_cache(w)
    q = to_torch(w.queries(), torch.float32)
    oa, la = a.decode(q)
    ob, lb = b.decode(q)
    torch.cuda.synchronize()
    assert torch.equal(oa, ob) and torch.equal(la, lb)


def test_split_count_invariance():
    """Reserving more pages changes how the pages are cut across SMs; results
    agree within tolerance."""
    w = W.make("long512k", ctx=40000, H_kv=2, H_q=8)
    q = w.queries()
    a = gpu_cache(w)
    oa, la = _decode(a, q)
    w2 = W.make("long512k", ctx=40000, H_kv=2, H_q=8, extra_pages=20000)
    b = gpu_cache(w2)
    ob, lb = _decode(b, q)
    assert a.total_pages != b.total_pages
    assert_close(oa, la, ob, lb, "split")
    ro, rl = oracle_unit(w, 0, 1, q)
    assert_close(oa[0, 4:8], la[0, 4:8], ro, rl, "split vs oracle")


# ------------------------------------------------------------- full size --
def _sampled_pages_bit_exact(w, cache, n_samples, rng):
    """Pick logical pages at random and check the library's bytes against the
    oracle's encoding of those 16 tokens."""
    table = cache.page_table.cpu().numpy()
    po = w.page_offsets
    pools = [None, None, None]
    checked = 0
    while checked < n_samples:
        b = int(rng.integers(w.B))
        n = int(w.seq_lens[b])
        if n == 0:
            continue
        g = int(rng.integers(w.H_kv))
        p = int(rng.integers((n + 15) // 16))
        e = int(table[g, po[b] + p]) & 0xFFFFFFFF
        t, phys = e >> 30, e & 0x3FFFFFFF
        if t == 0:
            continue
        if pools[t - 1] is None:
            pools[t - 1] = cache.pools[t - 1]
        got = pools[t - 1][phys].cpu().numpy()
        lo, hi = 16 * p, min(n, 16 * p + 16)
        K, V = w.dense_rows(b, lo, hi)
        c = oracle.encode(K[:, g], V[:, g], t)
        want = np.zeros(oracle.page_bytes(t), np.uint8)
        for i in range(hi - lo):
            oracle.pack_token(t, i, c["leaf"][i], c["up"][i], c["r16"][i], c["s16"][i], c["vq"][i], want)
        assert np.array_equal(got, want), f"page (b={b}, g={g}, p={p}, tier {t}) differs"
        checked += 1


@pytest.mark.parametrize("name", ["llama32k", "ragged64", "long512k"])
def test_full_size_workloads(name):
    """Full-size workloads: sampled pages bit-exact, the page table equal to
    the oracle's, and the decode of every (sequence, kv head) unit within
    tolerance of the oracle."""
    w = W.make(name)
    cache = gpu_cache(w)
    assert np.array_equal(cache.page_table.cpu().numpy(), oracle.build_page_table(w.tiers, w.pool_perms()))
    rng = np.random.default_rng(123)
    _sampled_pages_bit_exact(w, cache, 40, rng)
    q = w.queries()
    out, lse = _decode(cache, q)
    del cache
    assert np.all(np.isfinite(out)) and np.all(np.isfinite(lse))
    ro, rl = oracle_all_units(w, q)
    for b in range(w.B):
        for g in range(w.H_kv):
            rows = slice(4 * g, 4 * g + 4)
            assert_close(out[b, rows], lse[b, rows], ro[b, rows], rl[b, rows], f"{name} unit {(b, g)}")


# ------------------------------------------------------------------- RDR --
EPS = (1.1e-4, 2.75e-2, 7.12e-2, 2.0)


@pytest.mark.parametrize("shape", [dict(B=3, ctx=1000, H_kv=2), dict(B=5, ctx=333, H_kv=8)])
def test_rdr_matches_oracle(shape):
    torch = _torch()
    w = W.make("e2e_rdr", B=shape["B"], ctx=shape["ctx"], H_kv=shape["H_kv"], H_q=4 * shape["H_kv"])
    util = w.utility()
    for frac in (0.1, 0.25, 0.6):
        budget = int(frac * 512 * w.H_kv * int(w.seq_lens.sum()))
        budget = max(budget, 12 * 4160 * w.B * w.H_kv)
        want_t, want_lam, want_b = oracle.rdr_assign(w.page_offsets, w.seq_lens, util, EPS, budget, 4, 8,
                                                     w.H_kv, tiers_init=w.tiers)
        cache = gpu_cache(w, encode=False)
        lam, nb = cache.rdr_assign(to_torch(util), EPS, budget, 4, 8)
        cache.check()
        assert np.array_equal(cache.tiers.cpu().numpy(), want_t)
        assert float(lam.item()) == want_lam and int(nb.item()) == want_b <= budget


def test_rdr_infeasible_budget_reports():
    from compressed_paged_kv_ada_b200 import SphkvError

    w = W.make("e2e_rdr", B=2, ctx=500, H_kv=2, H_q=8)
    cache = gpu_cache(w, encode=False)
    cache.rdr_assign(to_torch(w.utility()), EPS, 1000, 4, 8)
    with pytest.raises(SphkvError) as e:
        cache.check()
    assert e.value.code == 3


def test_e2e_rdr_full():
    """End-to-end: 16 x 32768 prefill, RDR at 25 % of the fp16 bytes (tiers
    bit-exact vs the oracle), encode into the chosen tiers, then 256 steps of
    append + decode.  Against the oracle: every unit at steps 0, 1 and 255,
    and every step for sequences 0 and 1."""
    from concurrent.futures import ThreadPoolExecutor

    torch = _torch()
    w = W.make("e2e_rdr")
    util = w.utility()
    budget = w.extra["budget"]
    cache = gpu_cache(w, encode=False)
    lam, nb = cache.rdr_assign(to_torch(util), EPS, budget, 4, 8)
    cache.check()
    want_t, want_lam, want_b = oracle.rdr_assign(w.page_offsets, w.seq_lens, util, EPS, budget, 4, 8,
                                                 w.H_kv, tiers_init=w.tiers)
    tiers = cache.tiers.cpu().numpy()
    assert np.array_equal(tiers, want_t)
    assert float(lam.item()) == want_lam and int(nb.item()) == want_b <= budget
    cache.reallocate_pools()
    for b in range(w.B):
        n = int(w.seq_lens[b])
        K, V = w.dense_rows(b, 0, n)
        Kt, Vt = dense_torch(w, K, V)
        cache.encode(Kt, Vt, torch.full((n,), b, dtype=torch.int32, device="cuda"),
                     torch.arange(n, dtype=torch.int32, device="cuda"))
    cache.check()
    steps = w.extra["steps"]
    prefill = w.seq_lens.copy()
    lens = prefill.copy()
    full_steps = (0, 1, steps - 1)
    got_full, got_seq01 = {}, []
    # the appended rows of every sequence, drawn once (a row is the same
    # whichever slice it is drawn in)
    app = [w.dense_rows(b, int(prefill[b]), int(prefill[b]) + steps) for b in range(w.B)]
    for step in range(steps):
        Kd, Vd = dense_torch(w, np.stack([a[0][step] for a in app]), np.stack([a[1][step] for a in app]))
        cache.encode(Kd, Vd, torch.arange(w.B, dtype=torch.int32, device="cuda"),
                     to_torch(lens.astype(np.int32)))
        lens += 1
        cache.seq_lens.copy_(to_torch(lens.astype(np.int32)))
        out, lse = cache.decode(to_torch(w.queries(step + 1), torch.float32))
        if step in full_steps:
            cache.check()
            got_full[step] = (out.cpu().numpy(), lse.cpu().numpy())
        got_seq01.append((out[:2].cpu().numpy(), lse[:2].cpu().numpy()))
    cache.check()
    del cache
    # every unit at steps 0, 1, 255
    for step in full_steps:
        o, l = got_full[step]
        ro, rl = oracle_all_units(w, w.queries(step + 1), lens=prefill + step + 1, tiers=tiers)
        for b in range(w.B):
            for g in range(w.H_kv):
                rs = slice(4 * g, 4 * g + 4)
                assert_close(o[b, rs], l[b, rs], ro[b, rs], rl[b, rs], f"step {step} unit {(b, g)}")
    # every step for sequences 0 and 1: each unit's keys decoded once and its
    # kept tokens packed in position order, so the prefix a step saw is a
    # contiguous slice (no copy); then dense attention over that prefix
    dense = {}
    for b in (0, 1):
        for g in range(w.H_kv):
            kh, vh, keep = oracle_unit_dense(w, b, g, int(lens[b]), tiers)
            dense[(b, g)] = (np.ascontiguousarray(kh[keep]), np.ascontiguousarray(vh[keep]), np.cumsum(keep))
    qs = [np.asarray(w.queries(step + 1), np.float64) for step in range(steps)]

    def ref(item):
        step, b, g = item
        kk, vk, n_kept = dense[(b, g)]
        m = int(n_kept[int(prefill[b]) + step])   # kept tokens among the first prefill + step + 1
        return item, oracle.attention(kk[:m], vk[:m], qs[step][b, 4 * g:4 * g + 4])

    items = [(step, b, g) for step in range(steps) for b in (0, 1) for g in range(w.H_kv)]
    with ThreadPoolExecutor(max_workers=max(1, oracle.num_threads())) as ex:
        for (step, b, g), (ro, rl) in ex.map(ref, items):
            o, l = got_seq01[step]
            rs = slice(4 * g, 4 * g + 4)
            assert_close(o[b, rs], l[b, rs], ro, rl, f"step {step} unit {(b, g)}")


# ---------------------------------------------------------------- errors --
def test_bad_page_id_reports_data_error():
    torch = _torch()
    from compressed_paged_kv_ada_b200 import SphkvError

    w = W.make("ragged64", seq_lens=[200], H_kv=1, H_q=4)
    cache = gpu_cache(w)
    t = cache.page_table.cpu().numpy()
    t[0, 3] = (1 << 30) | 999999   # pool page far out of range: checked before any read
    cache.page_table.copy_(to_torch(t))
    cache.decode(to_torch(w.queries(), torch.float32))
    with pytest.raises(SphkvError) as e:
        cache.check()
    assert e.value.code == 6


def test_encode_bad_position_reports_data_error():
    torch = _torch()
    from compressed_paged_kv_ada_b200 import SphkvError

    w = W.make("ragged64", seq_lens=[40], H_kv=1, H_q=4)
    cache = gpu_cache(w, encode=False)
    K, V = dense_torch(w, *w.dense_rows(0, 0, 2))
    cache.encode(K, V, torch.tensor([0, 7], dtype=torch.int32, device="cuda"),
                 torch.tensor([0, 1], dtype=torch.int32, device="cuda"))
    with pytest.raises(SphkvError) as e:
        cache.check()
    assert e.value.code == 6


def test_host_argument_errors():
    torch = _torch()
    from compressed_paged_kv_ada_b200 import SphkvError

    w = W.make("ragged64", seq_lens=[40], H_kv=1, H_q=4)
    cache = gpu_cache(w, encode=False)
    q = torch.zeros((1, 8, 128), dtype=torch.float32, device="cuda")
    with pytest.raises(SphkvError) as e:
        cache.decode(q)   # H_q / H_kv = 8 is not supported
    assert e.value.code == 1
