"""Pins for the fp64 CPU oracle, checked against things other than itself:
library routines (numpy's fp16 conversion), hand-worked cases, closed forms,
explicit small-d formulas, rigorous error bounds and brute force.

Each test names the fact it pins.  None of them needs a GPU.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest

import oracle
from compressed_paged_kv_ada_b200 import workloads as W

GOLD = os.path.join(os.path.dirname(__file__), "golden")
TIERS = oracle.TIER_BITS


def _dir_err(d, b_leaf, b_up):
    """Worst-case direction error: half a leaf step plus half an upper step per
    upper level (levels act on disjoint subspaces of total weight 1)."""
    levels = int(round(math.log2(d // 2)))
    return math.pi / 2 ** b_leaf + levels * (math.pi / 2) / (2 * (2 ** b_up - 1))


def _random_codes(rng, n, d, b_leaf, b_up, inner_only=False):
    L = d // 2
    leaf = rng.integers(0, 2 ** b_leaf, size=(n, L)).astype(np.uint8)
    lo, hi = (1, 2 ** b_up - 2) if inner_only else (0, 2 ** b_up - 1)
    up = rng.integers(lo, hi, size=(n, L - 1), endpoint=True).astype(np.uint8)
    # radii: random normal fp16 values in [0.25, 64)
    r = rng.uniform(0.25, 64.0, size=n)
    r16 = r.astype(np.float16).view(np.uint16)
    return leaf, up, r16


# ------------------------------------------------------------------ fp16 --
def test_fp16_rounding_matches_numpy():
    """Pin: the oracle's double->half RNE equals numpy's conversion (a library
    routine), on random values over the whole range, halfway ties, subnormals
    and the overflow edge."""
    rng = np.random.default_rng(1)
    xs = list(rng.standard_normal(3000) * np.exp(rng.uniform(-25, 12, 3000)))
    # exact ties between consecutive halves, subnormal ties and the overflow edge
    h = np.arange(0, 0x7bff, 7, dtype=np.uint16).view(np.float16).astype(np.float64)
    xs += list((h[:-1] + h[1:]) / 2)
    xs += [0.0, -0.0, 65504.0, 65519.99, 65520.0, 1e9, 2.0 ** -24, 2.0 ** -25, 3 * 2.0 ** -26,
           2.0 ** -26, 6.1e-5, -6.1e-5, 1 / 127, 2 / 127]
    for x in xs:
        want = int(np.array(x, np.float64).astype(np.float16).view(np.uint16))
        got = oracle.f64_to_f16_bits(x)
        assert got == want, (x, hex(got), hex(want))
    for bits in range(0, 0x10000, 3):
        want = float(np.array(bits, np.uint16).view(np.float16))
        got = oracle.f16_bits_to_f64(bits)
        if math.isnan(want):
            assert math.isnan(got)
        else:
            assert got == want


# -------------------------------------------------------------- hand case --
def test_hand_case():
    """Pin: the two-token d = 4 case worked by hand (tests/golden/hand_case.json)."""
    g = json.load(open(os.path.join(GOLD, "hand_case.json")))
    K = np.array(g["K"], np.float64)
    V = np.array(g["V"], np.float64)
    q = np.array(g["q"], np.float64)
    c = oracle.encode(K, V, bits=(8, 8, 8))
    assert c["leaf"].tolist() == g["leaf_codes"]
    assert c["up"].tolist() == g["up_codes"]
    assert [oracle.f16_bits_to_f64(x) for x in c["r16"]] == g["r"]
    assert [oracle.f16_bits_to_f64(x) for x in c["s16"]] == g["vscale"]
    assert c["vq"].tolist() == g["vq"]
    kh = oracle.decode_keys(c["leaf"], c["up"], c["r16"], 8, 8)
    np.testing.assert_allclose(kh, K, atol=1e-15)
    tl = oracle.tree_logits(c["leaf"], c["up"], c["r16"], 8, 8, q)
    np.testing.assert_allclose(tl, g["logits"], atol=1e-15)
    vh = oracle.decode_values(c["vq"], c["s16"])
    out, lse = oracle.attention(kh, vh, q[None])
    p1 = 1.0 / (1.0 + math.exp(0.5))
    p2 = 1.0 / (1.0 + math.exp(-0.5))
    s1, s2 = g["vscale"]
    want_out = [p1 * 127 * s1, -p1 * 127 * s1, p2 * 127 * s2, 0.0]
    want_lse = 1.0 + math.log(1.0 + math.exp(-0.5))
    np.testing.assert_allclose(out[0], want_out, rtol=0, atol=1e-14)
    assert abs(lse[0] - want_lse) < 1e-14
    # and the numbers written out in decimal in the derivation
    np.testing.assert_allclose(out[0], [0.3775176255444346, -0.3775176255444346,
                                        1.2448426785986308, 0.0], atol=1e-14)
    assert abs(lse[0] - 1.4740769841801067) < 1e-14


# ---------------------------------------------------------- tree identity --
@pytest.mark.parametrize("tier", [1, 2, 3])
@pytest.mark.parametrize("d", [4, 8, 16, 64, 128])
def test_tree_logit_equals_dense_dot(tier, d):
    """Pin: the bottom-up angle-domain tree (leaf q.(cos, sin), node
    cos psi S_L + sin psi S_R) equals q . decode(codes) / sqrt(d) to 1e-12,
    for random codes of every tier (both are the same multilinear form)."""
    b_leaf, b_up, _ = TIERS[tier]
    rng = np.random.default_rng(10 * tier + d)
    leaf, up, r16 = _random_codes(rng, 300, d, b_leaf, b_up)
    for _ in range(3):
        q = rng.standard_normal(d) * rng.uniform(0.1, 5)
        tl = oracle.tree_logits(leaf, up, r16, b_leaf, b_up, q)
        kh = oracle.decode_keys(leaf, up, r16, b_leaf, b_up)
        dense = kh @ q / math.sqrt(d)
        r = r16.view(np.float16).astype(np.float64)
        scale = np.maximum(1.0, r * np.linalg.norm(q) / math.sqrt(d))
        assert np.all(np.abs(tl - dense) <= 1e-12 * scale)


def test_decode_matches_explicit_small_d():
    """Pin: decode for d = 4 and d = 8 equals the recursive-polar direction
    written out by hand as products of cosines and sines."""
    rng = np.random.default_rng(3)
    for tier, (bl, bu, _) in TIERS.items():
        leaf, up, r16 = _random_codes(rng, 50, 4, bl, bu)
        kh = oracle.decode_keys(leaf, up, r16, bl, bu)
        for i in range(50):
            f0 = 2 * math.pi * leaf[i, 0] / 2 ** bl
            f1 = 2 * math.pi * leaf[i, 1] / 2 ** bl
            ps = (math.pi / 2) * up[i, 0] / (2 ** bu - 1)
            r = float(r16[i:i + 1].view(np.float16)[0])
            want = r * np.array([math.cos(ps) * math.cos(f0), math.cos(ps) * math.sin(f0),
                                 math.sin(ps) * math.cos(f1), math.sin(ps) * math.sin(f1)])
            np.testing.assert_allclose(kh[i], want, atol=1e-13 * r)
        leaf, up, r16 = _random_codes(rng, 50, 8, bl, bu)
        kh = oracle.decode_keys(leaf, up, r16, bl, bu)
        for i in range(50):
            f = [2 * math.pi * leaf[i, j] / 2 ** bl for j in range(4)]
            # level order: level-1 nodes (leaves 0,1) and (leaves 2,3), then the root
            a, b, root = [(math.pi / 2) * up[i, m] / (2 ** bu - 1) for m in range(3)]
            w = [math.cos(root) * math.cos(a), math.cos(root) * math.sin(a),
                 math.sin(root) * math.cos(b), math.sin(root) * math.sin(b)]
            r = float(r16[i:i + 1].view(np.float16)[0])
            want = r * np.array([w[j // 2] * (math.cos(f[j // 2]) if j % 2 == 0 else math.sin(f[j // 2]))
                                 for j in range(8)])
            np.testing.assert_allclose(kh[i], want, atol=1e-13 * r)


# ---------------------------------------------------------- encode checks --
@pytest.mark.parametrize("tier", [1, 2, 3])
def test_grid_points_reencode_exactly(tier):
    """Pin: a key placed exactly on the angle grid (decode of random codes)
    re-encodes to the same codes and radius."""
    bl, bu, vb = TIERS[tier]
    rng = np.random.default_rng(20 + tier)
    leaf, up, r16 = _random_codes(rng, 400, 128, bl, bu, inner_only=True)
    kh = oracle.decode_keys(leaf, up, r16, bl, bu)
    c = oracle.encode(kh, np.zeros_like(kh), bits=(bl, bu, vb))
    assert np.array_equal(c["leaf"], leaf)
    assert np.array_equal(c["up"], up)
    assert np.array_equal(c["r16"], r16)


def test_zero_subtrees_and_axis_keys():
    """Pin: with the end-inclusive upper grid a zero half of the key gives an
    exact 0 or pi/2 upper angle, zero pairs get code 0, and axis keys decode
    exactly."""
    d = 16
    K = np.zeros((4, d))
    K[0, 0] = 3.0           # all weight in the leftmost leaf
    K[1, d - 1] = -2.0      # all weight in the last coordinate
    K[2, 4:8] = [1, 1, 1, 1]
    K[3, :] = 0.0           # the zero key
    c = oracle.encode(K, np.zeros_like(K), bits=(8, 8, 8))
    assert c["up"][0].tolist() == [0] * 7
    assert c["leaf"][0].tolist() == [0] * 8
    assert c["up"][1].tolist() == [0, 0, 0, 255, 0, 255, 255]
    assert c["leaf"][1].tolist() == [0] * 7 + [192]  # atan2(-2, 0) = -pi/2 -> -64 mod 256
    assert c["up"][3].tolist() == [0] * 7 and c["leaf"][3].tolist() == [0] * 8
    assert oracle.f16_bits_to_f64(c["r16"][3]) == 0.0
    kh = oracle.decode_keys(c["leaf"], c["up"], c["r16"], 8, 8)
    np.testing.assert_allclose(kh[0], K[0], atol=1e-15)
    np.testing.assert_allclose(kh[1], K[1], atol=1e-15)
    np.testing.assert_allclose(kh[3], 0.0)


@pytest.mark.parametrize("tier", [1, 2, 3])
def test_encode_error_bounds(tier):
    """Pin: for every tier the decoded direction is within the worst-case
    angle error bound of the true direction, |v - v_hat| <= s/2, and the radius
    is the fp16 rounding of |k|."""
    bl, bu, vb = TIERS[tier]
    rng = np.random.default_rng(30 + tier)
    sig = rng.lognormal(0, 0.5, 128)
    sig[rng.choice(128, 4, replace=False)] *= 8
    K = rng.standard_normal((2000, 128)) * sig
    V = rng.standard_normal((2000, 128))
    c = oracle.encode(K, V, tier)
    kh = oracle.decode_keys(c["leaf"], c["up"], c["r16"], bl, bu)
    r = np.linalg.norm(K, axis=1)
    rh = c["r16"].view(np.float16).astype(np.float64)
    assert np.all(np.abs(r - rh) <= np.abs(r) * 2.0 ** -11 + 1e-300)
    u = K / r[:, None]
    uh = kh / rh[:, None]
    err = np.linalg.norm(u - uh, axis=1)
    assert err.max() <= _dir_err(128, bl, bu) + 1e-12
    vh = oracle.decode_values(c["vq"], c["s16"])
    s = c["s16"].view(np.float16).astype(np.float64)
    assert np.all(np.abs(V - vh) <= s[:, None] / 2 + 1e-15)
    Q = 127 if vb == 8 else 7
    assert np.abs(c["vq"]).max() <= Q


@pytest.mark.parametrize("tier", [1, 2, 3])
def test_logits_within_bound_of_dense(tier):
    """Pin: every code-domain logit is within delta_t = |q| (r e_dir + |r - r_hat|)
    / sqrt(d) of the exact dense logit q.k / sqrt(d); T1 attention stays within
    the derived bounds of exact dense fp64 attention (|dlse| <= max delta,
    |dout| <= (e^(2 max delta) - 1) max|v_hat| + max s / 2)."""
    bl, bu, _ = TIERS[tier]
    rng = np.random.default_rng(40 + tier)
    d = 128
    sig = rng.lognormal(0, 0.5, d)
    K = rng.standard_normal((2048, d)) * sig
    V = rng.standard_normal((2048, d))
    q = rng.standard_normal((4, d))
    c = oracle.encode(K, V, tier)
    kh = oracle.decode_keys(c["leaf"], c["up"], c["r16"], bl, bu)
    vh = oracle.decode_values(c["vq"], c["s16"])
    r = np.linalg.norm(K, axis=1)
    rh = c["r16"].view(np.float16).astype(np.float64)
    e = _dir_err(d, bl, bu)
    for h in range(4):
        delta = np.linalg.norm(q[h]) * (r * e + np.abs(r - rh)) / math.sqrt(d)
        l_ex = K @ q[h] / math.sqrt(d)
        l_or = oracle.tree_logits(c["leaf"], c["up"], c["r16"], bl, bu, q[h])
        assert np.all(np.abs(l_or - l_ex) <= delta + 1e-12)
        eps_max = delta.max()
        out_o, lse_o = oracle.attention(kh, vh, q[h:h + 1])
        m = l_ex.max()
        p = np.exp(l_ex - m)
        out_d = (p[:, None] * V).sum(0) / p.sum()
        lse_d = m + math.log(p.sum())
        assert abs(lse_o[0] - lse_d) <= eps_max + 1e-12
        s = c["s16"].view(np.float16).astype(np.float64)
        bound = (math.exp(2 * eps_max) - 1) * np.abs(vh).max() + s.max() / 2
        assert np.abs(out_o[0] - out_d).max() <= bound + 1e-12


# -------------------------------------------------------------- attention --
def _small_cache(rng, tiers_per_page, seq_len, H_kv=1, G=4):
    """A one-sequence cache built with the oracle's own encoder and packer."""
    n_pages = len(tiers_per_page)
    tiers = np.array([tiers_per_page] * H_kv, np.uint8)
    table = oracle.build_page_table(tiers)
    K = rng.standard_normal((seq_len, H_kv, 128)) * rng.lognormal(0, 0.5, 128)
    V = rng.standard_normal((seq_len, H_kv, 128))
    counts = [int((tiers == t).sum()) for t in (1, 2, 3)]
    pools = oracle.encode_cache(K, V, np.zeros(seq_len, np.int32), np.arange(seq_len),
                                np.array([0, n_pages]), table, counts)
    cache = dict(B=1, H_q=G * H_kv, H_kv=H_kv, page_offsets=np.array([0, n_pages], np.int32),
                 seq_lens=np.array([seq_len], np.int32), page_table=table, pools=pools)
    return cache, K, V


def test_dropped_pages_contribute_exactly_zero():
    """Pin: attention over a cache with dropped pages equals, bit for bit,
    attention over the same tokens with the dropped tokens deleted."""
    rng = np.random.default_rng(5)
    tiers = [1, 0, 2, 3, 0, 0, 1, 2]
    cache, K, V = _small_cache(rng, tiers, 8 * 16 - 5)
    q = rng.standard_normal((1, 4, 128))
    out, lse = oracle.cache_attention(cache, q, [(0, 0)])
    keep_k, keep_v = [], []
    for t in range(K.shape[0]):
        tier = tiers[t // 16]
        if tier == 0:
            continue
        c = oracle.encode(K[t:t + 1, 0], V[t:t + 1, 0], tier)
        bl, bu, _ = TIERS[tier]
        keep_k.append(oracle.decode_keys(c["leaf"], c["up"], c["r16"], bl, bu)[0])
        keep_v.append(oracle.decode_values(c["vq"], c["s16"])[0])
    out2, lse2 = oracle.attention(np.array(keep_k), np.array(keep_v), q[0])
    assert np.array_equal(out[0], out2)
    assert np.array_equal(lse[0], lse2)


def test_multi_query_is_causal_prefix_attention():
    """Pin (multi-token decode): query token i of n_q equals, bit for bit,
    attention over the kept tokens among the first seq_len - (n_q - 1 - i),
    each decoded on its own; n_q = 1 is plain single-query attention."""
    rng = np.random.default_rng(9)
    tiers = [1, 2, 0, 3, 1, 2, 3, 1]
    seq_len = 8 * 16 - 5
    cache, K, V = _small_cache(rng, tiers, seq_len)
    n_q = 3
    q = rng.standard_normal((1, n_q, 4, 128))
    out, lse = oracle.multi_query_attention(cache, q, [(0, 0)], n_q)
    o1, l1 = oracle.cache_attention(cache, q[:, n_q - 1], [(0, 0)])
    assert np.array_equal(out[n_q - 1], o1) and np.array_equal(lse[n_q - 1], l1)
    for i in range(n_q):
        n_i = seq_len - (n_q - 1 - i)
        keep_k, keep_v = [], []
        for t in range(n_i):
            tier = tiers[t // 16]
            if tier == 0:
                continue
            c = oracle.encode(K[t:t + 1, 0], V[t:t + 1, 0], tier)
            bl, bu, _ = TIERS[tier]
            keep_k.append(oracle.decode_keys(c["leaf"], c["up"], c["r16"], bl, bu)[0])
            keep_v.append(oracle.decode_values(c["vq"], c["s16"])[0])
        o2, l2 = oracle.attention(np.array(keep_k), np.array(keep_v), q[0, i])
        assert np.array_equal(out[i, 0], o2) and np.array_equal(lse[i, 0], l2), i
    # a sequence shorter than n_q: the early query tokens see nothing
    short = dict(cache, seq_lens=np.array([1], np.int32))
    o, l = oracle.multi_query_attention(short, q, [(0, 0)], n_q)
    assert np.all(np.isneginf(l[:n_q - 1])) and np.all(o[:n_q - 1] == 0) and np.all(np.isfinite(l[n_q - 1]))


def test_special_cases():
    """Pin: q = 0 gives the mean of the kept values and lse = ln(#kept); one
    kept token gives its value and its logit; no kept token gives out = 0,
    lse = -inf."""
    rng = np.random.default_rng(6)
    cache, K, V = _small_cache(rng, [2, 0, 3], 40)
    q = np.zeros((1, 4, 128))
    out, lse = oracle.cache_attention(cache, q, [(0, 0)])
    kept = [t for t in range(40) if (t // 16) != 1]
    vh = []
    for t in kept:
        tier = [2, 0, 3][t // 16]
        c = oracle.encode(K[t:t + 1, 0], V[t:t + 1, 0], tier)
        vh.append(oracle.decode_values(c["vq"], c["s16"])[0])
    np.testing.assert_allclose(out[0, 0], np.mean(vh, 0), atol=1e-14)
    assert abs(lse[0, 0] - math.log(len(kept))) < 1e-14

    cache, K, V = _small_cache(rng, [1], 1)
    q = rng.standard_normal((1, 4, 128))
    out, lse = oracle.cache_attention(cache, q, [(0, 0)])
    c = oracle.encode(K[:, 0], V[:, 0], 1)
    vh = oracle.decode_values(c["vq"], c["s16"])[0]
    for h in range(4):
        np.testing.assert_allclose(out[0, h], vh, atol=1e-15)
        lt = oracle.tree_logits(c["leaf"], c["up"], c["r16"], 8, 8, q[0, h])[0]
        assert abs(lse[0, h] - lt) < 1e-12

    cache, K, V = _small_cache(rng, [0, 0], 20)
    out, lse = oracle.cache_attention(cache, q, [(0, 0)])
    assert np.all(out == 0) and np.all(np.isneginf(lse))


# ------------------------------------------------------------ page format --
def test_page_layout_golden():
    """Pin: packed bytes equal the hand-worked bytes in tests/golden/page_layout.json."""
    g = json.load(open(os.path.join(GOLD, "page_layout.json")))
    for t in (1, 2, 3):
        assert oracle.page_bytes(t) == g["page_bytes"][str(t)]
    z_v = np.zeros(128, np.int8)
    u32 = lambda b: int.from_bytes(bytes(b), "little")
    # T1
    page = np.zeros(oracle.page_bytes(1), np.uint8)
    oracle.pack_token(1, 0, np.arange(64).astype(np.uint8), np.arange(63).astype(np.uint8), 0, 0, z_v, page)
    assert page[64:80].tolist() == g["t1_block0"]
    assert page[64 + 7 * 16:64 + 8 * 16].tolist() == g["t1_block7"]
    assert page[64 + 6 * 16 + 15] == g["t1_block6_last"]
    # T2
    page = np.zeros(oracle.page_bytes(2), np.uint8)
    oracle.pack_token(2, 0, (np.arange(64) % 16).astype(np.uint8), np.arange(63).astype(np.uint8), 0, 0,
                      z_v, page)
    assert [u32(page[64:68]), u32(page[68:72])] == g["t2_block0_words"]
    assert u32(page[64 + 1024:64 + 1026]) == g["t2_block0_high"]
    # T3
    page = np.zeros(oracle.page_bytes(3), np.uint8)
    oracle.pack_token(3, 0, (np.arange(64) % 8).astype(np.uint8), (np.arange(63) % 16).astype(np.uint8), 0,
                      0, z_v, page)
    assert u32(page[64:68]) == g["t3_block0_upper"]
    assert u32(page[64 + 512:64 + 514]) == g["t3_block0_leaf_low"]
    assert page[64 + 768] == g["t3_block0_leaf_high"]
    # values
    page = np.zeros(oracle.page_bytes(1), np.uint8)
    oracle.pack_token(1, 0, np.zeros(64, np.uint8), np.zeros(63, np.uint8), 0, 0,
                      (np.arange(128) - 64).astype(np.int8), page)
    assert page[2112:2115].tolist() == g["v_int8_first_bytes"]
    assert page[2112 + 16] == g["v_int8_byte16"]
    page = np.zeros(oracle.page_bytes(1), np.uint8)
    oracle.pack_token(1, 3, np.zeros(64, np.uint8), np.zeros(63, np.uint8), 0, 0,
                      (np.arange(128) - 64).astype(np.int8), page)
    at = g["v_int8_slot3_chunk0_at"]
    assert page[at:at + 3].tolist() == g["v_int8_first_bytes"]
    page = np.zeros(oracle.page_bytes(2), np.uint8)
    oracle.pack_token(2, 0, np.zeros(64, np.uint8), np.zeros(63, np.uint8), 0, 0,
                      ((np.arange(128) % 15) - 7).astype(np.int8), page)
    assert page[1344:1346].tolist() == g["v_int4_first_bytes"]
    page = np.zeros(oracle.page_bytes(2), np.uint8)
    oracle.pack_token(2, 3, np.zeros(64, np.uint8), np.zeros(63, np.uint8), 0, 0,
                      ((np.arange(128) % 15) - 7).astype(np.int8), page)
    at = g["v_int4_slot3_first_bytes_at"]
    assert page[at:at + 2].tolist() == g["v_int4_first_bytes"]


def _blocks(leaf, up):
    """Subtree blocks written out from the level-order definition."""
    L = [[int(leaf[8 * s + j]) for j in range(8)] for s in range(8)]
    U = []
    for s in range(8):
        u = [int(up[4 * s + j]) for j in range(4)] + [int(up[32 + 2 * s]), int(up[33 + 2 * s]), int(up[48 + s])]
        u.append(int(up[56 + s]) if s < 7 else 0)
        U.append(u)
    return L, U


def test_pack_unpack_roundtrip_and_independent_layout():
    """Pin: pack/unpack round-trips for every tier and slot, and every field
    equals the same codes assembled independently as Python integers from the
    layout description; other slots are untouched."""
    rng = np.random.default_rng(7)
    for t, (bl, bu, vb) in TIERS.items():
        page = np.zeros(oracle.page_bytes(t), np.uint8)
        rows = []
        for slot in rng.permutation(16):
            leaf = rng.integers(0, 2 ** bl, 64).astype(np.uint8)
            up = rng.integers(0, 2 ** bu, 63).astype(np.uint8)
            Q = 127 if vb == 8 else 7
            vq = rng.integers(-Q, Q, 128, endpoint=True).astype(np.int8)
            r16, s16 = int(rng.integers(0, 0x7bff)), int(rng.integers(0, 0x7bff))
            oracle.pack_token(t, int(slot), leaf, up, r16, s16, vq, page)
            rows.append((int(slot), leaf, up, r16, s16, vq))
        for slot, leaf, up, r16, s16, vq in rows:
            u = oracle.unpack_token(t, slot, page)
            assert np.array_equal(u["leaf"], leaf) and np.array_equal(u["up"], up)
            assert u["r16"] == r16 and u["s16"] == s16 and np.array_equal(u["vq"], vq)
            L, U = _blocks(leaf, up)
            rd = lambda off, n: int.from_bytes(bytes(page[off:off + n]), "little")
            for s in range(8):
                blk = slot * 8 + s
                if t == 1:
                    assert page[64 + 16 * blk:64 + 16 * blk + 16].tolist() == L[s] + U[s]
                elif t == 2:
                    assert rd(64 + 8 * blk, 4) == sum(L[s][j] << (4 * j) for j in range(8))
                    uf = sum(U[s][j] << (6 * j) for j in range(8))
                    assert rd(68 + 8 * blk, 4) == uf & 0xFFFFFFFF
                    assert rd(64 + 1024 + 2 * blk, 2) == uf >> 32
                else:
                    assert rd(64 + 4 * blk, 4) == sum(U[s][j] << (4 * j) for j in range(8))
                    lf = sum(L[s][j] << (3 * j) for j in range(8))
                    assert rd(64 + 512 + 2 * blk, 2) == lf & 0xFFFF
                    assert rd(64 + 768 + blk, 1) == lf >> 16
            voff = 64 + 16 * {1: 128, 2: 80, 3: 56}[t]
            for p in range(128):
                ch = 16 * ((p >> 1) & 7) + (p >> 4) + 8 * (p & 1)
                gq, j = p // 16, p % 16
                if vb == 8:
                    at = voff + slot * 128 + 16 * (gq ^ (slot & 6)) + j
                    assert int(page[at].astype(np.int8)) == vq[ch]
                else:
                    i = slot // 2
                    at = voff + i * 128 + 16 * (gq ^ ((2 * i) & 6)) + 8 * (slot % 2) + j // 2
                    nib = (int(page[at]) >> (4 * (p % 2))) & 15
                    assert (nib - 16 if nib >= 8 else nib) == vq[ch]
            assert int(page[2 * slot]) | int(page[2 * slot + 1]) << 8 == r16
            assert int(page[32 + 2 * slot]) | int(page[33 + 2 * slot]) << 8 == s16


def test_page_table_entries():
    """Pin: entry = tier << 30 | pool index; the k-th page of a tier in table
    order gets perm[k]."""
    tiers = np.array([[1, 0, 2, 1, 3, 2, 0, 1]], np.uint8)
    t = oracle.build_page_table(tiers).view(np.uint32)
    assert t.tolist() == [[(1 << 30) | 0, 0, (2 << 30) | 0, (1 << 30) | 1, (3 << 30) | 0,
                           (2 << 30) | 1, 0, (1 << 30) | 2]]
    p1 = np.array([2, 0, 1], np.int32)
    t = oracle.build_page_table(tiers, (p1, None, None)).view(np.uint32)
    assert [x & 0x3fffffff for x in t[0, [0, 3, 7]]] == [2, 0, 1]


# -------------------------------------------------------------------- RDR --
EPS = np.array([1.1e-4, 2.75e-2, 7.12e-2, 2.0])
RATE = [4160, 2368, 1984, 0]


def _rdr_small(U_pages, budget, n_sink=0, n_recent=0):
    """Units = pages of one sequence with one token each carrying utility U."""
    n = len(U_pages)
    util = np.zeros((1, n * 16), np.float32)
    util[0, ::16] = U_pages
    lens = np.array([16 * (n - 1) + 1], np.int32)
    return oracle.rdr_assign(np.array([0, n], np.int32), lens, util, EPS, budget, n_sink,
                             n_recent, 1)


def test_rdr_hand_case():
    """Pin: worked by hand.  Units U = 100 and U = 1, budget 4160 + 2368.
    The U = 1 unit leaves T1 for T2 at lambda = 1*(eps2 - eps1)/(4160 - 2368),
    the U = 100 unit only at 100x that, so the answer is (T1, T2) with lambda
    at the first breakpoint."""
    util = np.zeros((1, 32), np.float32)
    util[0, 0] = 100.0
    util[0, 16] = 1.0
    tiers, lam, nb = oracle.rdr_assign(np.array([0, 2], np.int32), np.array([17], np.int32),
                                       util, EPS, 4160 + 2368, 0, 0, 1)
    assert tiers[0].tolist() == [1, 2]
    assert nb == 4160 + 2368
    lam_star = (EPS[1] - EPS[0]) / (4160 - 2368)
    assert abs(lam - lam_star) <= 1e-12 * lam_star


def test_rdr_brute_force_optimality():
    """Pin: brute force over all 4^n assignments (n <= 8): the Lagrangian
    answer has the least total distortion among all assignments using no more
    bytes, it fits the budget, and forced units are T1."""
    rng = np.random.default_rng(8)
    for trial in range(25):
        n = int(rng.integers(2, 9))
        U = rng.lognormal(0, 1.5, n).astype(np.float32)
        n_sink = int(rng.integers(0, 2))
        total = sum(4160 for _ in range(n))
        budget = int(rng.integers(4160 * n_sink + 1, total + 1))
        tiers, lam, nb = _rdr_small(U, budget, n_sink=n_sink)
        t = tiers[0]
        idx = [0 if x == 1 else 1 if x == 2 else 2 if x == 3 else 3 for x in t]
        R = sum(RATE[i] for i in idx)
        assert R == nb <= budget
        assert all(x == 1 for x in t[:n_sink])
        D = sum(float(U[u]) * EPS[i] for u, i in enumerate(idx))
        best = math.inf
        for combo in itertools.product(range(4), repeat=n):
            if any(combo[u] != 0 for u in range(n_sink)):
                continue
            if sum(RATE[i] for i in combo) <= R:
                best = min(best, sum(float(U[u]) * EPS[i] for u, i in enumerate(combo)))
        assert D <= best * (1 + 1e-12) + 1e-300


def test_rdr_budget_monotone_and_infeasible():
    """Pin: more budget never costs distortion and never reduces bytes; a
    budget below the forced pages raises."""
    rng = np.random.default_rng(9)
    U = rng.lognormal(0, 1, 40).astype(np.float32)
    prev_b, prev_d = -1, math.inf
    for budget in np.linspace(4160 * 3, 4160 * 40, 25).astype(np.int64):
        tiers, lam, nb = _rdr_small(U, int(budget), n_sink=2, n_recent=1)
        idx = [{1: 0, 2: 1, 3: 2, 0: 3}[int(x)] for x in tiers[0]]
        D = sum(float(U[u]) * EPS[i] for u, i in enumerate(idx))
        # the Lagrangian path: a larger budget lowers lambda, and bytes(lambda)
        # is non-increasing, so the bytes chosen never drop as the budget grows
        assert nb <= budget and nb >= prev_b and D <= prev_d * (1 + 1e-12)
        prev_b, prev_d = nb, D
    with pytest.raises(OverflowError):
        _rdr_small(U, 4160 * 3 - 1, n_sink=2, n_recent=1)


def test_rdr_ties_go_to_higher_precision():
    """Pin: when several tiers cost exactly the same in fp64 (equal eps, and
    lambda*R below half an ulp of U*eps), the tie goes to the lower tier index,
    i.e. the higher precision.  A budget that fits every page at T1 drives
    lambda down to ~2^-100, where that happens."""
    util = np.zeros((1, 5 * 16), np.float32)
    util[0, ::16] = 1.0
    eps = np.array([0.5, 0.5, 0.5, 2.0])
    tiers, lam, nb = oracle.rdr_assign(np.array([0, 5], np.int32), np.array([65], np.int32),
                                       util, eps, 5 * 4160, 0, 0, 1)
    assert lam < 1e-20
    assert tiers[0].tolist() == [1] * 5 and nb == 5 * 4160


def test_merge_partials_is_attention_over_the_union():
    """Pin: the log-sum-exp combine of attention over disjoint key sets equals
    attention over their union (to fp64 rounding), whatever the split, with
    empty parts contributing nothing; every part empty gives out 0, lse -inf."""
    rng = np.random.default_rng(31)
    for trial in range(20):
        n = int(rng.integers(1, 300))
        k = rng.standard_normal((n, 128)) * rng.lognormal(0, 0.5, 128)
        v = rng.standard_normal((n, 128))
        q = rng.standard_normal((4, 128)) * 3.0
        o, l = oracle.attention(k, v, q)
        n_parts = int(rng.integers(1, 6))
        cuts = np.sort(rng.integers(0, n + 1, n_parts - 1))
        bounds = np.concatenate([[0], cuts, [n]])
        perm = rng.permutation(n)   # the parts need not be contiguous
        outs, lses = [], []
        for a, b in zip(bounds[:-1], bounds[1:]):
            idx = perm[a:b]
            oo, ll = oracle.attention(k[idx], v[idx], q)
            outs.append(oo)
            lses.append(ll)
        mo, ml = oracle.merge_partials(np.stack(outs), np.stack(lses))
        assert np.abs(ml - l).max() <= 1e-12 * max(1.0, np.abs(l).max())
        assert np.abs(mo - o).max() <= 1e-12 * max(1.0, np.abs(o).max())
    empty_o, empty_l = oracle.attention(np.zeros((0, 128)), np.zeros((0, 128)), np.ones((2, 128)))
    mo, ml = oracle.merge_partials(np.stack([empty_o, empty_o]), np.stack([empty_l, empty_l]))
    assert np.all(mo == 0) and np.all(np.isneginf(ml))


def _tiny_cache(seq_lens, H_kv=2, seed=5):
    """An oracle-encoded mixed-tier cache (its own encoder and packer)."""
    w = W.make("ragged64", seq_lens=seq_lens, H_kv=H_kv, H_q=4 * H_kv, seed=seed)
    K, V = w.dense(w.seq_lens)
    seq, pos = w.token_index(w.seq_lens)
    table = oracle.build_page_table(w.tiers)
    counts = [int((w.tiers == t).sum()) for t in (1, 2, 3)]
    pools = oracle.encode_cache(K, V, seq, pos, w.page_offsets, table, counts)
    return w, dict(B=w.B, H_q=w.H_q, H_kv=w.H_kv, page_offsets=w.page_offsets, seq_lens=w.seq_lens,
                   page_table=table, pools=pools)


def test_set_keep_flips_only_radius_sign_bits_and_is_reversible():
    """Pin: the drop flag is the sign bit of the stored radius; set_keep changes
    exactly those bits of the present tokens of kept pages, and keeping every
    token again restores the pages byte for byte."""
    w, c = _tiny_cache([40, 17, 33])
    before = [p.copy() for p in c["pools"]]
    rng = np.random.default_rng(2)
    keep = (rng.random((w.H_kv, w.total_pages * 16)) < 0.6).astype(np.uint8)
    oracle.set_keep(c, keep)
    po = w.page_offsets
    for g in range(w.H_kv):
        for b in range(w.B):
            for t in range(int(w.seq_lens[b])):
                lp = po[b] + t // 16
                e = int(c["page_table"][g, lp]) & 0xFFFFFFFF
                tier, phys = e >> 30, e & 0x3FFFFFFF
                if tier == 0:
                    continue
                off = 2 * (t % 16)
                r_new = int(c["pools"][tier - 1][phys, off]) | int(c["pools"][tier - 1][phys, off + 1]) << 8
                r_old = int(before[tier - 1][phys, off]) | int(before[tier - 1][phys, off + 1]) << 8
                assert r_old & 0x8000 == 0   # the encoder never writes a negative radius
                want = r_old | (0 if keep[g, lp * 16 + t % 16] else 0x8000)
                assert r_new == want
                c["pools"][tier - 1][phys, off:off + 2] = before[tier - 1][phys, off:off + 2]
    for p, q in zip(c["pools"], before):   # nothing else changed
        assert np.array_equal(p, q)
    oracle.set_keep(c, np.ones_like(keep))
    for p, q in zip(c["pools"], before):
        assert np.array_equal(p, q)


def test_dropped_tokens_are_exactly_deleted():
    """Pin: attention over a cache with tokens dropped by their flag equals,
    bit for bit, attention over the kept tokens alone (decoded the same way);
    keeping every token changes nothing; dropping all gives out 0, lse -inf."""
    w, c = _tiny_cache([70, 1, 45], seed=8)
    q = np.random.default_rng(4).standard_normal((w.B, w.H_q, 128))
    units = [(b, g) for b in range(w.B) for g in range(w.H_kv)]
    ro0, rl0 = oracle.cache_attention(c, q, units)
    oracle.set_keep(c, np.ones((w.H_kv, w.total_pages * 16), np.uint8))
    ro1, rl1 = oracle.cache_attention(c, q, units)
    assert np.array_equal(ro0, ro1) and np.array_equal(rl0, rl1)
    keep = (np.random.default_rng(9).random((w.H_kv, w.total_pages * 16)) < 0.5).astype(np.uint8)
    oracle.set_keep(c, keep)
    ro, rl = oracle.cache_attention(c, q, units)
    po = w.page_offsets
    for i, (b, g) in enumerate(units):
        n = int(w.seq_lens[b])
        K, V = w.dense_rows(b, 0, n)
        tt = np.repeat(w.tiers[g, po[b]:po[b] + (n + 15) // 16], 16)[:n]
        kh, vh = np.zeros((n, 128)), np.zeros((n, 128))
        for t in (1, 2, 3):
            idx = np.nonzero(tt == t)[0]
            if idx.size:
                cc = oracle.encode(K[idx, g], V[idx, g], t)
                bl, bu, _ = oracle.TIER_BITS[t]
                kh[idx] = oracle.decode_keys(cc["leaf"], cc["up"], cc["r16"], bl, bu)
                vh[idx] = oracle.decode_values(cc["vq"], cc["s16"])
        sel = (tt != 0) & (keep[g, po[b] * 16 + np.arange(n)] != 0)
        o, l = oracle.attention(kh[sel], vh[sel], q[b, 4 * g:4 * g + 4])
        assert np.array_equal(ro[i], o) and np.array_equal(rl[i], l)
    oracle.set_keep(c, np.zeros((w.H_kv, w.total_pages * 16), np.uint8))
    ro, rl = oracle.cache_attention(c, q, units)
    assert np.all(ro == 0) and np.all(np.isneginf(rl))


# --------------------------------------------- transcode / RDR re-run pins --
def _angle_dist_leaf(a, b):
    d = abs(a - b) % (2 * math.pi)
    return min(d, 2 * math.pi - d)


@pytest.mark.parametrize("pair", [(1, 2), (1, 3), (2, 3)])
def test_transcode_angles_are_nearest_coarse_grid_points(pair):
    """Pin (brute force over every code): a transcoded leaf code is the
    nearest point of the coarser periodic grid to the fine angle, ties to the
    even code; a transcoded upper code is the nearest point of the coarser
    end-inclusive grid (whose odd step count leaves no ties)."""
    a, b = pair
    bla, bua, _ = TIERS[a]
    blb, bub, _ = TIERS[b]
    for c in range(1 << bla):
        phi = 2 * math.pi * c / (1 << bla)
        dists = [_angle_dist_leaf(phi, 2 * math.pi * k / (1 << blb)) for k in range(1 << blb)]
        best = min(dists)
        cands = [k for k, dd in enumerate(dists) if dd <= best + 1e-12]
        got = oracle.transcode_token(a, b, np.full(64, c, np.uint8), np.zeros(63, np.uint8), 0,
                                     np.zeros(128, np.int8))["leaf"][0]
        assert got in cands and (len(cands) == 1 or got % 2 == 0), (c, cands, got)
    for c in range(1 << bua):
        psi = (math.pi / 2) * c / ((1 << bua) - 1)
        dists = [abs(psi - (math.pi / 2) * k / ((1 << bub) - 1)) for k in range(1 << bub)]
        got = oracle.transcode_token(a, b, np.zeros(64, np.uint8), np.full(63, c, np.uint8), 0,
                                     np.zeros(128, np.int8))["up"][0]
        assert dists[got] <= min(dists) + 1e-12 and sorted(dists)[1] > min(dists) + 1e-9


@pytest.mark.parametrize("pair", [(1, 2), (1, 3), (2, 3)])
def test_transcode_equals_reencoding_the_decoded_token(pair):
    """Pin: away from exact ties of the leaf grid, transcoding equals running
    the encoder on the decoded (fp64) key and values of the finer tier; value
    codes and scales agree always (the same fp64 quantiser on the same
    values)."""
    a, b = pair
    bla, bua, _ = TIERS[a]
    rng = np.random.default_rng(40 + a * 3 + b)
    K = rng.standard_normal((200, 128)) * rng.lognormal(0, 0.5, 128)
    V = rng.standard_normal((200, 128)) * np.where(rng.random((200, 1)) < 0.1, 50.0, 1.0)
    ca = oracle.encode(K, V, a)
    kh = oracle.decode_keys(ca["leaf"], ca["up"], ca["r16"], bla, bua)
    vh = oracle.decode_values(ca["vq"], ca["s16"])
    cb = oracle.encode(kh, vh, b)
    blb, bub, _ = TIERS[b]
    tie = (ca["leaf"].astype(np.int64) << blb) % (1 << bla) == (1 << bla) // 2
    n_cmp = 0
    for i in range(200):
        tc = oracle.transcode_token(a, b, ca["leaf"][i], ca["up"][i], ca["s16"][i], ca["vq"][i])
        # compare the keys the codes decode to: codes under a subtree whose
        # weight is exactly 0 (an upper code 0 gives sin = 0) do not matter,
        # and the encoder writes 0 there
        kt = oracle.decode_keys(tc["leaf"][None], tc["up"][None], ca["r16"][i:i + 1], blb, bub)[0]
        kr = oracle.decode_keys(cb["leaf"][i:i + 1], cb["up"][i:i + 1], cb["r16"][i:i + 1], blb, bub)[0]
        ok = np.repeat(~tie[i], 2)
        assert np.array_equal(kt[ok], kr[ok])
        assert tc["s16"] == cb["s16"][i] and np.array_equal(tc["vq"], cb["vq"][i])
        n_cmp += int(ok.sum())
    assert n_cmp > 200 * 128 * 0.4   # T2 -> T3: every odd leaf code is a tie


def test_transcode_direction_error_within_both_tiers_bounds():
    """Pin (triangle inequality): a key transcoded T1 -> T3 stays within the
    sum of the T1 and T3 worst-case angle bounds of the exact direction."""
    rng = np.random.default_rng(44)
    K = rng.standard_normal((300, 128)) * rng.lognormal(0, 0.5, 128)
    V = rng.standard_normal((300, 128))
    c1 = oracle.encode(K, V, 1)

    def bound(t):
        bl, bu, _ = TIERS[t]
        return math.pi / 2 ** bl + 6 * (math.pi / 2) / (2 * (2 ** bu - 1))

    for i in range(300):
        tc = oracle.transcode_token(1, 3, c1["leaf"][i], c1["up"][i], c1["s16"][i], c1["vq"][i])
        u = oracle.decode_keys(tc["leaf"][None], tc["up"][None], np.array([0x3C00], np.uint16), 3, 4)[0]
        k = K[i] / np.linalg.norm(K[i])
        assert np.linalg.norm(u - k) <= bound(1) + bound(3) + 1e-12


def test_rdr_rerun_uncapped_equals_assign_and_respects_caps():
    """Pin: with every page at T1 (nothing to cap) the re-run is RDR itself;
    with caps, no page becomes finer than it was, forced pages keep the finest
    tier allowed, and the bytes fit the budget."""
    rng = np.random.default_rng(12)
    po = np.array([0, 30, 45, 90], np.int32)
    lens = np.array([400, 150, 600], np.int32)     # 25, 10, 38 pages of 30, 15, 45 reserved
    util = rng.lognormal(0, 1, (2, 90 * 16)).astype(np.float32)
    budget = 400_000
    t_all1 = np.ones((2, 90), np.uint8)
    a = oracle.rdr_assign(po, lens, util, EPS, budget, 4, 8, 2, tiers_init=t_all1)
    b = oracle.rdr_rerun(po, lens, util, EPS, budget, 4, 8, t_all1)
    assert np.array_equal(a[0], b[0]) and a[1] == b[1] and a[2] == b[2]
    cur = a[0]
    lens2 = lens + 40
    # a larger budget than before: unconstrained, many pages would become finer
    new, lam, nb = oracle.rdr_rerun(po, lens2, util, EPS, 600_000, 4, 8, cur)
    idx = lambda t: np.where(t == 0, 3, t.astype(np.int64) - 1)   # noqa: E731
    for g in range(2):
        for s in range(3):
            npg = (int(lens2[s]) + 15) // 16
            for p in range(npg):
                e = po[s] + p
                assert idx(new[g, e]) >= idx(cur[g, e])
                if p < 4 or p >= npg - 8:
                    assert new[g, e] == cur[g, e]
    assert nb <= 600_000
    free = oracle.rdr_assign(po, lens2, util, EPS, 600_000, 4, 8, 2, tiers_init=np.ones((2, 90), np.uint8))[0]
    assert (idx(free) < idx(cur)).any()   # the caps did bind somewhere


def test_rdr_rerun_brute_force_optimal_under_caps():
    """Pin: brute force over every capped assignment (n <= 7 units): the
    re-run's choice has the least distortion among assignments that respect
    the caps and use no more bytes."""
    rng = np.random.default_rng(13)
    R = [4160, 2368, 1984, 0]
    for trial in range(20):
        n = int(rng.integers(2, 8))
        util = np.zeros((1, n * 16), np.float32)
        util[0] = rng.lognormal(0, 1.5, n * 16).astype(np.float32)
        cur = rng.choice(np.array([1, 2, 3, 0], np.uint8), size=(1, n))
        cidx = [3 if x == 0 else int(x) - 1 for x in cur[0]]
        floor = sum(R[i] for i in cidx)   # every unit at its finest allowed tier
        budget = int(rng.integers(0, floor + 1))
        t, lam, nb = oracle.rdr_rerun(np.array([0, n], np.int32), np.array([16 * n], np.int32), util, EPS, budget,
                                      0, 0, cur)
        got = [3 if x == 0 else int(x) - 1 for x in t[0]]
        assert all(got[u] >= cidx[u] for u in range(n))   # no unit became finer
        U = util[0].reshape(n, 16).astype(np.float64).sum(1)
        D = sum(U[u] * EPS[i] for u, i in enumerate(got))
        assert sum(R[i] for i in got) == nb <= budget
        best = math.inf
        for combo in itertools.product(range(4), repeat=n):
            if any(combo[u] < cidx[u] for u in range(n)):
                continue
            if sum(R[i] for i in combo) <= nb:
                best = min(best, sum(U[u] * EPS[i] for u, i in enumerate(combo)))
        assert D <= best * (1 + 1e-12) + 1e-300


def test_migrate_moves_unchanged_pages_byte_for_byte_and_transcodes_the_rest():
    """Pin: migrating to the same tiers reproduces every page byte for byte
    (pool ids may differ); with coarser tiers, every token unpacked from its new
    page equals the transcode of the token unpacked from its old page."""
    w, c = _tiny_cache([300, 77, 160], seed=21)
    counts = [int((w.tiers == t).sum()) for t in (1, 2, 3)]
    perm = [np.random.default_rng(t).permutation(counts[t]).astype(np.int32) for t in range(3)]
    table2 = oracle.build_page_table(w.tiers, perm)
    new = oracle.migrate(c, table2, counts)
    for t in range(3):
        for k in range(counts[t]):
            assert np.array_equal(new[t][perm[t][k]], c["pools"][t][k])
    coarse = w.tiers.copy()
    coarse[coarse == 1] = 2
    coarse[(coarse == 2) & (np.arange(coarse.shape[1]) % 3 == 0)] = 3
    counts2 = [int((coarse == t).sum()) for t in (1, 2, 3)]
    table3 = oracle.build_page_table(coarse)
    new3 = oracle.migrate(c, table3, counts2)
    po = w.page_offsets
    for g in range(w.H_kv):
        for b in range(w.B):
            for tok in range(int(w.seq_lens[b])):
                lp = po[b] + tok // 16
                eo, en = int(c["page_table"][g, lp]) & 0xFFFFFFFF, int(table3[g, lp]) & 0xFFFFFFFF
                to, tn = eo >> 30, en >> 30
                if tn == 0:
                    continue
                old = oracle.unpack_token(to, tok % 16, c["pools"][to - 1][eo & 0x3FFFFFFF])
                got = oracle.unpack_token(tn, tok % 16, new3[tn - 1][en & 0x3FFFFFFF])
                want = oracle.transcode_token(to, tn, old["leaf"], old["up"], old["s16"], old["vq"]) if tn != to else old
                assert got["r16"] == old["r16"]
                for f in ("leaf", "up", "vq"):
                    assert np.array_equal(got[f], want[f])
                assert got["s16"] == want["s16"]


def test_rdr_rerun_counts_forced_pages_at_their_capped_tier():
    """Pin: forced pages that a re-run caps below T1 cost their own tier's
    bytes; a budget that fits them at that tier (but not at T1) is feasible
    and keeps them there."""
    po = np.array([0, 12], np.int32)
    lens = np.array([12 * 16], np.int32)
    util = np.ones((1, 12 * 16), np.float32)
    cur = np.full((1, 12), 3, np.uint8)        # every page T3, all forced (4 sink + 8 recent)
    budget = 12 * 1984 + 100                   # fits 12 T3 pages, far below 12 T1 pages
    t, lam, nb = oracle.rdr_rerun(po, lens, util, EPS, budget, 4, 8, cur)
    assert t[0].tolist() == [3] * 12 and nb == 12 * 1984
    with pytest.raises(OverflowError):
        oracle.rdr_rerun(po, lens, util, EPS, 12 * 1984 - 1, 4, 8, cur)
