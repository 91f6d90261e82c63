"""Host-side logic of bench.py: the multi-rank reduction (world size 2 over
gloo on CPU), the throughput aggregate, the algorithmic byte count and the
profile staleness check.  No GPU."""
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp

import bench
from compressed_paged_kv_ada_b200 import workloads as W


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank_main(rank, world, port, q):
    import torch
    import torch.distributed as dist

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    ms = [2.0, 3.5][rank]
    units = [100.0, 300.0][rank]
    t, u = bench.reduce_over_ranks(ms, units, dist, torch.device("cpu"))
    value, tmax = bench.aggregate([t], [u], world)
    q.put((rank, t, u, value, tmax))
    dist.barrier()
    dist.destroy_process_group()


def test_reduce_over_ranks_gloo_world2():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    out = sorted(q.get(timeout=10) for _ in range(2))
    for rank, t, u, value, tmax in out:
        assert t == 3.5 and u == 400.0
        assert value == pytest.approx(400.0 / 3.5e-3) and tmax == 3.5


def test_rank_seeds_differ_and_shapes_match():
    a, b = W.make("llama32k", seed=bench.rank_seed(0), B=2, ctx=200), W.make("llama32k", seed=bench.rank_seed(1), B=2, ctx=200)
    ka, _ = a.dense_rows(0, 0, 20)
    kb, _ = b.dense_rows(0, 0, 20)
    assert ka.shape == kb.shape and not np.array_equal(ka, kb)


def test_algorithmic_bytes_counts_kept_bits():
    w = W.make("llama32k", B=1, ctx=40, H_kv=1, H_q=4)
    w.tiers[:] = 0
    w.tiers[0, 0] = 1          # 16 tokens of T1
    w.tiers[0, 2] = 3          # 8 tokens of T3 (partial last page)
    want = (16 * 259 * 8 + 8 * 988) // 8 + 4 * 3 + 4 * (128 * 8 + 4)
    assert bench.algorithmic_bytes(w) == want


def test_profiled_traffic_goes_stale(tmp_path):
    src = tmp_path / "k.cu"
    src.write_text("kernel v1")
    import hashlib

    h = hashlib.sha256(b"kernel v1").hexdigest()[:16]
    summ = tmp_path / "s.md"
    summ.write_text(f"decode.cu sha256 prefix: {h}\ntraffic_bytes_per_launch: 1234\n")
    assert bench.profiled_traffic(str(src), str(summ)) == 1234
    src.write_text("kernel v2")
    assert bench.profiled_traffic(str(src), str(summ)) is None


def test_served_units_count_each_query_tokens_prefix():
    """One query: all tokens of every sequence for every query head; n_q
    causal tokens: token i serves seq_len - (n_q - 1 - i), never below 0."""
    w = W.make("ragged64", seq_lens=[5, 1, 0, 40], H_kv=2, H_q=8)
    assert bench.served_units(w) == (5 + 1 + 0 + 40) * 8
    # n_q = 3: token 0 sees len - 2, token 1 len - 1, token 2 len
    per_seq = [max(5 - 2, 0) + 4 + 5, 0 + 0 + 1, 0, 38 + 39 + 40]
    assert bench.served_units(w, 3) == sum(per_seq) * 8


def test_kept_units_counts_tokens_on_kept_pages():
    """Kept-token rate: tokens on pages that are not dropped, times the query
    heads per kv head, per query token (a later causal query sees one more
    token).  Worked by hand on a two-sequence cache."""
    w = W.make("ragged64", seq_lens=[40, 17], H_kv=2, H_q=8)
    po = w.page_offsets               # sequence 0: pages 0..2, sequence 1: pages 3..4
    w.tiers[:] = 1
    w.tiers[0, po[0] + 1] = 0         # kv head 0, tokens 16..31 of sequence 0 dropped
    w.tiers[1, po[1] + 1] = 0         # kv head 1, token 16 of sequence 1 dropped
    # kv head 0: 40 - 16 + 17 = 41 tokens; kv head 1: 40 + 16 = 56; G = 4
    assert bench.kept_units(w) == (41 + 56) * 4
    # two causal queries: the first sees 39 and 16 tokens
    first = ((39 - 16) + 16) + (39 + 16)
    assert bench.kept_units(w, n_q=2) == (first + 41 + 56) * 4
    # with nothing dropped it equals the served units
    w.tiers[:] = 1
    assert bench.kept_units(w) == bench.served_units(w)
