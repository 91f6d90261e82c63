"""Split-KV of one long stream across ranks, host side (no GPU): the page-aligned
partition, and the gather + log-sum-exp combine over world size 2 on gloo.

Each rank attends to its own token range with the oracle (the GPU decode is
covered by tests/test_gpu_splitkv.py); merge_over_ranks all-gathers the parts
and combines them; the result must equal the oracle's attention over the whole
stream."""
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp

import oracle
from compressed_paged_kv_ada_b200 import splitkv
from compressed_paged_kv_ada_b200 import workloads as W


def test_split_stream_is_a_page_aligned_partition():
    for n, world in [(0, 2), (1, 2), (16, 3), (17, 2), (1000, 4), (524288, 8), (33, 8)]:
        parts = splitkv.split_stream(n, world)
        assert len(parts) == world
        assert parts[0][0] == 0 and parts[-1][1] == n
        pages = []
        for (a, b), (c, _) in zip(parts, parts[1:] + [(n, n)]):
            # contiguous; a range starts on a page boundary, or is empty at the end
            assert b == c and a <= b and (a % 16 == 0 or a == b == n)
            pages.append((b - a + 15) // 16)
        assert max(pages) - min(pages) <= 1 and sum(pages) == (n + 15) // 16
    with pytest.raises(ValueError):
        splitkv.split_stream(10, 0)


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _unit_dense(w, g, n):
    """The oracle's decoded keys/values of the first n tokens of sequence 0,
    kv head g, and the keep mask (page not dropped)."""
    K, V = w.dense_rows(0, 0, n)
    tt = np.repeat(w.tiers[g, : (n + 15) // 16], 16)[:n]
    kh, vh = np.zeros((n, 128)), np.zeros((n, 128))
    for t in (1, 2, 3):
        idx = np.nonzero(tt == t)[0]
        if idx.size:
            c = oracle.encode(K[idx, g], V[idx, g], t)
            bl, bu, _ = oracle.TIER_BITS[t]
            kh[idx] = oracle.decode_keys(c["leaf"], c["up"], c["r16"], bl, bu)
            vh[idx] = oracle.decode_values(c["vq"], c["s16"])
    return kh, vh, tt != 0


def _rank_main(rank, world, port, n, q_out):
    import torch
    import torch.distributed as dist

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    w = W.make("long512k", ctx=n, H_kv=2, H_q=8)
    t0, t1 = splitkv.split_stream(n, world)[rank]
    q = np.asarray(w.queries(), np.float64)[0]
    outs, lses = [], []
    for g in range(w.H_kv):
        kh, vh, keep = _unit_dense(w, g, n)
        sel = np.arange(t0, t1)[keep[t0:t1]]
        o, l = oracle.attention(kh[sel], vh[sel], q[4 * g:4 * g + 4])
        outs.append(o)
        lses.append(l)
    out = torch.from_numpy(np.concatenate(outs))   # [H_q, 128] of this rank's range
    lse = torch.from_numpy(np.concatenate(lses))

    def merge(op, lp):
        mo, ml = oracle.merge_partials(op.numpy(), lp.numpy())
        return torch.from_numpy(mo), torch.from_numpy(ml)

    mo, ml = splitkv.merge_over_ranks(out, lse, merge=merge)
    q_out.put((rank, mo.numpy(), ml.numpy()))
    dist.barrier()
    dist.destroy_process_group()


def test_merge_over_ranks_gloo_world2_equals_whole_stream():
    n = 3000   # 188 pages, mixed tiers and dropped pages, ragged last page
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, n, q)) for r in range(2)]
    for p in procs:
        p.start()
    got = [q.get(timeout=300) for _ in range(2)]
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    w = W.make("long512k", ctx=n, H_kv=2, H_q=8)
    qq = np.asarray(w.queries(), np.float64)[0]
    want_o, want_l = [], []
    for g in range(w.H_kv):
        kh, vh, keep = _unit_dense(w, g, n)
        o, l = oracle.attention(kh[keep], vh[keep], qq[4 * g:4 * g + 4])
        want_o.append(o)
        want_l.append(l)
    want_o, want_l = np.concatenate(want_o), np.concatenate(want_l)
    for rank, mo, ml in got:   # every rank ends with the whole stream's result
        assert np.abs(ml - want_l).max() <= 1e-12 * max(1.0, np.abs(want_l).max())
        assert np.abs(mo - want_o).max() <= 1e-12 * max(1.0, np.abs(want_o).max())
