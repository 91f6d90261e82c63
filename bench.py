"""Benchmark: ADA decode over the paged, tier-homogeneous compressed cache.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]

One step = one full decode-attention call (plan, decode, split merge) over one
batch of the llama32k workload: B 8, 32 query / 8 kv heads, d 128, context
32768 per sequence in 16-token pages, tiers T1/T2/T3/drop drawn 20/40/25/15 %
(first 4 and last 8 pages T1), bf16 K with 4 outlier channels x8, V ~ N(0,1),
pages written by the library's encode kernel.  All inputs are synthetic and
seeded.  The compressed cache read per step (~300 MB) is larger than the
126 MB L2, so no flush is done between steps.

value = token.heads/s = sum(seq_len) * H_q / time per step, aggregated over
all ranks (weak scaling: every rank decodes its own batch of 8 sequences,
with no exchange between ranks; time is the max over ranks).

--impl reference times the fp64 CPU oracle on the host cores, on a bounded
sample of the same workload.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "ADA decode token·heads/s and achieved HBM GB/s vs ~8 TB/s at ctx 32k"
UNIT = "token·heads/s"
WORKLOAD = "llama32k"
WORKLOAD_DESC = ("llama32k: B 8 per GPU, 32 q / 8 kv heads, d 128, ctx 32768, 16-token pages, "
                 "tiers T1/T2/T3/drop 20/40/25/15 % (first 4, last 8 pages T1), bf16 K/V encoded "
                 "by the library")
# exact bits per token of each tier: r 16 + vscale 16 + 64 b_leaf + 63 b_up + 128 v_bits
ALGO_TOKEN_BITS = {1: 16 + 16 + 64 * 8 + 63 * 8 + 128 * 8,
                   2: 16 + 16 + 64 * 4 + 63 * 6 + 128 * 4,
                   3: 16 + 16 + 64 * 3 + 63 * 4 + 128 * 4}


def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def rank_seed(rank: int) -> int:
    """Each rank decodes its own batch: rank r draws with seed r."""
    return rank


def aggregate(times_ms, units, world):
    """Whole-job throughput from per-rank step times and units: total units
    over all ranks divided by the slowest rank's time."""
    t = max(times_ms)
    return sum(units) / (t / 1e3), t


def reduce_over_ranks(ms_step: float, units: float, dist, device):
    """Max of the per-rank step times and sum of the per-rank units, over all
    ranks of the default process group (every rank calls this once)."""
    import torch

    tt = torch.tensor([ms_step], dtype=torch.float64, device=device)
    uu = torch.tensor([units], dtype=torch.float64, device=device)
    dist.all_reduce(tt, op=dist.ReduceOp.MAX)
    dist.all_reduce(uu, op=dist.ReduceOp.SUM)
    return float(tt.item()), float(uu.item())


def profiled_traffic(kernel_src: str, summary: str):
    """DRAM bytes per launch from a committed ncu summary, or None when the
    kernel source has changed since the counters were taken."""
    import hashlib

    if not (os.path.exists(kernel_src) and os.path.exists(summary)):
        return None
    digest = hashlib.sha256(open(kernel_src, "rb").read()).hexdigest()[:16]
    fields = {}
    for line in open(summary):
        if ":" in line:
            k, v = line.split(":", 1)
            fields[k.strip()] = v.strip()
    if fields.get("decode.cu sha256 prefix") != digest:
        return None
    try:
        return int(fields["traffic_bytes_per_launch"])
    except (KeyError, ValueError):
        return None


def served_units(w, n_q: int = 1) -> int:
    """Token-heads one step serves: query token i of n_q attends to the first
    seq_len - (n_q - 1 - i) tokens (all of them for a single query), for every
    query head; dropped tokens count as served work."""
    lens = np.asarray(w.seq_lens, np.int64)
    return int(sum(np.maximum(lens - (n_q - 1 - i), 0).sum() for i in range(n_q))) * w.H_q


def algorithmic_bytes(w) -> int:
    """Exact bytes the decode must move for one step: the bits of every kept
    token, one page-table entry per token-holding page, q, out and lse."""
    po = w.page_offsets
    tot_bits = 0
    entries = 0
    for b in range(w.B):
        n = int(w.seq_lens[b])
        npg = (n + 15) // 16
        entries += npg * w.H_kv
        valid = np.minimum(16, n - 16 * np.arange(npg))
        for g in range(w.H_kv):
            tiers = w.tiers[g, po[b]:po[b] + npg]
            for t in (1, 2, 3):
                tot_bits += int(valid[tiers == t].sum()) * ALGO_TOKEN_BITS[t]
    q_out = w.B * w.H_q * (128 * 4 * 2 + 4)
    return tot_bits // 8 + 4 * entries + q_out


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        d = json.load(open(path))
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.tmp = None

    def __enter__(self):
        try:
            self.tmp = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=self.tmp, stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        if self.proc is None or self.tmp is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.tmp.flush()
        rows = [r.split(",") for r in open(self.tmp.name).read().strip().splitlines() if r.strip()]
        os.unlink(self.tmp.name)
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            try:
                sm.append(float(r[1]))
                smax.append(float(r[2]))
            except (ValueError, IndexError):
                continue
            for name, v in zip(names, r[5:9]):
                if v.strip().lower() == "active":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm)}


def _oracle_seq_cache(w, b):
    """The oracle's own pages (its encoder and packer) for sequence b of w,
    all kv heads: a one-sequence cache."""
    import oracle

    n = int(w.seq_lens[b])
    po = w.page_offsets
    cap = int(po[b + 1] - po[b])
    tiers = np.ascontiguousarray(w.tiers[:, po[b]:po[b + 1]])
    table = oracle.build_page_table(tiers)
    K, V = w.dense_rows(b, 0, n)
    counts = [int((tiers == t).sum()) for t in (1, 2, 3)]
    pools = oracle.encode_cache(K, V, np.zeros(n, np.int32), np.arange(n), np.array([0, cap]), table,
                                counts)
    return dict(B=1, H_q=w.H_q, H_kv=w.H_kv, page_offsets=np.array([0, cap], np.int32),
                seq_lens=np.array([n], np.int32), page_table=table, pools=pools)


def _oracle_decode(c, q_row, n_tok):
    """Oracle decode attention of one sequence (all kv heads, in parallel over
    the host cores), its first n_tok tokens.  Returns (seconds, threads)."""
    import oracle

    c["seq_lens"] = np.array([n_tok], np.int32)
    units = [(0, g) for g in range(c["H_kv"])]
    t0 = time.perf_counter()
    oracle.cache_attention(c, q_row, units)
    return time.perf_counter() - t0, min(len(units), oracle.num_threads())


def cpu_baseline(w, q, budget_s: float = 10.0):
    """Time the fp64 oracle's decode attention on a bounded sample of the
    workload: whole sequences (all 8 kv heads over the full context, 32 query
    heads), until about budget_s seconds of oracle time."""
    done, spent, n_seq, thr = 0, 0.0, 0, 1
    for b in range(w.B):
        c = _oracle_seq_cache(w, b)
        dt, thr = _oracle_decode(c, np.asarray(q, np.float64)[b:b + 1], int(w.seq_lens[b]))
        spent += dt
        done += int(w.seq_lens[b]) * w.H_q
        n_seq += 1
        if spent >= budget_s:
            break
    return {"value": done / spent, "unit": UNIT, "cores": thr, "kind": "oracle",
            "sample": f"{n_seq} whole sequence(s) of {WORKLOAD} ({done // w.H_q} tokens x {w.H_q} query heads), "
                      f"{spent:.1f} s of oracle time"}


def run_reference(args):
    """The oracle, as it stands, on the host cores.  Each step decodes one
    bounded sample: the first n tokens of sequence 0 for all 32 query heads,
    n sized so that the whole run takes about two minutes."""
    rank, world, _ = dist_env()
    if rank != 0:
        return 0
    from compressed_paged_kv_ada_b200 import workloads as W

    w = W.make(WORKLOAD, seed=rank_seed(0))
    q_row = np.asarray(w.queries(), np.float64)[0:1]
    c = _oracle_seq_cache(w, 0)
    full = int(w.seq_lens[0])
    probe = min(full, 2048)
    per_tok = _oracle_decode(c, q_row, probe)[0] / probe
    step_budget = 120.0 / max(1, args.steps + args.warmup)
    n = int(min(full, max(16, step_budget / per_tok)))
    for _ in range(args.warmup):
        _oracle_decode(c, q_row, n)
    spent, thr = 0.0, 1
    for _ in range(args.steps):
        dt, thr = _oracle_decode(c, q_row, n)
        spent += dt
    value = args.steps * n * w.H_q / spent
    sample = (f"each step: first {n} of {full} tokens of sequence 0 of {WORKLOAD}, all {w.H_kv} kv heads "
              f"/ {w.H_q} query heads; {args.steps} steps in {spent:.1f} s")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": spent / args.steps * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": {"workload": WORKLOAD_DESC, "sample": sample},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": thr, "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def run_gpu(args):
    import torch
    import torch.distributed as dist

    from compressed_paged_kv_ada_b200 import _lib as L
    from compressed_paged_kv_ada_b200 import PagedCache
    from compressed_paged_kv_ada_b200 import workloads as W

    rank, world, local = dist_env()
    if world > 1:
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=__import__("datetime").timedelta(seconds=120))
    dev = torch.device("cuda", local if world > 1 else 0)
    L.lib()

    w = W.make(WORKLOAD, seed=rank_seed(rank))
    cache = PagedCache(w.page_offsets, w.seq_lens, w.tiers, device=str(dev))
    for b in range(w.B):
        n = int(w.seq_lens[b])
        K, V = w.dense_rows(b, 0, n)
        Kt = torch.from_numpy(K).to(dev).to(torch.bfloat16)
        Vt = torch.from_numpy(V).to(dev).to(torch.bfloat16)
        cache.encode(Kt, Vt, torch.full((n,), b, dtype=torch.int32, device=dev),
                     torch.arange(n, dtype=torch.int32, device=dev))
        del Kt, Vt
    cache.check()
    n_q = args.n_q
    desc = cache.descriptor()
    stream = torch.cuda.current_stream(dev)
    if n_q == 1:
        q_np = w.queries()
        out = torch.empty((w.B, w.H_q, 128), dtype=torch.float32, device=dev)
        lse = torch.empty((w.B, w.H_q), dtype=torch.float32, device=dev)
        ws = cache.workspace(w.H_q)
    else:   # n_q causal query tokens per sequence (seeded as decode steps 0 .. n_q-1)
        q_np = np.stack([w.queries(step=i) for i in range(n_q)], axis=1)
        out = torch.empty((w.B, n_q, w.H_q, 128), dtype=torch.float32, device=dev)
        lse = torch.empty((w.B, n_q, w.H_q), dtype=torch.float32, device=dev)
        ws = torch.empty(L.sphkv_decode_mq_workspace_bytes(w.B, w.H_q, w.H_kv, w.total_pages), dtype=torch.uint8,
                         device=dev)
    q = torch.from_numpy(q_np).to(dev)

    def step():
        if n_q == 1:
            L.sphkv_decode_attention(desc, w.H_q, q, out, lse, ws, status=cache.status, stream=stream)
        else:
            L.sphkv_decode_attention_mq(desc, n_q, w.H_q, q, out, lse, ws, status=cache.status, stream=stream)

    for _ in range(max(3, args.warmup)):
        step()
    cache.check()

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize(dev)

    # ---- timed region: K back-to-back steps, device events
    n_ev = min(args.steps, 200)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n_ev)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    with ClockSampler(dev.index) as clk:
        start.record(stream)
        for i in range(args.steps):
            if i < n_ev:
                ev[i][0].record(stream)
            step()
            if i < n_ev:
                ev[i][1].record(stream)
        end.record(stream)
        barrier()
    cache.check()
    ms_total = start.elapsed_time(end)
    call_ms = float(np.mean([a.elapsed_time(b) for a, b in ev]))
    ms_step = ms_total / args.steps
    units = served_units(w, n_q)
    t_all = [ms_step]
    u_all = [units]
    if world > 1:
        t_max_r, u_sum = reduce_over_ranks(ms_step, units, dist, dev)
        t_all, u_all = [t_max_r], [u_sum]
    value, t_max = aggregate(t_all, u_all, world)

    # ---- end to end through host buffers: q from pinned host memory in,
    # out + lse back to pinned host memory, every step
    q_host = torch.from_numpy(q_np).pin_memory()
    out_host = torch.empty(out.shape, dtype=torch.float32).pin_memory()
    lse_host = torch.empty(lse.shape, dtype=torch.float32).pin_memory()
    e2e_steps = min(args.steps, 500)
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(e2e_steps):
        q.copy_(q_host, non_blocking=True)
        step()
        out_host.copy_(out, non_blocking=True)
        lse_host.copy_(lse, non_blocking=True)
        stream.synchronize()
    e1.record(stream)
    barrier()
    e2e_ms = e0.elapsed_time(e1) / e2e_steps
    if world > 1:
        e2e_ms, _ = reduce_over_ranks(e2e_ms, 0.0, dist, dev)
    e2e_value = sum(u_all) / (e2e_ms / 1e3)

    line = None
    if rank == 0:
        # the cache once per step, plus the extra query tokens' q, out and lse
        algo = algorithmic_bytes(w) + (n_q - 1) * w.B * w.H_q * (128 * 4 * 2 + 4)
        peak, peak_kind = measured_peaks()
        achieved = algo / (call_ms / 1e3) / 1e9
        traffic = profiled_traffic(os.path.join(ROOT, "compressed_paged_kv_ada_b200", "csrc", "decode.cu"),
                                   os.path.join(ROOT, "profiles", "decode_kernel_llama32k.md")) if n_q == 1 else None
        cb = (cpu_baseline(w, q_np, budget_s=args.cpu_seconds)
              if (world == 1 and args.cpu_seconds > 0 and n_q == 1) else None)
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": t_max, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": {"workload": WORKLOAD_DESC + (f"; {n_q} causal query tokens per sequence" if n_q > 1 else ""),
                       "n_q": n_q, "global_batch": w.B * world, "seq_len": int(w.seq_lens[0]),
                       "parallelism": f"replicas x{world} (batch sharded, no exchange)",
                       "l2": "compressed cache per step larger than L2 (126 MB); no flush",
                       "algorithmic_bytes_per_step": algo,
                       "hbm_gbs_per_gpu": achieved, "hbm_frac_of_8tbs": achieved / 8000.0},
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                         "frac": achieved / peak, "traffic": traffic,
                         "peak_source": f"{peak_kind} hbm_gbs (copy, burst)",
                         "kernel": ("sphkv_decode_attention" if n_q == 1 else "sphkv_decode_attention_mq")
                                   + " call (plan + decode + merge per query pair), per-call CUDA events"},
            "cpu_baseline": cb,
            "e2e": {"value": e2e_value, "unit": UNIT,
                    "h2d_bytes_per_step": int(q.numel() * 4),
                    "d2h_bytes_per_step": int(out.numel() * 4 + lse.numel() * 4)},
            "gpu_launches": 3 * ((n_q + 1) // 2) * args.steps,
            "clocks": clk.summary(),
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--n-q", type=int, default=1,
                    help="query tokens per sequence and step (causal multi-token decode; 1 = the headline)")
    ap.add_argument("--cpu-seconds", type=float, default=10.0,
                    help="seconds of oracle time for the cpu_baseline field (0 to skip)")
    args = ap.parse_args(argv)
    if args.impl == "reference":
        return run_reference(args)
    return run_gpu(args)


if __name__ == "__main__":
    sys.exit(main())
