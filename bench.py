"""Benchmark: ADA decode over the paged, tier-homogeneous compressed cache.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]
                    [--workload NAME] [--n-q N]

One step = one full decode-attention call (plan, decode, split merge) over one
batch of the workload.  The headline workload is llama32k: B 8, 32 query /
8 kv heads, d 128, context 32768 per sequence in 16-token pages, tiers
T1/T2/T3/drop drawn 20/40/25/15 % (first 4 and last 8 pages T1), bf16 K with 4
outlier channels x8, V ~ N(0,1), pages written by the library's encode
kernel.  All inputs are synthetic and seeded.  The other workloads (--workload)
are the method's other published configurations:
  tiny      B 1, 4 / 1 heads, ctx 2048, all T1, fp32 K/V
  ragged64  B 64, ctx ~ U{1024..16384}, the same mix, permuted pool pages
  long512k  B 1, ctx 524288, the same mix (split-KV over every SM)
  e2e_rdr   B 16, ctx 32768 prefill: RDR at 25 % of the fp16 bytes, prefill
            encode into the chosen tiers, then append + decode steps (one new
            token per sequence each); a step is one append + one decode
The compressed cache read per step is larger than the 126 MB L2 for llama32k,
ragged64, long512k and e2e_rdr, so no flush is done between steps; tiny (0.5 MB)
fits in L2, which its line states.

value = token.heads/s = sum(seq_len) * H_q / time per step, aggregated over
all ranks (weak scaling: every rank decodes its own batch, with no exchange
between ranks; time is the max over ranks).  The line also gives the rate over
kept tokens only (config.kept_token_heads_per_s).

e2e = the same rate through host buffers: every step copies its inputs in from
pinned host memory, makes the C-ABI call and copies out and lse back, then
synchronises (one CUDA graph per step for the decode workloads; e2e_rdr also
copies the step's new K/V rows in and appends them).

--impl reference times the fp64 CPU oracle on the host cores, on a bounded
sample of the same workload.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "ADA decode token·heads/s and achieved HBM GB/s vs ~8 TB/s at ctx 32k"
UNIT = "token·heads/s"
WORKLOAD = "llama32k"
WORKLOADS = ("llama32k", "tiny", "ragged64", "long512k", "e2e_rdr")
WORKLOAD_DESC = {
    "llama32k": ("llama32k: B 8 per GPU, 32 q / 8 kv heads, d 128, ctx 32768, 16-token pages, "
                 "tiers T1/T2/T3/drop 20/40/25/15 % (first 4, last 8 pages T1), bf16 K/V encoded by the library"),
    "tiny": "tiny: B 1, 4 q / 1 kv head, d 128, ctx 2048, every page T1, fp32 K/V encoded by the library",
    "ragged64": ("ragged64: B 64 per GPU, ctx ~ U{1024..16384}, 32 q / 8 kv heads, d 128, the llama32k tier "
                 "mix, pool pages a seeded permutation, bf16 K/V encoded by the library"),
    "long512k": ("long512k: B 1 per GPU, ctx 524288, 32 q / 8 kv heads, d 128, the llama32k tier mix, "
                 "split-KV over every SM, bf16 K/V encoded by the library"),
    "e2e_rdr": ("e2e_rdr: B 16 per GPU, 32 q / 8 kv heads, d 128, 32768-token bf16 prefill, RDR at 25 % of the "
                "fp16 bytes, prefill encode, then append + decode steps (16 reserved T1 pages per sequence)"),
}
EPS = (1.1e-4, 2.75e-2, 7.12e-2, 2.0)   # distortion per unit utility of T1, T2, T3, drop
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


def served_units(w, n_q: int = 1, lens=None) -> int:
    """Token-heads one step serves: query token i of n_q attends to the first
    seq_len - (n_q - 1 - i) tokens (all of them for a single query), for every
    query head; dropped tokens count as served work."""
    lens = np.asarray(w.seq_lens if lens is None else lens, np.int64)
    return int(sum(np.maximum(lens - (n_q - 1 - i), 0).sum() for i in range(n_q))) * w.H_q


def kept_units(w, n_q: int = 1) -> int:
    """Token-heads of kept tokens only (pages not dropped) that one step
    serves: the other reading of the metric, which leaves dropped work out."""
    lens = np.asarray(w.seq_lens, np.int64)
    po = w.page_offsets
    G = w.H_q // w.H_kv
    total = 0
    for i in range(n_q):
        for b in range(w.B):
            n = max(int(lens[b]) - (n_q - 1 - i), 0)
            npg = (n + 15) // 16
            valid = np.minimum(16, n - 16 * np.arange(npg))
            for g in range(w.H_kv):
                total += int(valid[w.tiers[g, po[b]:po[b] + npg] != 0].sum()) * G
    return total


def algorithmic_bytes(w, lens=None, tiers=None) -> int:
    """Exact bytes the decode must move for one step: the bits of every kept
    token, one page-table entry per token-holding page, q, out and lse."""
    lens = np.asarray(w.seq_lens if lens is None else lens, np.int64)
    tiers = w.tiers if tiers is None else tiers
    po = w.page_offsets
    tot_bits = 0
    entries = 0
    for b in range(w.B):
        n = int(lens[b])
        npg = (n + 15) // 16
        entries += npg * w.H_kv
        valid = np.minimum(16, n - 16 * np.arange(npg))
        for g in range(w.H_kv):
            tt = tiers[g, po[b]:po[b] + npg]
            for t in (1, 2, 3):
                tot_bits += int(valid[tt == t].sum()) * ALGO_TOKEN_BITS[t]
    q_out = w.B * w.H_q * (128 * 4 * 2 + 4)
    return tot_bits // 8 + 4 * entries + q_out


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        d = json.load(open(path))
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


_SAMPLER = r"""
import sys, time
import pynvml as N
N.nvmlInit()
h = N.nvmlDeviceGetHandleByIndex(int(sys.argv[1]))
period = float(sys.argv[2])
get = getattr(N, "nvmlDeviceGetCurrentClocksEventReasons", None) or N.nvmlDeviceGetCurrentClocksThrottleReasons
print("max", N.nvmlDeviceGetMaxClockInfo(h, N.NVML_CLOCK_SM), flush=True)
while True:
    print(f"{time.time():.6f},{N.nvmlDeviceGetClockInfo(h, N.NVML_CLOCK_SM)},{int(get(h))},"
          f"{N.nvmlDeviceGetPowerUsage(h) / 1000.0}", flush=True)
    time.sleep(period)
"""


class ClockSampler:
    """SM clock, power and clock-event (throttle) reasons of one GPU, read
    through NVML (read-only queries) every `period` seconds by a separate
    sampler process (so that a busy launching thread cannot starve it).
    mark() records wall-clock time stamps so that the samples taken inside the
    timed region can be told apart from the rest."""

    REASONS = (("hw_slowdown", 0x8), ("hw_thermal_slowdown", 0x40), ("sw_thermal_slowdown", 0x20),
               ("sw_power_cap", 0x4))

    def __init__(self, gpu_index: int, period: float = 0.001):
        self.gpu, self.period = gpu_index, period
        self.marks = {}
        self.proc = None
        self.tmp = None
        self.err = None

    def __enter__(self):
        import subprocess
        import tempfile

        try:
            self.tmp = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
            self.proc = subprocess.Popen([sys.executable, "-c", _SAMPLER, str(self.gpu), str(self.period)],
                                         stdout=self.tmp, stderr=subprocess.DEVNULL)
            t0 = time.time()
            while time.time() - t0 < 20:   # wait for the first sample
                self.tmp.flush()
                if open(self.tmp.name).read().count("\n") >= 2 or self.proc.poll() is not None:
                    break
                time.sleep(0.05)
        except OSError as e:
            self.err = f"nvml sampler unavailable: {e}"
            self.proc = None
        return self

    def mark(self, name: str):
        self.marks[name] = time.time()

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self, t0: str = "timed_start", t1: str = "timed_end"):
        rows, max_mhz = [], None
        if self.tmp is not None:
            for line in open(self.tmp.name).read().splitlines():
                if line.startswith("max "):
                    max_mhz = float(line.split()[1])
                    continue
                try:
                    t, mhz, r, pw = line.split(",")
                    rows.append((float(t), float(mhz), int(r), float(pw)))
                except ValueError:
                    continue
            os.unlink(self.tmp.name)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": max_mhz, "reasons": [self.err or "no NVML samples"], "samples": 0}
        a, b = self.marks.get(t0, 0.0), self.marks.get(t1, float("inf"))
        scope = "timed region"
        inside = [x for x in rows if a <= x[0] <= b]
        if len(inside) < 3:   # a very short timed region: add the warm-up before it
            scope = "timed region and warm-up"
            inside = [x for x in rows if self.marks.get("warmup_start", a) <= x[0] <= b]
        if len(inside) < 3:   # still too short: the nearest samples around it
            scope = "the samples nearest the timed region"
            inside = sorted(rows, key=lambda x: min(abs(x[0] - a), abs(x[0] - b)))[:3]
        reasons = sorted({name for _, _, r, _ in inside for name, bit in self.REASONS if r & bit})
        return {"sm_mhz": statistics.median(x[1] for x in inside), "sm_max_mhz": max_mhz, "reasons": reasons,
                "samples": len(inside), "power_w_max": max(x[3] for x in inside), "scope": scope,
                "source": f"NVML every {self.period * 1e3:.0f} ms from a sampler process"}


# ----------------------------------------------------------- CPU (oracle) --
def _oracle_seq_cache(w, b, n=None, tiers=None):
    """The oracle's own pages (its encoder and packer) for sequence b of w,
    all kv heads: a one-sequence cache over its first n tokens."""
    import oracle

    n = int(w.seq_lens[b]) if n is None else n
    po = w.page_offsets
    cap = int(po[b + 1] - po[b])
    tiers = np.ascontiguousarray((w.tiers if tiers is None else tiers)[:, po[b]:po[b + 1]])
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


def cpu_baseline(w, q, budget_s: float = 10.0, name: str = WORKLOAD, tiers=None):
    """Time the fp64 oracle's decode attention on a bounded sample of the
    workload: whole sequences (all kv heads, every query head) while about
    budget_s seconds of oracle time last; a sequence too long for the budget
    is cut to its first tokens (the sample says how many)."""
    done, spent, n_seq, thr, parts = 0, 0.0, 0, 1, []
    for b in range(w.B):
        full = int(w.seq_lens[b])
        if full == 0:
            continue
        n = full
        if b == 0 and full > 65536:   # a long stream: time a prefix first, then size the sample
            c = _oracle_seq_cache(w, b, n=4096, tiers=tiers)
            dt, thr = _oracle_decode(c, np.asarray(q, np.float64)[b:b + 1], 4096)
            n = int(min(full, max(4096, budget_s / max(dt / 4096, 1e-12) * 0.8)))
        c = _oracle_seq_cache(w, b, n=n, tiers=tiers)
        dt, thr = _oracle_decode(c, np.asarray(q, np.float64)[b:b + 1], n)
        spent += dt
        done += n * w.H_q
        n_seq += 1
        parts.append(n if n < full else None)
        if spent >= budget_s:
            break
    cut = [p for p in parts if p is not None]
    what = f"{n_seq} sequence(s) of {name}" + (f" (the first {cut[0]} tokens of one)" if cut else " (whole)")
    return {"value": done / spent, "unit": UNIT, "cores": thr, "kind": "oracle",
            "sample": f"{what}: {done // w.H_q} tokens x {w.H_q} query heads, {spent:.1f} s of oracle time"}


def run_reference(args):
    """The oracle, as it stands, on the host cores.  Each step decodes one
    bounded sample: the first n tokens of sequence 0 for all query heads, n
    sized so that the whole run takes about two minutes."""
    rank, world, _ = dist_env()
    if rank != 0:
        return 0
    from compressed_paged_kv_ada_b200 import workloads as W

    name = args.workload
    w = W.make(name, seed=rank_seed(0))
    q_row = np.asarray(w.queries(), np.float64)[0:1]
    full = int(w.seq_lens[0])
    probe = min(full, 2048)
    c = _oracle_seq_cache(w, 0, n=min(full, 65536))
    per_tok = _oracle_decode(c, q_row, probe)[0] / probe
    step_budget = 120.0 / max(1, args.steps + args.warmup)
    n = int(min(full, 65536, max(16, step_budget / per_tok)))
    for _ in range(args.warmup):
        _oracle_decode(c, q_row, n)
    spent, thr = 0.0, 1
    for _ in range(args.steps):
        dt, thr = _oracle_decode(c, q_row, n)
        spent += dt
    value = args.steps * n * w.H_q / spent
    sample = (f"each step: first {n} of {full} tokens of sequence 0 of {name}, all {w.H_kv} kv heads "
              f"/ {w.H_q} query heads; {args.steps} steps in {spent:.1f} s")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": spent / args.steps * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": {"workload": WORKLOAD_DESC[name], "sample": sample},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": thr, "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------- GPU --
def _encode_all(cache, w, dev, lens=None):
    """Encode every present token of w with the library's encode kernel."""
    import torch

    lens = w.seq_lens if lens is None else lens
    dt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    for b in range(w.B):
        n = int(lens[b])
        if n == 0:
            continue
        for t0 in range(0, n, 65536):   # bounded host/device staging for long streams
            t1 = min(n, t0 + 65536)
            K, V = w.dense_rows(b, t0, t1)
            cache.encode(torch.from_numpy(K).to(dev).to(dt), torch.from_numpy(V).to(dev).to(dt),
                         torch.full((t1 - t0,), b, dtype=torch.int32, device=dev),
                         torch.arange(t0, t1, dtype=torch.int32, device=dev))
    cache.check()


def _roofline(algo_bytes, call_ms, traffic):
    peak, peak_kind = measured_peaks()
    achieved = algo_bytes / (call_ms / 1e3) / 1e9
    return {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
            "traffic": traffic, "peak_source": f"{peak_kind} hbm_gbs (copy, burst)"}


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
    name = args.workload
    if name == "e2e_rdr":
        return run_e2e(args, rank, world, dev, dist)

    w = W.make(name, seed=rank_seed(rank))
    cache = PagedCache(w.page_offsets, w.seq_lens, w.tiers, w.pool_perms(), device=str(dev))
    _encode_all(cache, w, dev)
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

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize(dev)

    with ClockSampler(dev.index) as clk:
        clk.mark("warmup_start")
        for _ in range(max(3, args.warmup)):
            step()
        cache.check()

        # ---- timed region: K back-to-back steps, device events
        n_ev = min(args.steps, 200)
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n_ev)]
        start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        barrier()
        clk.mark("timed_start")
        start.record(stream)
        for i in range(args.steps):
            if i < n_ev:
                ev[i][0].record(stream)
            step()
            if i < n_ev:
                ev[i][1].record(stream)
        end.record(stream)
        barrier()
        clk.mark("timed_end")
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
    # out + lse back to pinned host memory, every step.  The step (copy in,
    # the C-ABI call, copies out) is captured once as a CUDA graph and
    # replayed, one launch per step; eager calls if capture is refused.
    q_host = torch.from_numpy(q_np).pin_memory()
    out_host = torch.empty(out.shape, dtype=torch.float32).pin_memory()
    lse_host = torch.empty(lse.shape, dtype=torch.float32).pin_memory()
    e2e_steps = min(args.steps, 500)

    def io_step(s=None):
        q.copy_(q_host, non_blocking=True)
        if n_q == 1:
            L.sphkv_decode_attention(desc, w.H_q, q, out, lse, ws, status=cache.status, stream=s)
        else:
            L.sphkv_decode_attention_mq(desc, n_q, w.H_q, q, out, lse, ws, status=cache.status, stream=s)
        out_host.copy_(out, non_blocking=True)
        lse_host.copy_(lse, non_blocking=True)

    graph, e2e_path = None, "eager: copy in, one C-ABI call, copies out, per step"
    try:
        cap = torch.cuda.Stream(device=dev)
        cap.wait_stream(stream)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=cap):
            io_step()
        stream.wait_stream(cap)
        torch.cuda.synchronize(dev)
        graph = g
        e2e_path = "one CUDA graph per step: copy in, the C-ABI call's launches, copies out"
    except Exception as ex:   # capture refused: keep the eager loop
        torch.cuda.synchronize(dev)
        e2e_path += f" (graph capture refused: {type(ex).__name__})"
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(e2e_steps):
        if graph is not None:
            graph.replay()
        else:
            io_step(stream)
        stream.synchronize()
    e1.record(stream)
    barrier()
    e2e_ms = e0.elapsed_time(e1) / e2e_steps
    if world > 1:
        e2e_ms, _ = reduce_over_ranks(e2e_ms, 0.0, dist, dev)
    e2e_value = sum(u_all) / (e2e_ms / 1e3)

    if rank == 0:
        # the cache once per step, plus the extra query tokens' q, out and lse
        algo = algorithmic_bytes(w) + (n_q - 1) * w.B * w.H_q * (128 * 4 * 2 + 4)
        traffic = None
        if n_q == 1 and name == WORKLOAD:
            traffic = profiled_traffic(os.path.join(ROOT, "compressed_paged_kv_ada_b200", "csrc", "decode.cu"),
                                       os.path.join(ROOT, "profiles", "decode_kernel_llama32k.md"))
        roof = _roofline(algo, call_ms, traffic)
        roof["kernel"] = (("sphkv_decode_attention" if n_q == 1 else "sphkv_decode_attention_mq")
                          + " call (plan + decode + merge per query pair), per-call CUDA events")
        cb = (cpu_baseline(w, q_np, budget_s=args.cpu_seconds, name=name)
              if (world == 1 and args.cpu_seconds > 0 and n_q == 1) else None)
        fits_l2 = algo < 100e6
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": t_max, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": {"workload": WORKLOAD_DESC[name] + (f"; {n_q} causal query tokens per sequence" if n_q > 1 else ""),
                       "n_q": n_q, "global_batch": w.B * world, "seq_len": int(w.seq_lens.max()),
                       "parallelism": f"replicas x{world} (batch sharded, no exchange)",
                       "l2": ("the compressed cache (under 1 MB) fits in L2 and stays there between steps; no flush"
                              if fits_l2 else "compressed cache per step larger than L2 (126 MB); no flush"),
                       "algorithmic_bytes_per_step": algo,
                       "kept_token_heads_per_s": kept_units(w, n_q) * world / (t_max / 1e3),
                       "hbm_gbs_per_gpu": roof["achieved"], "hbm_frac_of_8tbs": roof["achieved"] / 8000.0},
            "roofline": roof,
            "cpu_baseline": cb,
            "e2e": {"value": e2e_value, "unit": UNIT,
                    "h2d_bytes_per_step": int(q.numel() * 4),
                    "d2h_bytes_per_step": int(out.numel() * 4 + lse.numel() * 4),
                    "path": e2e_path},
            "gpu_launches": 3 * ((n_q + 1) // 2) * args.steps,
            "clocks": clk.summary(),
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def run_e2e(args, rank, world, dev, dist):
    """RDR + prefill encode + append/decode steps.  The timed region is K steps
    (at most the workload's 256) of one append (one new token per sequence,
    encoded into its reserved T1 page) plus one decode; RDR and the prefill
    encode are timed separately with CUDA events, once each after a warm-up
    on a copy of the state."""
    import torch

    from compressed_paged_kv_ada_b200 import _lib as L
    from compressed_paged_kv_ada_b200 import PagedCache
    from compressed_paged_kv_ada_b200 import workloads as W

    w = W.make("e2e_rdr", seed=rank_seed(rank))
    stream = torch.cuda.current_stream(dev)
    util = torch.from_numpy(w.utility()).to(dev)
    budget = w.extra["budget"]
    cache = PagedCache(w.page_offsets, w.seq_lens, w.tiers, device=str(dev))
    ev = lambda: torch.cuda.Event(enable_timing=True)   # noqa: E731

    # RDR: one warm-up call, then the timed call
    cache.rdr_assign(util, EPS, budget, 4, 8)
    cache.check()
    tiers0 = w.tiers.copy()
    cache.tiers.copy_(torch.from_numpy(tiers0).to(dev))
    a, b = ev(), ev()
    a.record(stream)
    lam, nb = cache.rdr_assign(util, EPS, budget, 4, 8)
    b.record(stream)
    cache.check()
    rdr_ms = a.elapsed_time(b)
    tiers = cache.tiers.cpu().numpy()
    cache.reallocate_pools()

    # prefill encode: all sequences' K/V staged on the device, then one timed
    # encode call per sequence
    dt = torch.bfloat16
    Ks, Vs = [], []
    for s in range(w.B):
        K, V = w.dense_rows(s, 0, int(w.seq_lens[s]))
        Ks.append(torch.from_numpy(K).to(dev).to(dt))
        Vs.append(torch.from_numpy(V).to(dev).to(dt))
    seqs = [torch.full((int(w.seq_lens[s]),), s, dtype=torch.int32, device=dev) for s in range(w.B)]
    poss = [torch.arange(int(w.seq_lens[s]), dtype=torch.int32, device=dev) for s in range(w.B)]
    for s in range(w.B):   # warm-up pass writes the same bytes the timed pass writes
        cache.encode(Ks[s], Vs[s], seqs[s], poss[s])
    cache.check()
    a, b = ev(), ev()
    a.record(stream)
    for s in range(w.B):
        cache.encode(Ks[s], Vs[s], seqs[s], poss[s])
    b.record(stream)
    cache.check()
    enc_ms = a.elapsed_time(b)
    del Ks, Vs, seqs, poss

    # append + decode steps, tokens and queries staged on the device up front
    steps = min(args.steps, w.extra["steps"])
    warm = min(max(3, args.warmup), w.extra["steps"] - steps)
    n_all = warm + steps
    lens0 = w.seq_lens.astype(np.int32).copy()
    rows = [w.dense_rows(s, int(lens0[s]), int(lens0[s]) + n_all) for s in range(w.B)]
    Kap = torch.from_numpy(np.stack([r[0] for r in rows], axis=1)).to(dev).to(dt)   # [n_all, B, H_kv, 128]
    Vap = torch.from_numpy(np.stack([r[1] for r in rows], axis=1)).to(dev).to(dt)
    qs = torch.from_numpy(np.stack([w.queries(i + 1) for i in range(n_all)])).to(dev)
    pos = torch.from_numpy(np.stack([lens0 + i for i in range(n_all)])).to(dev)      # [n_all, B]
    lens_dev = torch.from_numpy(np.stack([lens0 + i + 1 for i in range(n_all)])).to(dev)
    seq_idx = torch.arange(w.B, dtype=torch.int32, device=dev)
    out = torch.empty((w.B, w.H_q, 128), dtype=torch.float32, device=dev)
    lse = torch.empty((w.B, w.H_q), dtype=torch.float32, device=dev)
    ws = cache.workspace(w.H_q)
    desc = cache.descriptor()

    # with --rerun-every R: after every R-th step RDR runs again under the same
    # budget (each page capped at its tier) and the pools are rewritten; the
    # utilities for those points are computed before the timed region
    every = args.rerun_every
    utils = {}
    if every > 0:
        for i in range(n_all):
            if (i + 1) % every == 0:
                utils[i] = torch.from_numpy(w.utility(lens0 + i + 1)).to(dev)
    n_reruns = [0]

    def step(i):
        nonlocal desc
        L.sphkv_encode(desc, Kap[i], Vap[i], seq_idx, pos[i], status=cache.status, stream=stream)
        cache.seq_lens.copy_(lens_dev[i], non_blocking=True)
        L.sphkv_decode_attention(desc, w.H_q, qs[i], out, lse, ws, status=cache.status, stream=stream)
        if i in utils:
            cache.rdr_rerun(utils[i], EPS, budget, 4, 8)
            desc = cache.descriptor()
            n_reruns[0] += 1

    with ClockSampler(dev.index) as clk:
        clk.mark("warmup_start")
        for i in range(warm):
            step(i)
        cache.check()
        torch.cuda.synchronize(dev)
        clk.mark("timed_start")
        s0, s1 = ev(), ev()
        s0.record(stream)
        for i in range(warm, n_all):
            step(i)
        s1.record(stream)
        torch.cuda.synchronize(dev)
        clk.mark("timed_end")
    cache.check()
    step_ms = s0.elapsed_time(s1) / steps
    # decode alone on the final cache, for the roofline
    d0, d1 = ev(), ev()
    d0.record(stream)
    for _ in range(20):
        L.sphkv_decode_attention(desc, w.H_q, qs[n_all - 1], out, lse, ws, status=cache.status, stream=stream)
    d1.record(stream)
    cache.check()
    dec_ms = d0.elapsed_time(d1) / 20
    lens_end = lens0 + n_all

    # end to end through host buffers: every step copies its new K/V rows and
    # q in from pinned host memory, appends them (the last token of every
    # sequence again, at its own position, which leaves the cache as it is),
    # decodes, and reads out + lse back to pinned host memory
    Kh, Vh = Kap[n_all - 1].cpu().pin_memory(), Vap[n_all - 1].cpu().pin_memory()
    qh = qs[n_all - 1].cpu().pin_memory()
    Kd, Vd, qd = torch.empty_like(Kap[n_all - 1]), torch.empty_like(Vap[n_all - 1]), torch.empty_like(qs[0])
    out_h = torch.empty(out.shape, dtype=torch.float32).pin_memory()
    lse_h = torch.empty(lse.shape, dtype=torch.float32).pin_memory()
    e2e_steps = min(steps, 100)
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    x0, x1 = ev(), ev()
    x0.record(stream)
    for _ in range(e2e_steps):
        Kd.copy_(Kh, non_blocking=True)
        Vd.copy_(Vh, non_blocking=True)
        qd.copy_(qh, non_blocking=True)
        L.sphkv_encode(desc, Kd, Vd, seq_idx, pos[n_all - 1], status=cache.status, stream=stream)
        L.sphkv_decode_attention(desc, w.H_q, qd, out, lse, ws, status=cache.status, stream=stream)
        out_h.copy_(out, non_blocking=True)
        lse_h.copy_(lse, non_blocking=True)
        stream.synchronize()
    x1.record(stream)
    torch.cuda.synchronize(dev)
    cache.check()
    e2e_ms = x0.elapsed_time(x1) / e2e_steps
    e2e_units = served_units(w, 1, lens_end)
    if world > 1:
        e2e_ms, e2e_units = reduce_over_ranks(e2e_ms, e2e_units, dist, dev)
    e2e_value = e2e_units / (e2e_ms / 1e3)
    h2d = int(Kh.numel() * Kh.element_size() + Vh.numel() * Vh.element_size() + qh.numel() * 4)
    d2h = int(out_h.numel() * 4 + lse_h.numel() * 4)
    units = sum(served_units(w, 1, lens0 + i + 1) for i in range(warm, n_all)) / steps
    value = units / (step_ms / 1e3)
    if world > 1:
        t_max_r, u_sum = reduce_over_ranks(step_ms, units, dist, dev)
        value, step_ms = u_sum / (t_max_r / 1e3), t_max_r
    # residency: stored bytes of the pages holding tokens vs dense fp16 K/V
    cache.seq_lens.copy_(torch.from_numpy(lens_end.astype(np.int32)).to(dev))
    stored = cache.compressed_bytes()
    fp16 = int(lens_end.sum()) * w.H_kv * 128 * 2 * 2
    tiers = cache.tiers.cpu().numpy()   # after any re-runs
    if rank == 0:
        algo = algorithmic_bytes(w, lens=lens_end, tiers=tiers)
        roof = _roofline(algo, dec_ms, None)
        roof["kernel"] = "sphkv_decode_attention call on the final cache, CUDA events over 20 calls"
        cb = None
        if world == 1 and args.cpu_seconds > 0:
            w_end = W.make("e2e_rdr", seed=rank_seed(rank))
            w_end.seq_lens = lens_end.astype(np.int32)
            cb = cpu_baseline(w_end, np.asarray(qs[n_all - 1].cpu().numpy()), budget_s=args.cpu_seconds,
                              name="e2e_rdr (final cache)", tiers=tiers)
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": steps, "warmup": warm,
            "ms_per_step": step_ms, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "f32", "data": "synthetic",
            "config": {"workload": WORKLOAD_DESC["e2e_rdr"], "global_batch": w.B * world,
                       "seq_len": int(lens_end.max()), "parallelism": f"replicas x{world} (batch sharded, no exchange)",
                       "l2": "compressed cache per step larger than L2 (126 MB); no flush",
                       "step": "one append (one token per sequence) + one decode call"
                               + (f"; every {every} steps RDR runs again under the budget and the pools are "
                                  "rewritten (sphkv_rdr_rerun + sphkv_migrate), inside the timed region"
                                  if every > 0 else ""),
                       "algorithmic_bytes_per_decode": algo},
            "rerun_every": every, "reruns_in_run": n_reruns[0],
            "phases": {"rdr_ms": rdr_ms, "rdr_lambda": float(lam.item()), "rdr_bytes": int(nb.item()),
                       "rdr_budget": budget, "prefill_encode_ms": enc_ms,
                       "prefill_tokens": int(lens0.sum()), "append_decode_step_ms": step_ms,
                       "decode_alone_ms": dec_ms,
                       "end_to_end_ms": rdr_ms + enc_ms + step_ms * w.extra["steps"],
                       "end_to_end_note": "RDR + prefill encode + 256 x (append + decode), from the timed parts"},
            "residency": {"stored_bytes": stored, "fp16_bytes": fp16, "frac": stored / fp16,
                          "note": "pages holding tokens after the steps, all tiers, vs dense fp16 K and V"},
            "roofline": roof,
            "cpu_baseline": cb,
            "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "note": "each step: new K/V rows and q from pinned host memory, append, decode, out and lse "
                            "back to pinned host memory, on the final cache"},
            "gpu_launches": 4 * steps,
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
    ap.add_argument("--workload", default=WORKLOAD, choices=WORKLOADS,
                    help="llama32k (the headline), tiny, ragged64, long512k or e2e_rdr")
    ap.add_argument("--n-q", type=int, default=1,
                    help="query tokens per sequence and step (causal multi-token decode; 1 = the headline)")
    ap.add_argument("--rerun-every", type=int, default=0,
                    help="e2e_rdr: run RDR again every N append steps (0 = never, the published configuration)")
    ap.add_argument("--cpu-seconds", type=float, default=10.0,
                    help="seconds of oracle time for the cpu_baseline field (0 to skip)")
    args = ap.parse_args(argv)
    if args.impl == "reference":
        return run_reference(args)
    return run_gpu(args)


if __name__ == "__main__":
    sys.exit(main())
