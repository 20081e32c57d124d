"""Benchmark of the paged KV-cache attention hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl npv|reference] [--workload NAME]

One step = one decode step of the workload: npv_store_kvcache_and_decode_attention
(the store of this step's new K/V rows inside the split-KV kernel, then the merge
kernel) over every sequence; --separate-store runs npv_store_kvcache then
npv_paged_decode_attention instead.  The default workload is the Qwen3-0.6B-shaped decode
batch (256 sequences, 16 Q / 8 KV heads, head_dim 128, 256-token blocks,
contexts U[100, 2048] growing by one token per step, cycling through its 64
steps).  Inputs are synthetic and seeded; the KV read per step (about 1.16 GB)
is far larger than the 126 MB L2, so no explicit flush is needed.

`value` is algorithmic HBM bytes per step / device time per step (GB/s), summed
over ranks for N > 1 (each rank runs its own replica; no collective on the data
path) and divided by the slowest rank's time.  Prints one JSON line on rank 0.

At N = 1 the default run then times every other named workload (GQA 4:1 with
shared prefixes, long-context decode, the chunked-prefill mix, speculative-decode
verification) and the decode step with RoPE, one short loop each, in the line's
`secondary` block.

--impl reference times the fp64 CPU oracle (the only reference this method
has) on a bounded sample of the same workload, on rank 0 only.
"""

from __future__ import annotations

import argparse
import csv
import hashlib
import io
import json
import math
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "paged GQA decode attention: achieved HBM GB/s (% of peak), tokens/s"
MIXED_METRIC = "chunked-prefill mixed batch attention: HBM GB/s, tokens/s, prefill TFLOP/s"
SPEC_METRIC = "speculative-decode verify attention (multi-row decode over the paged cache): HBM GB/s, tokens/s"
FALLBACK_HBM_GBS = 6650.0
PROFILE_DIR = os.path.join(ROOT, "profiles")
KERNEL_SRC = os.path.join(ROOT, "paged_kv_cache_bf16_b200", "csrc", "decode_attention.cuh")
PREFILL_SRC = os.path.join(ROOT, "paged_kv_cache_bf16_b200", "csrc", "prefill_attention.cuh")


def parse_args(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["npv", "reference"], default="npv")
    ap.add_argument("--workload", default="qwen3_decode")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--separate-store", action="store_true",
                    help="decode steps as npv_store_kvcache + npv_paged_decode_attention instead of the fused call")
    ap.add_argument("--graph", action="store_true",
                    help="time the fused decode steps replayed from one CUDA graph of the workload's step cycle")
    ap.add_argument("--no-secondary", action="store_true",
                    help="skip the other workloads' block in the headline line")
    ap.add_argument("--cpu-seconds", type=float, default=12.0, help="CPU-baseline budget")
    ap.add_argument("--ref-seconds", type=float, default=150.0, help="reference-arm budget")
    return ap.parse_args(argv)


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except (OSError, KeyError, ValueError):
        return FALLBACK_HBM_GBS, "fallback"


def measured_tflops():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["bf16_tflops"]), "measured burst bf16 (MEASURED_PEAKS.json bf16_tflops)"
    except (OSError, KeyError, ValueError):
        return 1590.0, "fallback 1590 TFLOP/s"


def metric_for(wl) -> str:
    """The metric string of a workload's JSON line (the same for both arms)."""
    if wl.spec.prefill_seqs == 0:
        return METRIC
    if wl.spec.prefill_seqs == wl.B and wl.spec.prefill_len <= 8:
        return SPEC_METRIC
    return MIXED_METRIC


def kernel_source_hash(src: str = None) -> str:
    with open(src or KERNEL_SRC, "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()[:16]


def profiled_traffic(workload: str, kernel: str = "decode_split", src: str = None):
    """DRAM bytes per launch of `kernel` from the committed ncu summary
    profiles/<kernel>_<workload>.txt, or None if there is none or the kernel's
    source (`src`, default the decode kernel's) changed since the capture."""
    path = os.path.join(PROFILE_DIR, f"{kernel}_{workload}.txt")
    try:
        text = open(path).read()
    except OSError:
        return None
    vals = {}
    for line in text.splitlines():
        if ":" in line:
            k, v = line.split(":", 1)
            vals[k.strip()] = v.strip()
    if vals.get("kernel_source_sha256_16") != kernel_source_hash(src):
        return None
    try:
        return float(vals["dram_bytes_per_launch_full_workload"])
    except (KeyError, ValueError):
        return None


# ---------------------------------------------------------------------------
# ranks: one process per GPU; timing is a max over ranks, work a sum
# ---------------------------------------------------------------------------

class Ranks:
    """Barrier and reductions over the job's ranks (NCCL on GPUs, gloo on CPU).

    The data path has no collective: each rank runs its own replica of the
    workload; only timings and counts cross ranks."""

    def __init__(self, world: int, device=None):
        self.world = world
        self.device = device

    def _dist(self):
        import torch.distributed as dist

        return dist

    def barrier(self):
        if self.world > 1:
            self._dist().barrier()

    def _reduce(self, x: float, op) -> float:
        if self.world == 1:
            return float(x)
        import torch

        t = torch.tensor([float(x)], dtype=torch.float64, device=self.device)
        self._dist().all_reduce(t, op=op)
        return float(t.item())

    def max(self, x: float) -> float:
        return self._reduce(x, self._dist().ReduceOp.MAX) if self.world > 1 else float(x)

    def sum(self, x: float) -> float:
        return self._reduce(x, self._dist().ReduceOp.SUM) if self.world > 1 else float(x)


def whole_job_rate(ranks: Ranks, local_units: float, local_ms: float) -> tuple:
    """(units of all ranks per second, slowest rank's ms): the job is as fast as its slowest rank."""
    ms = ranks.max(local_ms)
    units = ranks.sum(local_units)
    return units / (ms * 1e-3), ms


# ---------------------------------------------------------------------------
# workload bookkeeping (host side)
# ---------------------------------------------------------------------------

def kv_tokens(wl, step, seqs):
    """(logical, unique) K/V token rows the attention of `seqs` reads: a physical block
    shared by several sequences counts once in `unique`, for the most tokens any of
    them reads from it."""
    L = wl.context_lens(step).astype(np.int64)
    logical = int(L[seqs].sum())
    used = {}
    for b in seqs:
        nblk = -(-int(L[b]) // wl.BS)
        for i, blk in enumerate(wl.seq_blocks[b][:nblk]):
            n = min(wl.BS, int(L[b]) - i * wl.BS)
            used[int(blk)] = max(used.get(int(blk), 0), n)
    return logical, int(sum(used.values()))


def step_bytes(wl, step, seqs=None, logical=False):
    """Algorithmic HBM bytes of one step over `seqs` (default all): (store, attention).

    Attention reads each live K/V row once (a block shared by several sequences
    once, unless `logical`), reads q, writes out and reads the metadata; the store
    reads and writes each new K/V row once."""
    seqs = np.arange(wl.B) if seqs is None else np.asarray(seqs)
    row = wl.Hkv * wl.D * 2
    nq = int(wl.query_lens[seqs].sum())
    store = 2 * nq * row * 2
    L = wl.context_lens(step).astype(np.int64)[seqs]
    qo = 2 * nq * wl.Hq * wl.D * 2
    meta = len(seqs) * 8 + int(sum(-(-int(x) // wl.BS) for x in L)) * 4
    n_log, n_uni = kv_tokens(wl, step, seqs)
    attn = (n_log if logical else n_uni) * 2 * row + qo + meta
    return store, attn


def prefill_flops(wl, step=0, seqs=None):
    """Algorithmic FLOPs of the attention of `seqs`: 4 * D per (query head, visible key) pair
    (2 * D for q.k, 2 * D for p.v)."""
    seqs = np.arange(wl.B) if seqs is None else np.asarray(seqs)
    L = wl.context_lens(step).astype(np.int64)
    total = 0
    for b in seqs:
        n = int(wl.query_lens[b])
        prior = int(L[b]) - n
        total += n * prior + n * (n + 1) // 2
    return 4 * wl.D * wl.Hq * total


class ClockSampler:
    """nvidia-smi clock/throttle sampling while the GPU is under load."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.t0 = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        self.t0 = time.time()

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.05)
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        rows = [r for r in csv.reader(io.StringIO(out)) if len(r) >= 9]
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].strip().replace(".", "").isdigit()]
        smax = [float(r[2]) for r in rows if r[2].strip().replace(".", "").isdigit()]
        reasons = set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            for i, n in enumerate(names):
                if r[5 + i].strip().lower() == "active":
                    reasons.add(n)
        # samples under load: the upper half of the observed clocks
        loaded = sorted(sm)[len(sm) // 2:] if sm else []
        return {"sm_mhz": statistics.median(loaded) if loaded else None,
                "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(rows)}


# ---------------------------------------------------------------------------
# CPU oracle timing (baseline leg and the reference arm)
# ---------------------------------------------------------------------------

class OracleRunner:
    """Times the fp64 oracle on this workload's sequences, a sample at a time."""

    def __init__(self, wl):
        from oracle import oracle as O

        self.O = O
        self.wl = wl
        self.threads = O.default_threads()
        # compact pool: every block any step references, relabelled in order
        last = wl.spec.num_steps - 1
        bt = wl.block_tables(last)
        used = np.unique(bt[bt >= 0])
        self.lut = np.full(wl.NB, -1, dtype=np.int64)
        self.lut[used] = np.arange(len(used))
        shape = (len(used), wl.BS, wl.Hkv, wl.D)
        self.kp = np.full(shape, 0x7FC0, dtype=np.uint16)
        self.vp = np.full(shape, 0x7FC0, dtype=np.uint16)
        ids, K, V = wl.prior_blocks_dense()
        self.kp[self.lut[ids]] = K
        self.vp[self.lut[ids]] = V
        self.step_cache = {}

    def inputs(self, step):
        if step not in self.step_cache:
            wl = self.wl
            k, v = wl.new_kv(step)
            slots = wl.slot_mapping(step).astype(np.int64)
            cslots = (self.lut[slots // wl.BS] * wl.BS + slots % wl.BS).astype(np.int32)
            bt = wl.block_tables(step)
            btc = np.where(bt >= 0, self.lut[np.maximum(bt, 0)], -1).astype(np.int32)
            self.step_cache[step] = (k, v, cslots, btc, wl.context_lens(step), wl.q(step))
        return self.step_cache[step]

    def run(self, step, seqs):
        """Oracle store of every sequence's new token (so later steps read a
        complete cache), then attention for the sampled sequences.  Returns the
        algorithmic bytes of that work."""
        wl = self.wl
        k, v, cslots, btc, L, q = self.inputs(step)
        seqs = np.asarray(seqs)
        self.O.store_kvcache(k, v, self.kp, self.vp, cslots)
        self.O.decode_attention(q[seqs], self.kp, self.vp, btc[seqs], L[seqs], threads=self.threads)
        row = wl.Hkv * wl.D * 2
        return (wl.B * 4 * row + len(seqs) * 2 * wl.Hq * wl.D * 2 +
                int(L[seqs].astype(np.int64).sum()) * 2 * row)


def cpu_baseline(wl, seconds: float):
    runner = OracleRunner(wl)
    # all sequences of successive steps, until the budget is spent
    t0 = time.perf_counter()
    nbytes = 0
    steps = 0
    while True:
        nbytes += runner.run(steps % wl.spec.num_steps, np.arange(wl.B))
        steps += 1
        if time.perf_counter() - t0 >= seconds or steps >= wl.spec.num_steps:
            break
    dt = time.perf_counter() - t0
    return {"value": nbytes / dt / 1e9, "unit": "GB/s", "cores": runner.threads, "kind": "oracle",
            "tokens_per_s": steps * wl.B / dt,
            "sample": f"fp64 C oracle (store + decode attention) on steps 0..{steps - 1} of {wl.spec.name}, "
                      f"all {wl.B} sequences, {runner.threads} threads, {dt:.1f} s"}


def reference_arm(args, rank, world):
    from paged_kv_cache_bf16_b200 import workloads as W

    if rank != 0:
        return 0
    wl = W.workload(args.workload)
    runner = OracleRunner(wl)
    # calibrate: seconds per sequence of oracle work
    t0 = time.perf_counter()
    runner.run(0, np.arange(min(8, wl.B)))
    per_seq = (time.perf_counter() - t0) / min(8, wl.B)
    total_steps = args.steps + args.warmup
    n = int(max(1, min(wl.B, args.ref_seconds / max(1e-9, per_seq * total_steps))))
    for i in range(args.warmup):
        runner.run(i % wl.spec.num_steps, np.arange(i * n, i * n + n) % wl.B)
    t0 = time.perf_counter()
    nbytes = 0
    for i in range(args.steps):
        j = args.warmup + i
        nbytes += runner.run(j % wl.spec.num_steps, (np.arange(n) + j * n) % wl.B)
    dt = time.perf_counter() - t0
    value = nbytes / dt / 1e9
    sample = (f"each step: the fp64 C oracle's store + decode attention for {n} of the {wl.B} sequences of "
              f"{wl.spec.name} ({runner.threads} threads)")
    line = {"metric": metric_for(wl), "value": value, "unit": "GB/s", "impl": "reference", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": workload_config(wl),
            "cpu_baseline": {"value": value, "unit": "GB/s", "cores": runner.threads, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def workload_config(wl):
    s = wl.spec
    if s.prefill_seqs:
        lens = (f"{s.prefill_seqs} sequences x {s.prefill_len} query rows over prior U[{s.prior_lo},{s.prior_hi}]"
                + (f" + {s.num_seqs - s.prefill_seqs} decode rows over U[{s.ctx_lo},{s.ctx_hi}]"
                   if s.num_seqs > s.prefill_seqs else ""))
    else:
        lens = f"U[{s.ctx_lo},{s.ctx_hi}]" + (" +1 per step" if s.num_steps > 1 else "")
    return {"workload": s.name, "num_seqs": s.num_seqs, "num_q_heads": s.num_q_heads,
            "num_kv_heads": s.num_kv_heads, "head_dim": s.head_dim, "block_size": s.block_size,
            "num_blocks": s.num_blocks, "context_lens": lens,
            "steps_cycle": s.num_steps,
            "l2": "not flushed: inputs larger than L2 (K/V read per step %.2f GB vs 126 MB L2)"
                  % (step_bytes(wl, 0)[1] / 1e9)}


# ---------------------------------------------------------------------------
# the npv arm
# ---------------------------------------------------------------------------

def npv_arm(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist

    from paged_kv_cache_bf16_b200 import ops
    from paged_kv_cache_bf16_b200 import workloads as W

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    ops.lib()
    wl = W.workload(args.workload)
    nsteps = wl.spec.num_steps
    mixed = wl.spec.prefill_seqs > 0
    st = W.DeviceState(wl, dev, steps=list(range(nsteps)))
    if mixed:
        ws = ops.alloc_workspace(ops.prefill_workspace_size(wl.B, wl.total_q, wl.Hq, wl.Hkv, wl.D), dev)
        out = torch.empty((wl.total_q, wl.Hq, wl.D), dtype=torch.bfloat16, device=dev)
    else:
        ws = ops.alloc_workspace(ops.decode_workspace_size(wl.B, wl.Hq, wl.Hkv, wl.D), dev)
        out = torch.empty((wl.B, wl.Hq, wl.D), dtype=torch.bfloat16, device=dev)
    stream = torch.cuda.current_stream(dev)

    def attend(i):
        s = st.steps[i % nsteps]
        if mixed:
            ops.paged_prefill_attention(s["q"], st.k_cache, st.v_cache, s["cu_seqlens_q"], s["max_seqlen_q"],
                                        s["block_tables"], s["context_lens"], out=out, workspace=ws)
        elif args.separate_store:
            ops.paged_decode_attention(s["q"], st.k_cache, st.v_cache, s["block_tables"], s["context_lens"],
                                       out=out, workspace=ws)
        else:
            ops.store_kvcache_and_decode_attention(s["q"], s["key"], s["value"], st.k_cache, st.v_cache,
                                                   s["slot_mapping"], s["block_tables"], s["context_lens"],
                                                   out=out, workspace=ws)

    def step(i):
        if mixed or args.separate_store:
            s = st.steps[i % nsteps]
            ops.store_kvcache(s["key"], s["value"], st.k_cache, st.v_cache, s["slot_mapping"])
        attend(i)

    launches_per_step = (5 if mixed else (3 if args.separate_store else 2))

    ranks = Ranks(world, dev)
    barrier = ranks.barrier
    max_over_ranks = ranks.max

    per_step = [step_bytes(wl, i) for i in range(nsteps)]
    bytes_steps = [per_step[i % nsteps] for i in range(args.steps)]
    store_bytes = sum(b[0] for b in bytes_steps)
    attn_bytes = sum(b[1] for b in bytes_steps)
    logical_attn = sum(step_bytes(wl, i, logical=True)[1] for i in range(nsteps)) / nsteps

    for i in range(args.warmup):
        step(i)
    ops.check_device_errors()

    sampler = ClockSampler(local_rank) if rank == 0 else None
    if sampler:
        sampler.start()
        time.sleep(0.3)

    def timed(fn, n):
        barrier()
        torch.cuda.synchronize(dev)
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for i in range(n):
            fn(i)
        e1.record(stream)
        torch.cuda.synchronize(dev)
        barrier()
        return max_over_ranks(e0.elapsed_time(e1))

    # ---- timed region 1: the step loop -> value
    graph = None
    if args.graph:
        if mixed or args.separate_store:
            raise SystemExit("--graph times the fused decode step only")
        # one graph holds the workload's whole step cycle (its per-step inputs are
        # distinct device tensors); replays repeat the cycle, re-storing the same
        # tokens into the same slots exactly as the eager loop does
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            for i in range(nsteps):
                step(i)
        reps = max(1, -(-args.steps // nsteps))
        args.steps = reps * nsteps
        bytes_steps = [per_step[i % nsteps] for i in range(args.steps)]
        store_bytes = sum(b[0] for b in bytes_steps)
        attn_bytes = sum(b[1] for b in bytes_steps)
        graph.replay()
        torch.cuda.synchronize(dev)
        ms = timed(lambda i: graph.replay(), reps)
    else:
        ms = timed(step, args.steps)

    # ---- timed region 2: events around each attention call -> kernel roofline
    barrier()
    torch.cuda.synchronize(dev)
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    for i in range(args.steps):
        if mixed or args.separate_store:
            s = st.steps[i % nsteps]
            ops.store_kvcache(s["key"], s["value"], st.k_cache, st.v_cache, s["slot_mapping"])
        evs[i][0].record(stream)
        attend(i)
        evs[i][1].record(stream)
    torch.cuda.synchronize(dev)
    barrier()
    call_ms = max_over_ranks(sum(a.elapsed_time(b) for a, b in evs) / args.steps)

    extra = {}
    if mixed:
        extra = mixed_subbatches(args.steps, wl, st, dev, stream, ops, W, timed)

    # keep the GPU loaded long enough for the clock sampler to see it
    t_end = time.time() + 1.5
    i = 0
    while time.time() < t_end:
        for _ in range(20):
            step(i)
            i += 1
        torch.cuda.synchronize(dev)
    clocks = sampler.stop() if sampler else None
    ops.check_device_errors()

    e2e = None
    if not args.no_e2e:
        e2e = npv_e2e(args, wl, st, ws, dev, stream, ops, W, barrier, max_over_ranks, step_fn_kind(args, mixed))

    peak, peak_kind = measured_peaks()
    # value: bytes of all ranks over the slowest rank's time (ms is already the max)
    rate, _ = whole_job_rate(ranks, store_bytes + attn_bytes, ms)
    value = rate / 1e9
    call_bytes = attn_bytes / args.steps + (0 if (mixed or args.separate_store) else store_bytes / args.steps)
    # With the fused call every step is exactly one call, so its mean duration over
    # the timed region is the step time (back-to-back calls overlap their launch
    # with programmatic dependent launch; the per-call events of region 2 break
    # that overlap and are reported as isolated_call_ms).
    launch_ms = (ms / args.steps) if not (mixed or args.separate_store) else call_ms
    achieved = call_bytes / (launch_ms * 1e-3) / 1e9
    line = {
        "metric": metric_for(wl),
        "value": value, "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": workload_config(wl),
        "tokens_per_s": ranks.sum(args.steps * wl.total_q) / (ms * 1e-3),
        "pct_of_peak_hbm": 100.0 * value / world / peak,
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clocks,
    }
    if graph is not None:
        line["config"]["cuda_graph"] = f"{nsteps} steps per graph, {args.steps // nsteps} replays"
    if wl.spec.share_group:
        # prefix-shared blocks: the GB/s above count each shared block once
        line["kv_bytes_per_step"] = {"unique": attn_bytes / args.steps, "logical": logical_attn}
        line["logical_gb_s"] = ranks.sum((logical_attn + store_bytes / args.steps) * args.steps) / (ms * 1e-3) / 1e9
    if not mixed:
        line["roofline"] = {
            "kernel": ("npv_paged_decode_attention" if args.separate_store else
                       "npv_store_kvcache_and_decode_attention") + " (split-KV kernel + merge kernel)",
            "bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
            "peak_source": f"{peak_kind}: MEASURED_PEAKS.json hbm_gbs" if peak_kind == "measured"
            else "fallback 6650 GB/s",
            "traffic": profiled_traffic(args.workload) if not args.separate_store else None,
            "traffic_source": (f"copied from the ncu capture in profiles/decode_split_{args.workload}.txt "
                               "(kept only while the kernel source hash matches the capture's)"),
            "algorithmic_bytes_per_launch": call_bytes, "mean_launch_ms": launch_ms,
            "isolated_call_ms": call_ms}
    else:
        line["roofline"] = extra.pop("roofline")
        line.update(extra)
    if e2e is not None:
        line["e2e"] = e2e
    if world == 1 and not args.no_secondary and args.workload == W.HEADLINE and not args.graph:
        del st, ws, out
        torch.cuda.empty_cache()
        line["secondary"] = secondary(args, dev, stream, ops, W, timed)
    if rank == 0 and not args.no_cpu_baseline and not mixed:
        line["cpu_baseline"] = cpu_baseline(wl, args.cpu_seconds)
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


# The other named workloads, measured in the headline run (one GPU) so that each
# has a record beside the headline: GQA 4:1 decode with prefix-shared blocks,
# long-context split-KV decode, the chunked-prefill mix and speculative-decode
# verification.
SECONDARY = ("llama8b_prefix_decode", "long_context_decode", "chunked_prefill_mixed", "spec_verify_decode")


def secondary(args, dev, stream, ops, W, timed):
    """One short timed loop per secondary workload (inputs resident; CUDA events)."""
    import torch

    hbm_peak, _ = measured_peaks()
    steps = max(3, min(args.steps, 30))
    res = {"steps": steps, "warmup": 3,
           "note": "each workload's own step (decode: fused store + decode call; mixed and verify: store + "
                   "prefill call), timed like the headline; bytes as the headline counts them"}
    for name in SECONDARY:
        wl = W.workload(name)
        st = W.DeviceState(wl, dev)
        s = st.steps[0]
        mixed = wl.spec.prefill_seqs > 0
        if mixed:
            ws = ops.alloc_workspace(ops.prefill_workspace_size(wl.B, wl.total_q, wl.Hq, wl.Hkv, wl.D), dev)
        else:
            ws = ops.alloc_workspace(ops.decode_workspace_size(wl.B, wl.Hq, wl.Hkv, wl.D), dev)
        out = torch.empty((wl.total_q, wl.Hq, wl.D), dtype=torch.bfloat16, device=dev)

        def step(i):
            if mixed:
                ops.store_kvcache(s["key"], s["value"], st.k_cache, st.v_cache, s["slot_mapping"])
                ops.paged_prefill_attention(s["q"], st.k_cache, st.v_cache, s["cu_seqlens_q"], s["max_seqlen_q"],
                                            s["block_tables"], s["context_lens"], out=out, workspace=ws)
            else:
                ops.store_kvcache_and_decode_attention(s["q"], s["key"], s["value"], st.k_cache, st.v_cache,
                                                       s["slot_mapping"], s["block_tables"], s["context_lens"],
                                                       out=out, workspace=ws)

        for i in range(3):
            step(i)
        ops.check_device_errors()
        ms = timed(step, steps) / steps
        store_b, attn_b = step_bytes(wl, 0)
        gbs = (store_b + attn_b) / (ms * 1e-3) / 1e9
        r = {"metric": metric_for(wl), "ms_per_step": ms, "gb_s": gbs, "frac_of_hbm": gbs / hbm_peak,
             "tokens_per_s": wl.total_q / (ms * 1e-3), "config": workload_config(wl)}
        if wl.spec.share_group:
            _, logical = step_bytes(wl, 0, logical=True)
            r["logical_gb_s"] = (store_b + logical) / (ms * 1e-3) / 1e9
            r["bytes"] = "gb_s counts each prefix-shared block once; logical_gb_s once per reading sequence"
        if mixed:
            r.update(mixed_subbatches(steps, wl, st, dev, stream, ops, W, timed))
        ops.check_device_errors()
        res[name] = r
        del st, ws, out, s
        torch.cuda.empty_cache()
    res["qwen3_decode_rope"] = rope_decode(steps, dev, ops, W, timed)
    return res


ROPE_BASE = 1.0e6  # Qwen3's rotary base


def rope_decode(steps, dev, ops, W, timed):
    """The headline decode step with RoPE: npv_rope_store_kvcache (rotate q in place,
    rotate k, store k and v) then npv_paged_decode_attention, two launches per step."""
    import torch

    hbm_peak, _ = measured_peaks()
    wl = W.workload(W.HEADLINE)
    st = W.DeviceState(wl, dev)
    s = st.steps[0]
    _, pos = wl.token_positions(0)
    positions = torch.from_numpy(pos.astype(np.int32)).to(dev)
    q = s["q"].clone()
    ws = ops.alloc_workspace(ops.decode_workspace_size(wl.B, wl.Hq, wl.Hkv, wl.D), dev)
    out = torch.empty((wl.B, wl.Hq, wl.D), dtype=torch.bfloat16, device=dev)

    def step(i):
        ops.rope_store_kvcache(q, s["key"], s["value"], positions, st.k_cache, st.v_cache, s["slot_mapping"],
                               ROPE_BASE)
        ops.paged_decode_attention(q, st.k_cache, st.v_cache, s["block_tables"], s["context_lens"], out=out,
                                   workspace=ws)

    for i in range(3):
        step(i)
    ops.check_device_errors()
    ms = timed(step, steps) / steps
    ops.check_device_errors()
    store_b, attn_b = step_bytes(wl, 0)
    q_rt = 2 * wl.B * wl.Hq * wl.D * 2  # q read and rewritten by the rotation
    gbs = (store_b + attn_b + q_rt) / (ms * 1e-3) / 1e9
    r = {"metric": metric_for(wl), "ms_per_step": ms, "gb_s": gbs, "frac_of_hbm": gbs / hbm_peak,
         "tokens_per_s": wl.B / (ms * 1e-3), "rope_base": ROPE_BASE,
         "config": dict(workload_config(wl), workload="qwen3_decode with RoPE on q and k before the store"),
         "bytes": "headline step bytes + the q rows read and rewritten by the rotation"}
    del st, ws, out, s, q
    torch.cuda.empty_cache()
    return r


def step_fn_kind(args, mixed):
    return "mixed" if mixed else ("separate" if args.separate_store else "fused")


def mixed_subbatches(steps, wl, st, dev, stream, ops, W, timed):
    """Time the prefill-only and decode-only parts of the mixed batch as their own calls."""
    import torch

    tflops_peak, tf_kind = measured_tflops()
    hbm_peak, _ = measured_peaks()
    s = st.steps[0]
    cu = wl.cu_seqlens_q()
    res = {}
    for kind in ("prefill", "decode"):
        seqs = [b for b in range(wl.B) if (wl.query_lens[b] > 1) == (kind == "prefill")]
        if not seqs:
            continue
        rows = np.concatenate([np.arange(cu[b], cu[b + 1]) for b in seqs])
        ridx = torch.from_numpy(rows).to(dev)
        bidx = torch.from_numpy(np.array(seqs)).to(dev)
        q = s["q"].index_select(0, ridx).contiguous()
        bt = s["block_tables"].index_select(0, bidx).contiguous()
        cl = s["context_lens"].index_select(0, bidx).contiguous()
        cus = np.zeros(len(seqs) + 1, dtype=np.int32)
        cus[1:] = np.cumsum(wl.query_lens[seqs])
        cut = torch.from_numpy(cus).to(dev)
        o = torch.empty_like(q)
        wsz = ops.prefill_workspace_size(len(seqs), int(cus[-1]), wl.Hq, wl.Hkv, wl.D)
        w = ops.alloc_workspace(wsz, dev)
        mq = int(wl.query_lens[seqs].max())

        def call(i, q=q, cut=cut, mq=mq, bt=bt, cl=cl, o=o, w=w):
            ops.paged_prefill_attention(q, st.k_cache, st.v_cache, cut, mq, bt, cl, out=o, workspace=w)

        for i in range(3):
            call(i)
        ms = timed(call, steps) / steps
        _, nbytes = step_bytes(wl, 0, seqs)
        fl = prefill_flops(wl, 0, seqs)
        res[kind] = {"ms": ms, "gb_s": nbytes / (ms * 1e-3) / 1e9, "tflop_s": fl / (ms * 1e-3) / 1e12,
                     "rows": int(cus[-1]), "seqs": len(seqs)}
    pre = res["prefill"]
    pre_seqs = [b for b in range(wl.B) if wl.query_lens[b] > 1]
    name = f"npv_paged_prefill_attention on the {len(pre_seqs)} multi-row sequences (plan + tcgen05 kernel)"
    # the binding resource of the multi-row part: tensor pipe (long chunks) or HBM
    # (a few rows per sequence, e.g. speculative-decode verification)
    if pre["tflop_s"] / tflops_peak >= pre["gb_s"] / hbm_peak:
        traffic = profiled_traffic(wl.spec.name, "prefill_attention", PREFILL_SRC)
        roof = {"kernel": name, "bound": "tensor", "achieved": pre["tflop_s"], "peak": tflops_peak,
                "unit": "TFLOP/s", "frac": pre["tflop_s"] / tflops_peak, "peak_source": tf_kind,
                "traffic": traffic,
                "traffic_source": (f"copied from the ncu capture in profiles/prefill_attention_{wl.spec.name}.txt "
                                   "(kept only while the kernel source hash matches the capture's)"),
                "algorithmic_flops_per_launch": prefill_flops(wl, 0, pre_seqs), "mean_launch_ms": pre["ms"]}
    else:
        _, hbm_kind = measured_peaks()
        roof = {"kernel": name, "bound": "hbm", "achieved": pre["gb_s"], "peak": hbm_peak, "unit": "GB/s",
                "frac": pre["gb_s"] / hbm_peak,
                "peak_source": "measured: MEASURED_PEAKS.json hbm_gbs" if hbm_kind == "measured"
                else "fallback 6650 GB/s",
                "traffic": None, "algorithmic_bytes_per_launch": step_bytes(wl, 0, pre_seqs)[1],
                "mean_launch_ms": pre["ms"]}
    out = {"roofline": roof, "prefill_part": pre}
    if "decode" in res:
        out["decode_part"] = dict(res["decode"], pct_of_peak_hbm=100 * res["decode"]["gb_s"] / hbm_peak)
    return out


def npv_e2e(args, wl, st, ws, dev, stream, ops, W, barrier, max_over_ranks, kind):
    """End to end through the public API with host-resident inputs and outputs.

    Each step's inputs (q, the new K/V rows and the metadata) sit packed in one
    pinned host buffer; every step copies its buffer to the device with one
    host-to-device copy, runs the step's library calls on views of the device
    buffer, and copies the output back with one device-to-host copy.  The
    copies run on their own streams, double-buffered, so step i+1's upload and
    step i-1's download overlap step i's kernels; every copy of every timed
    step lies inside the timed region."""
    import torch

    nsteps = wl.spec.num_steps
    keys = ["q", "key", "value", "slot_mapping", "block_tables", "context_lens", "cu_seqlens_q"]
    used = keys if kind == "mixed" else keys[:-1]
    layout, off = [], 0
    for k in used:
        t = st.steps[0][k]
        nb = t.numel() * t.element_size()
        layout.append((k, off, nb, t.dtype, tuple(t.shape)))
        off = (off + nb + 255) // 256 * 256
    total = off
    host = []
    for i in range(nsteps):
        h = torch.empty(total, dtype=torch.uint8).pin_memory()
        for k, o, nb, _, _ in layout:
            h[o:o + nb].copy_(st.steps[i][k].contiguous().view(torch.uint8).reshape(-1).cpu())
        host.append(h)
    nbuf = 2
    dbufs = [torch.empty(total, dtype=torch.uint8, device=dev) for _ in range(nbuf)]
    views = [{k: d[o:o + nb].view(dt).view(shp) for k, o, nb, dt, shp in layout} for d in dbufs]
    out_dev = [torch.empty((wl.total_q, wl.Hq, wl.D), dtype=torch.bfloat16, device=dev) for _ in range(nbuf)]
    out_host = [torch.empty((wl.total_q, wl.Hq, wl.D), dtype=torch.bfloat16).pin_memory() for _ in range(nbuf)]
    h2d = total
    d2h = out_host[0].numel() * out_host[0].element_size()
    mq = st.steps[0]["max_seqlen_q"]
    up, down = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev = lambda: torch.cuda.Event()  # noqa: E731
    uploaded = [ev() for _ in range(nbuf)]
    computed = [ev() for _ in range(nbuf)]
    downloaded = [ev() for _ in range(nbuf)]
    started = [False] * nbuf

    def compute(v, o):
        if kind == "fused":
            ops.store_kvcache_and_decode_attention(v["q"], v["key"], v["value"], st.k_cache, st.v_cache,
                                                   v["slot_mapping"], v["block_tables"], v["context_lens"],
                                                   out=o, workspace=ws)
        else:
            ops.store_kvcache(v["key"], v["value"], st.k_cache, st.v_cache, v["slot_mapping"])
            if kind == "mixed":
                ops.paged_prefill_attention(v["q"], st.k_cache, st.v_cache, v["cu_seqlens_q"], mq,
                                            v["block_tables"], v["context_lens"], out=o, workspace=ws)
            else:
                ops.paged_decode_attention(v["q"], st.k_cache, st.v_cache, v["block_tables"], v["context_lens"],
                                           out=o, workspace=ws)

    def step(i):
        j = i % nbuf
        with torch.cuda.stream(up):
            if started[j]:
                up.wait_event(computed[j])  # the kernels of step i - nbuf have read this buffer
            dbufs[j].copy_(host[i % nsteps], non_blocking=True)
            uploaded[j].record(up)
        stream.wait_event(uploaded[j])
        if started[j]:
            stream.wait_event(downloaded[j])  # step i - nbuf's output has left this buffer
        compute(views[j], out_dev[j])
        computed[j].record(stream)
        with torch.cuda.stream(down):
            down.wait_event(computed[j])
            out_host[j].copy_(out_dev[j], non_blocking=True)
            downloaded[j].record(down)
        started[j] = True

    def drain():
        for j in range(nbuf):
            if started[j]:
                stream.wait_event(downloaded[j])

    for i in range(args.warmup):
        step(i)
    drain()
    barrier()
    torch.cuda.synchronize(dev)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    up.wait_event(e0)
    down.wait_event(e0)
    for i in range(args.steps):
        step(i)
    drain()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    barrier()
    ms = max_over_ranks(e0.elapsed_time(e1))
    nbytes = sum(sum(step_bytes(wl, i % nsteps)) for i in range(args.steps))
    world = 1 if not torch.distributed.is_initialized() else torch.distributed.get_world_size()
    return {"value": world * nbytes / (ms * 1e-3) / 1e9, "unit": "GB/s", "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "ms_per_step": ms / args.steps,
            "tokens_per_s": world * args.steps * wl.total_q / (ms * 1e-3),
            "copies_per_step": {"h2d": 1, "d2h": 1},
            "pipelining": "uploads and downloads on their own streams, two buffers deep"}


def main(argv=None):
    args = parse_args(argv)
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        return reference_arm(args, rank, world)
    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist

        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    try:
        return npv_arm(args, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist

            dist.destroy_process_group()


if __name__ == "__main__":
    sys.exit(main())
