"""Benchmark of the paged decode step (cache write of one new token per
sequence + decode attention over the block tables) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload 70b|7b|long|tiny]
    python bench.py --impl reference ...      # the CPU oracle, same workload

Prints one JSON line.  ``value`` is KV bytes read per second over the whole
step (cache write + plan in one kernel, decode, reduce: pa_write_decode),
inputs resident in HBM, L2 flushed between steps (the flush is outside the
per-step events).  ``e2e`` is the same metric through ``pa_step`` with pinned
host buffers, host<->device copies inside each step's events, measured like
``value``; ``e2e.pipelined`` is the overlapped serving loop (pa_pipeline)
beside the device-only step over the same continuous loop.  ``roofline`` is
the decode kernel's achieved bandwidth (algorithmic bytes / its average
event-timed duration) against the measured HBM copy bandwidth.  On the
default run the other configurations follow as sub-objects: ``workloads``
(7B-shaped and long split-K decode), ``trace`` (per-step time of the
continuous-batching trace) and ``verify_q6`` (the verification pass of six
candidate tokens).  N > 1 runs independent replicas (one per GPU, no
data-path collective; weak scaling).
"""

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from paged_kv_cache_381_b200 import workloads as wl  # noqa: E402

WORKLOAD_NAMES = {
    "70b": "llama3-70b-shaped decode layer: bf16, 64 q / 8 kv heads (GQA 8), head_dim 128, block 16, "
           "256 seqs, contexts ~ Zipf(1.2) on [16, 8192], shuffled physical blocks",
    "7b": "llama2-7b-shaped decode layer: fp16, 32 q / 32 kv heads, head_dim 128, block 16, 64 seqs, "
          "contexts ~ U[128, 2048]",
    "long": "long-context split-K: bf16, 64 q / 8 kv heads, head_dim 128, block 16, 8 seqs x 32768 tokens, "
            "512-token partitions, 1% of K rows x8",
    "tiny": "tiny fp32 paged decode: 4 seqs {1,16,17,90}, 4/4 heads, head_dim 64, block 16, 32-block pool",
}
METRIC = "paged decode attention: KV GB/s read (% of B200 HBM peak); decode tokens/s"
VERIFY_METRIC = "paged verification attention (speculative decoding): KV GB/s read; verified tokens/s"
SPEC_HBM_GBS = 8000.0          # B200 HBM3e data-sheet bandwidth, reported beside the measured peak
_DEV = "paged_kv_cache_381_b200/csrc/device/"
# the sources each timed kernel is built from: a recorded ncu traffic figure is
# reported only while their hash is the one it was taken on
KERNEL_SOURCES = {
    "decode": [_DEV + "decode.cuh", _DEV + "common.cuh"],
    "verify": [_DEV + "verify.cuh", _DEV + "decode.cuh", _DEV + "common.cuh"],
    "verify_tc": [_DEV + "verify_tc.cuh", _DEV + "tcgen05.cuh", _DEV + "decode.cuh", _DEV + "common.cuh"],
}


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=300)
    p.add_argument("--warmup", type=int, default=10)
    p.add_argument("--impl", default="native", choices=["native", "reference"])
    p.add_argument("--workload", default="70b", choices=list(WORKLOAD_NAMES))
    p.add_argument("--seed", type=int, default=0)
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--no-extra", action="store_true",
                   help="time the 70b workload only (no 7b / long / trace / verification sub-objects)")
    p.add_argument("--math", default="auto", choices=["auto", "simt"],
                   help="decode arithmetic: tensor cores for fp16/bf16 (auto), CUDA cores (simt)")
    p.add_argument("--merge", default="kernel", choices=["kernel", "fused"],
                   help="merge split partitions with the reduce kernel or inside the decode kernel")
    p.add_argument("--num-seqs", type=int, default=0,
                   help="keep only the first N sequences (smaller cases for profiling)")
    p.add_argument("--swap-mb", type=int, default=0,
                   help="> 0: time pa_swap_blocks moving this many MiB of blocks (K and V) between the "
                        "device pool and a pinned host pool, against one contiguous copy of the same bytes")
    p.add_argument("--verify-kernel", default="auto", choices=["auto", "mma_sync", "tcgen05"],
                   help="tensor-core path of the verification pass (with --queries > 1)")
    p.add_argument("--partition-size", type=int, default=0,
                   help="split-K partition in tokens (power of two >= the block size); 0: the workload's (512)")
    p.add_argument("--profile-all", action="store_true",
                   help="event-time every library launch (kernel_ms per kernel); the events between "
                        "dependent launches cost the step its launch overlap, so ms_per_step rises")
    p.add_argument("--queries", type=int, default=1,
                   help="candidate tokens per sequence: > 1 times the verification pass (pa_verify) "
                        "of speculative decoding instead of decode")
    return p.parse_args()


def kernel_hash(kernel="decode"):
    """Hash of the kernel's sources without // comments and blank lines, so that a
    comment edit does not void a recorded traffic figure."""
    h = hashlib.sha256()
    for rel in KERNEL_SOURCES[kernel]:
        with open(os.path.join(ROOT, rel), encoding="utf-8") as f:
            for line in f:
                code = line.split("//", 1)[0].rstrip()
                if code:
                    h.update(code.encode() + b"\n")
    return h.hexdigest()[:16]


def traffic_profile_name(kernel, workload, queries):
    return f"{kernel}_{workload}_traffic.json" if queries == 1 else f"{kernel}_{workload}_q{queries}_traffic.json"


def _current_record(kernel, workload, queries):
    path = os.path.join(ROOT, "profiles", traffic_profile_name(kernel, workload, queries))
    if not os.path.exists(path):
        return None
    with open(path) as f:
        j = json.load(f)
    if j.get("kernel_source_sha256_16") != kernel_hash(kernel):
        return None
    return j


def recorded_traffic(kernel, workload, queries=1):
    """DRAM bytes per launch of `kernel` from the committed ncu summary for this
    workload, if it was taken on the current kernel source; else None."""
    j = _current_record(kernel, workload, queries)
    return None if j is None else j.get("dram_bytes_per_launch")


def recorded_dram_pct(kernel, workload, queries=1):
    """ncu's dram__throughput.avg.pct_of_peak_sustained_elapsed for `kernel` on
    this workload (mean over the captured launches), under the same gate."""
    j = _current_record(kernel, workload, queries)
    return None if j is None else j.get("dram_throughput_pct_of_peak_ncu")


def elt_bytes(dtype):
    return wl.ELEMENT_BYTES[dtype]


def kv_bytes(cfg, lens):
    return int(np.sum(lens)) * 2 * cfg.num_kv_heads * cfg.head_dim * elt_bytes(cfg.dtype)


def decode_kernel_bytes(cfg, lens, partition, fused=False):
    """Algorithmic bytes one decode-kernel launch must move: live K/V rows, q,
    the final rows it writes (all of them when partitions are merged in the
    kernel, else those of one-partition sequences), the fp32 partials (o, m, l)
    of split sequences (written, and read back when merged in the kernel), and
    the block-table entries each kv head reads."""
    e = elt_bytes(cfg.dtype)
    S, Hq, Hkv, D, bs = len(lens), cfg.num_heads, cfg.num_kv_heads, cfg.head_dim, cfg.block_size
    P = partition or 512
    maxc = int(np.max(lens)) if S else 0
    nparts = np.where(lens <= P, 1, -(-lens // P)) if maxc > P else np.ones(S, dtype=np.int64)
    single = nparts == 1
    b = kv_bytes(cfg, lens)
    b += S * Hq * D * e                                   # q
    b += (S * Hq * D * e if fused else int(single.sum()) * Hq * D * e)   # final rows
    b += (2 if fused else 1) * int(nparts[~single].sum()) * Hq * (D + 2) * 4   # partials (+ read back when fused)
    b += int(np.sum(-(-lens // bs))) * Hkv * 4            # block-table entries
    return int(b)


def verify_kernel_bytes(cfg, lens, partition, Q):
    """decode_kernel_bytes for the verification pass: Q query and output rows
    per sequence and head (partials likewise)."""
    e = elt_bytes(cfg.dtype)
    S, Hq, Hkv, D, bs = len(lens), cfg.num_heads, cfg.num_kv_heads, cfg.head_dim, cfg.block_size
    P = partition or 512
    maxc = int(np.max(lens)) if S else 0
    nparts = np.where(lens <= P, 1, -(-lens // P)) if maxc > P else np.ones(S, dtype=np.int64)
    single = nparts == 1
    b = kv_bytes(cfg, lens)
    b += S * Q * Hq * D * e
    b += int(single.sum()) * Q * Hq * D * e
    b += int(nparts[~single].sum()) * Q * Hq * (D + 2) * 4
    b += int(np.sum(-(-lens // bs))) * Hkv * 4
    return int(b)


def verify_flops(cfg, lens, Q):
    """Multiply-adds x 2 of S = QK^T and O = PV over the causal prefix of every
    query row: 4 * D * Hq * sum_s sum_i (ctx_s - Q + i + 1)."""
    seen = sum(max(0, int(n) - Q + i + 1) for n in lens for i in range(Q))
    return 4.0 * cfg.head_dim * cfg.num_heads * seen


def measured_tensor_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            return float(json.load(f)["bf16_tflops"]), "measured"
    return 1590.0, "fallback"


class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled every 200 ms."""

    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.idx = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.idx}", f"--query-gpu={self.QUERY}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=self.f, stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.f.close()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows)}


# ---------------------------------------------------------------------------
# CPU oracle timing (baseline leg and reference arm)
# ---------------------------------------------------------------------------

def _oracle_sample(cfg, seed, seqs, lens):
    """Host histories for the sampled sequences (numpy draws of the same shape)."""
    r = np.random.default_rng([seed, 7])
    Hq, Hkv, D = cfg.num_heads, cfg.num_kv_heads, cfg.head_dim
    items = []
    for s in seqs:
        n = int(lens[s])
        q = wl.normal_storage(r, (Hq, D), cfg.dtype)
        k = wl.normal_storage(r, (n, Hkv, D), cfg.dtype)
        v = wl.normal_storage(r, (n, Hkv, D), cfg.dtype)
        items.append((q, k, v))
    return items


def _time_oracle(cfg, items):
    from oracle import attention as oa
    from oracle.numerics import widen
    t0 = time.perf_counter()
    for q, k, v in items:
        oa.decode_history(widen(q, cfg.dtype), widen(k, cfg.dtype), widen(v, cfg.dtype), cfg.scale)
    return time.perf_counter() - t0


def _single_thread():
    """Context manager limiting BLAS to one thread (no-op if unavailable)."""
    try:
        from threadpoolctl import threadpool_limits
        return threadpool_limits(limits=1)
    except ImportError:
        import contextlib
        return contextlib.nullcontext()


def cpu_baseline(cfg, seed, lens, unit_scale, min_seconds=10.0, max_rounds=200):
    """The oracle, as it stands, on every 4th sequence of the workload, repeated
    until at least ``min_seconds`` of CPU work have been timed."""
    seqs = list(range(0, len(lens), 4)) or [0]
    items = _oracle_sample(cfg, seed, seqs, lens)
    secs, rounds = 0.0, 0
    with _single_thread():
        while secs < min_seconds and rounds < max_rounds:
            secs += _time_oracle(cfg, items)
            rounds += 1
    b = kv_bytes(cfg, lens[seqs]) * rounds
    return {"value": b / secs / unit_scale, "unit": "GB/s", "cores": 1, "kind": "oracle",
            "sample": f"{len(seqs)} of {len(lens)} sequences (every 4th), all {cfg.num_heads} query heads, "
                      f"{rounds} rounds, float64 numpy, 1 BLAS thread, {secs:.1f} s"}


def _oracle_worker(task):
    """One process of the all-cores baseline: its share of the sampled
    sequences (drawn here with the same shapes), timed after a start barrier."""
    cfg_name, seed, seqs, lens, rounds, barrier = task
    cfg = wl.CONFIGS[cfg_name]
    items = _oracle_sample(cfg, seed + 1000 + int(seqs[0]), seqs, lens)
    with _single_thread():
        _time_oracle(cfg, items[:1])                 # imports and first-touch outside the timing
        barrier.wait()
        secs = 0.0
        for _ in range(rounds):
            secs += _time_oracle(cfg, items)
    return secs


def cpu_baseline_all_cores(cfg_name, seed, lens, unit_scale, single, min_seconds=8.0):
    """The same oracle on every host core: one process per core (spawned; one
    BLAS thread each), the sampled sequences dealt round-robin, all started
    together; throughput = all bytes / the slowest process's time.  ``single``
    is the one-thread result, used to size the rounds."""
    import multiprocessing as mp
    cfg = wl.CONFIGS[cfg_name]
    seqs = list(range(0, len(lens), 4)) or [0]
    cores = len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else (os.cpu_count() or 1)
    cores = max(1, min(cores, len(seqs)))
    shares = [seqs[w::cores] for w in range(cores)]
    sample_bytes = kv_bytes(cfg, lens[seqs])
    per_round_1 = sample_bytes / (single * unit_scale)          # seconds per round on one thread
    # processes sharing the host's cores (and its hyperthreads) ran about 4x slower
    # each than one alone on a 16-core box: size for a third of the single rate
    rounds = max(1, min(200, int(np.ceil(min_seconds * cores / (3.0 * per_round_1)))))
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        barrier = mgr.Barrier(cores)
        with ctx.Pool(cores) as pool:
            secs = pool.map(_oracle_worker, [(cfg_name, seed, sh, lens, rounds, barrier) for sh in shares])
    t = max(secs)
    return {"value": sample_bytes * rounds / t / unit_scale, "unit": "GB/s", "cores": cores, "kind": "oracle",
            "sample": f"{len(seqs)} of {len(lens)} sequences (every 4th) dealt over {cores} processes, "
                      f"{rounds} rounds, float64 numpy, 1 BLAS thread each, slowest process {t:.1f} s"}


def workload_config(args, cfg, lens, P, world):
    """The ``config`` object of the JSON line: the same keys and values for the
    native arm and the reference arm of one workload."""
    return {"workload": WORKLOAD_NAMES[args.workload], "num_seqs": len(lens),
            "context_tokens": int(np.sum(lens)), "kv_bytes_per_step": kv_bytes(cfg, lens),
            "partition_size": P or 512, "decode_math": args.math, "split_merge": args.merge,
            "l2": "flushed between steps (256 MiB write, outside step events)",
            "parallelism": "replicas" if world > 1 else "single"}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    world = int(os.environ.get("WORLD_SIZE", "1"))
    cfg = wl.CONFIGS[args.workload]
    lens = wl.context_lengths(cfg, wl.rng(args.seed))
    seqs = list(range(0, len(lens), 4)) or [0]
    items = _oracle_sample(cfg, args.seed, seqs, lens)
    sample_bytes = kv_bytes(cfg, lens[seqs])
    with _single_thread():
        for _ in range(args.warmup):
            _time_oracle(cfg, items[:1])
        times = [_time_oracle(cfg, items) for _ in range(args.steps)]
    secs = sum(times) / len(times)
    value = sample_bytes / secs / 1e9
    full_ms = kv_bytes(cfg, lens) / (value * 1e9) * 1e3          # the whole batch at the sample's rate
    sample = (f"{len(seqs)} of {len(lens)} sequences (every 4th) per step, all {cfg.num_heads} query heads, "
              f"float64 numpy, 1 BLAS thread, {secs * 1e3:.1f} ms per sample step")
    P = args.partition_size or cfg.partition_size
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": full_ms, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": cfg.dtype, "data": "synthetic",
            "config": workload_config(args, cfg, lens, P, world),
            "tokens_per_s": len(lens) / (full_ms * 1e-3),
            "cpu_baseline": {"value": value, "unit": "GB/s", "cores": 1, "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line))
    return 0


# ---------------------------------------------------------------------------
# native arm
# ---------------------------------------------------------------------------

def max_over_ranks(values, device):
    """Each value's maximum over the ranks of the default process group (the
    values themselves without one): a multi-GPU time is the slowest rank's."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return [float(v) for v in values]
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t.cpu()]


def whole_job_gbs(world, bytes_per_rank, ms):
    """Whole-job throughput: every rank moved bytes_per_rank in the slowest
    rank's ms (replicas: weak scaling)."""
    return world * bytes_per_rank / (ms * 1e-3) / 1e9


def hbm_peak(dev):
    """HBM copy bandwidth to divide by: MEASURED_PEAKS.json when present, else
    measured here the same way (a device-to-device copy of 2 GiB, best of 10
    event-timed copies, read + written bytes)."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            return float(json.load(f)["hbm_gbs"]), "measured (MEASURED_PEAKS.json)"
    import torch
    n = 2 << 30
    a = torch.empty(n, dtype=torch.uint8, device=dev)
    b = torch.empty_like(a)
    a.fill_(1)
    best = float("inf")
    for i in range(13):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        b.copy_(a)
        e1.record()
        e1.synchronize()
        if i >= 3:
            best = min(best, e0.elapsed_time(e1))
    del a, b
    return 2 * n / (best * 1e-3) / 1e9, "measured in this run (2 GiB device copy, best of 10)"


def decode_case(pa, cfg, seed, dev, P, num_seqs=0, queries=1):
    """A full-size batch resident in HBM: pools filled, new rows held back."""
    import torch
    from paged_kv_cache_381_b200.batch import PagedBatch
    lens_override = wl.context_lengths(cfg, wl.rng(seed))[:num_seqs] if num_seqs else None
    d = wl.draw_device(cfg, seed, device=dev, context_lens=lens_override)
    batch = PagedBatch(d.k_hist, d.v_hist, d.offsets, d.context_lens, d.num_blocks, cfg.block_size, d.free_order,
                       new_tokens=queries)
    q = d.q
    if queries > 1:
        gq = torch.Generator(device=dev).manual_seed(seed * 7919 + queries)
        q = torch.randn((len(d.context_lens), queries, cfg.num_heads, cfg.head_dim), generator=gq, device=dev,
                        dtype=torch.float32).to(d.q.dtype)
    del d.k_hist, d.v_hist
    return batch, q, np.asarray(d.context_lens)


def time_steps(pa, step, steps, warmup, flush, kernel, profile_all=False, world=1):
    """Warm up, then time `steps` calls of step() each between two CUDA events
    on the current stream, L2 flushed between them outside the events; the
    library's own events time `kernel` (or every kernel) inside."""
    import torch
    import torch.distributed as dist
    for _ in range(max(warmup, 3)):
        step()
        flush.zero_()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    launches0 = pa.launch_count()
    pa.profile_begin(None if profile_all else [kernel])
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    wall0 = time.perf_counter()
    for i in range(steps):
        ev[i][0].record()
        step()
        ev[i][1].record()
        flush.zero_()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    wall = time.perf_counter() - wall0
    prof = pa.profile_end()
    step_ms = [a.elapsed_time(b) for a, b in ev]
    return {"step_ms": step_ms, "prof": prof, "launches": pa.launch_count() - launches0, "wall": wall}


def roofline(bytes_per_launch, ms, peak, peak_kind, kernel, traffic, ncu_dram_pct=None):
    achieved = bytes_per_launch / (ms * 1e-3) / 1e9
    return {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
            "traffic": traffic, "kernel": kernel, "algorithmic_bytes": int(bytes_per_launch), "peak_source": peak_kind,
            "spec_peak": SPEC_HBM_GBS, "spec_frac": achieved / SPEC_HBM_GBS,
            "ncu_dram_throughput_pct": ncu_dram_pct}


def sub_decode(pa, name, seed, dev, flush, peak, peak_kind, steps=100, warmup=5):
    """One more decode workload at full size: its step and decode-kernel roofline."""
    import torch
    cfg = wl.CONFIGS[name]
    P = cfg.partition_size
    batch, q, lens = decode_case(pa, cfg, seed, dev, P)
    out = torch.empty_like(q)
    batch.ensure_workspace(cfg.num_heads, P)
    r = time_steps(pa, lambda: batch.step(out, q, cfg.scale, partition_size=P), steps, warmup, flush, "decode")
    ms = statistics.mean(r["step_ms"])
    dec_ms = r["prof"]["decode"][0] / max(1, r["prof"]["decode"][1])
    step_kv = kv_bytes(cfg, lens)
    res = {"workload": WORKLOAD_NAMES[name], "dtype": cfg.dtype, "steps": steps, "ms_per_step": ms,
           "ms_per_step_median": statistics.median(r["step_ms"]), "value": step_kv / (ms * 1e-3) / 1e9,
           "unit": "GB/s", "pct_of_hbm_peak": step_kv / (ms * 1e-3) / 1e9 / peak, "kv_bytes_per_step": step_kv,
           "tokens_per_s": len(lens) / (ms * 1e-3), "kernel_ms": {"decode": dec_ms},
           "roofline": roofline(decode_kernel_bytes(cfg, lens, P), dec_ms, peak, peak_kind, "decode_kernel",
                                recorded_traffic("decode", name), recorded_dram_pct("decode", name))}
    del batch, q, out
    torch.cuda.empty_cache()
    return res


def sub_verify(pa, name, seed, dev, flush, peak, peak_kind, Q=6, steps=100, warmup=5, verify_kernel="auto"):
    """The verification pass of speculative decoding (Q candidate tokens per
    sequence) on a decode workload: step, kernel roofline and tensor work."""
    import torch
    cfg = wl.CONFIGS[name]
    batch, q, lens = decode_case(pa, cfg, seed, dev, 0, queries=Q)
    out = torch.empty_like(q)
    P = pa.pa_verify_partition_size(len(lens), Q, cfg.num_heads, cfg.num_kv_heads, batch.max_context_len,
                                    cfg.block_size, 0)
    batch.ensure_workspace(cfg.num_heads, 0)

    def step():
        batch.write_new_tokens()
        batch.verify(out, q, cfg.scale)
    r = time_steps(pa, step, steps, warmup, flush, "verify")
    ms = statistics.mean(r["step_ms"])
    k_ms = r["prof"]["verify"][0] / max(1, r["prof"]["verify"][1])
    kname = "verify_tc" if verify_kernel in ("auto", "tcgen05") else "verify"
    step_kv = kv_bytes(cfg, lens)
    tpeak, tkind = measured_tensor_peak()
    fl = verify_flops(cfg, lens, Q)
    res = {"workload": WORKLOAD_NAMES[name], "queries_per_seq": Q, "verify_kernel": verify_kernel,
           "partition_size": P, "steps": steps, "ms_per_step": ms, "ms_per_step_median": statistics.median(r["step_ms"]),
           "value": step_kv / (ms * 1e-3) / 1e9, "unit": "GB/s", "tokens_per_s": len(lens) * Q / (ms * 1e-3),
           "kernel_ms": {"verify": k_ms},
           "roofline": roofline(verify_kernel_bytes(cfg, lens, P, Q), k_ms, peak, peak_kind, f"{kname}_kernel",
                                recorded_traffic(kname, name, Q), recorded_dram_pct(kname, name, Q)),
           "tensor": {"flops_per_launch": fl, "achieved_tflops": fl / (k_ms * 1e-3) / 1e12, "peak_tflops": tpeak,
                      "frac": fl / (k_ms * 1e-3) / 1e12 / tpeak, "peak_source": tkind,
                      "note": "plain flops; P.V runs as two products (16-bit value + remainder) for bf16"}}
    del batch, q, out
    torch.cuda.empty_cache()
    return res


def sub_trace(dev, peak):
    """Per-step time of the continuous-batching trace (the serving loop): device
    work of each step and the host scheduler's time, separately."""
    import torch
    from paged_kv_cache_381_b200 import trace
    r = trace.run(wl.TRACE, seed=5, device=dev)
    d = np.asarray(r["device_ms"])
    h = np.asarray(r["host_ms"])
    tc = wl.TRACE
    res = {"workload": (f"continuous-batching trace: fp16, block 8, {tc.num_heads} q / {tc.num_kv_heads} kv heads, "
                        f"head_dim {tc.head_dim}, <= {tc.max_running} running, {tc.steps} steps, "
                        f"{tc.prefix_len}-token shared prefix for half the requests, prompts U[1, 512], "
                        "outputs geometric (mean 256), pool 75% of the unbounded peak"),
           "steps_timed": int(r["steps"]), "device_ms_median": float(np.median(d)), "device_ms_p90": float(np.percentile(d, 90)),
           "device_ms_mean": float(d.mean()), "host_sched_ms_median": float(np.median(h)),
           "host_sched_ms_p90": float(np.percentile(h, 90)),
           "kv_gbs": float(np.sum(r["kv_bytes"]) / (d.sum() * 1e-3) / 1e9),
           "pct_of_hbm_peak": float(np.sum(r["kv_bytes"]) / (d.sum() * 1e-3) / 1e9 / peak),
           "preemptions": int(r["preempted"]), "admissions": int(r["admitted"]), "num_blocks": int(r["num_blocks"]),
           "how": ("device: each step's metadata H2D (pinned), copy-on-write copies, prompt writes and "
                   "pa_write_decode between two events, L2 flushed between steps; host: pa_sched_step + "
                   "table packing through the Python binding")}
    torch.cuda.empty_cache()
    return res


def run_native(args):
    import torch
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        torch.cuda.set_device(local)
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120))
    dev = torch.device("cuda", local if world > 1 else 0)
    torch.cuda.set_device(dev)

    from paged_kv_cache_381_b200 import build
    if rank == 0:
        build.build()
    if world > 1:
        dist.barrier()
    import paged_kv_cache_381_b200 as pa
    pa.set_decode_math(pa.MATH_AUTO if args.math == "auto" else pa.MATH_SIMT)
    pa.set_split_merge(pa.MERGE_KERNEL if args.merge == "kernel" else pa.MERGE_FUSED)
    pa.set_verify_kernel({"auto": pa.VERIFY_AUTO, "tcgen05": pa.VERIFY_TCGEN05,
                          "mma_sync": pa.VERIFY_MMA_SYNC}[args.verify_kernel])
    peak, peak_kind = hbm_peak(dev)

    cfg = wl.CONFIGS[args.workload]
    seed = args.seed + rank                       # independent replica per rank
    Q = args.queries
    # decode: the workload's partition; verification: the one pa_verify picks
    # (partition_size 0) unless --partition-size names one
    P = args.partition_size or (0 if Q > 1 else cfg.partition_size)
    batch, q, lens = decode_case(pa, cfg, seed, dev, P, num_seqs=args.num_seqs, queries=Q)
    P_used = (pa.pa_verify_partition_size(len(lens), Q, cfg.num_heads, cfg.num_kv_heads, batch.max_context_len,
                                          cfg.block_size, P) if Q > 1 else P)
    out = torch.empty_like(q)
    batch.ensure_workspace(cfg.num_heads, P)
    step_kv = kv_bytes(cfg, lens)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    torch.cuda.synchronize()
    pa.pa_get_device_error()

    kernel = "verify" if Q > 1 else "decode"      # the library's launch-profile id
    if Q == 1:
        kname = "decode"
    elif args.verify_kernel in ("tcgen05", "auto"):
        kname = "verify_tc"       # the choice pa_verify makes for VERIFY_AUTO
    else:
        kname = "verify"

    def step():
        if Q > 1:
            batch.write_new_tokens()
            batch.verify(out, q, cfg.scale, partition_size=P)
        else:
            batch.step(out, q, cfg.scale, partition_size=P)      # pa_write_decode

    clocks = ClockSampler(dev.index)
    clocks.start()
    time.sleep(0.3)
    r = time_steps(pa, step, args.steps, args.warmup, flush, kernel, args.profile_all, world)
    clk = clocks.stop()
    err = pa.pa_get_device_error()
    prof = r["prof"]
    ms = sum(r["step_ms"]) / len(r["step_ms"])
    ms_median = statistics.median(r["step_ms"])
    dec_ms = prof[kernel][0] / max(1, prof[kernel][1])
    ms, dec_ms = max_over_ranks([ms, dec_ms], dev)

    # ---- e2e: the same step through the library's host-buffer calls
    e2e = None
    if not args.no_e2e and Q == 1:
        S, Hq, D = q.shape
        host = {"q": q.cpu().pin_memory(), "k": batch.k_new.cpu().pin_memory(), "v": batch.v_new.cpu().pin_memory(),
                "slot_mapping": batch.slot_mapping.cpu().pin_memory(),
                "block_tables": batch.block_tables.cpu().pin_memory(),
                "context_lens": batch.context_lens.cpu().pin_memory(),
                "out": torch.empty_like(q, device="cpu").pin_memory()}
        sets = []
        for _ in range(2):
            dset = {k: torch.empty_like(v, device=dev) for k, v in host.items()}
            dset["workspace"] = batch.workspace
            sets.append(dset)
        h2d = sum(host[k].numel() * host[k].element_size() for k in host if k != "out")
        d2h = host["out"].numel() * host["out"].element_size()
        # (1) like `value`: pa_step per step (copy in, compute, copy out on one
        # stream) between two events, L2 flushed between steps outside them
        er = time_steps(pa, lambda: pa.pa_step(host, sets[0], batch.k_cache, batch.v_cache, cfg.scale,
                                               batch.max_context_len, P),
                        args.steps, args.warmup, flush, "decode", False, world)
        ems = statistics.mean(er["step_ms"])
        (ems,) = max_over_ranks([ems], dev)
        # (2) a continuous serving loop without flushes (1.1 GB of K/V per step is
        # larger than L2): pa_pipeline overlaps step i's copies with its neighbours'
        # compute; the device-only step is timed over the same kind of loop
        pipe = pa.Pipeline(2)
        n = args.steps

        def pipe_run(k):
            pipe.begin(q)
            for i in range(k):
                pipe.step(i % 2, host, sets[i % 2], batch.k_cache, batch.v_cache, cfg.scale, batch.max_context_len, P)
            pipe.end(q)

        def loop_ms(fn):
            fn(3)
            torch.cuda.synchronize()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            fn(n)
            e1.record()
            torch.cuda.synchronize()
            return e0.elapsed_time(e1) / n

        def dev_run(k):
            for _ in range(k):
                step()
        pms, dcont = max_over_ranks([loop_ms(pipe_run), loop_ms(dev_run)], dev)
        e2e = {"value": whole_job_gbs(world, step_kv, ems), "unit": "GB/s", "h2d_bytes_per_step": int(h2d),
               "d2h_bytes_per_step": int(d2h), "ms_per_step": ems, "tokens_per_s": world * len(lens) / (ems * 1e-3),
               "copy_ms_per_step": ems - ms,
               "how": ("pa_step per step: H2D of q, k, v, slots, tables and lengths from pinned memory, the step, "
                       "D2H of out, on one stream between two events; L2 flushed between steps outside them, "
                       "as for value"),
               "pipelined": {"value": whole_job_gbs(world, step_kv, pms), "ms_per_step": pms,
                             "device_only_ms_per_step": dcont, "copy_ms_per_step": pms - dcont,
                             "how": ("continuous loop, no flush: pa_pipeline (two staging sets, copies on their "
                                     "own streams) against the device-only step over the same loop")}}

    dec_bytes = (verify_kernel_bytes(cfg, lens, pa.pa_verify_partition_size(len(lens), Q, cfg.num_heads,
                                                                           cfg.num_kv_heads, batch.max_context_len,
                                                                           cfg.block_size, P), Q)
                 if Q > 1 else decode_kernel_bytes(cfg, lens, P, fused=args.merge == "fused"))
    traffic = None if args.num_seqs else recorded_traffic(kname, args.workload, Q)
    dram_pct = None if args.num_seqs else recorded_dram_pct(kname, args.workload, Q)
    value = whole_job_gbs(world, step_kv, ms)
    result = {
        "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": max(args.warmup, 3), "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": cfg.dtype, "data": "synthetic",
        "config": workload_config(args, cfg, lens, P_used, world),
        "pct_of_hbm_peak": value / world / peak,
        "ms_per_step_median": ms_median,
        "pct_of_spec_peak": value / world / SPEC_HBM_GBS,
        "tokens_per_s": world * len(lens) / (ms * 1e-3),
        "kernel_ms": {k: v[0] / max(1, v[1]) for k, v in prof.items() if v[1]},
        "roofline": roofline(dec_bytes, dec_ms, peak, peak_kind, f"{kname}_kernel", traffic, dram_pct),
        "gpu_launches": int(r["launches"]), "device_error_flags": err, "wall_s": r["wall"],
        "e2e": e2e, "clocks": clk,
    }
    if Q > 1:
        tpeak, tkind = measured_tensor_peak()
        fl = verify_flops(cfg, lens, Q)
        result["metric"] = VERIFY_METRIC
        result["tokens_per_s"] = world * len(lens) * Q / (ms * 1e-3)
        result["config"]["queries_per_seq"] = Q
        result["config"]["verify_kernel"] = args.verify_kernel
        result["tensor"] = {"flops_per_launch": fl, "achieved_tflops": fl / (dec_ms * 1e-3) / 1e12,
                            "peak_tflops": tpeak, "frac": fl / (dec_ms * 1e-3) / 1e12 / tpeak,
                            "peak_source": tkind, "note": "plain flops; P.V runs as two mma (16-bit value + remainder)"}
    del batch, q, out
    torch.cuda.empty_cache()
    # the other configurations of the path, on the default run (one GPU)
    if world == 1 and Q == 1 and not args.no_extra and args.workload == "70b" and not args.num_seqs:
        result["workloads"] = {w: sub_decode(pa, w, args.seed, dev, flush, peak, peak_kind) for w in ("7b", "long")}
        result["trace"] = sub_trace(dev, peak)
        result["verify_q6"] = sub_verify(pa, "70b", args.seed, dev, flush, peak, peak_kind)
        result["device_error_flags"] |= pa.pa_get_device_error()
    if rank == 0 and world == 1 and not args.no_cpu_baseline and Q == 1:
        result["cpu_baseline"] = cpu_baseline(cfg, args.seed, lens, 1e9)
        try:        # a host without process spawning must not cost the run its line
            result["cpu_baseline_all_cores"] = cpu_baseline_all_cores(args.workload, args.seed, lens, 1e9,
                                                                      result["cpu_baseline"]["value"])
        except Exception as e:
            result["cpu_baseline_all_cores"] = {"unavailable": f"{type(e).__name__}: {e}"}
    if rank == 0:
        print(json.dumps(result))
    if world > 1:
        dist.destroy_process_group()
    return 0


def run_swap(args):
    """Host-link throughput of pa_swap_blocks: random (source, destination)
    block pairs of the 70B-shaped pool (16 tokens x 8 kv heads x 128 x bf16 =
    32 KiB per block and pool), device -> pinned host and back, against a
    single contiguous cudaMemcpyAsync of the same byte count (the copy engine
    over the same link) as the reference."""
    import torch
    from paged_kv_cache_381_b200 import build
    build.build()
    import paged_kv_cache_381_b200 as pa
    dev = torch.device("cuda", 0)
    blk = (16, 8, 128)
    block_bytes = 2 * 16 * 8 * 128 * 2                      # K and V
    n = max(1, (args.swap_mb << 20) // block_bytes)
    nb_dev, nb_host = 2 * n, 2 * n
    dk = torch.randn((nb_dev,) + blk, device=dev).to(torch.bfloat16)
    dv = torch.randn((nb_dev,) + blk, device=dev).to(torch.bfloat16)
    hk = torch.empty((nb_host,) + blk, dtype=torch.bfloat16).pin_memory()
    hv = torch.empty_like(hk).pin_memory()
    r = np.random.default_rng(args.seed)
    out_pairs = torch.from_numpy(np.stack([r.choice(nb_dev, n, replace=False),
                                           r.choice(nb_host, n, replace=False)], 1).astype(np.int32)).to(dev)
    in_pairs = torch.from_numpy(np.stack([out_pairs[:, 1].cpu().numpy(),
                                          r.choice(nb_dev, n, replace=False)], 1).astype(np.int32)).to(dev)
    flat_d = torch.empty(n * block_bytes, dtype=torch.uint8, device=dev)
    flat_h = torch.empty(n * block_bytes, dtype=torch.uint8).pin_memory()

    def timed(fn):
        for _ in range(3):
            fn()
        torch.cuda.synchronize()
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
        for a, b in ev:
            a.record()
            fn()
            b.record()
        torch.cuda.synchronize()
        return sorted(a.elapsed_time(b) for a, b in ev)[len(ev) // 2]

    steps = max(5, min(args.steps, 50))
    args.steps = steps
    t_out = timed(lambda: pa.pa_swap_blocks(hk, hv, dk, dv, out_pairs))
    t_in = timed(lambda: pa.pa_swap_blocks(dk, dv, hk, hv, in_pairs))
    t_d2h = timed(lambda: flat_h.copy_(flat_d, non_blocking=True))
    t_h2d = timed(lambda: flat_d.copy_(flat_h, non_blocking=True))
    err = pa.pa_get_device_error()
    gb = n * block_bytes / 1e9
    res = {"metric": "swap: GB/s of K/V blocks moved over the host link (pa_swap_blocks)", "unit": "GB/s",
           "value": gb / (t_out * 1e-3), "n_gpus": 1, "steps": steps, "higher_is_better": True,
           "blocks": int(n), "bytes_per_call": int(n * block_bytes),
           "swap_out": {"ms": t_out, "gbs": gb / (t_out * 1e-3), "copy_engine_gbs": gb / (t_d2h * 1e-3)},
           "swap_in": {"ms": t_in, "gbs": gb / (t_in * 1e-3), "copy_engine_gbs": gb / (t_h2d * 1e-3)},
           "reference": "one contiguous cudaMemcpyAsync of the same bytes (copy engine), median of the steps",
           "device_error_flags": err, "dtype": "bf16", "data": "synthetic"}
    print(json.dumps(res))
    return 0


def main():
    args = parse()
    if args.impl == "reference":
        return run_reference(args)
    if args.swap_mb > 0:
        return run_swap(args)
    return run_native(args)


if __name__ == "__main__":
    sys.exit(main())
