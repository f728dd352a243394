"""Benchmark of the paged decode hot path on B200.

One step = one decode step of one attention layer over a seeded synthetic
batch resident in HBM: ``copy_blocks`` for the batch's copy-on-write pairs
(none in the default workload), ``reshape_and_cache`` of every sequence's new
token, then ``paged_attention_decode`` (split-K attention kernel plus, when a
sequence spans several partitions, the log-sum-exp merge kernel).

Default workload: Llama-7B-shaped multi-head decode layer (64 sequences,
32 q = 32 kv heads, head_dim 128, 16-token blocks, fp16, context lengths
uniform on [128, 2048], pool = needed blocks + 10 %, shuffled).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME] [--kv-dtype auto|e4m3]

The same run also times a companion batch (default gqa_write, the GQA decode
+ cache-write batch) with the same step and protocol and reports it under
"companion" with its own clocks and roofline.  Beside the back-to-back timed
steps (inputs larger than L2), each batch's attention call is also timed
--flush-reps times with L2 flushed before every call (median, p10, p90).

Workloads prefill_llama7b, prefill_gqa_chunked and prefill_mixed time the
chunked-prefill path instead (cache write of the chunks + tcgen05 prefill attention; metric
TFLOP/s against the measured bf16 tensor peak).

Under torchrun every rank runs its own batch (weak scaling, seed + rank);
ranks share no data and the only collectives are the barrier and the max of
the timings.  Rank 0 prints one JSON line.
"""

from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

METRIC = "paged decode attention KV GB/s and tokens/s on 1 B200; % of HBM roofline"
PREFILL_METRIC = "paged prefill attention TFLOP/s (causal, algorithmic FLOPs) on 1 B200; % of tensor roofline"
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
NOMINAL_HBM_GBS = 8000.0       # HBM3e, 8 TB/s per GPU (the figure the roofline is also quoted against)
NOMINAL_BF16_TFLOPS = 2250.0   # dense bf16 / fp16 tensor rate per GPU
PROFILE_DIR = os.path.join(ROOT, "profiles")
KERNEL_SOURCES = ["paged_kv_cache_407_b200/csrc/pkv_host.cu",
                  "paged_kv_cache_407_b200/csrc/paged_attention.cu",
                  "paged_kv_cache_407_b200/csrc/decode_core.cuh",
                  "paged_kv_cache_407_b200/csrc/pkv_device.cuh"]
PREFILL_SOURCES = ["paged_kv_cache_407_b200/csrc/pkv_host.cu",
                   "paged_kv_cache_407_b200/csrc/paged_prefill.cu",
                   "paged_kv_cache_407_b200/csrc/tcgen05.cuh",
                   "paged_kv_cache_407_b200/csrc/pkv_device.cuh"]


def parse_args(argv=None):
    p = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=3000)
    p.add_argument("--warmup", type=int, default=20)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--workload", default="llama7b_mha")
    p.add_argument("--kv-dtype", choices=["auto", "e4m3"], default="auto",
                   help="auto: the workload's fp16/bf16 pools; e4m3: 8-bit pools (quantising write)")
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--cpu-seconds", type=float, default=12.0, help="target CPU time of the oracle sample")
    p.add_argument("--companion", default="gqa_write",
                   help="second decode batch timed in the same run and reported under its own key "
                        "(the other batch the ≥70%% HBM target names); 'none' to skip")
    p.add_argument("--flush-reps", type=int, default=100,
                   help="per-call timings with L2 flushed before each call (median, p10, p90)")
    return p.parse_args(argv)


def kernel_source_hash(sources=None) -> str:
    h = hashlib.sha256()
    for rel in sources or KERNEL_SOURCES:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def measured_peak(key: str = "hbm_gbs"):
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d[key]), "measured"
    except (OSError, KeyError, ValueError):
        return (FALLBACK_HBM_GBS if key == "hbm_gbs" else FALLBACK_BF16_TFLOPS), "fallback"


def profiled_traffic(workload: str, kv_dtype: str = "f16", kernel: str = "paged_decode_kernel"):
    """DRAM bytes per launch of the attention kernel from the committed ncu
    summary, if it was taken on the current kernel source; else None."""
    suffix = "_e4m3" if kv_dtype == "e4m3" else ""
    sources = PREFILL_SOURCES if kernel == "paged_prefill_kernel" else KERNEL_SOURCES
    path = os.path.join(PROFILE_DIR, f"{kernel}{suffix}_{workload}.txt")
    try:
        kv = {}
        with open(path, encoding="utf-8") as f:
            for line in f:
                if ":" in line and not line.startswith("#"):
                    k, v = line.split(":", 1)
                    kv[k.strip()] = (v.split() or [""])[0]
        if kv.get("kernel_source_sha256_16") != kernel_source_hash(sources):
            return None
        return float(kv["dram_bytes_per_launch_full_workload"])
    except (OSError, KeyError, ValueError):
        return None


# ---------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons while running."""

    FIELDS = ["timestamp", "uuid", "clocks.sm", "clocks.max.sm", "power.draw", "clocks_event_reasons.hw_slowdown",
              "clocks_event_reasons.hw_thermal_slowdown", "clocks_event_reasons.sw_thermal_slowdown",
              "clocks_event_reasons.sw_power_cap"]

    def __init__(self, uuid: str | None):
        self.uuid = uuid
        self.proc = None
        self.path = None
        self.window = None  # wall-clock (start, end) of the timed region

    def mark(self, start: float, end: float):
        self.window = (start, end)

    def __enter__(self):
        try:
            fd, self.path = tempfile.mkstemp(prefix="pkv_clocks_", suffix=".csv")
            self.fh = os.fdopen(fd, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={','.join(self.FIELDS)}", "--format=csv,noheader,nounits",
                 "-lms", "50"], stdout=self.fh, stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except (OSError, FileNotFoundError):
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.1)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.fh.close()
        return False

    def summary(self):
        if self.proc is None or self.path is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) != len(self.FIELDS):
                    continue
                if self.uuid and self.uuid not in parts[1]:
                    continue
                try:
                    ts = time.mktime(time.strptime(parts[0].split(".")[0], "%Y/%m/%d %H:%M:%S"))
                    ts += float("0." + parts[0].split(".")[1]) if "." in parts[0] else 0.0
                except (ValueError, IndexError):
                    ts = None
                rows.append((ts, parts))
        os.unlink(self.path)
        if self.window is not None:
            lo, hi = self.window
            inside = [r for ts, r in rows if ts is not None and lo - 0.06 <= ts <= hi + 0.06]
        else:
            inside = []
        used = inside if inside else [r for _, r in rows]
        if not used:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}

        def num(x):
            try:
                return float(x)
            except ValueError:
                return None

        sm = [v for v in (num(r[2]) for r in used) if v is not None]
        mx = [v for v in (num(r[3]) for r in used) if v is not None]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in used for i in range(4) if r[5 + i].lower().startswith("active")})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(used),
                "samples_in_timed_window": len(inside)}


# ----------------------------------------------------------------- helpers
def step_bytes(batch, kv_bytes=2):
    from paged_kv_cache_407_b200 import accounting as A

    att = A.decode_bytes(batch.context_lens, batch.num_q_heads, batch.num_kv_heads, batch.head_dim,
                         batch.block_size, kv_elem_bytes=kv_bytes)
    write = A.reshape_and_cache_bytes(batch.num_tokens, batch.num_kv_heads, batch.head_dim,
                                      cache_elem_bytes=kv_bytes)
    copy = A.copy_blocks_bytes(batch.cow_pairs.shape[0], batch.num_kv_heads, batch.block_size, batch.head_dim,
                               elem_bytes=kv_bytes)
    return att, write, copy


def split_partials_bytes(batch, partition_tokens: int) -> int:
    from paged_kv_cache_407_b200 import accounting as A

    return A.split_partials_bytes(batch.context_lens, batch.num_q_heads, batch.head_dim, partition_tokens)


def decode_accounting(batch, kv_bytes: int, ms_step: float) -> dict:
    """Side figures of a decode step beside the headline GB/s: internal
    fragmentation of the pool's used blocks, K/V bytes counted whole-block and
    per distinct physical block (a shared prefix once), and the rates those
    give, plus the cache write + attention rate."""
    from paged_kv_cache_407_b200 import accounting as A

    att, write, copy = step_bytes(batch, kv_bytes=kv_bytes)
    padded = A.decode_bytes_padded_kv(batch.context_lens, batch.num_kv_heads, batch.head_dim, batch.block_size,
                                      elem_bytes=kv_bytes)
    unique = A.unique_kv_bytes(batch.block_tables, batch.context_lens, batch.num_kv_heads, batch.head_dim,
                               batch.block_size, elem_bytes=kv_bytes)
    other = att["total"] - att["kv"]
    sec = ms_step * 1e-3
    return {
        "pool_fragmentation": round(A.block_fragmentation(batch.context_lens, batch.block_size), 5),
        "kv_bytes_logical": att["kv"],
        "kv_bytes_padded_to_blocks": padded,
        "kv_bytes_unique_blocks": unique,
        "unique_gbs": round((unique + other) / sec / 1e9, 2),
        "write_plus_attention_gbs": round((att["total"] + write) / sec / 1e9, 2),
    }


def blas_threads():
    try:
        from threadpoolctl import threadpool_info

        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:  # noqa: BLE001
        return 1


def host_cores() -> dict:
    """Cores of the host: all it has, and those this process may run on."""
    try:
        usable = len(os.sched_getaffinity(0))
    except (AttributeError, OSError):
        usable = os.cpu_count() or 1
    return {"cpu_count": os.cpu_count() or 1, "usable": usable}


def oracle_sample_rate(batch, seconds: float, f8=None, threads: int | None = None):
    """Time the oracle's decode over whole sequences of the batch (of its 8-bit
    variant ``f8`` when given) until about ``seconds`` of CPU work, with the
    BLAS limited to ``threads`` threads when given; returns (GB/s,
    description, threads used, seconds)."""
    import oracle as O
    from paged_kv_cache_407_b200 import accounting as A

    limit = None
    if threads is not None:
        from threadpoolctl import threadpool_limits

        limit = threadpool_limits(limits=threads)
    try:
        used = blas_threads()
        order = np.random.default_rng(12345).permutation(batch.num_seqs)
        done, t0 = [], time.perf_counter()
        while len(done) < len(order) and time.perf_counter() - t0 < seconds:
            s = int(order[len(done)])
            if f8 is None:
                O.decode_sequence(batch.q[s], batch.k_cache, batch.v_cache, batch.block_tables[s],
                                  int(batch.context_lens[s]), batch.block_size, batch.scale, batch.dtype)
            else:
                O.paged_attention_decode_fp8(batch.q, f8.k_cache, f8.v_cache, batch.block_tables,
                                             batch.context_lens, batch.block_size, batch.scale, f8.k_scale,
                                             f8.v_scale, batch.dtype, seqs=[s])
            done.append(s)
        dt = time.perf_counter() - t0
    finally:
        if limit is not None:
            limit.unregister()
    b = A.decode_bytes(batch.context_lens[done], batch.num_q_heads, batch.num_kv_heads, batch.head_dim,
                       batch.block_size, kv_elem_bytes=1 if f8 is not None else 2)["total"]
    desc = (f"oracle decode (fp64 NumPy) of {len(done)} of {batch.num_seqs} sequences of the "
            f"{batch.name} batch ({int(batch.context_lens[done].sum())} tokens), {dt:.1f} s")
    return b / dt / 1e9, desc, used, dt


def cpu_baseline_decode(batch, seconds: float, f8=None) -> dict:
    """The oracle on every core the BLAS uses, then on one core; both on a
    bounded sample of the batch (about ``seconds`` each)."""
    rate, desc, used, _ = oracle_sample_rate(batch, seconds, f8=f8)
    rate1, desc1, _, _ = oracle_sample_rate(batch, seconds, f8=f8, threads=1)
    return {"value": round(rate, 4), "unit": "GB/s", "cores": used, "kind": "oracle", "sample": desc,
            "blas_threads": used, **host_cores(),
            "one_core": {"value": round(rate1, 4), "cores": 1, "sample": desc1}}


def is_prefill(name: str) -> bool:
    import workloads as W

    return name in W.PREFILL_WORKLOADS


def build_prefill(name: str, rank: int):
    import workloads as W

    base = {"prefill_llama7b": 6, "prefill_gqa_chunked": 7, "prefill_mixed": 11}[name]
    return W.PREFILL_WORKLOADS[name](seed=base + 1000 * rank)


def oracle_prefill_rate(b, seconds: float):
    """Time the oracle's prefill on growing samples of one sequence's chunk
    (its last k tokens) until about ``seconds`` of CPU work; returns
    (TFLOP/s, description, cores, seconds)."""
    import oracle.prefill as PO
    import workloads as W
    from paged_kv_cache_407_b200 import accounting as A

    L = int(b.context_lens[0])
    k, spent, flop, done = 1, 0.0, 0.0, 0
    while spent < seconds and k <= int(b.chunk_lens[0]):
        sub = W.PrefillBatch(**{**b.__dict__, "q": b.q[b.query_start[1] - k: b.query_start[1]],
                                "context_lens": b.context_lens[:1], "block_tables": b.block_tables[:1],
                                "query_start": np.array([0, k], np.int32)})
        t0 = time.perf_counter()
        PO.paged_prefill(sub.q, b.k_cache, b.v_cache, sub.block_tables, sub.query_start, sub.context_lens,
                         b.block_size, b.scale, b.dtype)
        spent += time.perf_counter() - t0
        flop += A.prefill_flops([L], [k], b.num_q_heads, b.head_dim)
        done += k
        k *= 2
    desc = (f"oracle prefill (fp64 NumPy) of the last {done} query tokens (in growing slices) of sequence 0 "
            f"of the {b.name} batch (context {L}), {spent:.1f} s")
    return flop / spent / 1e12, desc, blas_threads(), spent


def build_workload(name: str, rank: int):
    import workloads as W

    fn = W.WORKLOADS[name]
    base = {"tiny": 1, "llama7b_mha": 2, "gqa_write": 3, "prefix_share": 4, "long_context": 5}[name]
    return fn(seed=base + 1000 * rank)


def workload_config(batch, args, n_gpus):
    lens = batch.context_lens
    return {
        "workload": batch.name,
        "num_seqs_per_gpu": batch.num_seqs,
        "global_batch": batch.num_seqs * n_gpus,
        "num_q_heads": batch.num_q_heads,
        "num_kv_heads": batch.num_kv_heads,
        "head_dim": batch.head_dim,
        "block_size": batch.block_size,
        "context_len_mean": float(lens.mean()),
        "context_len_max": int(lens.max()),
        "pool_blocks": batch.num_blocks,
        "pool_bytes": int(batch.k_cache.nbytes * 2),
        "new_tokens_per_step": batch.num_tokens,
        "cow_pairs_per_step": int(batch.cow_pairs.shape[0]),
        "parallelism": f"dp{n_gpus} (independent sequences per GPU)",
        "l2": "inputs larger than L2: the KV pool is re-read every step",
    }


def reduce_across_ranks(maxima, sums, device):
    """Max of the timings and sum of the byte/sequence counts over all ranks
    (identity on one process).  Every rank calls it once, in the same order."""
    import torch
    import torch.distributed as dist

    t_max = torch.tensor(list(maxima), dtype=torch.float64, device=device)
    t_sum = torch.tensor(list(sums), dtype=torch.float64, device=device)
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.all_reduce(t_max, op=dist.ReduceOp.MAX)
        dist.all_reduce(t_sum, op=dist.ReduceOp.SUM)
    return t_max.tolist(), t_sum.tolist()


# --------------------------------------------------------------- reference
def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0  # the reference arm runs on rank 0 only
    if is_prefill(args.workload):
        return run_reference_prefill(args)
    batch = build_workload(args.workload, 0)
    per_step = max(0.5, args.cpu_seconds / max(1, args.steps + args.warmup))
    for _ in range(args.warmup):
        oracle_sample_rate(batch, per_step)
    rates, secs = [], 0.0
    desc = ""
    cores = 1
    for _ in range(args.steps):
        r, desc, cores, dt = oracle_sample_rate(batch, per_step)
        rates.append(r)
        secs += dt
    value = float(statistics.median(rates))
    att, _, _ = step_bytes(batch)
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": "GB/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(secs / args.steps * 1e3, 3), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded)",
        "config": workload_config(batch, args, 1),
        "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": cores, "kind": "oracle",
                         "sample": desc + "; each step a bounded sample of this workload",
                         "blas_threads": cores, **host_cores()},
        "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "decode_tokens_per_s": round(value * 1e9 / att["total"] * batch.num_seqs, 2),
    }
    print(json.dumps(line), flush=True)
    return 0


def prefill_config(b, n_gpus):
    return {
        "workload": b.name, "num_seqs_per_gpu": b.num_seqs, "global_batch": b.num_seqs * n_gpus,
        "num_q_heads": b.num_q_heads, "num_kv_heads": b.num_kv_heads, "head_dim": b.head_dim,
        "block_size": b.block_size, "context_len_max": b.max_context_len,
        "chunk_tokens_per_seq": int(b.max_query_len), "query_tokens_per_step": b.num_tokens,
        "pool_blocks": int(b.k_cache.shape[0]), "pool_bytes": int(b.k_cache.nbytes * 2),
        "parallelism": f"dp{n_gpus} (independent sequences per GPU)",
        "l2": "compute-bound; K/V of a sequence are re-read from L2 by its query tiles",
    }


def run_reference_prefill(args):
    b = build_prefill(args.workload, 0)
    per_step = max(0.5, args.cpu_seconds / max(1, args.steps + args.warmup))
    for _ in range(args.warmup):
        oracle_prefill_rate(b, per_step)
    rates, secs, desc, cores = [], 0.0, "", 1
    for _ in range(args.steps):
        r, desc, cores, dt = oracle_prefill_rate(b, per_step)
        rates.append(r)
        secs += dt
    value = float(statistics.median(rates))
    line = {
        "impl": "reference", "metric": PREFILL_METRIC, "value": round(value, 6), "unit": "TFLOP/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(secs / args.steps * 1e3, 3), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded)", "config": prefill_config(b, 1),
        "cpu_baseline": {"value": round(value, 6), "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                         "sample": desc + "; each step a bounded sample of this workload",
                         "blas_threads": cores, **host_cores()},
        "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def run_prefill(args):
    """Chunked prefill step: write the chunks' K/V (reshape_and_cache), then
    paged_prefill; the metric is causal attention FLOPs per second."""
    import torch
    import torch.distributed as dist

    import paged_kv_cache_407_b200 as pkv
    from paged_kv_cache_407_b200 import accounting as A
    from paged_kv_cache_407_b200.build import build
    from workloads.device import upload_prefill

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        torch.cuda.set_device(local)
        from datetime import timedelta

        dist.init_process_group("nccl", timeout=timedelta(seconds=300), device_id=torch.device("cuda", local))
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    if rank == 0:
        build()
    if world > 1:
        dist.barrier()
    pkv.library()
    b = build_prefill(args.workload, rank)
    db = upload_prefill(b, dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    stream = torch.cuda.current_stream(dev)
    from paged_kv_cache_407_b200 import binding as bd
    prefill_ws = torch.empty(bd.PREFILL_WORKSPACE_BYTES, dtype=torch.uint8, device=dev)  # the item counter

    def step(q=db.q, out=db.out, key=db.key, value=db.value, slots=db.slot_mapping, tables=db.block_tables,
             qs=db.query_start, lens=db.context_lens, ev=None):
        pkv.reshape_and_cache(key, value, db.k_cache, db.v_cache, slots, d_status=status, stream=stream)
        if ev is not None:
            ev[0].record(stream)
        pkv.paged_prefill(out, q, db.k_cache, db.v_cache, tables, qs, lens, b.max_query_len, b.scale,
                          d_status=status, stream=stream, workspace=prefill_ws)
        if ev is not None:
            ev[1].record(stream)

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize(dev)
    if int(status.item()) != 0:
        raise RuntimeError(f"device status {int(status.item())} during warm-up")
    uuid = None
    try:
        uuid = str(torch.cuda.get_device_properties(dev).uuid)
    except Exception:  # noqa: BLE001
        pass
    K = args.steps
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(uuid) as clocks:
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize(dev)
        wall0 = time.time()
        t0.record(stream)
        for i in range(K):
            step(ev=evs[i])
        t1.record(stream)
        torch.cuda.synchronize(dev)
        clocks.mark(wall0, time.time())
        if world > 1:
            dist.barrier()
    ms_total = t0.elapsed_time(t1)
    pre_ms = float(np.mean([x.elapsed_time(y) for x, y in evs]))
    clock = clocks.summary()

    e2e = None
    if not args.no_e2e:  # inputs from pinned host memory, output back, every step
        names = ("q", "key", "value", "slots", "tables", "qs", "lens")
        srcs = (db.q, db.key, db.value, db.slot_mapping, db.block_tables, db.query_start, db.context_lens)
        h_in = {n: t.detach().cpu().pin_memory() for n, t in zip(names, srcs)}
        d_in = {n: torch.empty_like(t, device=dev) for n, t in h_in.items()}
        h_out = torch.empty(db.out.shape, dtype=db.out.dtype).pin_memory()
        h2d = sum(t.numel() * t.element_size() for t in h_in.values())
        d2h = h_out.numel() * h_out.element_size()

        def e2e_step():
            for n in names:
                d_in[n].copy_(h_in[n], non_blocking=True)
            step(q=d_in["q"], out=db.out, key=d_in["key"], value=d_in["value"], slots=d_in["slots"],
                 tables=d_in["tables"], qs=d_in["qs"], lens=d_in["lens"])
            h_out.copy_(db.out, non_blocking=True)

        for _ in range(max(3, args.warmup)):
            e2e_step()
        torch.cuda.synchronize(dev)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        if world > 1:
            dist.barrier()
        e0.record(stream)
        for _ in range(K):
            e2e_step()
        e1.record(stream)
        torch.cuda.synchronize(dev)
        e2e = {"ms": e0.elapsed_time(e1), "h2d": h2d, "d2h": d2h}
    if int(status.item()) != 0:
        raise RuntimeError(f"device status {int(status.item())} in the timed region")

    flop = A.prefill_flops(b.context_lens, b.chunk_lens, b.num_q_heads, b.head_dim)
    (ms_total, pre_max, e2e_ms), (flop_all,) = reduce_across_ranks(
        [ms_total, pre_ms, e2e["ms"] if e2e else 0.0], [flop], dev)
    ms_step = ms_total / K
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        rate, desc, cores, _ = oracle_prefill_rate(b, args.cpu_seconds)
        cpu = {"value": round(rate, 6), "unit": "TFLOP/s", "cores": cores, "kind": "oracle", "sample": desc,
               "blas_threads": cores, **host_cores()}
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return 0
    peak, peak_kind = measured_peak("bf16_tflops")
    achieved = flop / (pre_max * 1e-3) / 1e12
    line = {
        "metric": PREFILL_METRIC,
        "value": round(flop_all / (ms_step * 1e-3) / 1e12, 2),
        "unit": "TFLOP/s",
        "n_gpus": world, "steps": K, "warmup": args.warmup, "ms_per_step": round(ms_step, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": b.dtype,
        "data": "synthetic (seeded generator, inputs resident in HBM)",
        "config": prefill_config(b, world),
        "prefill_tokens_per_s": round(b.num_tokens * world / (ms_step * 1e-3), 1),
        "prefill_ms_per_call": round(pre_max, 5),
        "flop_per_step": flop,
        "bytes_per_step_min": A.prefill_bytes(b.context_lens, b.chunk_lens, b.num_q_heads, b.num_kv_heads,
                                              b.head_dim),
        "roofline": {
            "bound": "tensor",
            "kernel": "paged_prefill (tcgen05, 128x128 tiles)",
            "achieved": round(achieved, 1), "peak": peak,
            "peak_source": (f"{peak_kind} (MEASURED_PEAKS.json bf16_tflops; fp16 has the same nominal rate)"
                            if peak_kind == "measured" else "fallback"),
            "unit": "TFLOP/s", "frac": round(achieved / peak, 4),
            "traffic": profiled_traffic(b.name, kernel="paged_prefill_kernel"),
            "nominal": NOMINAL_BF16_TFLOPS,
            "frac_of_nominal": round(achieved / NOMINAL_BF16_TFLOPS, 4),
        },
        "clocks": clock,
        "gpu_launches": 2 * K,
    }
    if e2e:
        line["e2e"] = {"value": round(flop_all / (e2e_ms / K * 1e-3) / 1e12, 2), "unit": "TFLOP/s",
                       "h2d_bytes_per_step": e2e["h2d"], "d2h_bytes_per_step": e2e["d2h"],
                       "ms_per_step": round(e2e_ms / K, 5)}
    if cpu:
        line["cpu_baseline"] = cpu
    print(json.dumps(line), flush=True)
    return 0


# --------------------------------------------------------------------- ours
L2_FLUSH_BYTES = 256 * 1024 * 1024  # twice the 126 MB L2


class DecodeRunner:
    """One decode batch resident on the device, and the step the benchmark
    times: copy-on-write pairs (if any), the cache write of the step's new
    tokens, then decode attention (+ merge)."""

    def __init__(self, batch, e4m3: bool, rank: int, dev, status, stream):
        import torch

        import paged_kv_cache_407_b200 as pkv
        from workloads.device import upload

        self.batch, self.e4m3, self.dev, self.status, self.stream = batch, e4m3, dev, status, stream
        self.f8 = None
        if e4m3:
            import workloads as W
            from workloads.device import upload_fp8

            self.f8 = W.fp8_variant(batch, 777 + rank)
            self.db = upload_fp8(self.f8, dev)
        else:
            self.db = upload(batch, dev)
        self.ws_bytes = pkv.workspace_size(batch.num_seqs, batch.num_q_heads, batch.num_kv_heads, batch.head_dim,
                                           batch.block_size, batch.max_context_len, batch.partition_size)
        self.workspace = torch.empty(max(self.ws_bytes, 16), dtype=torch.uint8, device=dev)
        self.P = pkv.partition_size(batch.num_seqs, batch.num_kv_heads, batch.block_size, batch.max_context_len,
                                    batch.partition_size)
        self.split = batch.max_context_len > self.P
        nb_max = -(-batch.max_context_len // batch.block_size)
        self.max_parts = -(-nb_max // (self.P // batch.block_size))
        self.has_cow = batch.cow_pairs.shape[0] > 0
        # cache write + attention kernel (+ plan kernel for 3..32 partitions)
        # (+ merge kernel for more than 32) (+ block copy)
        self.attention_launches = 1 + (1 if 3 <= self.max_parts <= 32 else 0) + (1 if self.max_parts > 32 else 0)
        self.launches_per_step = 1 + self.attention_launches + (1 if self.has_cow else 0)
        self._calls, self._att = self.prepare()

    def prepare(self, q=None, out=None, key=None, value=None, slots=None, tables=None, lens=None):
        """The step's library calls on these buffers (default: the batch's
        own), each prepared once through the public API: (calls of the whole
        step, the attention call).  A serving loop that reuses its buffers
        calls the library this way."""
        import paged_kv_cache_407_b200 as pkv

        db, b = self.db, self.batch
        q = db.q if q is None else q
        out = db.out if out is None else out
        key = db.key if key is None else key
        value = db.value if value is None else value
        slots = db.slot_mapping if slots is None else slots
        tables = db.block_tables if tables is None else tables
        lens = db.context_lens if lens is None else lens
        kw = dict(d_status=self.status, stream=self.stream, prepare=True)
        calls = []
        if self.has_cow:
            calls.append(pkv.copy_blocks(db.k_cache, db.v_cache, db.cow_pairs, **kw))
        if self.e4m3:
            calls.append(pkv.reshape_and_cache_fp8(key, value, db.k_cache, db.v_cache, slots, self.f8.k_scale,
                                                   self.f8.v_scale, **kw))
            att = pkv.paged_attention_decode_fp8(out, q, db.k_cache, db.v_cache, tables, lens, b.max_context_len,
                                                 b.scale, self.f8.k_scale, self.f8.v_scale,
                                                 partition_size=b.partition_size, workspace=self.workspace, **kw)
        else:
            calls.append(pkv.reshape_and_cache(key, value, db.k_cache, db.v_cache, slots, **kw))
            att = pkv.paged_attention_decode(out, q, db.k_cache, db.v_cache, tables, lens, b.max_context_len,
                                             b.scale, partition_size=b.partition_size, workspace=self.workspace,
                                             **kw)
        calls.append(att)
        return tuple(calls), att

    def attention(self):
        self._att()

    def step(self):
        for c in self._calls:
            c()

    def check_status(self, where):
        if int(self.status.item()) != 0:
            raise RuntimeError(f"device status {int(self.status.item())} {where}")

    # ------------------------------------------------------------ timings
    def timed_steps(self, K: int, warmup: int, world: int, uuid):
        """Two timed regions, each bracketed by a barrier and a synchronize,
        with clocks sampled by nvidia-smi over both: K back-to-back steps
        (inputs larger than L2), then K back-to-back attention calls alone.
        Only the regions' ends carry CUDA events: an event recorded between
        two kernels would stop the second from launching while the first
        finishes (programmatic dependent launch), so per-call events would
        time the launch gap too.  Returns (ms of the K steps, ms per
        attention call, clocks)."""
        import torch
        import torch.distributed as dist

        for _ in range(max(3, warmup)):
            self.step()
        torch.cuda.synchronize(self.dev)
        self.check_status("during warm-up")
        t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a_start, a_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with ClockSampler(uuid) as clocks:
            if world > 1:
                dist.barrier()
            torch.cuda.synchronize(self.dev)
            wall0 = time.time()
            t_start.record(self.stream)
            for _ in range(K):
                self.step()
            t_end.record(self.stream)
            torch.cuda.synchronize(self.dev)
            if world > 1:
                dist.barrier()
            a_start.record(self.stream)
            for _ in range(K):
                self.attention()
            a_end.record(self.stream)
            torch.cuda.synchronize(self.dev)
            clocks.mark(wall0, time.time())
            if world > 1:
                dist.barrier()
        self.check_status("in the timed regions")
        return t_start.elapsed_time(t_end), a_start.elapsed_time(a_end) / K, clocks.summary()

    def graph_steps(self, K: int) -> dict:
        """The same step captured once in a CUDA graph and replayed K times
        back to back between two events: the launch cost a serving loop saves
        on small steps.  The capture issues plain library calls (they run on
        the current stream, which inside the capture is the capturing one)."""
        import torch

        import paged_kv_cache_407_b200 as pkv

        db, b = self.db, self.batch
        kw = dict(d_status=self.status)

        def step():
            if self.has_cow:
                pkv.copy_blocks(db.k_cache, db.v_cache, db.cow_pairs, **kw)
            if self.e4m3:
                pkv.reshape_and_cache_fp8(db.key, db.value, db.k_cache, db.v_cache, db.slot_mapping,
                                          self.f8.k_scale, self.f8.v_scale, **kw)
                pkv.paged_attention_decode_fp8(db.out, db.q, db.k_cache, db.v_cache, db.block_tables,
                                               db.context_lens, b.max_context_len, b.scale, self.f8.k_scale,
                                               self.f8.v_scale, partition_size=b.partition_size,
                                               workspace=self.workspace, **kw)
            else:
                pkv.reshape_and_cache(db.key, db.value, db.k_cache, db.v_cache, db.slot_mapping, **kw)
                pkv.paged_attention_decode(db.out, db.q, db.k_cache, db.v_cache, db.block_tables, db.context_lens,
                                           b.max_context_len, b.scale, partition_size=b.partition_size,
                                           workspace=self.workspace, **kw)

        torch.cuda.synchronize(self.dev)
        graph = torch.cuda.CUDAGraph()
        try:
            # thread-local capture: other threads' CUDA calls (NCCL's
            # watchdog under torchrun) do not break it
            with torch.cuda.graph(graph, capture_error_mode="thread_local"):
                step()
        except RuntimeError as e:
            torch.cuda.synchronize(self.dev)
            return {"unavailable": f"capture failed: {str(e).splitlines()[0][:160]}"}
        for _ in range(3):
            graph.replay()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize(self.dev)
        e0.record()
        for _ in range(K):
            graph.replay()
        e1.record()
        torch.cuda.synchronize(self.dev)
        self.check_status("in the graph replays")
        del graph
        return {"ms_per_step": round(e0.elapsed_time(e1) / K, 5), "steps": K,
                "kernels_per_step": self.launches_per_step,
                "how": "the step captured once in a CUDA graph (torch.cuda.CUDAGraph), replayed back to back"}

    def flushed_calls(self, reps: int) -> dict:
        """Per-call attention time with L2 flushed before every call (a write
        of 256 MB between calls, outside the events): median, p10, p90."""
        import torch

        if reps <= 0:
            return None
        flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=self.dev)
        clean = torch.zeros(L2_FLUSH_BYTES // 4, dtype=torch.int32, device=self.dev)
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(reps)]
        for i in range(reps + 3):
            # write 256 MB (evicts the inputs), then read another 256 MB so that
            # the dirty lines are written back before the call, not during it
            flush.fill_(i & 0xFF)
            torch.amax(clean)
            if i >= 3:
                evs[i - 3][0].record(self.stream)
            self.attention()
            if i >= 3:
                evs[i - 3][1].record(self.stream)
        torch.cuda.synchronize(self.dev)
        self.check_status("in the L2-flushed calls")
        ms = np.array([a.elapsed_time(b) for a, b in evs])
        del flush, clean
        return {"reps": reps, "l2_flushed": "256 MB written, then 256 MB read, before every call",
                "median_ms": round(float(np.median(ms)), 5),
                "p10_ms": round(float(np.percentile(ms, 10)), 5), "p90_ms": round(float(np.percentile(ms, 90)), 5),
                "mean_ms": round(float(ms.mean()), 5)}

    def host_submit_us(self, calls: int = 400) -> dict:
        """Host time per decode call: the Python binding (argument checks,
        marshalling, the C call), the binding's prepared call (checks and
        marshalling done once; what the timed steps use) and the bare C-ABI
        call; CPU wall clock around the calls, no synchronisation inside (the
        GPU drains them afterwards)."""
        import ctypes

        import torch

        import paged_kv_cache_407_b200 as pkv
        from paged_kv_cache_407_b200 import binding as bd

        db, b = self.db, self.batch
        torch.cuda.synchronize(self.dev)
        t0 = time.perf_counter()
        for _ in range(calls):
            if self.e4m3:
                pkv.paged_attention_decode_fp8(db.out, db.q, db.k_cache, db.v_cache, db.block_tables,
                                               db.context_lens, b.max_context_len, b.scale, self.f8.k_scale,
                                               self.f8.v_scale, partition_size=b.partition_size,
                                               workspace=self.workspace, d_status=self.status,
                                               stream=self.stream)
            else:
                pkv.paged_attention_decode(db.out, db.q, db.k_cache, db.v_cache, db.block_tables, db.context_lens,
                                           b.max_context_len, b.scale, partition_size=b.partition_size,
                                           workspace=self.workspace, d_status=self.status, stream=self.stream)
        t_binding = (time.perf_counter() - t0) / calls * 1e6
        torch.cuda.synchronize(self.dev)
        t0 = time.perf_counter()
        for _ in range(calls):
            self._att()
        t_prepared = (time.perf_counter() - t0) / calls * 1e6
        torch.cuda.synchronize(self.dev)
        lib = pkv.library()
        stream = ctypes.c_void_p(self.stream.cuda_stream)
        ptr = lambda t: ctypes.c_void_p(t.data_ptr())  # noqa: E731
        ws = ctypes.c_size_t(self.workspace.numel())
        if self.e4m3:
            desc = bd.fp8_cache_desc(db.k_cache, db.v_cache)
            fn = lib.pkv_paged_attention_decode_fp8
            argv = (ptr(db.out), ptr(db.q), bd._DTYPES[db.q.dtype], ptr(db.k_cache), ptr(db.v_cache), desc,
                    ptr(db.block_tables), db.block_tables.shape[1], ptr(db.context_lens), b.num_seqs,
                    b.num_q_heads, b.max_context_len, ctypes.c_float(b.scale), ctypes.c_float(self.f8.k_scale),
                    ctypes.c_float(self.f8.v_scale), b.partition_size, ptr(self.workspace), ws, ptr(self.status),
                    stream)
        else:
            desc = bd.cache_desc(db.k_cache)
            fn = lib.pkv_paged_attention_decode
            argv = (ptr(db.out), ptr(db.q), ptr(db.k_cache), ptr(db.v_cache), desc, ptr(db.block_tables),
                    db.block_tables.shape[1], ptr(db.context_lens), b.num_seqs, b.num_q_heads, b.max_context_len,
                    ctypes.c_float(b.scale), b.partition_size, ptr(self.workspace), ws, ptr(self.status), stream)
        t0 = time.perf_counter()
        for _ in range(calls):
            if fn(*argv) != 0:
                raise RuntimeError("decode call failed while timing the host submit")
        t_cabi = (time.perf_counter() - t0) / calls * 1e6
        torch.cuda.synchronize(self.dev)
        self.check_status("while timing the host submit")
        return {"binding": round(t_binding, 2), "binding_prepared": round(t_prepared, 2),
                "c_abi": round(t_cabi, 2), "calls": calls}

    def e2e(self, K: int, warmup: int, world: int) -> dict:
        """End to end through the public API from host buffers.  Every step
        copies its inputs from pinned host memory to the device and its output
        back.  As a serving loop would, the copies run on their own streams
        with double-buffered device tensors, so step i's upload and step
        i-1's read-back overlap step i-1's and step i's compute; every copy
        is inside the timed region."""
        import torch
        import torch.distributed as dist

        db, dev, stream = self.db, self.dev, self.stream
        names = ("q", "key", "value", "slots", "tables", "lens")
        srcs = (db.q, db.key, db.value, db.slot_mapping, db.block_tables, db.context_lens)
        h_in = {n: t.detach().cpu().pin_memory() for n, t in zip(names, srcs)}
        d_in = [{n: torch.empty_like(t, device=dev) for n, t in h_in.items()} for _ in range(2)]
        d_out = [torch.empty_like(db.out) for _ in range(2)]
        h_out = [torch.empty(db.out.shape, dtype=db.out.dtype).pin_memory() for _ in range(2)]
        h2d = sum(t.numel() * t.element_size() for t in h_in.values())
        d2h = h_out[0].numel() * h_out[0].element_size()
        up, down = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        ev_in = [torch.cuda.Event() for _ in range(2)]
        ev_done = [torch.cuda.Event() for _ in range(2)]
        ev_out = [torch.cuda.Event() for _ in range(2)]

        steps = [self.prepare(q=d_in[b]["q"], out=d_out[b], key=d_in[b]["key"], value=d_in[b]["value"],
                              slots=d_in[b]["slots"], tables=d_in[b]["tables"], lens=d_in[b]["lens"])[0]
                 for b in range(2)]

        def e2e_step(i):
            b = i % 2
            up.wait_event(ev_done[b])  # step i-2 has consumed input buffer b
            with torch.cuda.stream(up):
                for n in names:
                    d_in[b][n].copy_(h_in[n], non_blocking=True)
                ev_in[b].record(up)
            stream.wait_event(ev_in[b])
            stream.wait_event(ev_out[b])  # step i-2's output has been read back
            for c in steps[b]:
                c()
            ev_done[b].record(stream)
            down.wait_event(ev_done[b])
            with torch.cuda.stream(down):
                h_out[b].copy_(d_out[b], non_blocking=True)
                ev_out[b].record(down)

        for i in range(max(3, warmup)):
            e2e_step(i)
        torch.cuda.synchronize(dev)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize(dev)
        e0.record(stream)
        up.wait_event(e0)
        for i in range(K):
            e2e_step(i)
        stream.wait_stream(down)
        e1.record(stream)
        torch.cuda.synchronize(dev)
        if not torch.equal(h_out[(K - 1) % 2].view(torch.int16), db.out.view(torch.int16).cpu()):
            raise RuntimeError("end-to-end output differs from the device-resident run")
        self.check_status("in the end-to-end run")
        # the same copies with no kernel between them: the host link's share
        c0, c1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        c0.record(stream)
        up.wait_event(c0)
        down.wait_event(c0)
        for i in range(K):
            b = i % 2
            with torch.cuda.stream(up):
                for n in names:
                    d_in[b][n].copy_(h_in[n], non_blocking=True)
            with torch.cuda.stream(down):
                h_out[b].copy_(d_out[b], non_blocking=True)
        stream.wait_stream(up)
        stream.wait_stream(down)
        c1.record(stream)
        torch.cuda.synchronize(dev)
        return {"ms": e0.elapsed_time(e1), "h2d": h2d, "d2h": d2h, "copies_ms": c0.elapsed_time(c1)}


def read_stream_gbs(dev, nbytes: int = 2 << 30, reps: int = 10) -> float:
    """Context for the roofline: the rate of a plain read-only stream (a
    torch max-reduction over a 2 GiB buffer, one read per byte), beside the
    copy rate the roofline uses as its peak."""
    import torch

    buf = torch.zeros(nbytes // 4, dtype=torch.int32, device=dev)
    for _ in range(3):
        torch.amax(buf)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize(dev)
    e0.record()
    for _ in range(reps):
        torch.amax(buf)
    e1.record()
    torch.cuda.synchronize(dev)
    ms = e0.elapsed_time(e1) / reps
    del buf
    return nbytes / (ms * 1e-3) / 1e9


def decode_roofline(att_bytes_total: float, att_ms: float, e4m3: bool, workload: str) -> dict:
    peak, peak_kind = measured_peak()
    achieved = att_bytes_total / (att_ms * 1e-3) / 1e9
    return {
        "bound": "hbm",
        "kernel": "paged_attention_decode (planning + attention + merge kernels of one call; calls back to back)",
        "achieved": round(achieved, 1),
        "peak": peak,
        "peak_source": f"{peak_kind} (MEASURED_PEAKS.json hbm_gbs)" if peak_kind == "measured" else "fallback",
        "unit": "GB/s",
        "frac": round(achieved / peak, 4),
        "traffic": profiled_traffic(workload, "e4m3" if e4m3 else "f16"),
        "nominal": NOMINAL_HBM_GBS,
        "frac_of_nominal": round(achieved / NOMINAL_HBM_GBS, 4),
    }


def run_ours(args):
    import torch
    import torch.distributed as dist

    import paged_kv_cache_407_b200 as pkv
    from paged_kv_cache_407_b200.build import build

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        torch.cuda.set_device(local)
        from datetime import timedelta

        dist.init_process_group("nccl", timeout=timedelta(seconds=300), device_id=torch.device("cuda", local))
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    if rank == 0:
        build()
    if world > 1:
        dist.barrier()
    pkv.library()

    uuid = None
    try:
        uuid = str(torch.cuda.get_device_properties(dev).uuid)
    except Exception:  # noqa: BLE001
        pass
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    stream = torch.cuda.current_stream(dev)
    e4m3 = args.kv_dtype == "e4m3"
    K = args.steps

    batch = build_workload(args.workload, rank)
    run = DecodeRunner(batch, e4m3, rank, dev, status, stream)
    ms_total, att_ms, clock = run.timed_steps(K, args.warmup, world, uuid)
    flushed = run.flushed_calls(args.flush_reps)
    graph = run.graph_steps(K)
    host_us = run.host_submit_us()
    read_gbs = read_stream_gbs(dev)
    e2e = None if args.no_e2e else run.e2e(K, args.warmup, world)

    att_bytes, write_bytes, copy_bytes = step_bytes(batch, kv_bytes=1 if e4m3 else 2)
    (ms_total, att_ms_max, e2e_ms), (bytes_all, seqs_all) = reduce_across_ranks(
        [ms_total, att_ms, e2e["ms"] if e2e else 0.0], [att_bytes["total"], batch.num_seqs], dev)
    ms_step = ms_total / K

    # the companion batch: same step, same protocol, its own clocks and roofline
    companion = None
    if args.companion not in ("none", "", args.workload):
        cb = build_workload(args.companion, rank)
        crun = DecodeRunner(cb, e4m3, rank, dev, status, stream)
        c_total, c_att, c_clock = crun.timed_steps(K, args.warmup, world, uuid)
        c_flushed = crun.flushed_calls(args.flush_reps)
        c_att_bytes, c_write, _ = step_bytes(cb, kv_bytes=1 if e4m3 else 2)
        (c_total, c_att_max), (c_bytes_all, c_seqs_all) = reduce_across_ranks(
            [c_total, c_att], [c_att_bytes["total"], cb.num_seqs], dev)
        c_step = c_total / K
        companion = {
            "workload": cb.name,
            "value": round(c_bytes_all / (c_step * 1e-3) / 1e9, 2), "unit": "GB/s",
            "ms_per_step": round(c_step, 5),
            "decode_tokens_per_s": round(c_seqs_all / (c_step * 1e-3), 1),
            "attention_ms_per_call": round(c_att_max, 5),
            "bytes_per_step": {"attention": c_att_bytes["total"], "cache_write": c_write},
            "config": workload_config(cb, args, world),
            "split_k": {"partition_tokens": crun.P, "split": bool(crun.split), "workspace_bytes": crun.ws_bytes},
            "roofline": decode_roofline(c_att_bytes["total"], c_att_max, e4m3, cb.name),
            "per_call_l2_flushed": c_flushed,
            "clocks": c_clock,
            "gpu_launches": crun.launches_per_step * K,
            "gpu_launches_attention_region": crun.attention_launches * K,
        }
        del crun

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline_decode(batch, args.cpu_seconds, f8=run.f8)

    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return 0

    value = bytes_all / (ms_step * 1e-3) / 1e9  # every rank's own batch, summed
    config = workload_config(batch, args, world)
    config["kv_cache_dtype"] = "e4m3 (8-bit pools, fp16 MMA operands)" if e4m3 else batch.dtype
    if e4m3:
        config["pool_bytes"] = int(run.f8.k_cache.nbytes + run.f8.v_cache.nbytes)
    line = {
        "metric": METRIC,
        "value": round(value, 2),
        "unit": "GB/s",
        "n_gpus": world,
        "steps": K,
        "warmup": args.warmup,
        "ms_per_step": round(ms_step, 5),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f16" if e4m3 else batch.dtype,
        "data": "synthetic (seeded generator, inputs resident in HBM)",
        "config": config,
        "decode_tokens_per_s": round(seqs_all / (ms_step * 1e-3), 1),
        "decode_tokens_per_s_32_layer_attention_only": round(seqs_all / (ms_step * 1e-3) / 32, 1),
        "bytes_per_step": {"attention": att_bytes["total"], "attention_kv": att_bytes["kv"],
                           "cache_write": write_bytes, "block_copy": copy_bytes},
        "attention_ms_per_call": round(att_ms_max, 5),
        "per_call_l2_flushed": flushed,
        "graph_replay": graph,
        "host_submit_us_per_call": host_us,
        "context_read_stream_gbs": round(read_gbs, 1),
        "kv_accounting": decode_accounting(batch, 1 if e4m3 else 2, ms_step),
        "split_k": {"partition_tokens": run.P, "split": bool(run.split), "workspace_bytes": run.ws_bytes,
                    "partials_bytes_moved": split_partials_bytes(batch, run.P)},
        "roofline": decode_roofline(att_bytes["total"], att_ms_max, e4m3, batch.name),
        "clocks": clock,
        "gpu_launches": run.launches_per_step * K,
        "gpu_launches_attention_region": run.attention_launches * K,
    }
    if e2e:
        line["e2e"] = {"value": round(bytes_all / (e2e_ms / K * 1e-3) / 1e9, 2), "unit": "GB/s",
                       "h2d_bytes_per_step": e2e["h2d"], "d2h_bytes_per_step": e2e["d2h"],
                       "ms_per_step": round(e2e_ms / K, 5),
                       "copies_only_ms_per_step": round(e2e["copies_ms"] / K, 5),
                       "pipelining": "inputs uploaded and outputs read back on two copy streams, "
                                     "double-buffered, overlapping compute of neighbouring steps"}
    if cpu:
        line["cpu_baseline"] = cpu
    if companion:
        line["companion"] = companion
    print(json.dumps(line), flush=True)
    return 0


def main(argv=None):
    args = parse_args(argv)
    if args.impl == "reference":
        return run_reference(args)
    if is_prefill(args.workload):
        return run_prefill(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
