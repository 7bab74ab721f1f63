#!/usr/bin/env python3
"""Benchmark of the paged decode-attention hot path on B200 (sm_100a).

One step = one decode step of one layer over a synthetic batch already resident
in HBM, all through libpa's C ABI:
  1. copy-on-write block copies (when the workload plans any),
  2. scatter of the step's new K/V into the paged pool (one token per sequence),
  3. paged decode attention: plan, attend, partition merge.

Metric: paged decode attention KV GB/s (algorithmic bytes / step time; also as
% of 8 TB/s and of the measured HBM copy bandwidth) and seq-tokens/s per layer
(context tokens attended per second).  Algorithmic bytes of a step:
  sum_s ctx_s*Hkv*d*2*e + 2*S*Hq*d*e + sum_s ceil(ctx_s/B)*4 + 4*S
(shared prefix blocks counted once).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config NAME|decode] [--impl ours|reference]

Default (--config decode): every decode workload in one run.  The JSON line's
headline is the GQA batch (256 sequences, 32 q / 8 kv heads, head_dim 128,
block_size 16, log-normal context lengths with median 1000, a 90 % occupied
pool), the largest batch of the suite, timed over exactly K steps; its
``per_config`` object holds the same measurements for every decode workload:
Llama-7B-like, GQA, parallel sampling with a shared 512-token prompt (and the
520-token prompt's copy-on-write step) and long context at block size 8, 16
and 32.  Workloads whose unique bytes fit the 126 MB L2 (the copy-on-write
step) have L2 flushed (a 256 MB write) before every timed step, outside
per-step CUDA events; the others are larger than L2 and run back to back
(an ncu capture of one cold-L2 attend launch takes no less time than the
warm back-to-back average on each of them).  With N > 1 ranks
(torchrun) every rank runs its own batches (seed + rank): weak scaling, no
collective on the data path.

Rank 0 prints one JSON line.
"""

from __future__ import annotations

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

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "paged decode attention KV GB/s (% of 8 TB/s HBM) and seq-tokens/s per layer"
UNIT = "GB/s"
NOMINAL_HBM_GBS = 8000.0
FALLBACK_HBM_GBS = 6650.0

CONFIGS = {
    "llama7b": dict(max_len=2048, builder="llama7b", kwargs={},
                    desc="Llama-7B-like decode layer bf16: 64 seqs, 32 q = 32 kv heads, head_dim 128, "
                         "block_size 16, context lens uniform [128, 2048], 8192-block shuffled pool, "
                         "+ reshape_and_cache of 64 new tokens"),
    "gqa": dict(max_len=8192, builder="gqa", kwargs={},
                desc="GQA decode bf16: 256 seqs, 32 q / 8 kv heads, head_dim 128, block_size 16, "
                     "context lens log-normal (median 1000, sigma 1.0, capped 8192), 90% occupied pool"),
    "shared_prefix": dict(max_len=1025, builder="shared_prefix", kwargs=dict(prompt_len=512, suffix_max=512),
                          desc="parallel sampling bf16: 16 prompts x 8 samples, 512-token prompt in "
                               "shared blocks, suffix uniform [0, 512], 32 q / 8 kv heads, head_dim 128"),
    "shared_prefix_cow": dict(max_len=521, builder="shared_prefix", kwargs=dict(prompt_len=520, suffix_max=0),
                              desc="parallel sampling bf16, first decode step after a 520-token prompt: "
                                   "112 copy-on-write block copies, 32 q / 8 kv heads, head_dim 128"),
    "long_context_b8": dict(max_len=131072, builder="long_context", kwargs=dict(block_size=8),
                            desc="long-context decode bf16: 8 seqs, context lens uniform [32768, 131072], "
                                 "64 q / 8 kv heads, head_dim 128, block_size 8, partitions of 512"),
    "long_context_b16": dict(max_len=131072, builder="long_context", kwargs=dict(block_size=16),
                             desc="long-context decode bf16: 8 seqs, context lens uniform [32768, 131072], "
                                  "64 q / 8 kv heads, head_dim 128, block_size 16, partitions of 512"),
    "long_context_b32": dict(max_len=131072, builder="long_context", kwargs=dict(block_size=32),
                             desc="long-context decode bf16: 8 seqs, context lens uniform [32768, 131072], "
                                  "64 q / 8 kv heads, head_dim 128, block_size 32, partitions of 512"),
}
CONFIGS["prefill_chunk"] = dict(
    max_len=1280, builder="prefill_chunk", kwargs={},
    desc="chunked prefill bf16: 16 seqs x (1024 cached + 256 new tokens), causal, 32 q / 8 kv heads, "
         "head_dim 128, block_size 16, + reshape_and_cache of the 4096 new tokens")
CONFIGS["host_block_manager"] = dict(
    max_len=0, builder=None, kwargs={},
    desc="host block manager (pa_bm_*, C++): 256 requests with a 512-token shared system prompt + "
         "64 user tokens, then 256 decode steps of one token each, block_size 16")
DECODE_SUITE = ["llama7b", "gqa", "shared_prefix", "shared_prefix_cow", "long_context_b8", "long_context_b16",
                "long_context_b32"]
SUITE_HEADLINE = "gqa"
DEFAULT_CONFIG = "decode"
L2_BYTES = 126 * 1024 * 1024
# per-config entries other than the headline run enough steps to fill this much
# device time (at least K), so that short steps are not timed over a few ms only
PER_CONFIG_MIN_SECONDS = 0.25
# sources that make up each profiled kernel: a committed ncu summary counts only
# while their hash is the one it records
KERNEL_SOURCES = {
    "attend": ["paged_kv_cache_382_b200/csrc/decode.cu", "paged_kv_cache_382_b200/csrc/attend_bf16.cuh",
               "paged_kv_cache_382_b200/csrc/pa_device.cuh"],
    "prefill_tc": ["paged_kv_cache_382_b200/csrc/prefill_tc.cu", "paged_kv_cache_382_b200/csrc/pa_umma.cuh",
                   "paged_kv_cache_382_b200/csrc/pa_device.cuh"],
}


def parse_args(argv=None):
    p = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=5000)
    p.add_argument("--warmup", type=int, default=50)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--config", choices=sorted(CONFIGS) + [DEFAULT_CONFIG], default=DEFAULT_CONFIG)
    p.add_argument("--seed", type=int, default=0)
    p.add_argument("--partition-size", type=int, default=None,
                   help="tokens per split-context partition (default: the workload's own, 512 unless stated)")
    p.add_argument("--cpu-core-seconds", type=float, default=15.0,
                   help="CPU work of the oracle baseline sample, in core-seconds")
    p.add_argument("--reference-seconds", type=float, default=150.0,
                   help="wall-time budget of the whole --impl reference run")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--no-clocks", action="store_true")
    p.add_argument("--no-flush", action="store_true",
                   help="run every workload's steps back to back, without L2 flushes (comparisons only)")
    p.add_argument("--eager", action="store_true",
                   help="time eager pa_decode_step calls instead of replays of captured CUDA graphs")
    return p.parse_args(argv)


# ---------------------------------------------------------------------------
# small helpers (no torch at module level: spawned oracle workers import this file)
# ---------------------------------------------------------------------------

def measured_hbm_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            v = float(json.load(f)["hbm_gbs"])
        return v, "measured"
    except (OSError, KeyError, ValueError):
        return FALLBACK_HBM_GBS, "fallback"


def kernel_source_hash(kernel: str = "attend") -> str:
    h = hashlib.sha256()
    for rel in KERNEL_SOURCES[kernel]:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def profiled_traffic(config: str, kernel: str = "attend"):
    """dram bytes per launch of the kernel from the committed ncu summary of this
    workload (profiles/<kernel>_<config>.ncu.md), or None if there is none or the
    kernel source changed since it was taken."""
    path = os.path.join(ROOT, "profiles", f"{kernel}_{config}.ncu.md")
    if not os.path.exists(path):
        return None
    fields = {}
    with open(path) as f:
        for line in f:
            if ":" in line and line.lstrip().startswith("- "):
                k, v = line.strip()[2:].split(":", 1)
                fields[k.strip()] = v.strip().strip("`")
    try:
        if fields.get("kernel_source_sha256") != kernel_source_hash(kernel):
            return None
        return int(float(fields["dram_bytes_per_launch"]))
    except (KeyError, ValueError):
        return None


class ClockSampler:
    """nvidia-smi clock / throttle samples taken while the timed region runs."""

    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    REASONS = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]

    def __init__(self, device_id: str, enabled: bool = True):
        self.device_id = device_id
        self.enabled = enabled
        self.proc = None
        self.path = None

    def __enter__(self):
        if self.enabled:
            fd, self.path = tempfile.mkstemp(prefix="pa_clocks_", suffix=".csv")
            os.close(fd)
            try:
                self.proc = subprocess.Popen(
                    ["nvidia-smi", f"--id={self.device_id}", f"--query-gpu={self.QUERY}",
                     "--format=csv,noheader,nounits", "-lms", "100"],
                    stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
                time.sleep(0.3)
            except OSError:
                self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.15)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        if not self.path or not os.path.exists(self.path):
            return None
        sm, mx, reasons = [], None, set()
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    sm.append(float(parts[1]))
                    mx = float(parts[2])
                except ValueError:
                    continue
                for name, flag in zip(self.REASONS, parts[5:9]):
                    if flag.lower() == "active":
                        reasons.add(name)
        os.unlink(self.path)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# ---------------------------------------------------------------------------
# oracle timing (CPU baseline and the reference arm): spawn workers, fp64 numpy
# ---------------------------------------------------------------------------

def _oracle_task(task):
    """Runs in a spawned worker: decode attention of one sequence by the oracle,
    over its blocks stored as .npy files (table = their order)."""
    import numpy as np

    import oracle

    kpath, vpath, q, ctx, scale = task
    k = np.load(kpath, mmap_mode="r")
    v = np.load(vpath, mmap_mode="r")
    table = np.arange(k.shape[0])[None]
    t0 = time.perf_counter()
    oracle.decode_attention(q[None], k, v, table, np.array([ctx]), scale)
    return time.perf_counter() - t0


class OracleSample:
    """Stages the blocks of some sequences of a step on the host (not timed) and
    times the oracle over them with a process pool of the machine's host cores."""

    def __init__(self, step, seqs, pool, tmpdir):
        import numpy as np
        import torch

        self.step, self.seqs, self.pool = step, list(seqs), pool
        self.tasks = []
        B = step.block_size
        for s in self.seqs:
            c = int(step.context_lens[s])
            ids = torch.from_numpy(step.block_tables[s, : -(-c // B)].astype(np.int64)).to(step.k_cache.device)
            kp = os.path.join(tmpdir, f"k{s}.npy")
            vp = os.path.join(tmpdir, f"v{s}.npy")
            np.save(kp, step.k_cache.index_select(0, ids).float().cpu().numpy())
            np.save(vp, step.v_cache.index_select(0, ids).float().cpu().numpy())
            q = step.q[s].double().cpu().numpy()
            self.tasks.append((kp, vp, q, c, step.scale))

    def bytes(self):
        st = self.step
        e = st.element_bytes
        kv = sum(int(st.context_lens[s]) for s in self.seqs) * st.num_kv_heads * st.head_dim * 2 * e
        qo = 2 * len(self.seqs) * st.num_heads * st.head_dim * e
        tb = sum(-(-int(st.context_lens[s]) // st.block_size) for s in self.seqs) * 4 + 4 * len(self.seqs)
        return kv + qo + tb

    def tokens(self):
        return sum(int(self.step.context_lens[s]) for s in self.seqs)

    def run(self, repeats=1):
        t0 = time.perf_counter()
        busy = 0.0
        for _ in range(repeats):
            busy += sum(self.pool.map(_oracle_task, self.tasks, chunksize=1))
        return time.perf_counter() - t0, busy


def make_oracle_pool():
    import multiprocessing as mp

    os.environ.setdefault("OMP_NUM_THREADS", "1")
    os.environ.setdefault("OPENBLAS_NUM_THREADS", "1")
    os.environ.setdefault("MKL_NUM_THREADS", "1")
    cores = len(os.sched_getaffinity(0))
    return mp.get_context("spawn").Pool(cores), cores


# ---------------------------------------------------------------------------
# the GPU path
# ---------------------------------------------------------------------------

class DeviceStep:
    """One step's inputs resident on the device plus the preallocated outputs."""

    def __init__(self, pa, step, partition_size):
        import numpy as np
        import torch

        dev = step.k_cache.device
        self.pa, self.step = pa, step
        self.kc, self.vc = step.k_cache, step.v_cache
        self.q, self.new_key, self.new_value = step.q, step.new_key, step.new_value
        self.slots = torch.from_numpy(step.slot_mapping).to(dev)
        self.pairs = torch.from_numpy(np.ascontiguousarray(step.copy_pairs)).to(dev)
        self.tables = torch.from_numpy(step.block_tables.astype(np.int32)).to(dev)
        self.ctx = torch.from_numpy(step.context_lens.astype(np.int32)).to(dev)
        self.out = torch.empty(step.num_seqs, step.num_heads, step.head_dim, dtype=step.dtype, device=dev)
        self.P = partition_size
        self.cap = pa.decode_capacity(self.tables, step.block_size, step.max_context_len)
        self.ws = pa.alloc_workspace(step.num_seqs, step.num_heads, step.head_dim, self.cap, partition_size,
                                     dev)
        self.err = torch.zeros(1, dtype=torch.int32, device=dev)
        self.prefill = step.query_start is not None
        if self.prefill:
            T = step.q.shape[0]
            self.qs = torch.from_numpy(step.query_start.astype(np.int32)).to(dev)
            self.out = torch.empty(T, step.num_heads, step.head_dim, dtype=step.dtype, device=dev)
            n = pa.lib.pa_prefill_workspace_bytes(T, step.num_heads, step.head_dim, self.cap, partition_size)
            self.ws = torch.empty(n, dtype=torch.uint8, device=dev)
        self.tensor_core_prefill = self.prefill and pa.prefill_uses_tensor_cores(
            step.dtype, step.num_heads, step.num_kv_heads, step.head_dim, step.block_size)
        # Decode: one pa_decode_step call -- copy_blocks (if any pairs), the prologue
        # (plan + scatter of the new tokens), attend, reduce.  Prefill: copy_blocks,
        # reshape_and_cache, then rows/plan/attend/reduce (prefill by decode rows) or
        # plan/attend (tensor-core prefill).
        copies = 1 if len(step.copy_pairs) else 0
        if self.prefill:
            self.launches_per_step = copies + 1 + (2 if self.tensor_core_prefill else 4)
        else:
            self.launches_per_step = copies + 3

    def capture(self, n):
        """A CUDA graph of n consecutive decode steps (one pa_decode_step call each,
        on these buffers), as a serving loop replays its decode step: the same
        kernels and work as eager calls, without the host's per-call cost."""
        import torch

        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, capture_error_mode="relaxed"):
            for _ in range(n):
                self.run()
        return g

    def run(self, ev_attend=None, q=None, new_key=None, new_value=None, slots=None, tables=None, ctx=None,
            out=None):
        """One step.  A decode step without ``ev_attend`` is the single fused call
        (pa_decode_step); with it, the same work runs phase by phase so that events
        can bracket the attend kernel."""
        pa = self.pa
        if not self.prefill and ev_attend is None:
            pa.decode_step(out if out is not None else self.out, q if q is not None else self.q,
                           new_key if new_key is not None else self.new_key,
                           new_value if new_value is not None else self.new_value, self.kc, self.vc,
                           slots if slots is not None else self.slots,
                           tables if tables is not None else self.tables, ctx if ctx is not None else self.ctx,
                           self.step.scale, copy_pairs=self.pairs if len(self.step.copy_pairs) else None,
                           max_context_len=self.cap, partition_size=self.P, workspace=self.ws, dev_err=self.err)
            return
        if len(self.step.copy_pairs):
            pa.copy_blocks(self.kc, self.vc, self.pairs, dev_err=self.err)
        pa.reshape_and_cache(new_key if new_key is not None else self.new_key,
                             new_value if new_value is not None else self.new_value,
                             self.kc, self.vc, slots if slots is not None else self.slots, dev_err=self.err)
        args = (out if out is not None else self.out, q if q is not None else self.q, self.kc, self.vc,
                tables if tables is not None else self.tables, ctx if ctx is not None else self.ctx,
                self.step.scale)
        kw = dict(max_context_len=self.cap, partition_size=self.P, workspace=self.ws, dev_err=self.err)
        if self.prefill:
            if ev_attend is not None:
                ev_attend[0].record()
            pa.prefill(*args[:6], self.qs, self.step.scale, **kw)
            if ev_attend is not None:
                ev_attend[1].record()
            return
        pa.decode(*args, phases=pa.PHASE_PLAN, **kw)
        if ev_attend is not None:
            ev_attend[0].record()
        pa.decode(*args, phases=pa.PHASE_ATTEND, **kw)
        if ev_attend is not None:
            ev_attend[1].record()
        pa.decode(*args, phases=pa.PHASE_REDUCE, **kw)


def nvsmi_id(local_index: int) -> str:
    """nvidia-smi's name for torch device ``local_index`` (its UUID), robust to
    CUDA_VISIBLE_DEVICES remapping."""
    import torch

    try:
        return "GPU-" + str(torch.cuda.get_device_properties(local_index).uuid)
    except Exception:
        return str(local_index)


def kv_utilisation_summary(step, max_len):
    """Tokens held / KV slots reserved for this batch: paged blocks against a
    contiguous reservation of the workload's maximum length per sequence."""
    from paged_kv_cache_382_b200.utilization import kv_utilisation

    u = kv_utilisation(step.context_lens, step.block_size, max_len)
    return {"paged": round(u["paged"], 4), "contiguous_max_len": round(u["contiguous"], 4),
            "block_size": u["block_size"], "max_len": u["max_len"]}


def partition_for(args, config: str) -> int:
    """The partition size a workload runs with: --partition-size if given, else its own."""
    return args.partition_size or CONFIGS[config].get("partition_size", 512)


def build_step(config: str, seed: int, device, partition_size: int):
    from paged_kv_cache_382_b200 import workloads as W

    spec = CONFIGS[config]
    fn = W.WORKLOADS[spec["builder"]]
    return fn(seed=seed, device=device, partition_size=partition_size, **spec["kwargs"])


def dist_setup():
    import torch

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime

        import torch.distributed as dist

        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(local)
    return world, rank, local


def reduce_over_ranks(values, ops):
    """All-reduce a few scalars over the ranks (SUM or MAX each); identity at N=1."""
    import torch
    import torch.distributed as dist

    if not (dist.is_available() and dist.is_initialized()):
        return list(values)
    dev = torch.device("cuda", torch.cuda.current_device()) if dist.get_backend() == "nccl" else "cpu"
    out = []
    for v, op in zip(values, ops):
        t = torch.tensor([float(v)], dtype=torch.float64, device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX if op == "max" else dist.ReduceOp.SUM)
        out.append(float(t.item()))
    return out


def barrier():
    import torch.distributed as dist

    if dist.is_available() and dist.is_initialized():
        dist.barrier()


def config_dict(name, step, world, partition_size, flushed):
    """The line's ``config`` (the same keys in both arms)."""
    from paged_kv_cache_382_b200 import workloads as W

    alg = W.algorithmic_bytes(step, unique=True)
    if flushed:
        l2 = (f"L2 flushed before every timed step (a 256 MB write outside the per-step CUDA events): "
              f"{alg / 1e6:.1f} MB of unique K/V+q/out per step fits the 126 MB L2")
    else:
        l2 = f"inputs larger than L2: {alg / 1e9:.3f} GB of K/V+q/out per step vs 126 MB L2, steps back to back"
    return {
        "workload": CONFIGS[name]["desc"],
        "name": name,
        "num_seqs_per_gpu": step.num_seqs,
        "context_tokens_per_gpu": int(step.context_lens.sum()),
        "partition_size": partition_size,
        "parallelism": f"replicas x{world} (independent batches, no collective)",
        "l2": l2,
    }


def needs_flush(step) -> bool:
    from paged_kv_cache_382_b200 import workloads as W

    return W.algorithmic_bytes(step, unique=True) < L2_BYTES


GRAPH_CHUNK = 16   # steps per replayed CUDA graph when steps run back to back


class StepGraphs:
    """CUDA graphs of 1 and GRAPH_CHUNK decode steps; n steps replay
    n // GRAPH_CHUNK large graphs and n % GRAPH_CHUNK small ones."""

    def __init__(self, ds, warmup):
        import torch

        self.one = ds.capture(1)
        self.chunk = ds.capture(GRAPH_CHUNK)
        for _ in range(max(warmup, 1)):
            self.one.replay()
            self.chunk.replay()
        torch.cuda.synchronize()

    def replay(self, n):
        for _ in range(n // GRAPH_CHUNK):
            self.chunk.replay()
        for _ in range(n % GRAPH_CHUNK):
            self.one.replay()


def time_steps(ds, n, flush, stream, graphs=None):
    """Device time (ms) of n steps, and the host time (ms) spent enqueueing them:
    back to back between two events, or, with a flush buffer, each step between
    its own events after an L2 flush.  With ``graphs`` the steps are replays of
    captured CUDA graphs, otherwise eager pa_decode_step calls."""
    import torch

    if flush is None:
        start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t0 = time.perf_counter()
        start.record(stream)
        if graphs is not None:
            graphs.replay(n)
        else:
            for _ in range(n):
                ds.run()
        stop.record(stream)
        host_ms = (time.perf_counter() - t0) * 1e3
        torch.cuda.synchronize()
        return start.elapsed_time(stop), host_ms
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n)]
    t0 = time.perf_counter()
    for i in range(n):
        flush.fill_(i & 0xFF)
        ev[i][0].record(stream)
        if graphs is not None:
            graphs.one.replay()
        else:
            ds.run()
        ev[i][1].record(stream)
    host_ms = (time.perf_counter() - t0) * 1e3
    torch.cuda.synchronize()
    return sum(a.elapsed_time(b) for a, b in ev), host_ms


def time_attend(ds, n, flush):
    """Mean device time (ms) of the attend kernel alone: the step runs phase by
    phase with events around the attend launch (after an L2 flush if given)."""
    import torch

    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n)]
    for i in range(n):
        if flush is not None:
            flush.fill_(i & 0xFF)
        ds.run(ev_attend=ev[i])
    torch.cuda.synchronize()
    return statistics.fmean(a.elapsed_time(b) for a, b in ev)


def measure_decode(pa, args, name, dev, world, rank, local, steps, warmup, pool=None, cores=None):
    """Every measurement of one decode workload; ``steps`` None picks a count that
    fills PER_CONFIG_MIN_SECONDS of device time (at least --steps)."""
    import torch

    from paged_kv_cache_382_b200 import workloads as W

    P = partition_for(args, name)
    step = build_step(name, args.seed + rank, dev, P)
    ds = DeviceStep(pa, step, P)
    alg_bytes = W.algorithmic_bytes(step, unique=True)
    logical_bytes = W.algorithmic_bytes(step, unique=False)
    ctx_tokens = int(step.context_lens.sum())
    flush = (torch.empty(256 << 20, dtype=torch.uint8, device=dev)
             if needs_flush(step) and not args.no_flush else None)
    stream = torch.cuda.current_stream()
    for _ in range(warmup):
        ds.run()
    torch.cuda.synchronize()
    if int(ds.err.item()) != 0:
        raise RuntimeError(f"{name}: device error word {int(ds.err.item()):#x}")
    graphs = None if args.eager else StepGraphs(ds, warmup)
    if steps is None:
        est = time_steps(ds, 5, flush, stream, graphs)[0] / 5
        want = int(math.ceil(PER_CONFIG_MIN_SECONDS * 1e3 / max(est, 1e-4)))
        steps = int(reduce_over_ranks([min(5000, max(args.steps, want))], ["max"])[0])
    K = steps
    with ClockSampler(nvsmi_id(local), enabled=not args.no_clocks) as clocks:
        barrier()
        torch.cuda.synchronize()
        elapsed_ms, host_ms = time_steps(ds, K, flush, stream, graphs)
        torch.cuda.synchronize()
        barrier()
    # the same steps as eager calls (host-side cost per step included), for reference
    eager_ms, eager_host_ms = time_steps(ds, K, flush, stream) if graphs is not None else (elapsed_ms, host_ms)
    n_att = min(K, 500)
    attend_ms = time_attend(ds, n_att, flush)
    clock_info = clocks.summary()
    e2e = None
    if not args.no_e2e:
        e2e = run_e2e(ds, step, alg_bytes, warmup, min(K, 1000), flush)
    tot_bytes, max_ms, tot_tokens, tot_seqs = reduce_over_ranks(
        [alg_bytes * K, elapsed_ms, ctx_tokens * K, step.num_seqs * K], ["sum", "max", "sum", "sum"])
    e2e_line = None
    if e2e is not None:
        e2e_bytes, e2e_ms = reduce_over_ranks([e2e["bytes"], e2e["ms"]], ["sum", "max"])
        e2e_line = {"value": round(e2e_bytes / (e2e_ms * 1e-3) / 1e9, 2), "unit": UNIT,
                    "h2d_bytes_per_step": e2e["h2d"], "d2h_bytes_per_step": e2e["d2h"],
                    "ms_per_step": round(e2e_ms / e2e["steps"], 5), "steps": e2e["steps"],
                    "timing": e2e["timing"]}
    peak, peak_kind = measured_hbm_peak()
    achieved_attend = alg_bytes / (attend_ms * 1e-3) / 1e9
    value = tot_bytes / (max_ms * 1e-3) / 1e9
    traffic = profiled_traffic(name)
    cpu = None
    if pool is not None:
        cpu = cpu_baseline(step, pool, cores, args.cpu_core_seconds)
    res = {
        "value": round(value, 2),
        "unit": UNIT,
        "steps": K,
        "ms_per_step": round(max_ms / K, 5),
        "config": config_dict(name, step, world, P, flush is not None),
        "pct_of_8tbs": round(100.0 * value / NOMINAL_HBM_GBS, 2),
        "pct_of_measured_hbm": round(100.0 * value / peak, 2),
        "seq_tokens_per_s": round(tot_tokens / (max_ms * 1e-3), 1),
        "decode_tokens_per_s": round(tot_seqs / (max_ms * 1e-3), 1),
        "algorithmic_bytes_per_step": alg_bytes,
        "logical_bytes_per_step": logical_bytes,
        "effective_logical_gbs": round(logical_bytes * K * world / (max_ms * 1e-3) / 1e9, 2),
        "gpu_launches": ds.launches_per_step * K,
        "step_call": "pa_decode_step: " + ("copy_blocks, " if len(step.copy_pairs) else "")
                     + "plan+scatter prologue, attend, reduce",
        "step_timing": ("replays of CUDA graphs captured from pa_decode_step calls "
                        f"({GRAPH_CHUNK} steps per graph back to back, 1 per graph between flushes)"
                        if graphs is not None else "eager pa_decode_step calls"),
        "host_enqueue_ms_per_step": round(host_ms / K, 5),
        "eager": {"ms_per_step": round(eager_ms / K, 5), "host_enqueue_ms_per_step": round(eager_host_ms / K, 5),
                  "value": round(alg_bytes * K / (eager_ms * 1e-3) / 1e9, 2)},
        "kv_utilisation": kv_utilisation_summary(step, CONFIGS[name]["max_len"]),
        "roofline": {
            "kernel": "attend_bf16_kernel" if step.dtype == torch.bfloat16 else "attend_f32_kernel",
            "bound": "hbm",
            "achieved": round(achieved_attend, 2),
            "peak": peak,
            "peak_kind": f"{peak_kind} HBM copy bandwidth (MEASURED_PEAKS.json hbm_gbs)"
                         if peak_kind == "measured" else "fallback 6.65 TB/s",
            "unit": "GB/s",
            "frac": round(achieved_attend / peak, 4),
            "traffic": traffic,
            "traffic_source": (f"read from profiles/attend_{name}.ncu.md (an ncu capture of this kernel source, "
                               "dram__bytes_read.sum + dram__bytes_write.sum per launch), not measured in this run"
                               if traffic is not None else
                               "null: no ncu summary of the current attend kernel source for this workload"),
            "attend_ms": round(attend_ms, 5),
            "attend_timing": "CUDA events around each attend launch, in a pass after the timed steps "
                             f"({n_att} launches" + (", L2 flushed before each)" if flush is not None else ")"),
            "bytes_per_launch": alg_bytes,
        },
        "clocks": clock_info,
        "e2e": e2e_line,
        "cpu_baseline": cpu,
        "dtype": "bf16" if step.dtype == torch.bfloat16 else "f32",
    }
    del ds, step, flush, graphs
    torch.cuda.empty_cache()
    return res


def run_ours(args):
    import torch

    from paged_kv_cache_382_b200 import build as _build

    world, rank, local = dist_setup()
    if world != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE {world}")
    # the oracle pool is spawned before any CUDA work
    pool = cores = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        pool, cores = make_oracle_pool()
    _build.build()
    from paged_kv_cache_382_b200 import pa

    dev = torch.device("cuda", local)
    warmup = max(args.warmup, 3)
    if args.config != DEFAULT_CONFIG and CONFIGS[args.config]["builder"] == "prefill_chunk":
        run_prefill(args, pa, dev, world, rank, local, pool)
        return
    names = ([SUITE_HEADLINE] + [n for n in DECODE_SUITE if n != SUITE_HEADLINE]
             if args.config == DEFAULT_CONFIG else [args.config])
    results = {}
    for i, name in enumerate(names):
        results[name] = measure_decode(pa, args, name, dev, world, rank, local, args.steps if i == 0 else None,
                                       warmup, pool if i == 0 else None, cores)
    if pool is not None:
        pool.close()
    if rank != 0:
        return
    head = results[names[0]]
    line = {
        "metric": METRIC,
        "value": head["value"],
        "unit": UNIT,
        "n_gpus": world,
        "steps": args.steps,
        "warmup": warmup,
        "ms_per_step": head["ms_per_step"],
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": head["dtype"],
        "data": "synthetic (seeded; K/V ~ N(0,1) generated on the device by torch, no dataset)",
        "config": head["config"],
    }
    for k in ("pct_of_8tbs", "pct_of_measured_hbm", "seq_tokens_per_s", "decode_tokens_per_s",
              "algorithmic_bytes_per_step", "logical_bytes_per_step", "effective_logical_gbs", "gpu_launches",
              "step_call", "step_timing", "host_enqueue_ms_per_step", "eager", "kv_utilisation", "roofline",
              "clocks", "e2e", "cpu_baseline"):
        line[k] = head[k]
    if len(names) > 1:
        line["per_config"] = {n: {k: v for k, v in r.items() if k not in ("cpu_baseline", "dtype")}
                              for n, r in results.items()}
        line["per_config_note"] = (f"every decode workload measured in this run on this GPU; the headline is "
                                   f"{names[0]} over exactly --steps steps, the others over enough steps to "
                                   f"fill {PER_CONFIG_MIN_SECONDS} s of device time (at least --steps), stated "
                                   "per entry")
    print(json.dumps(line), flush=True)


def run_prefill(args, pa, dev, world, rank, local, pool):
    """The chunked-prefill workload (tensor-core prefill), L2 flushed before every step."""
    import torch

    from paged_kv_cache_382_b200 import workloads as W

    P = partition_for(args, args.config)
    step = build_step(args.config, args.seed + rank, dev, P)
    ds = DeviceStep(pa, step, P)
    alg_bytes = W.algorithmic_bytes(step, unique=True)
    alg_bytes += 2 * (step.q.shape[0] - step.num_seqs) * step.num_heads * step.head_dim * step.element_bytes
    for _ in range(max(args.warmup, 3)):
        ds.run()
    torch.cuda.synchronize()
    if int(ds.err.item()) != 0:
        raise RuntimeError(f"device error word {int(ds.err.item()):#x}")
    K = args.steps
    stream = torch.cuda.current_stream()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    ev_step = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    # The chunked-prefill K/V (84 MB) fits the 126 MB L2: flush L2 before every
    # step (a 256 MB write) and time the steps alone with per-step events.
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    with ClockSampler(nvsmi_id(local), enabled=not args.no_clocks) as clocks:
        barrier()
        torch.cuda.synchronize()
        for i in range(K):
            flush.fill_(i & 0xFF)
            ev_step[i][0].record(stream)
            ds.run(ev_attend=ev[i])
            ev_step[i][1].record(stream)
        torch.cuda.synchronize()
        barrier()
    elapsed_ms = sum(a.elapsed_time(b) for a, b in ev_step)
    prefill_ms = statistics.fmean(a.elapsed_time(b) for a, b in ev)
    clock_info = clocks.summary()
    (max_ms,) = reduce_over_ranks([elapsed_ms], ["max"])
    if pool is not None:
        pool.close()
    if rank != 0:
        return
    print(json.dumps(prefill_line(args, step, world, K, max_ms, prefill_ms, alg_bytes, clock_info, ds)),
          flush=True)


def measured_tensor_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["bf16_tflops_sustained"]), "measured sustained cuBLAS bf16"
    except (OSError, KeyError, ValueError):
        return 1400.0, "fallback sustained bf16"


def prefill_line(args, step, world, K, max_ms, prefill_ms, alg_bytes, clock_info, ds):
    """The chunked-prefill workload: useful attention FLOP/s against the tensor roofline."""
    from paged_kv_cache_382_b200 import workloads as W

    flops = W.prefill_flops(step)
    peak, kind = measured_tensor_peak()
    tflops_step = flops * K * world / (max_ms * 1e-3) / 1e12
    tflops_call = flops / (prefill_ms * 1e-3) / 1e12
    return {
        "metric": "paged prefill attention TFLOP/s (causal, useful flops) and KV GB/s",
        "value": round(tflops_step, 2), "unit": "TFLOP/s", "n_gpus": world, "steps": K,
        "warmup": max(args.warmup, 3), "ms_per_step": round(max_ms / K, 5), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded; K/V/q ~ N(0,1) generated on the device by torch, no dataset)",
        "config": {"workload": CONFIGS[args.config]["desc"], "name": args.config,
                   "new_tokens_per_gpu": int(step.q.shape[0]), "partition_size": ds.P,
                   "l2": "flushed before every step (256 MB write, outside the per-step CUDA events); "
                         "ms_per_step is the sum of the per-step event times"},
        "kv_gbs": round(alg_bytes * K * world / (max_ms * 1e-3) / 1e9, 2),
        "flops_per_step": flops,
        "gpu_launches": ds.launches_per_step * K,
        "roofline": {"kernel": ("pa_prefill (tcgen05: plan, attend)" if ds.tensor_core_prefill
                                else "pa_prefill (decode rows: rows, plan, attend, reduce)"),
                     "bound": "tensor",
                     "achieved": round(tflops_call, 2), "peak": peak, "peak_kind": kind, "unit": "TFLOP/s",
                     "frac": round(tflops_call / peak, 4),
                     "traffic": (profiled_traffic(args.config, "prefill_tc") if ds.tensor_core_prefill else None),
                     "prefill_ms": round(prefill_ms, 5),
                     "mma_flops_issued": (W.prefill_tc_mma_flops(step) if ds.tensor_core_prefill else None)},
        "clocks": clock_info, "e2e": None, "cpu_baseline": None,
    }


def run_e2e(ds, step, alg_bytes, warmup, steps, flush=None):
    """The same step through the binding, fed from the host: each step's inputs
    (q, new K/V, slot mapping, block tables, context lens) are packed in one
    pinned host buffer and copied in, the step runs, and its output is copied
    back to pinned host memory.  Copies and compute overlap across steps on
    three streams (H2D, compute, D2H) with double-buffered device inputs and
    outputs, the way a serving loop would feed the kernels.  With ``flush`` (a
    buffer larger than L2) every step instead runs alone after an L2 flush,
    between its own events: H2D copy, step and D2H copy in series."""
    import torch

    parts = dict(q=ds.q, new_key=ds.new_key, new_value=ds.new_value, slots=ds.slots, tables=ds.tables,
                 ctx=ds.ctx)
    offsets, off = {}, 0
    for name, t in parts.items():
        offsets[name] = off
        off += (t.numel() * t.element_size() + 255) // 256 * 256
    h2d = sum(t.numel() * t.element_size() for t in parts.values())
    host_in, dev_in, views, out_dev, out_host = [], [], [], [], []
    for b in range(2):
        hb = torch.empty(off, dtype=torch.uint8).pin_memory()
        db = torch.empty(off, dtype=torch.uint8, device=ds.q.device)
        v = {}
        for name, t in parts.items():
            n = t.numel() * t.element_size()
            hb[offsets[name]:offsets[name] + n].copy_(t.reshape(-1).view(torch.uint8).cpu())
            v[name] = db[offsets[name]:offsets[name] + n].view(t.dtype).view(t.shape)
        host_in.append(hb)
        dev_in.append(db)
        views.append(v)
        out_dev.append(torch.empty_like(ds.out))
        out_host.append(torch.empty(ds.out.shape, dtype=ds.out.dtype).pin_memory())
    d2h = out_host[0].numel() * out_host[0].element_size()
    compute = torch.cuda.current_stream()
    copy_in, copy_out = torch.cuda.Stream(), torch.cuda.Stream()
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_done = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]
    for b in range(2):
        ev_done[b].record(compute)
        ev_out[b].record(compute)

    def one(i):
        b = i % 2
        copy_in.wait_event(ev_done[b])               # inputs of step i-2 consumed
        with torch.cuda.stream(copy_in):
            dev_in[b].copy_(host_in[b], non_blocking=True)
        ev_in[b].record(copy_in)
        compute.wait_event(ev_in[b])
        compute.wait_event(ev_out[b])                # output of step i-2 read back
        v = views[b]
        ds.run(q=v["q"], new_key=v["new_key"], new_value=v["new_value"], slots=v["slots"],
               tables=v["tables"], ctx=v["ctx"], out=out_dev[b])
        ev_done[b].record(compute)
        copy_out.wait_event(ev_done[b])
        with torch.cuda.stream(copy_out):
            out_host[b].copy_(out_dev[b], non_blocking=True)
        ev_out[b].record(copy_out)

    for i in range(warmup):
        one(i)
    torch.cuda.synchronize()
    if flush is not None:
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
        barrier()
        torch.cuda.synchronize()
        for i in range(steps):
            for b in range(2):
                compute.wait_event(ev_out[b])
            flush.fill_(i & 0xFF)
            ev[i][0].record(compute)
            ev_done[i % 2].record(compute)
            one(i)
            compute.wait_event(ev_out[i % 2])
            ev[i][1].record(compute)
        torch.cuda.synchronize()
        barrier()
        return {"ms": sum(a.elapsed_time(b) for a, b in ev), "bytes": alg_bytes * steps, "h2d": h2d, "d2h": d2h,
                "steps": steps, "timing": "per step after an L2 flush: H2D copy, step, D2H copy in series, "
                                          "between events on the compute stream"}
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    start.record(compute)
    copy_in.wait_event(start)
    for i in range(steps):
        one(i)
    for b in range(2):
        compute.wait_event(ev_out[b])
    stop.record(compute)
    torch.cuda.synchronize()
    barrier()
    return {"ms": start.elapsed_time(stop), "bytes": alg_bytes * steps, "h2d": h2d, "d2h": d2h,
            "steps": steps, "timing": "steps pipelined over H2D, compute and D2H streams between two events"}


def cpu_baseline(step, pool, cores, core_seconds):
    """The oracle timed on the host cores over a bounded sample of the same batch."""
    with tempfile.TemporaryDirectory(prefix="pa_oracle_") as tmp:
        sample = OracleSample(step, range(step.num_seqs), pool, tmp)
        wall1, busy1 = sample.run(1)            # first pass also warms the workers
        repeats = max(1, int(math.ceil(core_seconds / max(busy1, 1e-3))))
        wall, busy = sample.run(repeats)
        return {
            "value": round(sample.bytes() * repeats / wall / 1e9, 4),
            "unit": UNIT,
            "cores": cores,
            "kind": "oracle",
            "sample": f"all {len(sample.seqs)} sequences of the batch (every head, "
                      f"{sample.tokens()} context tokens) x {repeats} passes, decode attention only, "
                      f"fp64 numpy, one sequence per task; {busy:.1f} core-s of work in {wall:.2f} s",
            "seq_tokens_per_s": round(sample.tokens() * repeats / wall, 1),
        }


def run_reference(args):
    """The reference arm: the fp64 oracle as it stands, on the host cores."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    pool, cores = make_oracle_pool()
    import torch

    from paged_kv_cache_382_b200 import workloads as W

    del W
    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", "0"))) if torch.cuda.is_available() else "cpu"
    name = SUITE_HEADLINE if args.config == DEFAULT_CONFIG else args.config
    P = partition_for(args, name)
    step = build_step(name, args.seed, dev, P)
    with tempfile.TemporaryDirectory(prefix="pa_oracle_") as tmp:
        full = OracleSample(step, range(step.num_seqs), pool, tmp)
        wall1, busy1 = full.run(1)
        per_seq = busy1 / len(full.seqs)
        # sequences per step so that warmup + steps fit the time budget
        n_steps = max(args.warmup, 3) + args.steps
        per_step_budget = args.reference_seconds / n_steps
        n_seq = max(1, min(len(full.seqs), int(per_step_budget * cores / max(per_seq, 1e-6))))
        total_wall, total_bytes, total_tokens = 0.0, 0, 0
        for i in range(n_steps):
            seqs = [(i * n_seq + j) % len(full.seqs) for j in range(n_seq)]
            sub = OracleSample.__new__(OracleSample)
            sub.step, sub.seqs, sub.pool = step, seqs, pool
            sub.tasks = [full.tasks[s] for s in seqs]
            wall, _ = sub.run(1)
            if i >= max(args.warmup, 3):
                total_wall += wall
                total_bytes += sub.bytes()
                total_tokens += sub.tokens()
    pool.close()
    value = total_bytes / total_wall / 1e9
    line = {
        "impl": "reference",
        "metric": METRIC,
        "value": round(value, 4),
        "unit": UNIT,
        "n_gpus": world,
        "steps": args.steps,
        "warmup": max(args.warmup, 3),
        "ms_per_step": round(1e3 * total_wall / args.steps, 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f64",
        "data": "synthetic (seeded, same batch as the GPU arm)",
        "config": config_dict(name, step, world, P, needs_flush(step)),
        "seq_tokens_per_s": round(total_tokens / total_wall, 1),
        "cpu_baseline": {"value": round(value, 4), "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": f"{n_seq} of {len(full.seqs)} sequences per step (every head), "
                                   f"decode attention by the fp64 numpy oracle, one sequence per task"},
        "e2e": {"value": round(value, 4), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def run_block_manager(args):
    """Tokens per second through the library's host block manager: prompt
    admission with and without prefix caching, then single-token decode
    appends (CPU only)."""
    import numpy as np

    from paged_kv_cache_382_b200 import build as _build

    _build.build()
    from paged_kv_cache_382_b200 import pa

    rng = np.random.default_rng(args.seed)
    R, P_SYS, USER, STEPS, B = 256, 512, 64, 256, 16
    system = rng.integers(0, 32000, size=P_SYS).astype(np.int32)
    prompts = [np.concatenate([system, rng.integers(0, 32000, size=USER).astype(np.int32)]) for _ in range(R)]
    res = {}
    for cache in (False, True):
        m = pa.NativeBlockManager(R * ((P_SYS + USER + STEPS) // B + 2), B, prefix_cache=cache)
        t0 = time.perf_counter()
        cached = 0
        for r in range(R):
            m.add(r)
            _, _, c = m.append(r, prompts[r] if cache else len(prompts[r]))
            cached += c
        t1 = time.perf_counter()
        one = np.zeros(1, dtype=np.int32)
        half = STEPS // 2
        for _ in range(half):                      # one call per sequence and step
            for r in range(R):
                m.append(r, one if cache else 1)
        t2 = time.perf_counter()
        ids = np.arange(R, dtype=np.int64)
        counts = np.ones(R, dtype=np.int32)
        step_tokens = np.zeros(R, dtype=np.int32) if cache else None
        for _ in range(STEPS - half):              # one call per step (pa_bm_append_batch), flat arrays
            m.append_batch(ids, step_tokens, counts=counts)
        t3 = time.perf_counter()
        key = "prefix_cache" if cache else "no_cache"
        res[key] = {"admit_tokens_per_s": round(R * (P_SYS + USER) / (t1 - t0), 1),
                    "decode_appends_per_s": round(R * half / (t2 - t1), 1),
                    "decode_appends_per_s_batched": round(R * (STEPS - half) / (t3 - t2), 1),
                    "decode_step_us_batched": round((t3 - t2) / (STEPS - half) * 1e6, 2),
                    "cached_token_fraction": round(cached / (R * (P_SYS + USER)), 4),
                    "blocks_in_use": R * ((P_SYS + USER + STEPS) // B + 2) - m.num_free}
    line = {"metric": "host block manager tokens/s (admission and decode appends)",
            "value": res["prefix_cache"]["admit_tokens_per_s"], "unit": "tokens/s", "n_gpus": 0,
            "higher_is_better": True, "data": "synthetic token ids (seeded)",
            "config": {"workload": CONFIGS["host_block_manager"]["desc"], "name": "host_block_manager"},
            "results": res,
            "note": "timed through the Python binding: one ctypes call per request for admission; decode "
                    "appends one call per sequence and step, then one pa_bm_append_batch call per step "
                    "over flat id / count / token arrays"}
    print(json.dumps(line), flush=True)


def main(argv=None):
    args = parse_args(argv)
    if args.config == "host_block_manager":
        run_block_manager(args)
        return
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)
    try:
        import torch.distributed as dist

        if dist.is_available() and dist.is_initialized():
            dist.destroy_process_group()
    except Exception:
        pass


if __name__ == "__main__":
    main()
