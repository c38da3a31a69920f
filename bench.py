#!/usr/bin/env python
"""Benchmark of one decode step of the paged KV cache hot path.

A step, for every sequence of the batch: the host pool reserves the new
token's slot (copy-on-write pairs where a block is shared), the new token's
K/V rows are written into the cache (pkv_write_slots), and paged decode
attention runs over the whole context through the Block Tables
(pkv_decode_attention: one pass, or split-K partitions plus a merge).  The
workload is the 7B-shaped decode batch: 256 sequences, 32 query = 32 KV
heads, head_dim 128, block size 16, context lengths U[128, 2048], bf16,
blocks scattered over a pool of 1.1x the blocks needed.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl pkv|reference]
                    [--workload NAME] [--kv-dtype auto|fp8]

With --kv-dtype fp8 the cache holds e4m3 codes with an fp32 scale per
(block, KV head) and the step calls the _fp8 entry points; queries, new rows
and outputs keep the workload's 16-bit type.

`value` is effective GB/s of algorithmic bytes (every context token's K and V
read once, plus queries, outputs, table rows, the slot write and any
workspace traffic) over device time, with all inputs resident in HBM; the
host pool's slot appends for the timed steps are made before timing.  `e2e`
is the same metric through the public step API (PagedKVCache) from pinned
host buffers, host pool and copies included, with the host time of each part
and the loop's mode.  `allocator` is the host pool's append latency.  With
the default workload the line also carries `workloads`: the 70B-shaped GQA
batch, the long split-K contexts at block sizes 32 and 64, both decode
shapes over e4m3 caches, the shared-prefix fork and steady steps and paged
prefill, each timed the same way in the same process.  `clocks` holds the
SM clock and clock-event reasons sampled every millisecond, from the
samples inside the timed region.  Under torchrun each rank runs its own
batch (weak scaling, no collective on the data path) and the time is the
maximum over ranks.
"""
import argparse
import gc
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

METRIC = "paged decode attention effective KV GB/s (% of HBM peak); decode tok/s"
# the committed ncu summaries that give a workload's DRAM bytes per launch of
# its dominant kernel, by workload name; other workloads report traffic null
PROFILE_TRAFFIC = {
    "7b_s256_h32_d128_bs16_bf16": os.path.join(ROOT, "profiles", "decode_attention_7b_s256.md"),
    "7b_s256_h32_d128_bs16_bf16_kv_e4m3": os.path.join(ROOT, "profiles",
                                                        "decode_attention_fp8_7b_s256.md"),
    "70b_gqa_s64_hq64_hkv8_d128_bs16_bf16": os.path.join(ROOT, "profiles",
                                                          "decode_attention_gqa_70b.md"),
    "70b_gqa_s64_hq64_hkv8_d128_bs16_bf16_kv_e4m3": os.path.join(
        ROOT, "profiles", "decode_attention_fp8_gqa_70b.md"),
    "long_s8_l32768_hq32_hkv8_d128_bs32_bf16": os.path.join(ROOT, "profiles",
                                                             "decode_attention_long_bs32.md"),
    "long_s8_l32768_hq32_hkv8_d128_bs64_bf16": os.path.join(ROOT, "profiles",
                                                             "decode_attention_long_bs64.md"),
    "prefill_s8_l2048_hq32_hkv8_d128_bs16_bf16": os.path.join(ROOT, "profiles",
                                                               "prefill_attention_s8_l2048.md"),
}
# the sources whose digest a summary records: the kernel's file and the
# headers it includes
KERNEL_SOURCES = {
    "decode": ("decode_attention.cu", "common.cuh"),
    "prefill": ("prefill_attention.cu", "common.cuh", "packed_f32.cuh", "tcgen05.cuh"),
}


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=400)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["pkv", "reference"], default="pkv")
    ap.add_argument("--workload", default="7b_s256_h32_d128_bs16_bf16")
    ap.add_argument("--partition-size", type=int, default=-1,
                    help="tokens per split-K partition (0: one pass; -1: the workload's)")
    ap.add_argument("--num-seqs", type=int, default=0,
                    help="profiling only: run the workload's first N sequences")
    ap.add_argument("--kv-dtype", choices=["auto", "fp8"], default="auto",
                    help="fp8: e4m3 cache with a scale per (block, KV head)")
    ap.add_argument("--work-list", default="auto",
                    choices=["auto", "longest_first", "sequences_longest_first", "batch_order",
                             "none"],
                    help="the decode grid: PagedKVCache's work_list (auto: the full grid for "
                         "one pass, a work list with split-K)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--e2e-mode", choices=["serial", "pipelined"], default="pipelined",
                    help="e2e loop: wait for each step's output before enqueueing the next "
                         "(serial) or after (pipelined)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--extra", choices=["all", "none"], default="all",
                    help="with the default workload: also measure the other decode "
                         "workloads, e4m3 caches, the shared prefix and prefill")
    return ap.parse_args()


# ---------------------------------------------------------------------------
# distributed plumbing
# ---------------------------------------------------------------------------
def dist_setup(backend=None):
    """One process per GPU: NCCL over the GPUs, or gloo on CPU (tests)."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime

        backend = backend or ("nccl" if torch.cuda.is_available() else "gloo")
        kw = {}
        if backend == "nccl":
            torch.cuda.set_device(local)
            kw["device_id"] = torch.device("cuda", local)
        torch.distributed.init_process_group(backend, timeout=datetime.timedelta(seconds=300),
                                             **kw)
    return world, rank, local


def barrier(world):
    if world > 1:
        torch.distributed.barrier()


def max_over_ranks(x, world, device):
    if world == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(x, world, device):
    if world == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.SUM)
    return float(t.item())


# ---------------------------------------------------------------------------
# byte accounting (algorithmic bytes, not DRAM traffic)
# ---------------------------------------------------------------------------
def decode_bytes(spec, lens, partition_size, fp8=False):
    """Bytes paged decode attention must move for one step: each context
    token's K and V once (one byte per value for an e4m3 cache, plus the K
    and V scale of each (block, KV head) visited), queries, outputs, the
    table entries it follows, the context lengths, and with split-K the fp32
    partials written and read back by the merge."""
    dtb = 2
    S, Hq, Hkv, D, bs = (spec.num_seqs, spec.num_q_heads, spec.num_kv_heads, spec.head_dim,
                         spec.block_size)
    kv = sum(lens) * Hkv * D * 2 * (1 if fp8 else dtb)
    if fp8:
        kv += sum(-(-L // bs) for L in lens) * Hkv * 2 * 4
    qo = 2 * S * Hq * D * dtb
    table = sum(-(-L // bs) for L in lens) * 4 + S * 4
    ws = 0
    maxlen = max(lens)
    if partition_size and partition_size < maxlen:
        nparts = sum(-(-L // partition_size) if L > partition_size else 0 for L in lens)
        ws = nparts * Hq * (D + 2) * 4 * 2
    return kv + qo + table + ws


def write_bytes(spec, num_tokens, fp8=False):
    """Slot write: new K and V rows read and written (written as one byte per
    value, after reading the row's scale, for an e4m3 cache), plus the
    slots."""
    row = num_tokens * spec.num_kv_heads * spec.head_dim * 2  # K and V values
    if fp8:
        return row * (2 + 1) + num_tokens * spec.num_kv_heads * 2 * 4 + num_tokens * 8
    return row * 2 * 2 + num_tokens * 8


def copy_bytes(spec, num_pairs, fp8=False):
    """Block copy: each pair's K and V blocks read and written (and their
    scales for an e4m3 cache)."""
    vals = num_pairs * spec.block_size * spec.num_kv_heads * spec.head_dim * 2 * 2
    if fp8:
        return vals + num_pairs * spec.num_kv_heads * 2 * 4 * 2
    return vals * 2


# ---------------------------------------------------------------------------
# clocks during the timed region
# ---------------------------------------------------------------------------
# A child process polls NVML (read-only queries) every millisecond and
# stamps each sample with CLOCK_MONOTONIC, which the parent shares, so the
# samples taken while the timed region ran can be picked out afterwards.
# It runs apart from the benchmark's interpreter so that the GIL never
# delays a sample or a launch.
_NVML_SAMPLER = r"""
import signal, sys, time
import pynvml
pynvml.nvmlInit()
path, dt, keys = sys.argv[1], float(sys.argv[2]), sys.argv[3:]
h = None
for key in keys:  # the device's UUID first, then its NVML index
    try:
        if key.startswith(("GPU-", "MIG-")):
            h = pynvml.nvmlDeviceGetHandleByUUID(key)
        else:
            h = pynvml.nvmlDeviceGetHandleByIndex(int(key))
        break
    except pynvml.NVMLError:
        pass
if h is None:
    sys.exit(1)
stop = []
signal.signal(signal.SIGTERM, lambda *a: stop.append(1))
with open(path, "w") as f:
    f.write("max %d\n" % pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM))
    f.flush()
    while not stop:
        t = time.monotonic()
        sm = pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM)
        why = pynvml.nvmlDeviceGetCurrentClocksEventReasons(h)
        f.write("%.6f %d %d\n" % (t, sm, why))
        time.sleep(dt)
"""
# NVML clock-event reason bits, by the names the clocks record uses
_REASON_BITS = {"sw_power_cap": 0x4, "hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20,
                "hw_thermal_slowdown": 0x40, "hw_power_brake_slowdown": 0x80}


class ClockSampler:
    """SM clock and clock-event reasons sampled during a timed region.

    start() launches the sampler, mark() brackets each timed region with
    host monotonic times (taken just before the first launch and just after
    the closing synchronize, so the device work lies inside), stop() returns
    the summary of the samples inside the marked windows."""

    INTERVAL_S = 0.001

    def __init__(self, local_rank):
        vis = os.environ.get("CUDA_VISIBLE_DEVICES")
        self.keys = [vis.split(",")[local_rank].strip() if vis else str(local_rank)]
        try:
            uuid = str(torch.cuda.get_device_properties(local_rank).uuid)
            self.keys.insert(0, uuid if uuid.startswith("GPU-") else "GPU-" + uuid)
        except (AttributeError, RuntimeError, AssertionError):
            pass
        self.proc = None
        self.path = None
        self.windows = []

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".clk")
            os.close(fd)
            self.proc = subprocess.Popen(
                [sys.executable, "-c", _NVML_SAMPLER, self.path, str(self.INTERVAL_S)] +
                self.keys, stdout=subprocess.DEVNULL, stderr=subprocess.DEVNULL)
        except (OSError, ValueError):
            self.proc = None
            return
        # wait (bounded) until the sampler has its handle and is polling
        t0 = time.monotonic()
        while time.monotonic() - t0 < 10.0 and self.proc.poll() is None:
            try:
                with open(self.path) as f:
                    if len(f.read().splitlines()) >= 3:
                        break
            except OSError:
                pass
            time.sleep(0.02)

    def window(self, t0, t1):
        self.windows.append((t0, t1))

    def stop(self):
        if self.proc is None:
            return None
        if self.proc.poll() is None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                self.proc.wait()
        smax, rows = None, []
        try:
            with open(self.path) as f:
                for line in f:
                    parts = line.split()
                    if parts[:1] == ["max"] and len(parts) == 2:
                        smax = float(parts[1])
                    elif len(parts) == 3:
                        rows.append((float(parts[0]), float(parts[1]), int(parts[2])))
            os.unlink(self.path)
        except (OSError, ValueError):
            return None
        inside = [r for r in rows if any(a <= r[0] <= b for a, b in self.windows)]
        use = inside or rows
        if not use:
            return None
        reasons = sorted(n for n, bit in _REASON_BITS.items() if any(r[2] & bit for r in use))
        return {"sm_mhz": statistics.median(r[1] for r in use), "sm_max_mhz": smax,
                "reasons": reasons, "samples": len(inside), "samples_total": len(rows),
                "interval_ms": 1e3 * self.INTERVAL_S,
                "source": "NVML, samples inside the timed region" if inside else
                          "NVML, no sample inside the timed region: all samples"}


def measured_peak():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except (OSError, KeyError, ValueError):
        return 6650.0, "fallback"


def profiled_traffic(source_digest, workload):
    """DRAM bytes per launch of the workload's dominant kernel from its
    committed ncu summary, or None when there is none or it was taken on
    other kernel source."""
    try:
        with open(PROFILE_TRAFFIC[workload]) as f:
            text = f.read()
    except (KeyError, OSError):
        return None
    vals = {}
    for line in text.splitlines():
        line = line.strip().strip("`").strip("-").strip()
        if ":" in line:
            k, v = line.split(":", 1)
            vals[k.strip()] = v.strip()
    if vals.get("kernel_source_sha256") != source_digest:
        return None
    try:
        return float(vals["dram_bytes_per_launch_full_size"])
    except (KeyError, ValueError):
        return None


def kernel_source_digest(kernel="decode"):
    import hashlib

    h = hashlib.sha256()
    for name in KERNEL_SOURCES[kernel]:
        with open(os.path.join(ROOT, "paged_kv_cache_337_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


# ---------------------------------------------------------------------------
# CPU oracle timing (baseline, not a target)
# ---------------------------------------------------------------------------
def oracle_sample_problem(spec, lens, seed, fp8=False):
    """A compact copy of the workload's first sequences for the CPU oracle:
    the same lengths and shapes, scattered over a small pool (e4m3 codes and
    per-(block, KV head) scales for an e4m3 cache)."""
    import numpy as np

    g = torch.Generator().manual_seed(seed)
    bs = spec.block_size
    need = sum(-(-L // bs) for L in lens)
    nb = need + 1
    perm = torch.randperm(nb, generator=g).tolist()
    mb = max(-(-L // bs) for L in lens)
    tables = np.full((len(lens), mb), -1, np.int32)
    i = 0
    for s, L in enumerate(lens):
        for j in range(-(-L // bs)):
            tables[s, j] = perm[i]
            i += 1
    dt = spec.torch_dtype
    shape = (nb, bs, spec.num_kv_heads, spec.head_dim)
    q = torch.randn(len(lens), spec.num_q_heads, spec.head_dim, generator=g).to(dt)
    prob = dict(q=q, tables=tables, lens=np.asarray(lens, np.int32))
    if not fp8:
        prob["kc"] = torch.randn(shape, generator=g).to(dt)
        prob["vc"] = torch.randn(shape, generator=g).to(dt)
        return prob
    for c in ("k", "v"):
        sc = (0.75 + 0.5 * torch.rand(nb, spec.num_kv_heads, generator=g)) * (4.0 / 448.0)
        x = (torch.randn(shape, generator=g) / sc[:, None, :, None]).clamp_(-448.0, 448.0)
        prob[c + "c"] = x.to(torch.float8_e4m3fn).view(torch.uint8)
        prob[c + "s"] = sc.numpy().astype(np.float32)
    return prob


def oracle_step(spec, prob, fp8=False):
    """One decode step of the oracle (all host cores) on a sample problem."""
    from oracle import reference as ref

    if fp8:
        return ref.decode_attention_fp8(prob["q"], prob["kc"], prob["vc"], prob["ks"],
                                        prob["vs"], prob["tables"], prob["lens"], spec.scale,
                                        spec.dtype, spec.num_kv_heads, spec.block_size)
    return ref.decode_attention(prob["q"], prob["kc"], prob["vc"], prob["tables"], prob["lens"],
                                spec.scale, spec.dtype, spec.num_kv_heads, spec.block_size,
                                num_threads=0)


def time_oracle(spec, lens, target_s, fp8=False):
    """Times the fp64 oracle (all host cores) on the first n sequences, n
    grown until one call takes about target_s seconds.  Returns (GB/s,
    seconds, n, reps, cores)."""
    from oracle import reference as ref

    n = 1
    while True:
        prob = oracle_sample_problem(spec, lens[:n], 7, fp8)
        t0 = time.perf_counter()
        oracle_step(spec, prob, fp8)
        dt = time.perf_counter() - t0
        if dt >= 0.5 * target_s or n >= len(lens):
            break
        n = min(len(lens), max(n + 1, int(n * target_s / max(dt, 1e-3))))
    # the whole batch may take less than the target: repeat the step
    reps, total = 1, dt
    while total < 0.8 * target_s:
        t0 = time.perf_counter()
        oracle_step(spec, prob, fp8)
        total += time.perf_counter() - t0
        reps += 1
    byts = decode_bytes(spec, list(lens[:n]), 0, fp8) * reps
    return byts / total / 1e9, total, n, reps, ref.max_threads()


def workload_name(spec, fp8):
    return spec.name + ("_kv_e4m3" if fp8 else "")


# ---------------------------------------------------------------------------
# the reference arm: the oracle as it stands, on the host cores
# ---------------------------------------------------------------------------
def run_reference(args, spec, world, rank):
    if rank != 0:
        return
    from paged_kv_cache_337_b200 import workloads as W

    gen = torch.Generator("cpu").manual_seed(spec.seed)
    lens = W.draw_lens(spec, gen).tolist()
    per_step = max(0.2, min(10.0, 120.0 / max(1, args.steps + args.warmup)))
    fp8 = args.kv_dtype == "fp8"
    gbs, dt, n, reps, cores = time_oracle(spec, lens, per_step, fp8)
    prob = oracle_sample_problem(spec, lens[:n], 11, fp8)

    times = []
    for i in range(args.warmup + args.steps):
        t0 = time.perf_counter()
        oracle_step(spec, prob, fp8)
        if i >= args.warmup:
            times.append(time.perf_counter() - t0)
    byts = decode_bytes(spec, lens[:n], 0, fp8)
    value = byts * len(times) / sum(times) / 1e9
    sample = "first %d of %d sequences (all %d query heads), one decode step each" % (
        n, spec.num_seqs, spec.num_q_heads)
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": "GB/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(1e3 * sum(times) / len(times), 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": workload_name(spec, fp8),
                   "oracle": "fp64 C oracle, OpenMP over (seq, head)", "sample": sample},
        "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": cores,
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------
# the product arm
# ---------------------------------------------------------------------------
def cache_work_list(args):
    return False if args.work_list == "none" else args.work_list


def grid_label(args, P, max_len, fp8):
    """What the decode launch runs over, as PagedKVCache's work_list picks
    it for this workload."""
    wl = args.work_list
    if wl == "auto":
        if not 0 < P < max_len:
            return "full grid (one pass per sequence)"
        wl = "sequences_longest_first"
    if wl == "none":
        return "full grid"
    return "work list of the (sequence, KV head, partition) items holding tokens, " + {
        "longest_first": "longest first",
        "sequences_longest_first": "sequences longest first",
        "batch_order": "sequences in batch order"}[wl]


def allocator_latency(spec, lens, order, rank):
    """Block-allocation latency of the host pool (the metric the "PagedAttention
    动态内存分页" page lists under 性能监控要点): microseconds per batched append
    (one token for every sequence of the batch, new blocks taken from the
    pool as they fill) and per single-sequence append, both through the
    Python binding, on a pool in the workload's state."""
    from paged_kv_cache_337_b200 import _abi

    S, bs = spec.num_seqs, spec.block_size
    nb = len(order)
    pool = _abi.BlockPool(nb, bs, order)
    for s in range(S):
        pool.add(s, int(lens[s]) - 1)
    ids = torch.arange(S, dtype=torch.int64)
    slots = torch.empty(S, dtype=torch.int64)
    pairs = torch.empty((S, 2), dtype=torch.int32)
    # stay within the pool's spare blocks: each round may take one per sequence
    spare = pool.num_free() // max(1, S)
    rounds = max(1, min(64, spare * bs // 2))
    for _ in range(2):
        pool.append_batch(ids, slots, pairs)
    t0 = time.perf_counter()
    for _ in range(rounds):
        pool.append_batch(ids, slots, pairs)
    batch_us = 1e6 * (time.perf_counter() - t0) / rounds
    singles = min(S * 4, max(1, (pool.num_free() // 2) * bs))
    t0 = time.perf_counter()
    for i in range(singles):
        pool.append(i % S)
    single_us = 1e6 * (time.perf_counter() - t0) / singles
    pool.close()
    return {"append_batch_us": round(batch_us, 2), "batch": S,
            "per_sequence_us": round(batch_us / S, 4), "append_single_us": round(single_us, 3),
            "batches_timed": rounds, "singles_timed": singles,
            "what": "host pool, Python binding included: one slot per sequence, a new block "
                    "from the pool when the last one is full"}


def run_e2e(args, spec, cache, ids, steps, stream, P, fp8, world, dev):
    """The decode step end to end through the public step API, from pinned
    host memory.  Per step: the step's q, k and v go up in one copy from
    pinned memory (on an upload stream, into one of two input buffers,
    issued while the previous step computes), the host pool reserves the
    slots and plans the work list (PagedKVCache.prepare_step, one native
    call), and one more native call (PagedKVCache.run_step) uploads the
    metadata on the upload stream, runs the kernels and copies the
    attention output back to pinned host memory on a readback stream,
    where the copy overlaps the next step's kernels; the host waits for it.
    (run_step can take the q/k/v copy too, `inputs=`; issued with the step
    rather than a step ahead, it measured slower on the shortest steps.)

    serial: the host waits for step i's output before it enqueues step i+1
    (the pool's work for step i+1 and its input upload still overlap step
    i on the GPU).  pipelined: step i+1 is enqueued before the host waits
    for step i's output (two output buffers), so the GPU goes from step to
    step without waiting for the host.  Returns the e2e record with the
    host time of each part."""
    S, Hq, Hkv, D = spec.num_seqs, spec.num_q_heads, spec.num_kv_heads, spec.head_dim
    dt = spec.torch_dtype
    pipelined = args.e2e_mode == "pipelined"
    nq, nk = S * Hq * D, S * Hkv * D
    h_in = [torch.randn(nq + 2 * nk).to(dt).pin_memory() for _ in range(2)]
    d_in = [torch.empty(nq + 2 * nk, dtype=dt, device=dev) for _ in range(2)]
    views = [(b[:nq].view(S, Hq, D), b[nq:nq + nk].view(S, Hkv, D),
              b[nq + nk:].view(S, Hkv, D)) for b in d_in]
    nout = 2 if pipelined else 1
    outs = [torch.empty((S, Hq, D), dtype=dt, device=dev) for _ in range(nout)]
    houts = [torch.empty((S, Hq, D), dtype=dt).pin_memory() for _ in range(nout)]
    upload_stream = torch.cuda.Stream(dev)
    readback_stream = torch.cuda.Stream(dev)
    ev_in = [torch.cuda.Event() for _ in range(2)]    # inputs of buffer b uploaded
    ev_used = [torch.cuda.Event() for _ in range(2)]  # the step using buffer b done
    ev_out = [torch.cuda.Event() for _ in range(nout)]  # a step's result on the host
    e2e_bytes = h2d = d2h = 0
    host = {"prepare": 0.0, "enqueue": 0.0, "input_upload_enqueue": 0.0, "wait": 0.0}

    def timed(key, fn, *a):
        t = time.perf_counter()
        r = fn(*a)
        host[key] += time.perf_counter() - t
        return r

    def enqueue(i, prep):
        b, o = i % 2, i % nout
        stream.wait_event(ev_in[b])
        if i >= nout:
            stream.wait_event(ev_out[o])  # step i - nout's readback has read outs[o]
        dq, dk, dv = views[b]
        # metadata upload, copies, slot write, attention and readback: one call
        cache.run_step(prep, dq, dk, dv, outs[o], out_host=houts[o], stream=stream,
                       readback_stream=readback_stream, upload_stream=upload_stream)
        ev_used[b].record(stream)
        ev_out[o].record(readback_stream)

    def upload_inputs(i):
        b = i % 2
        with torch.cuda.stream(upload_stream):
            if i >= 2:
                upload_stream.wait_event(ev_used[b])  # step i - 2 done with the buffer
            d_in[b].copy_(h_in[i % 2], non_blocking=True)
            ev_in[b].record(upload_stream)

    barrier(world)
    torch.cuda.synchronize(dev)
    # Python's collector runs before the timed loop, not inside it: a full
    # collection over this process's heap pauses the host for milliseconds
    gc.collect()
    gc.disable()
    t0 = time.perf_counter()
    timed("input_upload_enqueue", upload_inputs, 0)
    prep = timed("prepare", cache.prepare_step, ids)
    for i in range(steps):
        timed("enqueue", enqueue, i, prep)
        lens = prep["st"]["h_lens"].tolist()
        e2e_bytes += (decode_bytes(spec, lens, P, fp8) + write_bytes(spec, S, fp8) +
                      copy_bytes(spec, prep["num_pairs"], fp8))
        used = prep["st"]["items_off"] + max(prep["num_items"], 0)
        h2d = d_in[i % 2].numel() * 2 + used * 4
        d2h = houts[0].numel() * 2
        if pipelined and i >= 1:
            timed("wait", ev_out[(i - 1) % nout].synchronize)  # step i - 1's result
        if i + 1 < steps:
            timed("input_upload_enqueue", upload_inputs, i + 1)
            prep = timed("prepare", cache.prepare_step, ids)  # overlaps step i on the GPU
        if not pipelined:
            timed("wait", ev_out[0].synchronize)
    if pipelined:
        timed("wait", ev_out[(steps - 1) % nout].synchronize)
    e2e_s = time.perf_counter() - t0
    gc.enable()
    barrier(world)
    e2e_s = max_over_ranks(e2e_s, world, dev)
    e2e_total = sum_over_ranks(e2e_bytes, world, dev)
    return {"value": round(e2e_total / e2e_s / 1e9, 2), "unit": "GB/s",
            "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
            "steps": steps, "ms_per_step": round(1e3 * e2e_s / steps, 4), "mode": args.e2e_mode,
            "python_gc": "collected before the timed loop, paused during it",
            "host_ms_per_step": {
                "pool_append_tables_and_work_list": round(1e3 * host["prepare"] / steps, 4),
                "step_enqueue": round(1e3 * host["enqueue"] / steps, 4),
                "input_upload_enqueue": round(1e3 * host["input_upload_enqueue"] / steps, 4),
                "readback_wait": round(1e3 * host["wait"] / steps, 4)}}


def pool_memory(pool, ids, block_size, num_blocks, max_len):
    """KV memory of the host pool ("PagedAttention 动态内存分页" page, 性能监控要点:
    GPU memory utilisation): blocks handed out, the token slots they hold,
    the tokens the sequences have written (logical: a shared block counts
    once per sequence, so utilisation passes 1 with sharing), the slots of a
    sequence's last block that hold none (at most block_size - 1), and the
    slots a contiguous reservation of max_len tokens per sequence would
    hold ("一文读懂vLLM..." page: what paging replaces)."""
    free = pool.num_free()
    used_blocks = num_blocks - free
    tokens = sum(pool.num_tokens(s) for s in ids)
    slots = used_blocks * block_size
    waste = [(-pool.num_tokens(s)) % block_size for s in ids]
    contiguous = len(ids) * max_len
    return {"blocks_in_use": used_blocks, "blocks_free": free, "slots_in_use": slots,
            "tokens": tokens, "utilization": round(tokens / slots, 4) if slots else None,
            "empty_slots_per_sequence_max": max(waste) if waste else 0,
            "empty_slots_per_sequence_mean": round(sum(waste) / len(waste), 2) if waste else 0,
            "contiguous_prealloc_slots": contiguous,
            "contiguous_prealloc_utilization": round(tokens / contiguous, 4) if contiguous else None}


def run_pkv(args, spec, world, rank, local, fp8=False, with_cpu=True, with_alloc=True):
    """One decode workload: returns its JSON line (rank 0) or None."""
    from paged_kv_cache_337_b200 import _abi
    from paged_kv_cache_337_b200 import workloads as W
    from paged_kv_cache_337_b200.cache import PagedKVCache

    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    _abi.lib()
    P = spec.partition_for(fp8) if args.partition_size < 0 else args.partition_size

    # seeded shapes on the CPU; cache values drawn on the device (per rank)
    gen = torch.Generator("cpu").manual_seed(spec.seed)
    lens0 = W.draw_lens(spec, gen).tolist()
    nb = W.pool_size(spec, lens0)
    order = torch.randperm(nb, generator=gen, dtype=torch.int64).to(torch.int32)
    S, Hq, Hkv, D, bs = (spec.num_seqs, spec.num_q_heads, spec.num_kv_heads, spec.head_dim,
                         spec.block_size)
    n_states = 16  # decode steps whose metadata is prepared (one block's worth)
    e2e_steps = 0 if args.no_e2e else min(args.steps, 48)
    mb = spec.max_blocks_per_seq + -(-(n_states + e2e_steps + 2) // bs)
    cache = PagedKVCache(nb, bs, Hq, Hkv, D, spec.torch_dtype, dev, mb, P,
                         free_order=order.tolist(), scale=spec.scale,
                         kv_dtype=torch.uint8 if fp8 else None,
                         work_list=cache_work_list(args))
    if fp8:
        W.fill_device_scales_(cache.k_scale, spec.seed * 10 + 2 * rank + 5)
        W.fill_device_scales_(cache.v_scale, spec.seed * 10 + 2 * rank + 6)
        W.fill_device_cache_fp8_(cache.key_cache, cache.k_scale, spec.seed * 10 + 2 * rank)
        W.fill_device_cache_fp8_(cache.value_cache, cache.v_scale, spec.seed * 10 + 2 * rank + 1)
    else:
        W.fill_device_cache_(cache.key_cache, spec.seed * 10 + 2 * rank)
        W.fill_device_cache_(cache.value_cache, spec.seed * 10 + 2 * rank + 1)
    ids = list(range(S))
    for s in ids:
        cache.add_sequence(s, lens0[s] - 1)

    stream = torch.cuda.Stream(dev)
    dgen = torch.Generator(dev).manual_seed(spec.seed + 100 * rank)
    dt = spec.torch_dtype

    # prepare n_states consecutive steps: the host pool really appends one
    # token per sequence each time; the step replays them cyclically
    states = []
    for j in range(n_states):
        prep = cache.prepare_step(ids)
        st = prep["st"]
        npairs = prep["num_pairs"]
        lens = st["h_lens"].tolist()
        n_items = prep["num_items"]
        states.append(dict(
            slots=st["h_slots"].to(dev), pairs=st["h_pairs"][:npairs].to(dev),
            tables=st["h_tables"].to(dev), lens=st["h_lens"].to(dev), max_len=max(lens),
            items=st["h_items"][:n_items].to(dev) if n_items >= 0 else None,
            q=torch.randn((S, Hq, D), generator=dgen, device=dev).to(dt),
            k=torch.randn((S, Hkv, D), generator=dgen, device=dev).to(dt),
            v=torch.randn((S, Hkv, D), generator=dgen, device=dev).to(dt),
            bytes_decode=decode_bytes(spec, lens, P, fp8),
            bytes_step=decode_bytes(spec, lens, P, fp8) + write_bytes(spec, S, fp8) +
            copy_bytes(spec, npairs, fp8), npairs=npairs, lens_sum=sum(lens)))
    max_len_all = max(s["max_len"] for s in states)
    ws_bytes = _abi.pkv_decode_workspace_bytes(S, Hq, max_len_all, P, D)
    ws = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device=dev) if ws_bytes else None
    out = torch.empty((S, Hq, D), dtype=dt, device=dev)
    err = cache.dev_error
    kc, vc = cache.key_cache, cache.value_cache

    ks, vs = cache.k_scale, cache.v_scale

    def step(state, ev=None):
        if state["npairs"]:
            if fp8:
                _abi.pkv_copy_blocks_fp8(kc, vc, ks, vs, state["pairs"], dev_error=err,
                                         stream=stream)
            else:
                _abi.pkv_copy_blocks(kc, vc, state["pairs"], dev_error=err, stream=stream)
        if fp8:
            _abi.pkv_write_slots_fp8(state["k"], state["v"], kc, vc, ks, vs, state["slots"],
                                     dev_error=err, stream=stream)
        else:
            _abi.pkv_write_slots(state["k"], state["v"], kc, vc, state["slots"], dev_error=err,
                                 stream=stream)
        if ev is not None:
            ev[0].record(stream)
        if fp8:
            _abi.pkv_decode_attention_fp8(out, state["q"], kc, vc, ks, vs, state["tables"],
                                          state["lens"], state["max_len"], spec.scale, P, ws,
                                          dev_error=err, stream=stream,
                                          work_items=state["items"])
        else:
            _abi.pkv_decode_attention(out, state["q"], kc, vc, state["tables"], state["lens"],
                                      state["max_len"], spec.scale, P, ws, dev_error=err,
                                      stream=stream, work_items=state["items"])
        if ev is not None:
            ev[1].record(stream)
        # copy-on-write: a bytes kernel, plus a scale kernel for e4m3 caches
        return (((2 if fp8 else 1) if state["npairs"] else 0)) + 2

    # inputs and caches were made on the default stream; the timed
    # stream is not ordered after it
    torch.cuda.synchronize(dev)
    for i in range(args.warmup):
        step(states[i % n_states])
    torch.cuda.synchronize(dev)

    clocks = ClockSampler(local) if rank == 0 else None
    if clocks:
        clocks.start()
    K = args.steps
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(K)]
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    launches = 0
    bytes_step = bytes_decode = 0
    barrier(world)
    torch.cuda.synchronize(dev)
    h0 = time.monotonic()
    t_start.record(stream)
    for i in range(K):
        stt = states[(args.warmup + i) % n_states]
        launches += step(stt, evs[i])
        bytes_step += stt["bytes_step"]
        bytes_decode += stt["bytes_decode"]
    t_end.record(stream)
    torch.cuda.synchronize(dev)
    if clocks:
        clocks.window(h0, time.monotonic())
    barrier(world)
    clock_info = clocks.stop() if clocks else None
    elapsed_ms = t_start.elapsed_time(t_end)
    decode_ms = sum(a.elapsed_time(b) for a, b in evs)
    cache.check_errors()

    t_max = max_over_ranks(elapsed_ms, world, dev)
    total_bytes = sum_over_ranks(bytes_step, world, dev)
    value = total_bytes / (t_max * 1e-3) / 1e9
    ms_per_step = t_max / K
    decode_gbs = bytes_decode / (decode_ms * 1e-3) / 1e9
    peak, peak_kind = measured_peak()
    tok_s = world * S * K / (t_max * 1e-3)

    # ---- end to end through the public step API from pinned host memory ----
    e2e = None
    if e2e_steps:
        e2e = run_e2e(args, spec, cache, ids, e2e_steps, stream, P, fp8, world, dev)
        e2e["device_ms_per_step"] = round(ms_per_step, 4)
        cache.check_errors()

    cpu = None
    if rank == 0 and world == 1 and with_cpu and not args.no_cpu_baseline:
        gbs, secs, n, reps, cores = time_oracle(spec, lens0, 10.0, fp8)
        cpu = {"value": round(gbs, 4), "unit": "GB/s", "cores": cores, "kind": "oracle",
               "sample": "first %d of %d sequences (all %d query heads), decode step "
                         "repeated %d times, %.1f s" % (n, S, Hq, reps, secs)}
    alloc = allocator_latency(spec, lens0, order.tolist(), rank) if with_alloc else None
    memory = pool_memory(cache.pool, ids, bs, nb, spec.len_hi)

    if rank != 0:
        return None
    traffic = profiled_traffic(kernel_source_digest(), workload_name(spec, fp8))
    line = {
        "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world,
        "steps": K, "warmup": args.warmup, "ms_per_step": round(ms_per_step, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "e4m3" if fp8 else "bf16" if dt == torch.bfloat16 else "f16",
        "data": "synthetic",
        "config": {
            "workload": workload_name(spec, fp8), "num_seqs": S, "num_q_heads": Hq,
            "num_kv_heads": Hkv, "head_dim": D, "block_size": bs,
            "context_lens": "U[%d,%d]" % (spec.len_lo, spec.len_hi),
            "pool_blocks": nb, "partition_size": P,
            "grid": grid_label(args, P, max_len_all, fp8),
            "kv_cache": ("e4m3, fp32 scale per (block, KV head)" if fp8 else
                         "bf16" if dt == torch.bfloat16 else "f16"),
            "step": "slot write + paged decode attention (+ copy-on-write copies; split-K "
                    "partitions merged in-kernel); the host pool's slot appends are done "
                    "before timing, so value holds device work only and e2e holds the pool",
            "l2": "inputs larger than L2 (%.2f GB of K/V read per step)" % (
                states[0]["lens_sum"] * Hkv * D * (2 if fp8 else 4) / 1e9),
            "states": "%d consecutive decode steps prepared by the host pool, replayed "
                      "cyclically" % n_states},
        "pct_hbm_peak": round(100 * value / (world * peak), 2),
        "decode_tok_s": round(tok_s, 1),
        "roofline": {"bound": "hbm", "achieved": round(decode_gbs, 2), "peak": peak,
                     "unit": "GB/s", "frac": round(decode_gbs / peak, 4),
                     "traffic": traffic, "kernel": "paged_decode_kernel",
                     "peak_source": peak_kind},
        "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": launches, "clocks": clock_info,
        "memory": memory,
    }
    if alloc is not None:
        line["allocator"] = alloc
    return line


SWAP_WORKLOAD = "swap_7b_s256_q64_h32_d128_bs16_bf16"
COW_LAYERS_WORKLOAD = "cow_layers_l32_p112_h32_d128_bs16_bf16"


def run_cow_layers(args, world, rank, local):
    """Copy-on-write over a 32-layer cache: the shared-prefix fork step's 112
    (src, dst) pairs copied in every layer by one pkv_copy_blocks_layers
    launch, against 32 pkv_copy_blocks launches.  `value` is the bytes
    moved (each pair's K and V block read and written, every layer) over
    the device time of the one-launch copy; the roofline peak is HBM."""
    from paged_kv_cache_337_b200 import _abi

    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    _abi.lib()
    layers, pairs_n, nb, bs, hkv, d = 32, 112, 2048, 16, 32, 128
    dt = torch.bfloat16
    g = torch.Generator(dev).manual_seed(4000 + rank)
    ks = [torch.empty((nb, bs, hkv, d), dtype=dt, device=dev) for _ in range(layers)]
    vs = [torch.empty((nb, bs, hkv, d), dtype=dt, device=dev) for _ in range(layers)]
    for t in ks + vs:
        t.view(-1)[:: 4096].normal_(generator=g)
    perm = torch.randperm(nb, generator=torch.Generator().manual_seed(4100 + rank))
    pairs = torch.stack([perm[:pairs_n], perm[pairs_n:2 * pairs_n]], 1).to(torch.int32).to(dev)
    kp, vp = _abi.layer_pointers(ks, dev), _abi.layer_pointers(vs, dev)
    err = torch.zeros(2, dtype=torch.int32, device=dev)
    stream = torch.cuda.Stream(dev)
    step_bytes = pairs_n * layers * 2 * 2 * bs * hkv * d * 2

    def one_launch():
        _abi.pkv_copy_blocks_layers(ks, vs, pairs, dev_error=err, stream=stream, key_ptrs=kp,
                                    value_ptrs=vp)

    def per_layer():
        for l in range(layers):
            _abi.pkv_copy_blocks(ks[l], vs[l], pairs, dev_error=err, stream=stream)

    def timed(fn, K):
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(K)]
        # inputs and caches were made on the default stream; the timed
        # stream is not ordered after it
        torch.cuda.synchronize(dev)
        for _ in range(args.warmup):
            fn()
        torch.cuda.synchronize(dev)
        for a, b in evs:
            a.record(stream)
            fn()
            b.record(stream)
        torch.cuda.synchronize(dev)
        return sum(a.elapsed_time(b) for a, b in evs) / K

    clocks = ClockSampler(local) if rank == 0 else None
    if clocks:
        clocks.start()
    barrier(world)
    K = args.steps
    h0 = time.monotonic()
    ms = timed(one_launch, K)
    ms_layers = timed(per_layer, K)
    if clocks:
        clocks.window(h0, time.monotonic())
    barrier(world)
    clock_info = clocks.stop() if clocks else None
    t_max = max_over_ranks(ms, world, dev)
    value = sum_over_ranks(step_bytes, world, dev) / (t_max * 1e-3) / 1e9
    peak, peak_kind = measured_peak()
    if err.tolist() != [0, 0]:
        raise RuntimeError("device error %s" % err.tolist())
    if rank == 0:
        line = {
            "metric": "multi-layer copy-on-write GB/s (read + write)", "value": round(value, 2),
            "unit": "GB/s", "n_gpus": world, "steps": K, "warmup": args.warmup,
            "ms_per_step": round(t_max, 4), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": COW_LAYERS_WORKLOAD, "layers": layers, "pairs": pairs_n,
                       "block_bytes_kv": 2 * bs * hkv * d * 2, "step_gb": step_bytes / 1e9,
                       "per_layer_launches_ms": round(ms_layers, 4)},
            "roofline": {"bound": "hbm", "achieved": round(value, 2), "peak": peak,
                         "unit": "GB/s", "frac": round(value / peak, 4), "traffic": None,
                         "kernel": "copy_blocks_layers_kernel", "peak_source": peak_kind},
            "e2e": None, "cpu_baseline": None, "gpu_launches": K * (1 + layers),
            "clocks": clock_info,
        }
        print(json.dumps(line), flush=True)


def host_link_peak(dev, nbytes=1 << 30):
    """Copy-engine bandwidth of one large pinned <-> device copy each way
    (cudaMemcpyAsync through torch), GB/s: the host link's practical peak."""
    h = torch.empty(nbytes, dtype=torch.uint8).pin_memory()
    d = torch.empty(nbytes, dtype=torch.uint8, device=dev)
    out = {}
    for name, (dst, src) in (("d2h", (h, d)), ("h2d", (d, h))):
        dst.copy_(src, non_blocking=True)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        times = []
        for _ in range(3):
            a.record()
            dst.copy_(src, non_blocking=True)
            b.record()
            torch.cuda.synchronize(dev)
            times.append(a.elapsed_time(b))
        out[name] = nbytes / (min(times) * 1e-3) / 1e9
    del h, d
    return out


def run_swap(args, world, rank, local):
    """Block swap of the 7B-shaped batch: each step swaps the first 64 of
    the 256 sequences out to pinned host memory and back in
    (pkv_seq_swap_out / _in on the host pool, one pkv_swap_blocks launch
    per direction).  `value` is the bytes moved (K and V blocks, both
    directions) over the swap kernels' device time; the roofline peak is
    the copy engine's bandwidth for one 1 GiB pinned copy each way, measured
    in the same run.  `e2e` times PagedKVCache.swap_out / swap_in from the
    host, pool bookkeeping and pair upload included."""
    from paged_kv_cache_337_b200 import _abi
    from paged_kv_cache_337_b200 import workloads as W
    from paged_kv_cache_337_b200.cache import PagedKVCache

    spec = W.SPECS["7b_s256_h32_d128_bs16_bf16"]
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    _abi.lib()
    gen = torch.Generator("cpu").manual_seed(spec.seed)
    lens = W.draw_lens(spec, gen).tolist()
    nb = W.pool_size(spec, lens)
    order = torch.randperm(nb, generator=gen, dtype=torch.int64).to(torch.int32)
    S, Hq, Hkv, D, bs = (spec.num_seqs, spec.num_q_heads, spec.num_kv_heads, spec.head_dim,
                         spec.block_size)
    moved = list(range(64))
    host_blocks = sum(-(-lens[s] // bs) for s in moved)
    cache = PagedKVCache(nb, bs, Hq, Hkv, D, spec.torch_dtype, dev, spec.max_blocks_per_seq,
                         0, free_order=order.tolist(), scale=spec.scale)
    W.fill_device_cache_(cache.key_cache, spec.seed * 10 + 2 * rank)
    W.fill_device_cache_(cache.value_cache, spec.seed * 10 + 2 * rank + 1)
    cache.enable_swap(host_blocks)
    for s in range(S):
        cache.add_sequence(s, lens[s])
    block_bytes = bs * Hkv * D * cache.key_cache.element_size()
    stream = torch.cuda.Stream(dev)
    err = cache.dev_error
    kc, vc, hk, hv = cache.key_cache, cache.value_cache, cache.host_key_cache, cache.host_value_cache

    def step(ev=None):
        with torch.cuda.stream(stream):  # the pairs go up on the stream that reads them
            pairs = torch.cat([cache.pool.swap_out(s) for s in moved]).to(dev)
        if ev:
            ev[0].record(stream)
        _abi.pkv_swap_blocks(kc, vc, hk, hv, pairs, dev_error=err, stream=stream)
        if ev:
            ev[1].record(stream)
        with torch.cuda.stream(stream):
            pairs = torch.cat([cache.pool.swap_in(s) for s in moved]).to(dev)
        if ev:
            ev[2].record(stream)
        _abi.pkv_swap_blocks(hk, hv, kc, vc, pairs, dev_error=err, stream=stream)
        if ev:
            ev[3].record(stream)
        return 2 * pairs.shape[0] * 2 * block_bytes

    # inputs and caches were made on the default stream; the timed
    # stream is not ordered after it
    torch.cuda.synchronize(dev)
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    clocks = ClockSampler(local) if rank == 0 else None
    if clocks:
        clocks.start()
    K = args.steps
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(K)]
    barrier(world)
    torch.cuda.synchronize(dev)
    h0 = time.monotonic()
    total = 0
    for i in range(K):
        total += step(evs[i])
    torch.cuda.synchronize(dev)
    if clocks:
        clocks.window(h0, time.monotonic())
    barrier(world)
    clock_info = clocks.stop() if clocks else None
    out_ms = sum(e[0].elapsed_time(e[1]) for e in evs)
    in_ms = sum(e[2].elapsed_time(e[3]) for e in evs)
    cache.check_errors()
    t_max = max_over_ranks(out_ms + in_ms, world, dev)
    value = sum_over_ranks(total, world, dev) / (t_max * 1e-3) / 1e9
    per_dir = total / 2
    out_gbs = per_dir / (out_ms * 1e-3) / 1e9
    in_gbs = per_dir / (in_ms * 1e-3) / 1e9
    step_bytes = total // K  # both directions, one step

    # end to end through the driver: pool bookkeeping + pair upload + kernel
    e2e_steps = min(K, 10)
    barrier(world)
    torch.cuda.synchronize(dev)
    t0 = time.perf_counter()
    for _ in range(e2e_steps):
        cache.swap_out(moved, stream=stream)
        cache.swap_in(moved, stream=stream)
    torch.cuda.synchronize(dev)
    e2e_s = max_over_ranks(time.perf_counter() - t0, world, dev)
    cache.check_errors()
    peak = host_link_peak(dev)
    if rank == 0:
        peak_both = 2 / (1 / peak["d2h"] + 1 / peak["h2d"])  # same bytes each way
        line = {
            "metric": "block swap GB/s (K/V blocks to pinned host memory and back)",
            "value": round(value, 2), "unit": "GB/s", "n_gpus": world, "steps": K,
            "warmup": args.warmup, "ms_per_step": round(t_max / K, 4),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16", "data": "synthetic",
            "config": {"workload": SWAP_WORKLOAD, "num_seqs": S, "swapped_seqs": len(moved),
                       "blocks_per_direction": int(step_bytes // (2 * 2 * block_bytes)),
                       "block_bytes_kv": 2 * block_bytes, "pool_blocks": nb,
                       "step": "swap-out of 64 sequences then swap-in (new GPU blocks)"},
            "swap_out_gbs": round(out_gbs, 2), "swap_in_gbs": round(in_gbs, 2),
            "roofline": {"bound": "host-link", "achieved": round(value, 2),
                         "peak": round(peak_both, 2), "unit": "GB/s",
                         "frac": round(value / peak_both, 4), "traffic": None,
                         "kernel": "swap_blocks_kernel",
                         "peak_source": "measured in this run: 1 GiB pinned copy, "
                                        "d2h %.1f / h2d %.1f GB/s" % (peak["d2h"], peak["h2d"])},
            "e2e": {"value": round(e2e_steps * step_bytes / e2e_s / 1e9, 2), "unit": "GB/s",
                    "h2d_bytes_per_step": int(step_bytes // 2),
                    "d2h_bytes_per_step": int(step_bytes // 2)},
            "gpu_launches": 2 * K, "clocks": clock_info, "cpu_baseline": None,
        }
        print(json.dumps(line), flush=True)


PREFILL_WORKLOAD = "prefill_s8_l2048_hq32_hkv8_d128_bs16_bf16"


def prefill_flops(lens, n, Hq, D):
    """Algorithmic FLOPs of causal attention: for each query row at
    position p, S (p + 1 dot products) and P V (p + 1 axpys), 2 * D each."""
    f = 0
    for L, k in zip(lens, n):
        first = L - k  # positions L - k .. L - 1
        keys = k * (first + 1) + k * (k - 1) // 2
        f += 4 * D * Hq * keys
    return f


def run_prefill(args, world, rank, local, with_cpu=True):
    """Paged prefill of 8 prompts of 2048 tokens (Hq 32 / Hkv 8, head_dim
    128, block size 16, bf16) over scattered blocks: each step writes the
    prompts' K/V into their slots (pkv_write_slots) and runs causal paged
    attention (pkv_prefill_attention).  `value` is the attention's
    algorithmic TFLOP/s (S = QK^T and PV, causal) over its device time."""
    import numpy as np

    from paged_kv_cache_337_b200 import _abi
    from paged_kv_cache_337_b200.cache import PagedKVCache

    S, L, Hq, Hkv, D, bs = 8, 2048, 32, 8, 128, 16
    dt = torch.bfloat16
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    _abi.lib()
    gen = torch.Generator("cpu").manual_seed(2000 + rank)
    lens = [L] * S
    nb = int(math.ceil(1.1 * S * (L // bs)))
    order = torch.randperm(nb, generator=gen).tolist()
    cache = PagedKVCache(nb, bs, Hq, Hkv, D, dt, dev, L // bs, 0, free_order=order,
                         scale=1.0 / math.sqrt(D))
    for s in range(S):
        cache.pool.add(s, L)
    slots = torch.cat([cache.pool.slot_mapping(s, 0, L) for s in range(S)]).to(dev)
    tables, tl = cache.pool.block_tables(list(range(S)), L // bs)
    tables, tl = tables.to(dev), tl.to(dev)
    qs = torch.tensor(np.concatenate([[0], np.cumsum(lens)]), dtype=torch.int32, device=dev)
    dgen = torch.Generator(dev).manual_seed(3000 + rank)
    T = S * L
    q = torch.randn((T, Hq, D), generator=dgen, device=dev).to(dt)
    k = torch.randn((T, Hkv, D), generator=dgen, device=dev).to(dt)
    v = torch.randn((T, Hkv, D), generator=dgen, device=dev).to(dt)
    out = torch.empty_like(q)
    stream = torch.cuda.Stream(dev)
    err = cache.dev_error
    flops = prefill_flops(lens, lens, Hq, D)

    def step(ev=None):
        _abi.pkv_write_slots(k, v, cache.key_cache, cache.value_cache, slots, dev_error=err,
                             stream=stream)
        if ev:
            ev[0].record(stream)
        _abi.pkv_prefill_attention(out, q, cache.key_cache, cache.value_cache, tables, tl, qs, L,
                                   cache.scale, dev_error=err, stream=stream)
        if ev:
            ev[1].record(stream)

    # inputs and caches were made on the default stream; the timed
    # stream is not ordered after it
    torch.cuda.synchronize(dev)
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    clocks = ClockSampler(local) if rank == 0 else None
    if clocks:
        clocks.start()
    K = args.steps
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(K)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize(dev)
    h0 = time.monotonic()
    t0.record(stream)
    for i in range(K):
        step(evs[i])
    t1.record(stream)
    torch.cuda.synchronize(dev)
    if clocks:
        clocks.window(h0, time.monotonic())
    barrier(world)
    clock_info = clocks.stop() if clocks else None
    cache.check_errors()
    attn_ms = sum(a.elapsed_time(b) for a, b in evs) / K
    t_max = max_over_ranks(t0.elapsed_time(t1), world, dev)
    value = sum_over_ranks(flops * K, world, dev) / (t_max * 1e-3) / 1e12
    attn_tflops = flops / (attn_ms * 1e-3) / 1e12
    peak = measured_tensor_peak()

    cpu = None
    if rank == 0 and world == 1 and with_cpu and not args.no_cpu_baseline:
        from oracle import reference as ref

        n_rows = 64  # the last 64 rows of one prompt: the heaviest rows
        hq = q[L - n_rows:L].cpu()
        sub = torch.tensor([0, n_rows], dtype=torch.int32)
        kc, vc = cache.key_cache.cpu(), cache.value_cache.cpu()
        tc = time.perf_counter()
        reps = 0
        while time.perf_counter() - tc < 10.0:
            ref.prefill_attention(hq, kc, vc, tables[:1].cpu(), tl[:1].cpu(), sub, cache.scale,
                                  "bf16", Hkv, bs)
            reps += 1
        secs = time.perf_counter() - tc
        cpu = {"value": round(reps * prefill_flops([L], [n_rows], Hq, D) / secs / 1e12, 6),
               "unit": "TFLOP/s", "cores": ref.max_threads(), "kind": "oracle",
               "sample": "last %d rows of one 2048-token prompt (all 32 heads), %d times, "
                         "%.1f s" % (n_rows, reps, secs)}
    if rank == 0:
        line = {
            "metric": "paged prefill attention TFLOP/s (causal, algorithmic)",
            "value": round(value, 2), "unit": "TFLOP/s", "n_gpus": world, "steps": K,
            "warmup": args.warmup, "ms_per_step": round(t_max / K, 4),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic",
            "config": {"workload": PREFILL_WORKLOAD, "num_seqs": S, "prompt_len": L,
                       "num_q_heads": Hq, "num_kv_heads": Hkv, "head_dim": D,
                       "block_size": bs, "pool_blocks": nb,
                       "step": "prompt K/V slot write + causal paged prefill attention",
                       "l2": "K/V %.2f GB, Q %.2f GB per step" % (
                           2 * T * Hkv * D * 2 / 1e9, T * Hq * D * 2 / 1e9)},
            "roofline": {"bound": "tensor", "achieved": round(attn_tflops, 2),
                         "peak": peak[0], "unit": "TFLOP/s",
                         "frac": round(attn_tflops / peak[0], 4),
                         "traffic": profiled_traffic(kernel_source_digest("prefill"),
                                                     PREFILL_WORKLOAD),
                         "kernel": "paged_prefill_kernel", "peak_source": peak[1]},
            "cpu_baseline": cpu, "e2e": None, "gpu_launches": 2 * K, "clocks": clock_info,
        }
        return line
    return None


def measured_tensor_peak():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["bf16_tflops"]), "measured (bf16 burst)"
    except (OSError, KeyError, ValueError):
        return 1590.0, "fallback"


def run_shared_prefix(args, world, rank, local):
    """The shared-prefix parallel-sampling workload (16 prompts x 8 samples,
    1024-token prefix): the fork step (112 copy-on-write copies + slot write
    + decode) and a steady step after each sample has diverged.  A step's
    metadata comes from the host pool once and the step is replayed (the
    copies and writes are idempotent).  `value` counts logical bytes: every
    sequence's K/V once, although samples share the prefix blocks, so it may
    exceed the HBM peak; `unique_kv_gb` is the K/V a step must bring from
    HBM at least once."""
    from paged_kv_cache_337_b200 import _abi
    from paged_kv_cache_337_b200 import workloads as W
    from paged_kv_cache_337_b200.cache import PagedKVCache

    spec = W.SHARED_PREFIX
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    inp = W.make_shared_prefix_inputs(spec)
    Pn, N, bs = spec.num_prompts, spec.samples_per_prompt, spec.block_size
    Hq, Hkv, D, dt = spec.num_q_heads, spec.num_kv_heads, spec.head_dim, spec.torch_dtype
    S = Pn * N
    ids = list(range(S))
    mb = -(-(int(inp.prompt_lens.max()) + int(inp.diverge.max()) + 4) // bs)
    cache = PagedKVCache(inp.num_blocks, bs, Hq, Hkv, D, dt, dev, mb, 0,
                         free_order=inp.free_order.tolist(), scale=spec.scale,
                         work_list=cache_work_list(args))
    W.fill_device_cache_(cache.key_cache, inp.seed_values + rank)
    W.fill_device_cache_(cache.value_cache, inp.seed_values + rank + 1)
    for p in range(Pn):
        cache.add_sequence(p * N, int(inp.prompt_lens[p]))
        for c in range(1, N):
            cache.fork(p * N, p * N + c)
    dgen = torch.Generator(dev).manual_seed(inp.seed_values)
    stream = torch.cuda.Stream(dev)
    out = torch.empty((S, Hq, D), dtype=dt, device=dev)

    def snapshot():
        prep = cache.prepare_step(ids)
        st = prep["st"]
        n = prep["num_pairs"]
        lens = st["h_lens"].tolist()
        tables = st["h_tables"]
        used = set()
        for i in range(S):
            nblk = -(-lens[i] // bs)
            used.update(tables[i, :nblk].tolist())
        ni = prep["num_items"]
        return dict(slots=st["h_slots"].to(dev), pairs=st["h_pairs"][:n].to(dev), npairs=n,
                    tables=tables.to(dev), lens=st["h_lens"].to(dev), max_len=max(lens),
                    items=st["h_items"][:ni].to(dev) if ni >= 0 else None,
                    logical=decode_bytes(spec_like(spec), lens, 0) + write_bytes(spec, S) +
                    copy_bytes(spec, n),
                    unique=len(used) * bs * Hkv * D * 4,
                    q=torch.randn((S, Hq, D), generator=dgen, device=dev).to(dt),
                    k=torch.randn((S, Hkv, D), generator=dgen, device=dev).to(dt),
                    v=torch.randn((S, Hkv, D), generator=dgen, device=dev).to(dt))

    def time_state(stt):
        kc, vc, err = cache.key_cache, cache.value_cache, cache.dev_error

        def step():
            if stt["npairs"]:
                _abi.pkv_copy_blocks(kc, vc, stt["pairs"], dev_error=err, stream=stream)
            _abi.pkv_write_slots(stt["k"], stt["v"], kc, vc, stt["slots"], dev_error=err,
                                 stream=stream)
            _abi.pkv_decode_attention(out, stt["q"], kc, vc, stt["tables"], stt["lens"],
                                      stt["max_len"], spec.scale, 0, None, dev_error=err,
                                      stream=stream, work_items=stt["items"])
            return (1 if stt["npairs"] else 0) + 2

        # inputs and caches were made on the default stream; the timed
        # stream is not ordered after it
        torch.cuda.synchronize(dev)
        for _ in range(args.warmup):
            step()
        torch.cuda.synchronize(dev)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        barrier(world)
        torch.cuda.synchronize(dev)
        h0 = time.monotonic()
        e0.record(stream)
        launches = sum(step() for _ in range(args.steps))
        e1.record(stream)
        torch.cuda.synchronize(dev)
        if clocks:
            clocks.window(h0, time.monotonic())
        barrier(world)
        cache.check_errors()
        ms = max_over_ranks(e0.elapsed_time(e1), world, dev) / args.steps
        total = sum_over_ranks(stt["logical"], world, dev)
        return {"ms_per_step": round(ms, 4), "logical_gbs": round(total / ms / 1e6, 2),
                "unique_kv_gb": round(stt["unique"] / 1e9, 3), "cow_copies": stt["npairs"],
                "logical_gb": round(stt["logical"] / 1e9, 3)}, launches

    clocks = ClockSampler(local) if rank == 0 else None
    if clocks:
        clocks.start()
    fork = snapshot()
    fork_res, launches = time_state(fork)
    # every sample advances by its private tokens (host pool only; values
    # are whatever the cache holds: timing does not depend on them)
    for s in ids:
        for _ in range(int(inp.diverge[s])):
            cache.pool.append(s)
    steady = snapshot()
    steady_res, _ = time_state(steady)
    memory = pool_memory(cache.pool, ids, bs, inp.num_blocks,
                         int(inp.prompt_lens.max()) + int(inp.diverge.max()) + 1)
    clock_info = clocks.stop() if clocks else None
    peak, peak_kind = measured_peak()
    if rank == 0:
        line = {
            "metric": METRIC, "value": fork_res["logical_gbs"], "unit": "GB/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": fork_res["ms_per_step"], "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": spec.name, "num_seqs": S, "num_q_heads": Hq,
                       "num_kv_heads": Hkv, "head_dim": D, "block_size": bs,
                       "step": "fork step: copy-on-write copies + slot write + decode",
                       "bytes": "logical (shared prefix blocks counted per sequence)"},
            "fork_step": fork_res, "steady_step": steady_res,
            "decode_tok_s": round(world * S / (fork_res["ms_per_step"] * 1e-3), 1),
            "peak_gbs": peak, "peak_source": peak_kind, "gpu_launches": launches,
            "clocks": clock_info, "memory": memory,
        }
        return line
    return None


def spec_like(spec):
    """A decode-shaped view of the shared-prefix workload for byte counting."""
    from paged_kv_cache_337_b200 import workloads as W

    return W.DecodeSpec(spec.name, spec.seed, spec.num_seqs, spec.num_q_heads,
                        spec.num_kv_heads, spec.head_dim, spec.block_size, 1, 1, spec.dtype)


# The decode workloads measured beside the headline in the same process, with
# the same --steps / --warmup and the same device timing: the 70B-shaped GQA
# batch, the long split-K contexts at block sizes 32 and 64, both decode
# shapes over e4m3 caches, the shared-prefix fork and steady steps, and
# paged prefill.
EXTRA_DECODE = (("70b_gqa_s64_hq64_hkv8_d128_bs16_bf16", False),
                ("long_s8_l32768_hq32_hkv8_d128_bs32_bf16", False),
                ("long_s8_l32768_hq32_hkv8_d128_bs64_bf16", False),
                ("7b_s256_h32_d128_bs16_bf16", True),
                ("70b_gqa_s64_hq64_hkv8_d128_bs16_bf16", True))


def summary(line):
    """The fields of a workload's line kept under the headline's workloads."""
    keep = ("value", "unit", "ms_per_step", "roofline", "clocks", "e2e", "gpu_launches",
            "decode_tok_s", "pct_hbm_peak", "fork_step", "steady_step", "dtype")
    out = {k: line[k] for k in keep if k in line}
    cfg = line.get("config", {})
    out["config"] = {k: cfg[k] for k in ("workload", "partition_size", "grid", "step", "bytes")
                     if k in cfg}
    return out


def run_extra_workloads(args, world, rank, local):
    from paged_kv_cache_337_b200 import workloads as W

    sub = argparse.Namespace(**vars(args))
    sub.partition_size = -1
    out = {}
    runs = [(workload_name(W.SPECS[n], fp8),
             lambda n=n, fp8=fp8: run_pkv(sub, W.SPECS[n], world, rank, local, fp8=fp8,
                                          with_cpu=False, with_alloc=False))
            for n, fp8 in EXTRA_DECODE]
    runs.append((W.SHARED_PREFIX.name, lambda: run_shared_prefix(sub, world, rank, local)))
    runs.append((PREFILL_WORKLOAD, lambda: run_prefill(sub, world, rank, local, with_cpu=False)))
    for name, fn in runs:
        try:
            line = fn()
            if line is not None:
                out[name] = summary(line)
        except Exception as e:  # recorded; the headline line still prints
            if world > 1:
                raise
            out[name] = {"error": "%s: %s" % (type(e).__name__, e)}
        torch.cuda.synchronize()
        torch.cuda.empty_cache()
    return out


def main():
    args = parse_args()
    from paged_kv_cache_337_b200 import workloads as W

    special = {COW_LAYERS_WORKLOAD: run_cow_layers, SWAP_WORKLOAD: run_swap}
    returning = {PREFILL_WORKLOAD: run_prefill, W.SHARED_PREFIX.name: run_shared_prefix}
    if args.workload in special or args.workload in returning:
        world, rank, local = dist_setup()
        try:
            if args.workload in special:
                special[args.workload](args, world, rank, local)
            else:
                line = returning[args.workload](args, world, rank, local)
                if line is not None:
                    print(json.dumps(line), flush=True)
        finally:
            if world > 1:
                torch.distributed.destroy_process_group()
        return
    spec = W.SPECS[args.workload]
    if args.num_seqs:
        import dataclasses

        spec = dataclasses.replace(spec, num_seqs=args.num_seqs,
                                   name="%s_first%d" % (spec.name, args.num_seqs))
    world, rank, local = dist_setup()
    try:
        if args.impl == "reference":
            run_reference(args, spec, world, rank)
            return
        fp8 = args.kv_dtype == "fp8"
        line = run_pkv(args, spec, world, rank, local, fp8=fp8)
        if (args.extra == "all" and args.workload == W.DECODE_7B.name and not fp8 and
                not args.num_seqs):
            extra = run_extra_workloads(args, world, rank, local)
            if line is not None:
                line["workloads"] = extra
        if line is not None:
            print(json.dumps(line), flush=True)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
