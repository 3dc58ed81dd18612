#!/usr/bin/env python
"""Benchmark of the paged decode hot path on B200.

One step = one pass of the whole path over one synthetic batch, with every
input already resident in HBM:
  slot indexing of the new tokens -> reshape_and_cache -> decode plan ->
  decode (-> log-sum-exp merge when sequences are split)
The first three share one launch when the new tokens are one per sequence
or a short list (the fused prologues).  The shared-prefix workload runs
copy_blocks first and decodes with the shared-prefix plan: each prompt's
blocks read once for its samples, merged with each sample's own blocks.

The default workload is the Llama-3-8B-shaped GQA batch (256 sequences, 32 q /
8 kv heads, head_dim 128, bf16, lognormal context lengths with median 1000),
the batched bf16 GQA configuration the throughput target is stated on.  The
KV pools (about 2.3 GB) are far larger than the 126 MB L2, so no flush is
needed between steps.

Usage:
  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload c3|c2|c4|c5|...]
  python bench.py --impl reference ...      # the float64 CPU oracle, timed
For N > 1 launch one process per GPU with torch.distributed.run; every rank
decodes its own replica of the batch (the path has no exchange step), the
timed region is bracketed by barriers and the max over ranks is reported.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import workloads  # noqa: E402

METRIC = "paged decode attn: KV-read GB/s (% of B200 HBM peak), seqs/s at batch"
UNIT = "GB/s"
WORKLOADS = {"c3": "c3_llama3_8b_gqa", "c2": "c2_llama2_13b_mha", "c4": "c4_shared_prefix",
             "c5": "c5_long_splitk", "c1": "c1_tiny_fp32", "c3spec": "c3_spec_decode",
             "c3fp8": "c3_fp8", "c3specfp8": "c3_spec_fp8", "c3e5m2": "c3_fp8e5m2",
             "c3prefill": "c3_prefill"}
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0            # burst; about 1400 sustained under the power cap
FALLBACK_BF16_TFLOPS_SUSTAINED = 1400.0
# Chunks with more query rows per kv head than this run on the tcgen05 prefill kernel
# (128-row query tiles); shorter ones on the decode kernel (at most 16 rows per item).
PREFILL_MIN_ROWS = 64
L2_BYTES = 126 << 20       # B200 L2; working sets below 4x this are flushed between steps
# the sources of every kernel a step can launch and of their launch configuration: a
# recorded traffic figure holds only for the code it was taken on
DECODE_SOURCES = ["pkv_decode.cuh", "pkv_decode_warp.cuh", "pkv_decode_fp8tc.cuh",
                  "pkv_prefill.cuh", "pkv_device.cuh", "pkv_api.cu"]
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "decode_kernel_traffic.txt")  # JSON text


# ------------------------------------------------------------------ helpers
def hbm_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except (OSError, KeyError, ValueError):
        return FALLBACK_HBM_GBS, "fallback"


def tensor_peak():
    """(burst, sustained, kind) dense bf16 TFLOP/s of this machine's B200s."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        burst = float(d["bf16_tflops"])
        return burst, float(d.get("bf16_tflops_sustained", burst)), "measured"
    except (OSError, KeyError, ValueError):
        return FALLBACK_BF16_TFLOPS, FALLBACK_BF16_TFLOPS_SUSTAINED, "fallback"


def attention_flops(b: workloads.Batch) -> int:
    """Multiply-adds x 2 of S = q K^T and O = P V over the keys each query row can see:
    4 * head_dim per (query row, query head, visible key); chunk token i of an n-token
    chunk sees L - n + i + 1 keys."""
    lens = b.context_lens.astype(np.int64)
    if b.query_start_loc is None:
        visible = int(lens.sum())
    else:
        n = np.diff(b.query_start_loc).astype(np.int64)
        # sum over i < n of (L - n + i + 1) = n (L - n) + n (n + 1) / 2
        visible = int((n * (lens - n) + n * (n + 1) // 2).sum())
    return 4 * b.head_dim * b.num_q_heads * visible


def decode_source_hash() -> str:
    h = hashlib.sha256()
    for name in DECODE_SOURCES:
        with open(os.path.join(ROOT, "paged_kv_cache_375_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def traffic_key(workload: str, partition: int) -> str:
    """The traffic record of a workload (and an explicit partition size, when given)."""
    return workload if not partition else f"{workload}@{partition}"


def recorded_traffic(key: str):
    """DRAM bytes per launch of the step's dominant kernel from the committed ncu
    summary, if it was taken on the current kernel sources and this workload; else None."""
    try:
        with open(TRAFFIC_FILE) as f:
            rec = json.load(f)
    except (OSError, ValueError):
        return None
    entry = rec.get(key)
    if not entry or entry.get("source_hash") != decode_source_hash():
        return None
    return entry.get("dram_bytes_per_launch")


def algorithmic_bytes(b: workloads.Batch) -> dict:
    """Bytes a decode launch must move from HBM at least: every context token's K and V once
    per kv head (slots shared by several sequences once), q, out, the block-table entries
    in use and the context lengths."""
    lens = b.context_lens.astype(np.int64)
    table = int(((lens + 15) // 16).sum()) * 4
    qo = 2 * b.q.shape[0] * b.num_q_heads * b.head_dim * b.q_elem_bytes
    kv = b.unique_kv_bytes() if b.cow_pairs.shape[0] or b.name == "c4_shared_prefix" else b.kv_bytes()
    return {"kv": kv, "kv_logical": b.kv_bytes(), "q_out": qo, "table": table,
            "lens": 4 * b.num_seqs, "total": kv + qo + table + 4 * b.num_seqs}


class ClockSampler:
    """Samples the GPU's SM clock and clock-event reasons through NVML while running."""

    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
               0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
               0x100: "display_clock_setting"}

    def __init__(self, local_rank: int, period_s: float = 0.01):
        self.samples, self.reasons, self.period = [], 0, period_s
        self.ok = False
        try:
            import pynvml
            pynvml.nvmlInit()
            vis = os.environ.get("CUDA_VISIBLE_DEVICES")
            index = int(vis.split(",")[local_rank]) if vis else local_rank
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.nv = pynvml
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # no NVML: report no clocks rather than fail the run
            self.err = str(e)
        self._stop = threading.Event()

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
                get = getattr(self.nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                    self.nv.nvmlDeviceGetCurrentClocksThrottleReasons
                self.reasons |= get(self.h)
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *exc):
        if self.ok:
            self._stop.set()
            self.t.join()

    def summary(self):
        if not self.ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "note": "NVML unavailable"}
        names = [n for bit, n in self.REASONS.items() if self.reasons & bit and n != "gpu_idle"]
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": names, "samples": len(self.samples)}


def dist_init():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=300))
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, world: int, device) -> float:
    """The maximum of x over all ranks (the slowest rank sets the job's time)."""
    if world == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64,
                     device=device if dist.get_backend() == "nccl" else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_value(units_per_rank: float, world: int, seconds: float) -> float:
    """Aggregate throughput: units all ranks processed over the slowest rank's time."""
    return units_per_rank * world / seconds


# ------------------------------------------------------------------ our arm
# New tokens per step up to which the writes share a launch with the plan.
TOKEN_PROLOGUE_MAX = 4096
# The roofline's decode duration: at least this many bracketed launches and this many
# seconds after the timed region (at most ROOF_MAX_LAUNCHES).
ROOF_LAUNCHES = 200
ROOF_SECONDS = 0.3
ROOF_MAX_LAUNCHES = 5000


class Step:
    """The hot path over one batch through the public API (device-resident inputs)."""

    def __init__(self, b: workloads.Batch, partition_tokens: int, shared_prefix: bool = True,
                 token_prologue: bool = False, multi_kernel: str = "auto"):
        import paged_kv_cache_375_b200 as pkv
        self.pkv, self.b = pkv, b
        dev = b.q.device
        self.dev = dev
        self.bt = torch.from_numpy(b.block_tables).to(dev)
        self.cl = torch.from_numpy(b.context_lens).to(dev)
        self.out = torch.empty_like(b.q)
        self.mcl = max(b.max_context_len, 1)
        self.partition = partition_tokens
        self.dims = pkv.make_dims(b.num_seqs, b.num_q_heads, b.k_cache, b.max_blocks_per_seq)
        self.part_tokens = pkv.decode_partition_tokens(self.dims, self.mcl, partition_tokens)
        self.split = self.part_tokens < self.mcl
        self.multi = b.query_start_loc is not None
        # sequences that share a prompt's blocks: read those blocks once per group
        self.shared = shared_prefix and "group_start" in b.meta and not self.multi
        if self.shared:
            self.part_tokens = pkv.decode_shared_partition_tokens(self.dims, self.mcl,
                                                                  partition_tokens)
            self.group_start = torch.tensor(b.meta["group_start"], dtype=torch.int32, device=dev)
            self.shared_blocks = torch.tensor(b.meta["shared_blocks"], dtype=torch.int32,
                                              device=dev)
            self.split = True                           # prefix and own partials are merged
        # long chunks (chunked prefill) on the tcgen05 kernel, short ones on the decode kernel
        g = b.num_q_heads // b.num_kv_heads
        self.prefill = self.multi and b.dtype == "bf16" and (
            multi_kernel == "prefill" or
            (multi_kernel == "auto" and b.max_query_len * g > PREFILL_MIN_ROWS))
        if self.prefill:
            self.split = False
        if self.multi:
            self.qsl = torch.from_numpy(b.query_start_loc).to(dev)
            ws = pkv.load_library().pkv_multi_workspace_bytes(
                __import__("ctypes").byref(self.dims), b.q.shape[0], self.mcl, partition_tokens)
        elif self.shared:
            ws = pkv.decode_shared_workspace_bytes(self.dims, self.mcl, partition_tokens)
        else:
            ws = pkv.decode_workspace_bytes(self.dims, self.mcl, partition_tokens)
        self.ws = torch.empty(ws, dtype=torch.uint8, device=dev)
        self.T = int(b.new_seq.shape[0])
        self.decode_mode = (self.T == b.num_seqs
                            and np.array_equal(b.new_seq, np.arange(b.num_seqs))
                            and np.array_equal(b.new_pos, b.context_lens - 1))
        self.seq = torch.from_numpy(b.new_seq).to(dev)
        self.pos = torch.from_numpy(b.new_pos).to(dev)
        self.slots = torch.empty(max(self.T, 1), dtype=torch.int64, device=dev)
        self.pairs = torch.from_numpy(b.cow_pairs).to(dev) if b.cow_pairs.shape[0] else None
        # one new token per sequence at its last position, no copies: the fused prologue
        self.fused = (self.decode_mode and self.pairs is None and not self.multi
                      and not self.shared)
        # any other short list of new tokens (a few per sequence): written in the same
        # launch as the plan.  A long list (the parallel-sampling tails) keeps
        # reshape_and_cache, whose many small CTAs stream the rows at the copy bandwidth.
        self.fused_tokens = (self.T > 0 and not self.fused and not self.prefill
                             and (token_prologue or self.T <= TOKEN_PROLOGUE_MAX))
        if self.pairs is not None:
            pkv.validate_copy_pairs(torch.from_numpy(b.cow_pairs), b.num_blocks)

    def launches_per_step(self) -> int:
        if self.prefill:                               # slots, reshape, prefill
            return 1 + (2 if self.T else 0)
        n = 2 + (1 if self.split else 0)              # plan or prologue, decode (, merge)
        n += 2 if self.T and not (self.fused or self.fused_tokens) else 0  # slots, reshape
        n += 1 if self.pairs is not None else 0        # copy_blocks
        return n

    def cache_ops(self):
        pkv, b = self.pkv, self.b
        if self.fused:
            return                                     # done by the prologue in plan()
        if self.pairs is not None:
            pkv.copy_blocks(b.k_cache, b.v_cache, self.pairs, validate=False)
        if self.T and not self.fused_tokens:
            if self.decode_mode:
                pkv.slot_mapping(self.bt, b.num_blocks, context_lens=self.cl, out=self.slots)
            else:
                pkv.slot_mapping(self.bt, b.num_blocks, token_seq=self.seq, token_pos=self.pos,
                                 out=self.slots)
            self.write_new(self.slots[:self.T])

    def write_new(self, slots):
        b = self.b
        if workloads.fp8_format(b.dtype):
            self.pkv.reshape_and_cache_fp8(b.new_k, b.new_v, b.k_cache, b.v_cache, slots,
                                           b.k_scale, b.v_scale)
        else:
            self.pkv.reshape_and_cache(b.new_k, b.new_v, b.k_cache, b.v_cache, slots)

    def plan(self):
        b = self.b
        if self.prefill:
            return                                     # the prefill kernel needs no plan
        extra = {}
        if self.fused or self.fused_tokens:
            # one launch: the new tokens' slots and writes, and the plan
            extra = dict(new_k=b.new_k, new_v=b.new_v, v_cache=b.v_cache, k_scale=b.k_scale,
                         v_scale=b.v_scale, slot_mapping_out=self.slots[:self.T])
            if self.fused_tokens:
                extra.update(token_seq=self.seq, token_pos=self.pos)
        if self.shared:
            self.plan_obj = self.pkv.SharedDecodePlan(
                self.bt, self.cl, self.group_start, self.shared_blocks, b.num_q_heads, b.k_cache,
                max_context_len=self.mcl, partition_tokens=self.partition,
                workspace_tensor=self.ws, **extra)
            return
        self.plan_obj = self.pkv.DecodePlan(self.bt, self.cl, b.num_q_heads, b.k_cache,
                                            max_context_len=self.mcl,
                                            partition_tokens=self.partition,
                                            workspace_tensor=self.ws, **extra)

    def decode(self):
        if self.prefill:
            b = self.b
            self.pkv.paged_prefill(self.out, b.q, b.k_cache, b.v_cache, self.bt, self.cl,
                                   self.qsl, b.scale, b.num_kv_heads, max_context_len=self.mcl)
        elif self.multi and workloads.fp8_format(self.b.dtype):
            self.plan_obj.run_multi_fp8(self.out, self.b.q, self.b.k_cache, self.b.v_cache,
                                        self.qsl, self.b.max_query_len, self.b.scale,
                                        self.b.k_scale, self.b.v_scale)
        elif self.multi:
            self.plan_obj.run_multi(self.out, self.b.q, self.b.k_cache, self.b.v_cache, self.qsl,
                                    self.b.max_query_len, self.b.scale)
        elif workloads.fp8_format(self.b.dtype):
            self.plan_obj.run_fp8(self.out, self.b.q, self.b.k_cache, self.b.v_cache, self.b.scale,
                                  self.b.k_scale, self.b.v_scale)
        else:
            self.plan_obj.run(self.out, self.b.q, self.b.k_cache, self.b.v_cache, self.b.scale)

    def __call__(self):
        self.cache_ops()
        self.plan()
        self.decode()


def run_ours(args, world, rank, local):
    import paged_kv_cache_375_b200 as pkv
    from paged_kv_cache_375_b200 import build as pkv_build
    if not pkv_build.up_to_date():
        pkv_build.build()
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    name = WORKLOADS[args.workload]
    b = (workloads.BUILDERS[name](device=dev, num_seqs=args.batch) if args.batch else
         workloads.BUILDERS[name](device=dev))
    step = Step(b, args.partition, shared_prefix=not args.no_shared_prefix,
                token_prologue=args.token_prologue, multi_kernel=args.multi_kernel)
    alg = algorithmic_bytes(b)
    kv_bytes = b.kv_bytes() if name != "c4_shared_prefix" else b.unique_kv_bytes()
    stream = torch.cuda.current_stream(dev)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    pkv.check_device_error(dev)

    # Timed region: K steps back to back.  Events between launches would break
    # the overlap of consecutive launches (programmatic dependent launch), so
    # only every SAMPLE-th step has its decode launch bracketed by events (a
    # bracketed launch cannot overlap the plan kernel before it); the roofline's
    # decode duration comes from a longer loop right after the region.
    #
    # A working set that L2 could hold a good part of (the tiny fp32 batch, the
    # shared-prefix batch's unique bytes) is flushed before every step by a
    # write of twice the L2 size; each step is then bracketed by its own events
    # and the flush stays outside them.
    K = args.steps
    SAMPLE = 8
    flush = alg["total"] < 4 * L2_BYTES
    flush_buf = torch.empty(2 * L2_BYTES, dtype=torch.uint8, device=dev) if flush else None
    ev = {i: (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for i in range(0, K, SAMPLE)}
    step_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(K if flush else 1)]
    sampler = ClockSampler(local)
    barrier(world)
    torch.cuda.synchronize(dev)
    sampler.__enter__()
    try:
        step_ev[0][0].record(stream)
        for i in range(K):
            if flush:
                flush_buf.fill_(i & 0xff)
                step_ev[i][0].record(stream)
            step.cache_ops()
            step.plan()
            if i in ev:
                ev[i][0].record(stream)
                step.decode()
                ev[i][1].record(stream)
            else:
                step.decode()
            if flush:
                step_ev[i][1].record(stream)
        if not flush:
            step_ev[0][1].record(stream)
        torch.cuda.synchronize(dev)
        total_ms = sum(a.elapsed_time(z) for a, z in step_ev)
        # Roofline sample, right after the timed region and under the same clock
        # sampling: the decode launch of at least ROOF_LAUNCHES further steps (and
        # ROOF_SECONDS), each bracketed by events, so the duration does not rest on
        # the few launches a short timed region samples.  Each decode follows its
        # step's own cache ops and plan (the decode consumes the plan's work
        # counters) and, for flushed workloads, the L2 flush.
        n_roof = int(min(ROOF_MAX_LAUNCHES,
                         max(ROOF_LAUNCHES, ROOF_SECONDS * 1e3 / max(total_ms / K, 1e-3))))
        roof_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                   for _ in range(n_roof)]
        for i in range(n_roof):
            if flush:
                flush_buf.fill_(i & 0xff)
            step.cache_ops()
            step.plan()
            roof_ev[i][0].record(stream)
            step.decode()
            roof_ev[i][1].record(stream)
        torch.cuda.synchronize(dev)
    finally:
        sampler.__exit__(None, None, None)
    barrier(world)
    pkv.check_device_error(dev)
    region_samples = sorted(a.elapsed_time(z) for a, z in ev.values())
    decode_samples = sorted(a.elapsed_time(z) for a, z in roof_ev)
    decode_ms = statistics.mean(decode_samples)
    ops = None if args.no_breakdown else breakdown(step, stream, dev)
    total_ms = max_over_ranks(total_ms, world, dev)
    ms_per_step = total_ms / K
    seconds = total_ms / 1e3
    value = whole_job_value(kv_bytes * K / 1e9, world, seconds)
    peak, peak_kind = hbm_peak()

    # end to end through the public API with host buffers
    e2e = None
    if not args.no_e2e:
        e2e = run_e2e(step, args, world, dev, kv_bytes)

    result = {
        "metric": METRIC, "value": round(value, 2), "unit": UNIT, "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": round(ms_per_step, 5), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": b.dtype, "data": "synthetic",
        "config": {
            "workload": f"{name}: {workloads.CONFIGS[name]}; " + (
                f"split-K, {step.part_tokens}-token partitions this run" if step.split
                and not step.shared else "single pass this run" if not step.split else
                "shared-prefix plan this run"),
            "batch": b.num_seqs, "num_q_heads": b.num_q_heads, "num_kv_heads": b.num_kv_heads,
            "head_dim": b.head_dim, "block_size": 16, "num_blocks": b.num_blocks,
            "context_tokens": int(b.context_lens.sum()), "max_context_len": b.max_context_len,
            "new_tokens_per_step": step.T, "cow_pairs_per_step": int(b.cow_pairs.shape[0]),
            "partition_tokens": step.part_tokens, "split_k": step.split,
            **({"shared_prefix": "each prompt's full blocks read once per kv head for its "
                                 f"{b.meta['samples']} samples (shared-prefix items, "
                                 "log-sum-exp merge)"} if step.shared else {}),
            "kv_bytes_per_step": kv_bytes,
            # KV-block usage of the pool (blocks holding tokens / pool size)
            "blocks_in_use": int(b.meta.get("blocks_in_use", 0)),
            "pool_usage": round(int(b.meta.get("blocks_in_use", 0)) / b.num_blocks, 4),
            **({"batch_override": args.batch} if args.batch else {}),
            "l2": ("L2 flushed before every step (a 252 MB write outside the timed events; "
                   "the working set is under 4x L2)" if flush else
                   "inputs larger than L2 (KV pools >> 126 MB); no flush between steps"),
            "parallelism": f"replicas x{world} (no data-path collective)",
        },
        "pct_of_hbm_peak": round(100.0 * value / world / peak, 2),
        "seqs_per_s": round(whole_job_value(b.num_seqs * K, world, seconds), 1),
        "breakdown": {"decode_ms_mean": round(decode_ms, 5),
                      "decode_ms_median": round(statistics.median(decode_samples), 5),
                      "decode_ms_best": round(decode_samples[0], 5),
                      "decode_launches_sampled": len(decode_samples),
                      "decode_ms_in_region_mean": round(statistics.mean(region_samples), 5),
                      "decode_launches_in_region": len(region_samples), "ops_alone": ops,
                      "note": "decode: each of the roofline loop's launches after the timed "
                              "region bracketed by events (in the timed region, every 8th "
                              "step's decode is bracketed too: decode_ms_in_region_mean); "
                              "other ops: each timed alone (50 launches) after the timed region"},
        "roofline": roofline(step, alg, decode_ms, peak, peak_kind, args.workload),
        "gpu_launches": step.launches_per_step() * K,
        "clocks": sampler.summary(),
    }
    if e2e is not None:
        result["e2e"] = e2e
    if rank == 0 and not args.no_breakdown:
        result["host_block_manager"] = host_block_manager_cost(b)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        result["cpu_baseline"] = cpu_baseline(b, args.cpu_seconds)
    return result


def dominant_kernel(step: Step) -> str:
    """The kernel the library launches for the step's attention (the dispatch of
    run_decode and pkv_paged_prefill in pkv_api.cu, restated)."""
    b = step.b
    if step.prefill:
        return "prefill_kernel"
    g = b.num_q_heads // b.num_kv_heads
    one_token = not step.multi or b.max_query_len == 1
    chunk_rows = (b.max_query_len if step.multi else 1) * g
    if b.dtype in ("fp8", "fp8e5m2") and not step.shared and chunk_rows <= 16:
        return "decode_fp8tc_kernel"
    rows = (16 // g) * g if step.shared else g
    if (b.dtype == "bf16" and b.head_dim == 128 and one_token and rows <= 16
            and step.part_tokens // 16 <= 128 and (step.split or step.shared)):
        return "decode_warp_kernel"
    return "decode_kernel"


def roofline(step: Step, alg: dict, decode_ms: float, peak: float, peak_kind: str,
             workload: str) -> dict:
    """The dominant kernel against its roofline: HBM for decode (algorithmic bytes per
    launch / launch time), the bf16 tensor cores for the prefill kernel (attention
    flops per launch / launch time; its HBM bytes reported beside)."""
    gbs = alg["total"] / (decode_ms / 1e3) / 1e9
    if step.prefill:
        burst, sustained, kind = tensor_peak()
        flops = attention_flops(step.b)
        tf = flops / (decode_ms / 1e3) / 1e12
        return {"kernel": "prefill_kernel", "bound": "tensor",
                "achieved": round(tf, 2), "peak": burst,
                "peak_kind": f"{kind} bf16_tflops (dense, burst)", "unit": "TFLOP/s",
                "frac": round(tf / burst, 4), "frac_of_sustained": round(tf / sustained, 4),
                "peak_sustained": sustained,
                "traffic": recorded_traffic(traffic_key(workload, step.partition)),
                "algorithmic_flops_per_launch": flops,
                "hbm": {"achieved_GBps": round(gbs, 2), "peak": peak,
                        "frac": round(gbs / peak, 4)},
                "algorithmic_bytes_per_launch": alg}
    return {"kernel": dominant_kernel(step) + (" + merge_kernel" if step.split else ""),
            "bound": "hbm", "achieved": round(gbs, 2), "peak": peak,
            "peak_kind": f"{peak_kind} hbm_gbs (copy bandwidth)", "unit": "GB/s",
            "frac": round(gbs / peak, 4),
            "traffic": recorded_traffic(traffic_key(workload, step.partition)),
            "algorithmic_bytes_per_launch": alg}


def plan_items(step: Step) -> int:
    """Work items the plan writes: a (sequence, partition) each; with shared prefixes, each
    sequence's partitions after its prefix plus, per group, its prefix partitions times the
    items that take the group's members (16 query rows at most per item)."""
    b = step.b
    lens = b.context_lens.astype(np.int64)
    P = step.part_tokens

    def parts(n):
        return np.maximum(1, (n + P - 1) // P)

    if not step.shared:
        return int(parts(lens).sum())
    g = b.num_q_heads // b.num_kv_heads
    per_item = 16 // g if g <= 8 else 1
    gs, sb = b.meta["group_start"], b.meta["shared_blocks"]
    items = 0
    for i in range(len(sb)):
        members = lens[gs[i]:gs[i + 1]]
        pref = min([int(sb[i])] + [int(L) // 16 for L in members]) if len(members) >= 2 else 0
        items += int(parts(members - 16 * pref).sum())
        if pref:
            items += int(parts(np.int64(16 * pref))) * -(-len(members) // per_item)
    return items


def op_bytes(step: Step) -> dict:
    """Algorithmic bytes of each cache-maintenance op of one step (read + write)."""
    b = step.b
    row = b.num_kv_heads * b.head_dim * b.elem_bytes           # one token's cached K (or V)
    row_in = b.num_kv_heads * b.head_dim * b.q_elem_bytes      # one new token's K (or V)
    block = row * 16                                            # one K (or V) block
    T, P = step.T, int(b.cow_pairs.shape[0])
    out = {
        "slot_mapping": T * (4 + 4 + 8) + (4 * b.num_seqs if step.decode_mode else 8 * T),
        "reshape_and_cache": 2 * T * (row_in + row) + 8 * T,    # K and V, read and write
        "copy_blocks": 2 * 2 * P * block + 16 * P,              # K and V, read and write
        # reads the lengths (and the groups), writes one 32-byte work item per item
        "plan": 4 * b.num_seqs + 32 * plan_items(step) + (
            8 * len(step.b.meta["shared_blocks"]) + 4 if step.shared else 0),
    }
    out["decode_prologue"] = out["slot_mapping"] + out["reshape_and_cache"] + out["plan"]
    return out


def breakdown(step: Step, stream, dev, n: int = 50) -> dict:
    """Each op of the step timed alone with events after the timed region (launches
    here do not overlap), with achieved bandwidth against the HBM peak."""
    pkv, b = step.pkv, step.b

    def plan_only():
        if step.shared:
            pkv.SharedDecodePlan(step.bt, step.cl, step.group_start, step.shared_blocks,
                                 b.num_q_heads, b.k_cache, max_context_len=step.mcl,
                                 partition_tokens=step.partition, workspace_tensor=step.ws)
            return
        pkv.DecodePlan(step.bt, step.cl, b.num_q_heads, b.k_cache, max_context_len=step.mcl,
                       partition_tokens=step.partition, workspace_tensor=step.ws)

    ops = {} if step.prefill else {"plan": plan_only}
    if step.fused or step.fused_tokens:
        ops["decode_prologue"] = step.plan
    if step.T:
        if step.decode_mode:
            ops["slot_mapping"] = lambda: pkv.slot_mapping(step.bt, b.num_blocks,
                                                           context_lens=step.cl, out=step.slots)
        else:
            ops["slot_mapping"] = lambda: pkv.slot_mapping(step.bt, b.num_blocks,
                                                           token_seq=step.seq, token_pos=step.pos,
                                                           out=step.slots)
        ops["reshape_and_cache"] = lambda: step.write_new(step.slots[:step.T])
    if step.pairs is not None:
        ops["copy_blocks"] = lambda: pkv.copy_blocks(b.k_cache, b.v_cache, step.pairs,
                                                     validate=False)
    nbytes = op_bytes(step)
    peak, _ = hbm_peak()
    out = {}
    for name, fn in ops.items():
        a = torch.cuda.Event(enable_timing=True)
        z = torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize(dev)
        a.record(stream)
        for _ in range(n):
            fn()
        z.record(stream)
        torch.cuda.synchronize(dev)
        ms = a.elapsed_time(z) / n
        gbs = nbytes[name] / (ms / 1e3) / 1e9
        out[name] = {"ms": round(ms, 5), "bytes": nbytes[name], "GBps": round(gbs, 1),
                     "frac_of_hbm_peak": round(gbs / peak, 4)}
    step()  # leave a consistent state behind
    torch.cuda.synchronize(dev)
    return out


def host_block_manager_cost(b: workloads.Batch, steps: int = 50) -> dict:
    """Host time of the native block manager for one decode step of this batch: append
    one token to every sequence (slots, copy-on-write pairs) and export the block tables
    and lengths the decode call takes.  CPU only."""
    import paged_kv_cache_375_b200 as pkv
    rng = np.random.default_rng(0)
    bm = pkv.BlockManager(b.num_blocks, 16, seed=1, prefix_caching=True)
    ids = np.arange(b.num_seqs, dtype=np.int64)
    for s in range(b.num_seqs):
        bm.add_sequence(int(s), rng.integers(0, 32000, size=int(b.context_lens[s]) - 1))
    width = b.max_blocks_per_seq + (steps + 15) // 16 + 1
    toks = rng.integers(0, 32000, size=(steps, b.num_seqs)).astype(np.int32)
    slots = np.empty(b.num_seqs, dtype=np.int64)
    tables = np.empty((b.num_seqs, width), dtype=np.int32)
    lens = np.empty(b.num_seqs, dtype=np.int32)
    t0 = time.perf_counter()
    for i in range(steps):
        bm.append_tokens(ids, toks[i], out=slots)
        bm.take_copies()
        bm.block_tables(ids, width, tables=tables, lens=lens)
    el = time.perf_counter() - t0
    bm.close()
    return {"us_per_step": round(1e6 * el / steps, 2), "sequences": b.num_seqs,
            "what": "append one token per sequence + take copies + export tables and lengths"}


def run_e2e(step: Step, args, world, dev, kv_bytes):
    """Same step, but every step copies its inputs from pinned host memory to the device
    (q, the new tokens' K/V, context lengths, block tables) and reads the output back to
    pinned host memory, synchronising on it."""
    b = step.b
    ins = [("q", b.q), ("new_k", b.new_k), ("new_v", b.new_v), ("cl", step.cl), ("bt", step.bt)]
    if step.shared:
        ins += [("gs", step.group_start), ("sb", step.shared_blocks)]
    if step.fused_tokens:
        ins += [("seq", step.seq), ("pos", step.pos)]
    host = {name: t.detach().cpu().pin_memory() for name, t in ins}
    dst = dict(ins)
    out_host = torch.empty(step.out.shape, dtype=step.out.dtype).pin_memory()
    h2d = sum(t.numel() * t.element_size() for t in host.values())
    d2h = out_host.numel() * out_host.element_size()
    stream = torch.cuda.current_stream(dev)

    def inputs_in():
        for name, t in host.items():
            dst[name].copy_(t, non_blocking=True)

    def one():
        inputs_in()
        step()
        out_host.copy_(step.out, non_blocking=True)
        stream.synchronize()

    def timed(fn, K):
        for _ in range(max(3, args.warmup // 4)):
            fn()
        barrier(world)
        torch.cuda.synchronize(dev)
        s = torch.cuda.Event(enable_timing=True)
        e = torch.cuda.Event(enable_timing=True)
        s.record(stream)
        for _ in range(K):
            fn()
        e.record(stream)
        torch.cuda.synchronize(dev)
        barrier(world)
        return max_over_ranks(s.elapsed_time(e), world, dev)

    K = max(3, args.steps // 4)
    ms = timed(one, K)
    result = {"value": round(whole_job_value(kv_bytes * K / 1e9, world, ms / 1e3), 2),
              "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": K,
              "ms_per_step": round(ms / K, 5), "host_sync_per_step": True}
    # The same step captured once into a CUDA graph (copies in, kernels, copy out) and
    # replayed every step: what a serving loop that replays a captured step would see.
    try:
        graph_stream = torch.cuda.Stream(device=dev)
        graph_stream.wait_stream(stream)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.stream(graph_stream):
            with torch.cuda.graph(g, stream=graph_stream):
                inputs_in()
                step()
                out_host.copy_(step.out, non_blocking=True)
        torch.cuda.synchronize(dev)

        def replay():
            g.replay()
            torch.cuda.current_stream(dev).synchronize()

        gms = timed(replay, K)
        result["graph_replay"] = {
            "value": round(whole_job_value(kv_bytes * K / 1e9, world, gms / 1e3), 2),
            "ms_per_step": round(gms / K, 5)}
        del g
    except RuntimeError as ex:  # report, do not fail the bench
        result["graph_replay"] = {"error": str(ex)[:200]}
    return result


# ------------------------------------------------------------ oracle (CPU)
def oracle_step(b: workloads.Batch, host: dict, seqs: np.ndarray | None, threads: int):
    """The oracle's pass over (a sample of) the step: copies, writes, attention."""
    import oracle
    k, v = host["k_cache"], host["v_cache"]
    if b.cow_pairs.shape[0]:
        oracle.copy_blocks(k, v, b.cow_pairs)
    fmt = workloads.fp8_format(b.dtype)
    fp8 = fmt is not None
    if b.new_seq.shape[0]:
        slots = oracle.slot_mapping(b.block_tables, b.new_seq, b.new_pos)
        if fp8:
            oracle.reshape_and_cache_fp8(host["new_k"], host["new_v"], k, v, slots, b.k_scale,
                                         b.v_scale, fmt=fmt)
        else:
            oracle.reshape_and_cache(host["new_k"], host["new_v"], k, v, slots)
    if b.query_start_loc is not None:          # several query tokens per sequence
        sel = np.arange(b.num_seqs) if seqs is None else np.asarray(seqs)
        qsl = b.query_start_loc
        rows = np.concatenate([np.arange(qsl[s], qsl[s + 1]) for s in sel] + [np.zeros(0, int)])
        sub_qsl = np.concatenate([[0], np.cumsum(qsl[sel + 1] - qsl[sel])]).astype(np.int32)
        q = np.ascontiguousarray(host["q"][rows])
        if fp8:
            return oracle.paged_multi_fp8(q, k, v, b.k_scale, b.v_scale, b.block_tables[sel],
                                          b.context_lens[sel], sub_qsl, b.scale, threads=threads,
                                          fmt=fmt)
        return oracle.paged_multi(q, k, v, b.block_tables[sel], b.context_lens[sel], sub_qsl,
                                  b.scale, threads=threads)
    tasks = None if seqs is None else np.array([(s, h) for s in seqs
                                                for h in range(b.num_q_heads)], dtype=np.int32)
    if fp8:
        return oracle.paged_decode_fp8(host["q"], k, v, b.k_scale, b.v_scale, b.block_tables,
                                       b.context_lens, b.scale, tasks=tasks, threads=threads,
                                       fmt=fmt)
    return oracle.paged_decode(host["q"], k, v, b.block_tables, b.context_lens, b.scale,
                               tasks=tasks, threads=threads)


def cpu_baseline(b: workloads.Batch, seconds: float) -> dict:
    """The oracle, as it stands, on the host cores: whole steps of the workload repeated
    for about `seconds` (at least once)."""
    threads = len(os.sched_getaffinity(0))
    host = b.host()
    reps, t0 = 0, time.perf_counter()
    while True:
        oracle_step(b, host, None, threads)
        reps += 1
        el = time.perf_counter() - t0
        if el >= seconds:
            break
    kv = b.kv_bytes()
    # the same on one core, over a seeded sample of the sequences
    rng = np.random.default_rng(1)
    sample = np.sort(rng.choice(b.num_seqs, size=max(1, b.num_seqs // 16), replace=False))
    skv = int(b.context_lens[sample].astype(np.int64).sum()) * b.num_kv_heads * \
        b.head_dim * b.elem_bytes * 2
    reps1, t0 = 0, time.perf_counter()
    while True:
        oracle_step(b, host, sample, 1)
        reps1 += 1
        el1 = time.perf_counter() - t0
        if el1 >= seconds / 3:
            break
    return {"value": round(kv * reps / el / 1e9, 4), "unit": UNIT, "cores": threads,
            "kind": "oracle",
            "sample": f"{reps} full step(s) of {b.name} ({b.num_seqs} seqs x {b.num_q_heads} "
                      f"q heads, fp64) in {el:.1f} s",
            "seqs_per_s": round(b.num_seqs * reps / el, 2),
            "single_core": {"value": round(skv * reps1 / el1 / 1e9, 4), "unit": UNIT, "cores": 1,
                            "sample": f"{reps1} pass(es) over {sample.size} of {b.num_seqs} "
                                      f"sequences (seeded choice) in {el1:.1f} s"}}


def run_reference(args, world, rank, local):
    """The reference arm: the float64 oracle timed on the host cores, on this workload, each
    step a bounded sample of sequences so that the whole run takes a few minutes."""
    name = WORKLOADS[args.workload]
    b = workloads.BUILDERS[name](device="cpu")
    threads = len(os.sched_getaffinity(0))
    host = b.host()
    # size the per-step sample: calibrate on one sequence, aim at ~150 s for the whole run
    t0 = time.perf_counter()
    oracle_step(b, host, np.array([int(np.argmax(b.context_lens))]), threads)
    per_seq = max((time.perf_counter() - t0) * float(b.context_lens.mean())
                  / float(b.context_lens.max()), 1e-4)
    budget = 150.0 / max(1, args.steps + args.warmup)
    n = int(min(b.num_seqs, max(1, budget / per_seq)))
    rng = np.random.default_rng(0)
    sample = np.sort(rng.choice(b.num_seqs, size=n, replace=False))
    sample_kv = int(b.context_lens[sample].astype(np.int64).sum()) * b.num_kv_heads * \
        b.head_dim * b.elem_bytes * 2
    for _ in range(args.warmup):
        oracle_step(b, host, sample, threads)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle_step(b, host, sample, threads)
    el = time.perf_counter() - t0
    value = sample_kv * args.steps / el / 1e9
    peak, _ = hbm_peak()
    desc = f"{n} of {b.num_seqs} sequences (seeded choice) x {b.num_q_heads} q heads per step"
    return {
        "metric": METRIC, "value": round(value, 4), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(1e3 * el / args.steps, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "impl": "reference",
        "config": {"workload": f"{name}: {workloads.CONFIGS[name]}", "batch": b.num_seqs,
                   "sample_per_step": desc},
        "pct_of_hbm_peak": round(100.0 * value / peak, 4),
        "seqs_per_s": round(n * args.steps / el, 3),
        "cpu_baseline": {"value": round(value, 4), "unit": UNIT, "cores": threads,
                         "kind": "oracle", "sample": desc},
        "e2e": {"value": round(value, 4), "unit": UNIT, "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawTextHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=sorted(WORKLOADS), default="c3")
    ap.add_argument("--partition", type=int, default=0, help="partition tokens (0 = automatic)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-breakdown", action="store_true",
                    help="skip timing the cache ops and the plan alone after the timed region")
    ap.add_argument("--no-shared-prefix", action="store_true",
                    help="decode a batch with shared prompt blocks with the plain plan (every "
                         "sequence reads its whole table)")
    ap.add_argument("--token-prologue", action="store_true",
                    help="write any number of new tokens in the plan's launch (by default only "
                         f"up to {TOKEN_PROLOGUE_MAX} a step)")
    ap.add_argument("--multi-kernel", choices=["auto", "prefill", "decode"], default="auto",
                    help="several query tokens per sequence: the tcgen05 prefill kernel "
                         f"(auto: chunks of more than {PREFILL_MIN_ROWS} rows per kv head) or "
                         "the decode kernel's row groups")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--batch", type=int, default=0,
                    help="number of sequences (0 = the workload's own); a smaller batch of the "
                         "same shape, for profiler captures that must stay small")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        # rank 0 alone times the CPU oracle; other ranks have nothing to do
        if int(os.environ.get("RANK", "0")) != 0:
            return 0
        world = int(os.environ.get("WORLD_SIZE", "1"))
        print(json.dumps(run_reference(args, world, 0, 0)), flush=True)
        return 0
    world, rank, local = dist_init()
    if world != args.gpus:
        print(f"warning: --gpus {args.gpus} but WORLD_SIZE={world}", file=sys.stderr)
    try:
        result = run_ours(args, world, rank, local)
        if rank == 0:
            print(json.dumps(result), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
