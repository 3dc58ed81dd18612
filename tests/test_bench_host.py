"""Host logic of bench.py without a GPU: the max-over-ranks timing and whole-job
aggregation across two gloo ranks, the reference arm's JSON line, and the
algorithmic byte count."""
import json
import os
import socket
import subprocess
import sys

import numpy as np
import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402
import workloads  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    elapsed = [1.5, 2.5][rank]                 # the slower rank sets the job time
    bench.barrier(world)
    slowest = bench.max_over_ranks(elapsed, world, "cpu")
    value = bench.whole_job_value(10.0, world, slowest)
    q.put((rank, slowest, value))
    dist.destroy_process_group()


def test_max_over_ranks_and_aggregate_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=5) for _ in range(2))
    for rank, slowest, value in got:
        assert slowest == 2.5
        assert value == pytest.approx(10.0 * 2 / 2.5)


def test_reference_arm_json_line():
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--workload", "c1", "--steps", "3", "--warmup", "3"],
                         capture_output=True, text=True, timeout=300, check=True).stdout
    line = json.loads(out.strip().splitlines()[-1])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "impl", "cpu_baseline", "e2e", "config"):
        assert key in line
    assert line["impl"] == "reference" and line["metric"] == bench.METRIC
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["cpu_baseline"]["kind"] == "oracle"


def test_reference_arm_other_ranks_exit_quietly():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2")
    p = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--workload", "c1", "--steps", "3", "--warmup", "3"], env=env,
                       capture_output=True, text=True, timeout=120)
    assert p.returncode == 0 and p.stdout.strip() == ""


def test_algorithmic_bytes_count_every_context_token_once_per_kv_head():
    b = workloads.random_batch(1, [17, 40], 8, 2, 64, "bf16")
    a = bench.algorithmic_bytes(b)
    assert a["kv"] == (17 + 40) * 2 * 64 * 2 * 2
    assert a["table"] == (2 + 3) * 4
    assert a["total"] == a["kv"] + a["q_out"] + a["table"] + a["lens"]


def test_plan_item_accounting():
    """The bench's count of planned work items (the plan kernel's written bytes) for the
    plain and the shared-prefix plans of the parallel-sampling batch."""
    import types
    import bench
    import workloads
    b = workloads.c4_shared_prefix(prompts=4, samples=8, prefix=256, max_tail=100,
                                   num_blocks=2000)
    lens = b.context_lens.astype(np.int64)
    P = int(((int(lens.max()) + 15) // 16) * 16)          # single pass
    plain = types.SimpleNamespace(b=b, part_tokens=P, shared=False)
    assert bench.plan_items(plain) == b.num_seqs
    shared = types.SimpleNamespace(b=b, part_tokens=P, shared=True)
    # per prompt: 2 prefix items (4 samples x 4 heads = 16 rows each) + 8 own-block items
    assert bench.plan_items(shared) == 4 * (2 + 8)
    split = types.SimpleNamespace(b=b, part_tokens=64, shared=True)
    n_own = int(np.maximum(1, (lens - 256 + 63) // 64).sum())
    assert bench.plan_items(split) == 4 * (256 // 64) * 2 + n_own


def test_dominant_kernel_follows_the_dispatch():
    """The kernel bench.py names in `roofline` is the one pkv_api.cu launches: FP8
    units of up to 16 query rows (one token x g, or a few draft tokens x g) on the
    tensor-core kernel, longer chunks and shared-prefix plans on decode_kernel, short
    bf16 items on the warp kernel, long chunks on the prefill kernel."""
    from types import SimpleNamespace as NS

    def step(dtype, hq, hkv, qlen=None, shared=False, split=False, part_tokens=4096,
             prefill=False):
        b = NS(dtype=dtype, num_q_heads=hq, num_kv_heads=hkv, head_dim=128,
               max_query_len=qlen or 1)
        return NS(b=b, multi=qlen is not None, shared=shared, split=split,
                  part_tokens=part_tokens, prefill=prefill)

    dk = bench.dominant_kernel
    assert dk(step("fp8", 32, 8)) == "decode_fp8tc_kernel"                 # 4 rows
    assert dk(step("fp8e5m2", 32, 8)) == "decode_fp8tc_kernel"
    assert dk(step("fp8", 32, 8, qlen=4)) == "decode_fp8tc_kernel"         # 16 rows
    assert dk(step("fp8", 16, 1)) == "decode_fp8tc_kernel"                 # g = 16
    assert dk(step("fp8", 32, 8, qlen=5)) == "decode_kernel"               # row groups
    assert dk(step("fp8", 32, 8, shared=True)) == "decode_kernel"
    assert dk(step("bf16", 32, 8)) == "decode_kernel"                      # single pass
    assert dk(step("bf16", 32, 8, split=True, part_tokens=512)) == "decode_warp_kernel"
    assert dk(step("bf16", 32, 8, shared=True, part_tokens=512)) == "decode_warp_kernel"
    assert dk(step("bf16", 32, 8, qlen=4)) == "decode_kernel"
    assert dk(step("bf16", 32, 8, qlen=1024, prefill=True)) == "prefill_kernel"
