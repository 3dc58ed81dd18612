"""Every output of every full-size workload, in the launch configuration the
benchmark times, against the float64 oracle.

Each case builds the workload at its full size, runs one step through the
benchmark's own ``Step`` (the fused decode prologue for one new token per
sequence; the token prologue for draft verification; copy_blocks, slot
indexing and reshape_and_cache before the shared-prefix plan for parallel
sampling; the decode and, where sequences are split, the log-sum-exp merge;
slot indexing, reshape_and_cache and the tcgen05 prefill kernel for the
chunked-prefill step),
then runs the oracle's pass over the same step on all host cores.  Both pools
must equal the oracle's byte for byte (copy-on-write copies, the new tokens'
writes, FP8 quantisation), and every output row must meet the tolerance: max
|e| <= 1e-5 for fp32, |e| <= 2e-2 + 1e-2 |ref| element-wise otherwise.

The long-context batch runs twice: with the automatic partition and with the
512-token partitions its configuration states (about 1,300 partials per row,
all merged by the merge kernel).
"""
import os

import numpy as np
import pytest
import torch

import bench
import paged_kv_cache_375_b200 as pkv
import workloads
from gpu_util import check_close, host_bits

pytestmark = pytest.mark.gpu

CASES = [("c2", 0), ("c3", 0), ("c3", 512), ("c4", 0), ("c5", 0), ("c5", 512), ("c3fp8", 0),
         ("c3e5m2", 0), ("c3spec", 0), ("c3specfp8", 0), ("c3prefill", 0)]


@pytest.mark.parametrize("workload,partition", CASES)
def test_bench_step_every_output(cuda_device, workload, partition):
    name = bench.WORKLOADS[workload]
    b = workloads.BUILDERS[name](device=cuda_device)
    host = b.host()                                     # the pools before the step
    step = bench.Step(b, partition)
    if partition:
        assert step.part_tokens == partition and step.split
    assert step.prefill == (workload == "c3prefill")     # long chunks: the tcgen05 kernel
    step()
    torch.cuda.synchronize(cuda_device)
    assert pkv.device_error_bits(cuda_device) == 0
    # the oracle's pass over the same step updates host's pools in place
    ref = bench.oracle_step(b, host, None, len(os.sched_getaffinity(0)))
    assert np.array_equal(host_bits(b.k_cache), host["k_cache"]), "k_cache differs from the oracle"
    assert np.array_equal(host_bits(b.v_cache), host["v_cache"]), "v_cache differs from the oracle"
    assert ref.shape == tuple(step.out.shape)
    check_close(step.out, ref, "f32" if b.dtype == "f32" else "bf16",
                f"{name} partition {step.part_tokens}")
