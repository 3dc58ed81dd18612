"""Edge cases of the decode path on the GPU, against the float64 oracle.

The largest partition (8192 tokens = 512 blocks, the most an item stages in
shared memory), lengths on partition boundaries, one long sequence spread
over all SMs, the largest query group at fp32, a batch of empty contexts,
and a batch with many more work items than the scheduler's ring.
"""
import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_375_b200 as pkv
import workloads
from gpu_util import check_close, dev_i32, gpu_step, oracle_caches_after_step

pytestmark = pytest.mark.gpu


def run(b, partition_tokens=0, what=""):
    host = b.host()
    out, _, _ = gpu_step(b, partition_tokens)
    assert pkv.device_error_bits() == 0
    k, v = oracle_caches_after_step(b, host)
    ref = oracle.paged_decode(host["q"], k, v, b.block_tables, b.context_lens, b.scale)
    check_close(out, ref, b.dtype, what)
    return out


def test_largest_partition_and_items_of_512_blocks(cuda_device):
    lens = [8192, 8193, 12000, 16, 8191]
    b = workloads.random_batch(1001, lens, 8, 2, 128, "bf16", device=cuda_device, new_token=True)
    run(b, 8192, "partition 8192")


@pytest.mark.parametrize("partition", [512, 1024])
def test_lengths_on_partition_boundaries(cuda_device, partition):
    lens = [partition - 1, partition, partition + 1, 2 * partition, 2 * partition + 16, 1]
    b = workloads.random_batch(1002 + partition, lens, 32, 8, 128, "bf16", device=cuda_device,
                               new_token=True)
    run(b, partition, f"boundaries {partition}")


def test_one_long_sequence_spreads_over_the_sms(cuda_device):
    b = workloads.random_batch(1003, [60000], 32, 8, 128, "bf16", device=cuda_device,
                               new_token=True)
    dims = pkv.make_dims(1, 32, b.k_cache, b.max_blocks_per_seq)
    assert pkv.decode_partition_tokens(dims, 60000) < 60000     # split by the auto rule
    run(b, 0, "one long sequence")


def test_group_of_16_at_fp32(cuda_device):
    b = workloads.random_batch(1004, [1, 17, 300, 64], 16, 1, 64, "f32", device=cuda_device,
                               new_token=True)
    run(b, 0, "g16 fp32")


def test_batch_of_empty_contexts_gives_zeros(cuda_device):
    b = workloads.random_batch(1005, [0, 0, 0], 8, 8, 64, "bf16", device=cuda_device)
    out, _, _ = gpu_step(b, 0)
    assert pkv.device_error_bits() == 0
    assert torch.count_nonzero(out) == 0


def test_many_more_items_than_the_ring(cuda_device):
    rng = np.random.default_rng(1006)
    lens = rng.integers(0, 40, size=3000)
    b = workloads.random_batch(1006, lens, 8, 4, 64, "bf16", device=cuda_device, new_token=True)
    run(b, 0, "3000 short sequences")


def test_empty_step_launches_nothing(cuda_device):
    """No sequences and no new tokens: every call returns without a launch or an error."""
    dev = cuda_device
    kc = torch.zeros((4, 2, 16, 64), dtype=torch.bfloat16, device=dev)
    q = torch.zeros((0, 4, 64), dtype=torch.bfloat16, device=dev)
    bt = torch.zeros((0, 1), dtype=torch.int32, device=dev)
    cl = torch.zeros((0,), dtype=torch.int32, device=dev)
    pkv.paged_attention_decode(torch.empty_like(q), q, kc, kc, bt, cl, 0.125, 2,
                               max_context_len=16)
    empty = torch.zeros((0, 2, 64), dtype=torch.bfloat16, device=dev)
    pkv.reshape_and_cache(empty, empty, kc, kc, torch.zeros((0,), dtype=torch.int64, device=dev))
    assert pkv.device_error_bits() == 0
    assert torch.count_nonzero(kc) == 0


def test_fp8_largest_partition(cuda_device):
    lens = [8192, 9000, 5]
    b = workloads.random_batch(1007, lens, 32, 8, 128, "fp8", device=cuda_device)
    host = b.host()
    bt, cl = dev_i32(b.block_tables, cuda_device), dev_i32(b.context_lens, cuda_device)
    out = torch.empty_like(b.q)
    pkv.paged_attention_decode_fp8(out, b.q, b.k_cache, b.v_cache, bt, cl, b.scale, b.k_scale,
                                   b.v_scale, max_context_len=9000, partition_tokens=8192)
    assert pkv.device_error_bits() == 0
    ref = oracle.paged_decode_fp8(host["q"], host["k_cache"], host["v_cache"], b.k_scale,
                                  b.v_scale, b.block_tables, b.context_lens, b.scale)
    check_close(out, ref, "bf16", "fp8 partition 8192")
