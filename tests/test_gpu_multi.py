"""GPU parity of several causal query tokens per sequence (through the C ABI)
against the float64 oracle: chunks of new tokens written by reshape_and_cache,
each with its query row attending to the context up to its own position."""
import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_375_b200 as pkv
import workloads
from gpu_util import check_close, dev_i32, oracle_caches_after_step

pytestmark = pytest.mark.gpu


def gpu_multi(b, partition_tokens=0, max_query_len=None):
    dev = b.q.device
    bt = dev_i32(b.block_tables, dev)
    cl = dev_i32(b.context_lens, dev)
    qsl = dev_i32(b.query_start_loc, dev)
    if b.new_seq.shape[0]:
        slots = pkv.slot_mapping(bt, b.num_blocks, token_seq=dev_i32(b.new_seq, dev),
                                 token_pos=dev_i32(b.new_pos, dev))
        pkv.reshape_and_cache(b.new_k, b.new_v, b.k_cache, b.v_cache, slots)
    out = torch.empty_like(b.q)
    pkv.paged_attention_multi(out, b.q, b.k_cache, b.v_cache, bt, cl, qsl, b.scale,
                              b.num_kv_heads, max_query_len or b.max_query_len,
                              max_context_len=max(b.max_context_len, 1),
                              partition_tokens=partition_tokens)
    return out


def run_and_check(b, partition_tokens=0, what=""):
    host = b.host()
    out = gpu_multi(b, partition_tokens)
    assert pkv.device_error_bits() == 0
    k, v = oracle_caches_after_step(b, host)
    ref = oracle.paged_multi(host["q"], k, v, b.block_tables, b.context_lens,
                             b.query_start_loc, b.scale)
    check_close(out, ref, b.dtype, what)
    return out


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("hq,hkv,max_chunk", [(32, 8, 4), (8, 8, 16), (16, 2, 2), (6, 2, 5),
                                             (8, 4, 8)])
@pytest.mark.parametrize("d", [64, 128])
def test_random_chunks(cuda_device, dtype, hq, hkv, max_chunk, d):
    rng = np.random.default_rng(hq * 100 + hkv * 10 + max_chunk + d)
    lens = np.array([1, 2, 15, 16, 17, 33, 64, 100, 257, 300, 31, 48])
    chunks = np.minimum(rng.integers(1, max_chunk + 1, size=lens.shape[0]), lens)
    b = workloads.chunked_batch(500 + d, lens, chunks, hq, hkv, d, dtype, device=cuda_device,
                                extra_table=2)
    run_and_check(b, what=f"{dtype} {hq}/{hkv} chunks<={max_chunk} d{d}")


@pytest.mark.parametrize("partition", [16, 64, 256])
def test_chunks_with_split_k(cuda_device, partition):
    lens = np.array([40, 300, 1000, 2100, 5])
    chunks = np.array([4, 3, 4, 1, 2])
    b = workloads.chunked_batch(600 + partition, lens, chunks, 32, 8, 128, "bf16",
                                device=cuda_device)
    run_and_check(b, partition, f"split {partition}")


def test_one_token_chunks_equal_decode_bitwise(cuda_device):
    lens = np.array([3, 16, 17, 600, 1500])
    b = workloads.chunked_batch(700, lens, np.ones(5, dtype=np.int64), 32, 8, 128, "bf16",
                                device=cuda_device)
    multi = gpu_multi(b)
    out = torch.empty_like(b.q)
    pkv.paged_attention_decode(out, b.q, b.k_cache, b.v_cache,
                               dev_i32(b.block_tables, cuda_device),
                               dev_i32(b.context_lens, cuda_device), b.scale, b.num_kv_heads,
                               max_context_len=b.max_context_len)
    assert torch.equal(multi.view(torch.int16), out.view(torch.int16))


def test_empty_chunks_and_zero_length_sequences(cuda_device):
    lens = np.array([0, 20, 7, 0, 33])
    chunks = np.array([0, 3, 0, 0, 2])
    b = workloads.chunked_batch(701, lens, chunks, 8, 2, 64, "bf16", device=cuda_device)
    run_and_check(b, what="empty chunks")


def test_chunk_longer_than_its_context_is_flagged(cuda_device):
    lens = np.array([10, 40])
    b = workloads.chunked_batch(702, lens, np.array([2, 3]), 8, 8, 64, "bf16", device=cuda_device)
    b.query_start_loc = np.array([0, 2, 5], dtype=np.int32)
    gpu_multi(b, max_query_len=2)     # the second chunk (3 tokens) exceeds max_query_len
    assert pkv.device_error_bits() & pkv.DEVERR_LEN


def test_chunk_outside_the_query_rows_is_skipped_and_flagged(cuda_device):
    lens = np.array([10, 40])
    b = workloads.chunked_batch(703, lens, np.array([2, 3]), 8, 8, 64, "bf16", device=cuda_device)
    b.query_start_loc = np.array([0, 2, 9], dtype=np.int32)   # rows 2..8 but q has 5 rows
    gpu_multi(b, max_query_len=16)
    assert pkv.device_error_bits() & pkv.DEVERR_LEN


@pytest.mark.parametrize("hq,hkv,chunk_cap,partition", [(32, 8, 40, 0), (8, 8, 100, 0),
                                                       (6, 2, 17, 0), (32, 8, 64, 256),
                                                       (16, 1, 9, 48)])
def test_long_chunks_in_row_groups(cuda_device, hq, hkv, chunk_cap, partition):
    """Chunks longer than 16 query rows per kv head: split into row groups of whole
    tokens, each reading only the keys its rows can see."""
    rng = np.random.default_rng(hq * 13 + chunk_cap)
    lens = np.array([1, 17, 40, 64, 100, 300, 1000, 33])
    chunks = np.minimum(rng.integers(1, chunk_cap + 1, size=lens.shape[0]), lens)
    chunks[1] = min(chunk_cap, lens[1])            # at least one chunk at the cap
    b = workloads.chunked_batch(800 + hq + chunk_cap, lens, chunks, hq, hkv, 128, "bf16",
                                device=cuda_device)
    run_and_check(b, partition, f"rows in groups {hq}/{hkv} chunks<={chunk_cap} p{partition}")


def test_whole_prompt_prefill_matches_oracle(cuda_device):
    """Every sequence's whole context as its chunk (a prompt prefilled in one call)."""
    lens = np.array([5, 16, 31, 77, 128])
    b = workloads.chunked_batch(811, lens, lens.copy(), 8, 2, 64, "f32", device=cuda_device)
    run_and_check(b, 0, "whole-prompt prefill fp32")
