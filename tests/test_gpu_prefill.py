"""GPU parity of the tcgen05 prefill path (pkv_paged_prefill, through the C ABI)
against the float64 oracle.

Chunk token i of a sequence of context L with an n-token chunk attends to keys
0 .. L - n + i (the multi-token reading of the pages' decode: chunked prefill
splits long prompts into chunks).  Covers whole-prompt prefill for query heads
per kv head g in {1, 4, 8}, chunks over a cached context (random chunk mixes,
lengths around the 16-token block, the 128-row query tile and the 128-key KV
tile), other group sizes (2, 3, 6, 16) and head_dim 64, long prompts (many KV
tiles, so the running maximum moves and the output rows are rescaled in
tensor memory), empty chunks and sequences, zero and negative scales, NaN in
every unused slot, device-side errors, and agreement with the decode kernel's
multi-token path.  Tolerance: |e| <= 2e-2 + 1e-2 |ref| element-wise.
"""
import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_375_b200 as pkv
import workloads
from gpu_util import check_close, dev_i32, oracle_caches_after_step

pytestmark = pytest.mark.gpu


def write_chunks(b):
    dev = b.q.device
    if b.new_seq.shape[0]:
        slots = pkv.slot_mapping(dev_i32(b.block_tables, dev), b.num_blocks,
                                 token_seq=dev_i32(b.new_seq, dev), token_pos=dev_i32(b.new_pos, dev))
        pkv.reshape_and_cache(b.new_k, b.new_v, b.k_cache, b.v_cache, slots)


def gpu_prefill(b, scale=None, max_context_len=None):
    dev = b.q.device
    write_chunks(b)
    out = torch.full_like(b.q, float("nan"))
    pkv.paged_prefill(out, b.q, b.k_cache, b.v_cache, dev_i32(b.block_tables, dev),
                      dev_i32(b.context_lens, dev), dev_i32(b.query_start_loc, dev),
                      b.scale if scale is None else scale, b.num_kv_heads,
                      max_context_len=max(b.max_context_len, 1) if max_context_len is None
                      else max_context_len)
    return out


def run_and_check(b, what, scale=None):
    host = b.host()
    out = gpu_prefill(b, scale)
    assert pkv.device_error_bits() == 0
    k, v = oracle_caches_after_step(b, host)
    ref = oracle.paged_multi(host["q"], k, v, b.block_tables, b.context_lens, b.query_start_loc,
                             b.scale if scale is None else scale)
    return check_close(out, ref, "bf16", what), out


@pytest.mark.parametrize("hq,hkv", [(8, 8), (32, 8), (64, 8)])
def test_whole_prompt_prefill(cuda_device, hq, hkv):
    lens = np.array([1, 5, 16, 17, 100, 127, 128, 129, 300, 777])
    b = workloads.chunked_batch(2000 + hq, lens, lens.copy(), hq, hkv, 128, "bf16",
                                device=cuda_device)
    run_and_check(b, f"whole prompts {hq}/{hkv}")


@pytest.mark.parametrize("hq,hkv", [(8, 8), (32, 8), (64, 8)])
def test_random_chunk_mix_over_cached_context(cuda_device, hq, hkv):
    rng = np.random.default_rng(2100 + hq)
    lens = rng.integers(1, 1500, size=12)
    lens[:4] = [16, 33, 256, 1024]
    chunks = np.minimum(rng.integers(1, 400, size=lens.shape[0]), lens)
    chunks[0] = 16
    chunks[2] = 129
    b = workloads.chunked_batch(2200 + hq, lens, chunks, hq, hkv, 128, "bf16",
                                device=cuda_device, extra_table=3)
    run_and_check(b, f"chunk mix {hq}/{hkv}")


@pytest.mark.parametrize("hq,hkv,d", [(16, 8, 128), (6, 2, 128), (12, 2, 64), (16, 1, 128),
                                      (8, 8, 64), (32, 8, 64)])
def test_other_groups_and_head_dims(cuda_device, hq, hkv, d):
    lens = np.array([3, 64, 200, 513])
    chunks = np.array([3, 40, 200, 300])
    b = workloads.chunked_batch(2300 + hq + d, lens, chunks, hq, hkv, d, "bf16",
                                device=cuda_device)
    run_and_check(b, f"groups {hq}/{hkv} d{d}")


def test_long_prompt_many_kv_tiles(cuda_device):
    lens = np.array([4096, 2500])
    b = workloads.chunked_batch(2400, lens, lens.copy(), 32, 8, 128, "bf16", device=cuda_device)
    run_and_check(b, "long prompts")


def test_empty_chunks_and_zero_length_sequences(cuda_device):
    lens = np.array([0, 20, 7, 0, 300, 5])
    chunks = np.array([0, 20, 0, 0, 150, 5])
    b = workloads.chunked_batch(2500, lens, chunks, 32, 8, 128, "bf16", device=cuda_device)
    run_and_check(b, "empty chunks")


@pytest.mark.parametrize("scale", [0.0, -0.05])
def test_zero_and_negative_scale(cuda_device, scale):
    lens = np.array([40, 300])
    b = workloads.chunked_batch(2600, lens, np.array([40, 200]), 32, 8, 128, "bf16",
                                device=cuda_device)
    run_and_check(b, f"scale {scale}", scale=scale)


def test_agrees_with_the_decode_kernel_multi_path(cuda_device):
    lens = np.array([50, 600, 1000])
    chunks = np.array([50, 100, 300])
    b = workloads.chunked_batch(2700, lens, chunks, 32, 8, 128, "bf16", device=cuda_device)
    host = b.host()
    out = gpu_prefill(b)
    dev = cuda_device
    multi = torch.empty_like(b.q)
    pkv.paged_attention_multi(multi, b.q, b.k_cache, b.v_cache, dev_i32(b.block_tables, dev),
                              dev_i32(b.context_lens, dev), dev_i32(b.query_start_loc, dev),
                              b.scale, b.num_kv_heads, int(chunks.max()),
                              max_context_len=b.max_context_len)
    assert pkv.device_error_bits() == 0
    k, v = oracle_caches_after_step(b, host)
    ref = oracle.paged_multi(host["q"], k, v, b.block_tables, b.context_lens, b.query_start_loc,
                             b.scale)
    check_close(out, ref, "bf16", "prefill")
    check_close(multi, ref, "bf16", "multi")
    # the two paths differ only in rounding order
    d = (out.double() - multi.double()).abs().max().item()
    assert d < 2e-2


def test_bad_table_entry_is_flagged(cuda_device):
    lens = np.array([40, 100])
    b = workloads.chunked_batch(2800, lens, np.array([40, 50]), 8, 8, 64, "bf16",
                                device=cuda_device)
    b.block_tables[1, 1] = b.num_blocks + 3
    out = gpu_prefill(b)
    assert pkv.device_error_bits() & pkv.DEVERR_BLOCK
    assert torch.isfinite(out[:40]).all()          # sequence 0 is untouched by the bad entry


def test_chunk_outside_the_query_rows_is_skipped_and_flagged(cuda_device):
    lens = np.array([10, 40])
    b = workloads.chunked_batch(2900, lens, np.array([2, 3]), 8, 8, 64, "bf16",
                                device=cuda_device)
    b.query_start_loc = np.array([0, 2, 9], dtype=np.int32)   # rows 2..8 but q has 5 rows
    gpu_prefill(b)
    assert pkv.device_error_bits() & pkv.DEVERR_LEN


def test_rejects_what_it_does_not_run(cuda_device):
    """fp32 pools are refused by the C entry point itself (the binding checks first)."""
    lens = np.array([20])
    b = workloads.chunked_batch(3000, lens, np.array([20]), 8, 8, 64, "f32", device=cuda_device)
    dev = cuda_device
    bt, cl, qsl = (dev_i32(b.block_tables, dev), dev_i32(b.context_lens, dev),
                   dev_i32(b.query_start_loc, dev))
    out = torch.empty_like(b.q)
    dims = pkv.make_dims(1, 8, b.k_cache, bt.shape[1])
    lib = pkv.load_library()
    st = lib.pkv_paged_prefill(pkv._p(out), pkv._p(b.q), pkv._p(b.k_cache), pkv._p(b.v_cache),
                               pkv._p(bt), pkv._p(cl), pkv._p(qsl), 20, b.scale,
                               pkv.ctypes.byref(dims), 20, pkv._stream_ptr(dev))
    assert pkv.STATUS_NAMES[st] == "PKV_ERR_UNSUPPORTED"
    with pytest.raises(TypeError):
        gpu_prefill(b)


def test_many_sequences(cuda_device):
    """300 short sequences: many units per CTA, the per-CTA tile prefix over all of
    them, chunks from 1 token to 150."""
    rng = np.random.default_rng(3100)
    lens = rng.integers(1, 200, size=300)
    chunks = np.minimum(rng.integers(1, 150, size=300), lens)
    b = workloads.chunked_batch(3100, lens, chunks, 32, 8, 128, "bf16", device=cuda_device)
    run_and_check(b, "300 sequences")
