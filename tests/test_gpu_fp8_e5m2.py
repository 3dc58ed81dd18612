"""GPU parity of FP8 e5m2 pools through the C ABI against the oracle: quantising writes
bit for bit, decode and several query tokens within the bf16 tolerance, the fused
prologue equal to the separate calls, and every output of the full Llama-3-8B-shaped
batch."""
import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_375_b200 as pkv
import workloads
from gpu_util import check_close, dev_i32

pytestmark = pytest.mark.gpu


def codes(t):
    return t.detach().contiguous().cpu().view(torch.uint8).numpy()


def write_new(b):
    dev = b.q.device
    bt = dev_i32(b.block_tables, dev)
    if b.new_seq.shape[0]:
        slots = pkv.slot_mapping(bt, b.num_blocks, token_seq=dev_i32(b.new_seq, dev),
                                 token_pos=dev_i32(b.new_pos, dev))
        pkv.reshape_and_cache_fp8(b.new_k, b.new_v, b.k_cache, b.v_cache, slots, b.k_scale,
                                  b.v_scale)


def oracle_caches(b, host):
    k, v = host["k_cache"].copy(), host["v_cache"].copy()
    if b.new_seq.shape[0]:
        slots = oracle.slot_mapping(b.block_tables, b.new_seq, b.new_pos)
        oracle.reshape_and_cache_fp8(host["new_k"], host["new_v"], k, v, slots, b.k_scale,
                                     b.v_scale, fmt="e5m2")
    return k, v


@pytest.mark.parametrize("scale", [1.0, 1.0 / 64.0, 3.5])
def test_reshape_e5m2_bit_exact(cuda_device, scale):
    dev = cuda_device
    T, hkv, d, nb = 300, 8, 128, 64
    gen = torch.Generator(device=dev).manual_seed(41)
    mag = torch.exp2(torch.rand((T, hkv, d), generator=gen, device=dev) * 50 - 30)
    sign = torch.where(torch.rand((T, hkv, d), generator=gen, device=dev) < 0.5, -1.0, 1.0)
    k = (mag * sign).to(torch.bfloat16)
    v = (torch.randn((T, hkv, d), generator=gen, device=dev) * 3e4).to(torch.bfloat16)
    slots = np.random.default_rng(42).permutation(nb * 16)[:T].astype(np.int64)
    slots[::13] = -1
    kc = torch.full((nb, hkv, 16, d), 0x11, dtype=torch.uint8, device=dev)
    vc = torch.full_like(kc, 0x22)
    ref_k, ref_v = codes(kc).copy(), codes(vc).copy()
    pkv.reshape_and_cache_fp8(k, v, kc.view(torch.float8_e5m2), vc.view(torch.float8_e5m2),
                              torch.from_numpy(slots).to(dev), scale, scale * 2)
    assert pkv.device_error_bits() == 0
    oracle.reshape_and_cache_fp8(k.cpu().view(torch.int16).numpy().view(np.uint16),
                                 v.cpu().view(torch.int16).numpy().view(np.uint16),
                                 ref_k, ref_v, slots, scale, scale * 2, fmt="e5m2")
    np.testing.assert_array_equal(codes(kc), ref_k)
    np.testing.assert_array_equal(codes(vc), ref_v)


@pytest.mark.parametrize("hq,hkv,partition", [(32, 8, 0), (8, 8, 0), (16, 1, 0), (12, 4, 48),
                                              (32, 8, 256)])
def test_decode_e5m2_matches_oracle(cuda_device, hq, hkv, partition):
    lens = [1, 5, 16, 17, 31, 100, 257, 1000, 2049]
    b = workloads.random_batch(1200 + hq + hkv + partition, lens, hq, hkv, 128, "fp8e5m2",
                               device=cuda_device, new_token=True, extra_table=1)
    host = b.host()
    write_new(b)
    out = torch.empty_like(b.q)
    pkv.paged_attention_decode_fp8(out, b.q, b.k_cache, b.v_cache,
                                   dev_i32(b.block_tables, cuda_device),
                                   dev_i32(b.context_lens, cuda_device), b.scale, b.k_scale,
                                   b.v_scale, max_context_len=b.max_context_len,
                                   partition_tokens=partition)
    assert pkv.device_error_bits() == 0
    k, v = oracle_caches(b, host)
    np.testing.assert_array_equal(codes(b.k_cache), k)
    ref = oracle.paged_decode_fp8(host["q"], k, v, b.k_scale, b.v_scale, b.block_tables,
                                  b.context_lens, b.scale, fmt="e5m2")
    check_close(out, ref, "bf16", f"e5m2 {hq}/{hkv} p{partition}")


@pytest.mark.parametrize("hq,hkv,max_chunk", [(32, 8, 4), (16, 2, 9), (8, 8, 30)])
def test_multi_e5m2_matches_oracle(cuda_device, hq, hkv, max_chunk):
    rng = np.random.default_rng(hq + max_chunk)
    lens = np.array([1, 17, 40, 64, 100, 300, 33])
    chunks = np.minimum(rng.integers(1, max_chunk + 1, size=lens.shape[0]), lens)
    b = workloads.chunked_batch(1250 + hq + max_chunk, lens, chunks, hq, hkv, 128, "fp8e5m2",
                                device=cuda_device)
    host = b.host()
    write_new(b)
    out = torch.empty_like(b.q)
    pkv.paged_attention_multi_fp8(out, b.q, b.k_cache, b.v_cache,
                                  dev_i32(b.block_tables, cuda_device),
                                  dev_i32(b.context_lens, cuda_device),
                                  dev_i32(b.query_start_loc, cuda_device), b.scale, b.k_scale,
                                  b.v_scale, b.max_query_len, max_context_len=b.max_context_len)
    assert pkv.device_error_bits() == 0
    k, v = oracle_caches(b, host)
    ref = oracle.paged_multi_fp8(host["q"], k, v, b.k_scale, b.v_scale, b.block_tables,
                                 b.context_lens, b.query_start_loc, b.scale, fmt="e5m2")
    check_close(out, ref, "bf16", f"e5m2 multi {hq}/{hkv} <= {max_chunk}")


def test_prologue_e5m2_equals_separate_calls(cuda_device):
    b = workloads.random_batch(1270, [3, 40, 700, 1500], 32, 8, 128, "fp8e5m2",
                               device=cuda_device, new_token=True)
    dev = cuda_device
    bt, cl = dev_i32(b.block_tables, dev), dev_i32(b.context_lens, dev)
    k1, v1 = b.k_cache.clone(), b.v_cache.clone()
    slots = pkv.slot_mapping(bt, b.num_blocks, context_lens=cl)
    pkv.reshape_and_cache_fp8(b.new_k, b.new_v, k1, v1, slots, b.k_scale, b.v_scale)
    k2, v2 = b.k_cache.clone(), b.v_cache.clone()
    out2 = torch.empty_like(b.q)
    plan = pkv.DecodePlan(bt, cl, 32, k2, max_context_len=1500, new_k=b.new_k, new_v=b.new_v,
                          v_cache=v2, k_scale=b.k_scale, v_scale=b.v_scale)
    plan.run_fp8(out2, b.q, k2, v2, b.scale, b.k_scale, b.v_scale)
    out1 = torch.empty_like(b.q)
    pkv.paged_attention_decode_fp8(out1, b.q, k1, v1, bt, cl, b.scale, b.k_scale, b.v_scale,
                                   max_context_len=1500)
    assert pkv.device_error_bits() == 0
    np.testing.assert_array_equal(codes(k1), codes(k2))
    np.testing.assert_array_equal(codes(v1), codes(v2))
    assert torch.equal(out1.view(torch.int16), out2.view(torch.int16))


def test_c3_e5m2_full_size_every_output(cuda_device):
    """The full Llama-3-8B-shaped batch over e5m2 pools, through the fused decode prologue
    the benchmark times: the pools bit for bit and every output against the oracle."""
    b = workloads.c3_fp8e5m2(device=cuda_device)
    host = b.host()
    k_ref, v_ref = oracle_caches(b, host)
    dev = cuda_device
    bt, cl = dev_i32(b.block_tables, dev), dev_i32(b.context_lens, dev)
    plan = pkv.DecodePlan(bt, cl, b.num_q_heads, b.k_cache, max_context_len=b.max_context_len,
                          new_k=b.new_k, new_v=b.new_v, v_cache=b.v_cache, k_scale=b.k_scale,
                          v_scale=b.v_scale)
    out = torch.empty_like(b.q)
    plan.run_fp8(out, b.q, b.k_cache, b.v_cache, b.scale, b.k_scale, b.v_scale)
    assert pkv.device_error_bits() == 0
    np.testing.assert_array_equal(codes(b.k_cache), k_ref)
    np.testing.assert_array_equal(codes(b.v_cache), v_ref)
    ref = oracle.paged_decode_fp8(host["q"], k_ref, v_ref, b.k_scale, b.v_scale, b.block_tables,
                                  b.context_lens, b.scale, fmt="e5m2")
    check_close(out, ref, "bf16", "c3 e5m2, every output")
