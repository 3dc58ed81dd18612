"""GPU parity of the FP8 (e4m3) KV cache through the C ABI against the oracle.

reshape_and_cache_fp8 is compared bit for bit (the division by the scale in
float32, round to nearest even, saturation at +-448 are fixed on both sides).
Decode over e4m3 pools is compared with the float64 oracle under the bf16
tolerance: the codes widen exactly, q enters the products as f16 (exact for
the bf16 inputs used here), products accumulate in fp32 and the output is
rounded to bf16.
"""
import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_375_b200 as pkv
import workloads
from gpu_util import check_close, dev_i32

pytestmark = pytest.mark.gpu


def codes(t: torch.Tensor) -> np.ndarray:
    return t.detach().contiguous().cpu().view(torch.uint8).numpy()


def gpu_fp8_step(b, partition_tokens=0, max_context_len=None):
    dev = b.q.device
    bt = dev_i32(b.block_tables, dev)
    cl = dev_i32(b.context_lens, dev)
    if b.cow_pairs.shape[0]:
        pkv.copy_blocks(b.k_cache, b.v_cache, torch.from_numpy(b.cow_pairs))
    if b.new_seq.shape[0]:
        slots = pkv.slot_mapping(bt, b.num_blocks, token_seq=dev_i32(b.new_seq, dev),
                                 token_pos=dev_i32(b.new_pos, dev))
        pkv.reshape_and_cache_fp8(b.new_k, b.new_v, b.k_cache, b.v_cache, slots, b.k_scale,
                                  b.v_scale)
    out = torch.empty_like(b.q)
    pkv.paged_attention_decode_fp8(out, b.q, b.k_cache, b.v_cache, bt, cl, b.scale, b.k_scale,
                                   b.v_scale, max_context_len=max_context_len
                                   or max(b.max_context_len, 1),
                                   partition_tokens=partition_tokens)
    return out


def oracle_fp8_caches(b, host):
    k, v = host["k_cache"].copy(), host["v_cache"].copy()
    if b.cow_pairs.shape[0]:
        oracle.copy_blocks(k, v, b.cow_pairs)
    if b.new_seq.shape[0]:
        slots = oracle.slot_mapping(b.block_tables, b.new_seq, b.new_pos)
        oracle.reshape_and_cache_fp8(host["new_k"], host["new_v"], k, v, slots, b.k_scale,
                                     b.v_scale)
    return k, v


@pytest.mark.parametrize("scale", [1.0, 1.0 / 64.0, 0.0029296875, 3.5])
def test_reshape_and_cache_fp8_bit_exact(cuda_device, scale):
    dev = cuda_device
    T, hkv, d, nb = 300, 8, 128, 64
    gen = torch.Generator(device=dev).manual_seed(31)
    # magnitudes from 2^-30 to 2^12 so that subnormal codes, ties and saturation all occur
    mag = torch.exp2(torch.rand((T, hkv, d), generator=gen, device=dev) * 42 - 30)
    sign = torch.where(torch.rand((T, hkv, d), generator=gen, device=dev) < 0.5, -1.0, 1.0)
    k = (mag * sign).to(torch.bfloat16)
    v = (torch.randn((T, hkv, d), generator=gen, device=dev) * 300).to(torch.bfloat16)
    rng = np.random.default_rng(32)
    slots = rng.permutation(nb * 16)[:T].astype(np.int64)
    slots[::17] = -1
    kc = torch.full((nb, hkv, 16, d), 0x55, dtype=torch.uint8, device=dev)
    vc = torch.full_like(kc, 0x2a)
    k_host = k.cpu().view(torch.int16).numpy().view(np.uint16)
    v_host = v.cpu().view(torch.int16).numpy().view(np.uint16)
    ref_k, ref_v = codes(kc).copy(), codes(vc).copy()
    pkv.reshape_and_cache_fp8(k, v, kc.view(torch.float8_e4m3fn), vc.view(torch.float8_e4m3fn),
                              torch.from_numpy(slots).to(dev), scale, scale * 0.5)
    assert pkv.device_error_bits() == 0
    oracle.reshape_and_cache_fp8(k_host, v_host, ref_k, ref_v, slots, scale, scale * 0.5)
    np.testing.assert_array_equal(codes(kc), ref_k)
    np.testing.assert_array_equal(codes(vc), ref_v)


def test_reshape_and_cache_fp8_matches_torch_cast(cuda_device):
    """Cross-check with torch's own float32 -> float8_e4m3fn cast (round to nearest even)
    on values inside the e4m3 range, where torch and satfinite conversion agree."""
    dev = cuda_device
    gen = torch.Generator(device=dev).manual_seed(33)
    k = (torch.randn((64, 2, 128), generator=gen, device=dev) * 20).to(torch.bfloat16)
    kc = torch.zeros((8, 2, 16, 128), dtype=torch.float8_e4m3fn, device=dev)
    vc = torch.zeros_like(kc)
    slots = torch.arange(64, dtype=torch.int64, device=dev)
    pkv.reshape_and_cache_fp8(k, k, kc, vc, slots, 0.125, 0.125)
    want = (k.float() / 0.125).clamp(-448, 448).to(torch.float8_e4m3fn)
    got = kc.view(8, 2, 16, 128).permute(0, 2, 1, 3).reshape(128, 2, 128)[:64]
    assert torch.equal(got.view(torch.uint8), want.view(torch.uint8))


@pytest.mark.parametrize("hq,hkv", [(32, 8), (8, 8), (16, 1), (12, 4), (64, 8)])
def test_decode_fp8_matches_oracle(cuda_device, hq, hkv):
    lens = [1, 5, 16, 17, 31, 100, 257, 1000, 2049]
    b = workloads.random_batch(800 + hq + hkv, lens, hq, hkv, 128, "fp8", device=cuda_device,
                               new_token=True, extra_table=1)
    host = b.host()
    out = gpu_fp8_step(b)
    assert pkv.device_error_bits() == 0
    k, v = oracle_fp8_caches(b, host)
    np.testing.assert_array_equal(codes(b.k_cache), k)
    np.testing.assert_array_equal(codes(b.v_cache), v)
    ref = oracle.paged_decode_fp8(host["q"], k, v, b.k_scale, b.v_scale, b.block_tables,
                                  b.context_lens, b.scale)
    check_close(out, ref, "bf16", f"fp8 {hq}/{hkv}")


@pytest.mark.parametrize("partition", [16, 48, 256, 1024])
def test_decode_fp8_split_k(cuda_device, partition):
    lens = [3000, 17, 700, 4096, 1]
    b = workloads.random_batch(900 + partition, lens, 32, 8, 128, "fp8", device=cuda_device,
                               new_token=True)
    host = b.host()
    out = gpu_fp8_step(b, partition_tokens=partition)
    assert pkv.device_error_bits() == 0
    k, v = oracle_fp8_caches(b, host)
    ref = oracle.paged_decode_fp8(host["q"], k, v, b.k_scale, b.v_scale, b.block_tables,
                                  b.context_lens, b.scale)
    check_close(out, ref, "bf16", f"fp8 split {partition}")


def test_decode_fp8_scales_enter_linearly(cuda_device):
    """Doubling v_scale doubles the output (exactly, up to bf16 rounding of both);
    k_scale multiplies the scores like the softmax scale does."""
    b = workloads.random_batch(950, [40, 300, 77], 32, 8, 128, "fp8", device=cuda_device)
    bt, cl = dev_i32(b.block_tables, b.q.device), dev_i32(b.context_lens, b.q.device)
    o1 = torch.empty_like(b.q)
    o2 = torch.empty_like(b.q)
    o3 = torch.empty_like(b.q)
    pkv.paged_attention_decode_fp8(o1, b.q, b.k_cache, b.v_cache, bt, cl, b.scale, 0.5, 1.0,
                                   max_context_len=300)
    pkv.paged_attention_decode_fp8(o2, b.q, b.k_cache, b.v_cache, bt, cl, b.scale, 0.5, 2.0,
                                   max_context_len=300)
    pkv.paged_attention_decode_fp8(o3, b.q, b.k_cache, b.v_cache, bt, cl, b.scale * 2, 0.25,
                                   1.0, max_context_len=300)
    assert torch.equal(o2.float(), (o1.float() * 2).bfloat16().float())
    assert torch.equal(o1.view(torch.int16), o3.view(torch.int16))


def test_copy_blocks_on_fp8_pools(cuda_device):
    dev = cuda_device
    gen = torch.Generator(device=dev).manual_seed(34)
    kc = torch.randint(0, 256, (40, 8, 16, 128), generator=gen, device=dev, dtype=torch.uint8)
    vc = torch.randint(0, 256, (40, 8, 16, 128), generator=gen, device=dev, dtype=torch.uint8)
    pairs = np.array([[3, 7], [8, 9], [0, 39], [12, 13]], dtype=np.int64)
    rk, rv = codes(kc).copy(), codes(vc).copy()
    pkv.copy_blocks(kc.view(torch.float8_e4m3fn), vc.view(torch.float8_e4m3fn),
                    torch.from_numpy(pairs))
    assert pkv.device_error_bits() == 0
    oracle.copy_blocks(rk, rv, pairs)
    np.testing.assert_array_equal(codes(kc), rk)
    np.testing.assert_array_equal(codes(vc), rv)


def test_plan_run_fp8_equals_one_shot(cuda_device):
    b = workloads.random_batch(960, [2000, 33, 512, 900], 32, 8, 128, "fp8", device=cuda_device)
    bt, cl = dev_i32(b.block_tables, b.q.device), dev_i32(b.context_lens, b.q.device)
    a = torch.empty_like(b.q)
    pkv.paged_attention_decode_fp8(a, b.q, b.k_cache, b.v_cache, bt, cl, b.scale, b.k_scale,
                                   b.v_scale, max_context_len=2000, partition_tokens=256)
    plan = pkv.DecodePlan(bt, cl, 32, b.k_cache, max_context_len=2000, partition_tokens=256)
    c = torch.empty_like(b.q)
    plan.run_fp8(c, b.q, b.k_cache, b.v_cache, b.scale, b.k_scale, b.v_scale)
    assert torch.equal(a.view(torch.int16), c.view(torch.int16))


def test_fp8_dims_rejected_where_unsupported(cuda_device):
    b = workloads.random_batch(970, [20], 8, 8, 128, "fp8", device=cuda_device)
    bt, cl = dev_i32(b.block_tables, b.q.device), dev_i32(b.context_lens, b.q.device)
    out = torch.empty_like(b.q)
    # the plain decode call has no scales: it refuses FP8 pools
    dims = pkv.make_dims(1, 8, b.k_cache, bt.shape[1])
    ws = torch.empty(pkv.decode_workspace_bytes(dims, 20), dtype=torch.uint8, device=b.q.device)
    st = pkv.load_library().pkv_paged_attention_decode(
        pkv._p(out), pkv._p(b.q), pkv._p(b.k_cache), pkv._p(b.v_cache), pkv._p(bt), pkv._p(cl),
        b.scale, pkv.ctypes.byref(dims), 20, 0, pkv._p(ws), ws.numel(),
        pkv._stream_ptr(b.q.device))
    assert st == 3
    # head_dim 64 FP8 pools are not supported
    kc = torch.zeros((4, 8, 16, 64), dtype=torch.float8_e4m3fn, device=b.q.device)
    q = torch.zeros((1, 8, 64), dtype=torch.bfloat16, device=b.q.device)
    with pytest.raises(pkv.PkvError):
        pkv.paged_attention_decode_fp8(torch.empty_like(q), q, kc, kc, bt, cl, 0.125, 1.0, 1.0)
    with pytest.raises(pkv.PkvError):
        pkv.paged_attention_decode_fp8(out, b.q, b.k_cache, b.v_cache, bt, cl, b.scale, 0.0, 1.0)


def test_c3_fp8_full_size_every_output(cuda_device):
    """The full Llama-3-8B-shaped batch over FP8 pools, through the fused decode prologue
    the benchmark times: both pools bit for bit against the oracle's quantising writes,
    and every output against the oracle on all host cores."""
    b = workloads.c3_fp8(device=cuda_device)
    host = b.host()
    k_ref, v_ref = oracle_fp8_caches(b, host)
    dev = b.q.device
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
                                  b.context_lens, b.scale)
    check_close(out, ref, "bf16", "c3 fp8, every output")


def test_plain_multi_call_rejects_fp8_pools(cuda_device):
    b = workloads.random_batch(980, [20, 30], 8, 2, 128, "fp8", device=cuda_device)
    bt, cl = dev_i32(b.block_tables, b.q.device), dev_i32(b.context_lens, b.q.device)
    qsl = torch.tensor([0, 1, 2], dtype=torch.int32, device=b.q.device)
    out = torch.empty_like(b.q)
    dims = pkv.make_dims(2, 8, b.k_cache, bt.shape[1])
    lib = pkv.load_library()
    need = lib.pkv_multi_workspace_bytes(pkv.ctypes.byref(dims), 2, 30, 0)
    ws = torch.empty(need, dtype=torch.uint8, device=b.q.device)
    st = lib.pkv_paged_attention_multi(
        pkv._p(out), pkv._p(b.q), pkv._p(b.k_cache), pkv._p(b.v_cache), pkv._p(bt), pkv._p(cl),
        pkv._p(qsl), 2, 1, b.scale, pkv.ctypes.byref(dims), 30, 0, pkv._p(ws), ws.numel(),
        pkv._stream_ptr(b.q.device))
    assert st == 3


def gpu_fp8_multi(b, partition_tokens=0, plan=False):
    dev = b.q.device
    bt = dev_i32(b.block_tables, dev)
    cl = dev_i32(b.context_lens, dev)
    qsl = dev_i32(b.query_start_loc, dev)
    if b.new_seq.shape[0]:
        slots = pkv.slot_mapping(bt, b.num_blocks, token_seq=dev_i32(b.new_seq, dev),
                                 token_pos=dev_i32(b.new_pos, dev))
        pkv.reshape_and_cache_fp8(b.new_k, b.new_v, b.k_cache, b.v_cache, slots, b.k_scale,
                                  b.v_scale)
    out = torch.empty_like(b.q)
    mcl = max(b.max_context_len, 1)
    if plan:
        dims = pkv.make_dims(b.num_seqs, b.num_q_heads, b.k_cache, bt.shape[1])
        need = pkv.load_library().pkv_multi_workspace_bytes(pkv.ctypes.byref(dims), b.q.shape[0],
                                                            mcl, partition_tokens)
        ws = torch.empty(need, dtype=torch.uint8, device=dev)
        p = pkv.DecodePlan(bt, cl, b.num_q_heads, b.k_cache, max_context_len=mcl,
                           partition_tokens=partition_tokens, workspace_tensor=ws)
        p.run_multi_fp8(out, b.q, b.k_cache, b.v_cache, qsl, b.max_query_len, b.scale,
                        b.k_scale, b.v_scale)
    else:
        pkv.paged_attention_multi_fp8(out, b.q, b.k_cache, b.v_cache, bt, cl, qsl, b.scale,
                                      b.k_scale, b.v_scale, b.max_query_len,
                                      max_context_len=mcl, partition_tokens=partition_tokens)
    return out


# chunks x group <= 16 rows run on the tensor-core kernel (4-, 8- and 16-row units),
# longer chunks in row groups on decode_kernel
@pytest.mark.parametrize("hq,hkv,max_chunk", [(32, 8, 2), (8, 8, 8), (16, 8, 4), (24, 8, 2),
                                             (32, 8, 4), (8, 8, 16), (16, 2, 2), (12, 4, 5),
                                             (16, 1, 1), (32, 8, 20), (16, 1, 3)])
def test_fp8_multi_matches_oracle(cuda_device, hq, hkv, max_chunk):
    rng = np.random.default_rng(hq * 31 + hkv * 7 + max_chunk)
    lens = np.array([1, 2, 15, 16, 17, 33, 64, 100, 257, 300, 31, 48])
    chunks = np.minimum(rng.integers(1, max_chunk + 1, size=lens.shape[0]), lens)
    b = workloads.chunked_batch(990 + hq + max_chunk, lens, chunks, hq, hkv, 128, "fp8",
                                device=cuda_device, extra_table=2)
    b.k_scale, b.v_scale = workloads.FP8_K_SCALE, workloads.FP8_V_SCALE
    host = b.host()
    out = gpu_fp8_multi(b)
    assert pkv.device_error_bits() == 0
    k, v = oracle_fp8_caches(b, host)
    ref = oracle.paged_multi_fp8(host["q"], k, v, b.k_scale, b.v_scale, b.block_tables,
                                 b.context_lens, b.query_start_loc, b.scale)
    check_close(out, ref, "bf16", f"fp8 multi {hq}/{hkv} chunks<={max_chunk}")


@pytest.mark.parametrize("partition,chunks", [(16, (4, 3, 4, 1, 2)), (256, (4, 3, 4, 1, 2)),
                                              (16, (2, 1, 2, 2, 1)), (256, (2, 1, 2, 2, 1))])
def test_fp8_multi_split_k_and_plan_run(cuda_device, partition, chunks):
    """Split-K and plan/run for chunks of up to 4 tokens (16-row units) and of up to 2
    (8-row units), both on the tensor-core kernel."""
    lens = np.array([40, 300, 1000, 2100, 5])
    chunks = np.array(chunks)
    b = workloads.chunked_batch(995 + partition, lens, chunks, 32, 8, 128, "fp8",
                                device=cuda_device)
    b.k_scale, b.v_scale = workloads.FP8_K_SCALE, workloads.FP8_V_SCALE
    host = b.host()
    out = gpu_fp8_multi(b, partition)
    assert pkv.device_error_bits() == 0
    k, v = oracle_fp8_caches(b, host)
    ref = oracle.paged_multi_fp8(host["q"], k, v, b.k_scale, b.v_scale, b.block_tables,
                                 b.context_lens, b.query_start_loc, b.scale)
    check_close(out, ref, "bf16", f"fp8 multi split {partition}")
    again = gpu_fp8_multi(b, partition, plan=True)     # the K/V writes are idempotent
    assert torch.equal(out.view(torch.int16), again.view(torch.int16))


def test_fp8_one_token_chunks_equal_fp8_decode_bitwise(cuda_device):
    lens = np.array([3, 16, 17, 600, 1500])
    b = workloads.chunked_batch(997, lens, np.ones(5, dtype=np.int64), 32, 8, 128, "fp8",
                                device=cuda_device)
    b.k_scale, b.v_scale = workloads.FP8_K_SCALE, workloads.FP8_V_SCALE
    multi = gpu_fp8_multi(b)
    out = torch.empty_like(b.q)
    pkv.paged_attention_decode_fp8(out, b.q, b.k_cache, b.v_cache,
                                   dev_i32(b.block_tables, cuda_device),
                                   dev_i32(b.context_lens, cuda_device), b.scale, b.k_scale,
                                   b.v_scale, max_context_len=b.max_context_len)
    assert torch.equal(multi.view(torch.int16), out.view(torch.int16))


@pytest.mark.parametrize("hq,hkv,max_chunk", [(32, 8, 1), (32, 8, 4), (16, 1, 1), (8, 8, 16)])
def test_fp8_running_max_moves_in_later_tiles(cuda_device, hq, hkv, max_chunk):
    """Scores scaled up (softmax scale 1.0, about 11 times 1/sqrt(128)) over contexts of
    many 128-key tiles: the rows' maxima keep moving by more than the rescale slack after
    a unit's first tile, so the tensor-core kernel's softmax leaves its one-flag path and
    rescales O in tensor memory mid-unit (4- and 16-row units), beside units that never
    move."""
    lens = np.array([700, 1500, 2600, 4100, 130, 257, 16, 3000])
    chunks = np.minimum(np.full(lens.shape[0], max_chunk), lens)
    b = workloads.chunked_batch(1201 + hq + max_chunk, lens, chunks, hq, hkv, 128, "fp8",
                                device=cuda_device)
    b.k_scale, b.v_scale = workloads.FP8_K_SCALE, workloads.FP8_V_SCALE
    b.scale = 1.0
    host = b.host()
    out = gpu_fp8_multi(b)
    assert pkv.device_error_bits() == 0
    k, v = oracle_fp8_caches(b, host)
    ref = oracle.paged_multi_fp8(host["q"], k, v, b.k_scale, b.v_scale, b.block_tables,
                                 b.context_lens, b.query_start_loc, b.scale)
    check_close(out, ref, "bf16", f"fp8 moving maxima {hq}/{hkv} chunks {max_chunk}")
    split = gpu_fp8_multi(b, 256)
    assert pkv.device_error_bits() == 0
    check_close(split, ref, "bf16", f"fp8 moving maxima, 256-token partitions {hq}/{hkv}")
