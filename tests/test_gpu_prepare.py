"""The fused decode prologue (pkv_decode_prepare / _fp8 through DecodePlan with new
tokens) against the three separate calls it replaces -- slot indexing in
context-length mode, reshape_and_cache, the plan -- and against the oracle: the
pools and slots bit for bit, the decode output bit for bit (the plan is the same)."""
import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_375_b200 as pkv
import workloads
from gpu_util import check_close, dev_i32, oracle_caches_after_step

pytestmark = pytest.mark.gpu


def _bits(t):
    return t.detach().contiguous().cpu().view(torch.uint8).numpy()


def separate(b, kc, vc, partition=0):
    dev = b.q.device
    bt, cl = dev_i32(b.block_tables, dev), dev_i32(b.context_lens, dev)
    slots = pkv.slot_mapping(bt, b.num_blocks, context_lens=cl)
    if b.dtype == "fp8":
        pkv.reshape_and_cache_fp8(b.new_k, b.new_v, kc, vc, slots, b.k_scale, b.v_scale)
    else:
        pkv.reshape_and_cache(b.new_k, b.new_v, kc, vc, slots)
    plan = pkv.DecodePlan(bt, cl, b.num_q_heads, kc, max_context_len=max(b.max_context_len, 1),
                          partition_tokens=partition)
    out = torch.empty_like(b.q)
    if b.dtype == "fp8":
        plan.run_fp8(out, b.q, kc, vc, b.scale, b.k_scale, b.v_scale)
    else:
        plan.run(out, b.q, kc, vc, b.scale)
    return out, slots


def fused(b, kc, vc, partition=0):
    dev = b.q.device
    bt, cl = dev_i32(b.block_tables, dev), dev_i32(b.context_lens, dev)
    slots = torch.full((b.num_seqs,), -7, dtype=torch.int64, device=dev)
    plan = pkv.DecodePlan(bt, cl, b.num_q_heads, kc, max_context_len=max(b.max_context_len, 1),
                          partition_tokens=partition, new_k=b.new_k, new_v=b.new_v, v_cache=vc,
                          k_scale=b.k_scale, v_scale=b.v_scale, slot_mapping_out=slots)
    out = torch.empty_like(b.q)
    if b.dtype == "fp8":
        plan.run_fp8(out, b.q, kc, vc, b.scale, b.k_scale, b.v_scale)
    else:
        plan.run(out, b.q, kc, vc, b.scale)
    return out, slots


@pytest.mark.parametrize("dtype,hq,hkv,d,partition", [
    ("bf16", 32, 8, 128, 0), ("bf16", 40, 40, 128, 0), ("f32", 8, 8, 64, 0),
    ("bf16", 16, 2, 64, 48), ("fp8", 32, 8, 128, 0), ("fp8", 16, 1, 128, 256)])
def test_fused_prologue_equals_the_separate_calls(cuda_device, dtype, hq, hkv, d, partition):
    lens = [1, 2, 15, 16, 17, 33, 100, 257, 1000, 2049]
    b = workloads.random_batch(1100 + hq + d, lens, hq, hkv, d, dtype, device=cuda_device,
                               new_token=True, extra_table=1)
    host = b.host()
    k1, v1 = b.k_cache.clone(), b.v_cache.clone()
    k2, v2 = b.k_cache.clone(), b.v_cache.clone()
    out1, slots1 = separate(b, k1, v1, partition)
    out2, slots2 = fused(b, k2, v2, partition)
    assert pkv.device_error_bits() == 0
    assert torch.equal(slots1, slots2)
    np.testing.assert_array_equal(_bits(k1), _bits(k2))
    np.testing.assert_array_equal(_bits(v1), _bits(v2))
    assert torch.equal(out1.view(torch.uint8), out2.view(torch.uint8))
    # and the oracle
    if dtype == "fp8":
        kh, vh = host["k_cache"].copy(), host["v_cache"].copy()
        oracle.reshape_and_cache_fp8(host["new_k"], host["new_v"], kh, vh,
                                     oracle.slot_mapping(b.block_tables, b.new_seq, b.new_pos),
                                     b.k_scale, b.v_scale)
        ref = oracle.paged_decode_fp8(host["q"], kh, vh, b.k_scale, b.v_scale, b.block_tables,
                                      b.context_lens, b.scale)
    else:
        kh, vh = oracle_caches_after_step(b, host)
        ref = oracle.paged_decode(host["q"], kh, vh, b.block_tables, b.context_lens, b.scale)
    # the pools byte for byte against the oracle's writes, in every dtype
    np.testing.assert_array_equal(_bits(k2), kh.view(np.uint8))
    np.testing.assert_array_equal(_bits(v2), vh.view(np.uint8))
    check_close(out2, ref, "bf16" if dtype == "fp8" else dtype, f"fused {dtype}")


def test_empty_sequences_have_no_new_token(cuda_device):
    b = workloads.random_batch(1120, [0, 20, 0, 5], 8, 2, 64, "bf16", device=cuda_device)
    dev = cuda_device
    new_k = torch.randn((4, 2, 64), device=dev).to(torch.bfloat16)
    new_v = torch.randn((4, 2, 64), device=dev).to(torch.bfloat16)
    before_k, before_v = _bits(b.k_cache).copy(), _bits(b.v_cache).copy()
    slots = torch.zeros(4, dtype=torch.int64, device=dev)
    bt, cl = dev_i32(b.block_tables, dev), dev_i32(b.context_lens, dev)
    pkv.DecodePlan(bt, cl, 8, b.k_cache, max_context_len=20, new_k=new_k, new_v=new_v,
                   v_cache=b.v_cache, slot_mapping_out=slots)
    assert pkv.device_error_bits() == 0
    sl = slots.cpu().numpy()
    assert sl[0] == -1 and sl[2] == -1
    want = oracle.slot_mapping(b.block_tables, np.array([1, 3]), np.array([19, 4]))
    assert np.array_equal(sl[[1, 3]], want)
    # exactly the two slots changed, to the new rows
    k_after = b.k_cache.cpu()
    changed = np.nonzero((_bits(b.k_cache) != before_k).reshape(b.num_blocks, 2, 16, -1)
                         .any(axis=(1, 3)))
    got = sorted(int(x) * 16 + int(y) for x, y in zip(*changed))
    assert got == sorted(want.tolist())
    v_after = b.v_cache.cpu()
    for s, slot in zip([1, 3], want):
        blk, off = divmod(int(slot), 16)
        assert torch.equal(k_after[blk, :, off], new_k[s].cpu())
        assert torch.equal(v_after[blk, :, off], new_v[s].cpu())
    changed_v = (_bits(b.v_cache) != before_v).reshape(b.num_blocks, 2, 16, -1).any(axis=(1, 3))
    assert changed_v.sum() == 2


def test_bad_table_entry_is_flagged_and_not_written(cuda_device):
    b = workloads.random_batch(1121, [20, 40], 8, 8, 64, "bf16", device=cuda_device,
                               new_token=True)
    b.block_tables[1, 2] = b.num_blocks + 5          # the block of position 39
    before = _bits(b.k_cache).copy()
    slots = torch.zeros(2, dtype=torch.int64, device=cuda_device)
    bt, cl = dev_i32(b.block_tables, cuda_device), dev_i32(b.context_lens, cuda_device)
    pkv.DecodePlan(bt, cl, 8, b.k_cache, max_context_len=40, new_k=b.new_k, new_v=b.new_v,
                   v_cache=b.v_cache, slot_mapping_out=slots)
    assert pkv.device_error_bits() & pkv.DEVERR_BLOCK
    assert slots.cpu().numpy()[1] == -1
    diff = (_bits(b.k_cache) != before).reshape(b.num_blocks, -1).any(axis=1)
    assert diff.sum() == 1                            # only sequence 0's block changed


def test_full_size_batch_fused_equals_separate(cuda_device):
    """The full Llama-3-8B-shaped batch: the fused prologue and the three separate calls
    give the same pools, slots and outputs, and both meet the oracle: the pools byte for
    byte, the slots exactly, every output within the bf16 tolerance."""
    b = workloads.c3_llama3_8b_gqa(device=cuda_device)
    host = b.host()
    k_ref, v_ref = oracle_caches_after_step(b, host)
    k1, v1 = b.k_cache.clone(), b.v_cache.clone()
    out1, s1 = separate(b, k1, v1)
    k2, v2 = b.k_cache.clone(), b.v_cache.clone()
    out2, s2 = fused(b, k2, v2)
    assert torch.equal(k1.view(torch.int16), k2.view(torch.int16))
    assert torch.equal(v1.view(torch.int16), v2.view(torch.int16))
    assert pkv.device_error_bits() == 0
    assert torch.equal(s1, s2)
    assert torch.equal(out1.view(torch.int16), out2.view(torch.int16))
    np.testing.assert_array_equal(_bits(k2), k_ref.view(np.uint8))
    np.testing.assert_array_equal(_bits(v2), v_ref.view(np.uint8))
    np.testing.assert_array_equal(s2.cpu().numpy(),
                                  oracle.slot_mapping(b.block_tables, b.new_seq, b.new_pos))
    ref = oracle.paged_decode(host["q"], k_ref, v_ref, b.block_tables, b.context_lens, b.scale)
    check_close(out2, ref, "bf16", "c3 fused prologue, every output")


# ---------------------------------------------------------------- token lists
def _write_separately(b, kc, vc, seq, pos):
    dev = b.q.device
    bt = dev_i32(b.block_tables, dev)
    slots = pkv.slot_mapping(bt, b.num_blocks, token_seq=seq, token_pos=pos)
    if workloads.fp8_format(b.dtype):
        pkv.reshape_and_cache_fp8(b.new_k, b.new_v, kc, vc, slots, b.k_scale, b.v_scale)
    else:
        pkv.reshape_and_cache(b.new_k, b.new_v, kc, vc, slots)
    return slots


@pytest.mark.parametrize("dtype,hq,hkv,d", [("bf16", 32, 8, 128), ("f32", 8, 4, 64),
                                            ("fp8", 32, 8, 128), ("fp8e5m2", 16, 4, 128)])
def test_token_prologue_for_chunks_equals_the_separate_calls(cuda_device, dtype, hq, hkv, d):
    """Chunks of several query tokens: the token prologue's pools, slots and plan against
    slot indexing (token mode) + reshape_and_cache + the plan; the decode over either is
    bitwise equal, and within tolerance of the oracle."""
    lens = np.array([5, 40, 300, 17, 1000, 64])
    chunks = np.array([1, 4, 4, 3, 7, 2])
    b = workloads.chunked_batch(1300 + hq, lens, chunks, hq, hkv, d, dtype, device=cuda_device)
    dev = cuda_device
    host = b.host()
    bt, cl = dev_i32(b.block_tables, dev), dev_i32(b.context_lens, dev)
    seq, pos = dev_i32(b.new_seq, dev), dev_i32(b.new_pos, dev)
    qsl = dev_i32(b.query_start_loc, dev)
    fp8 = workloads.fp8_format(dtype) is not None
    mcl = b.max_context_len
    ws_bytes = pkv.load_library().pkv_multi_workspace_bytes(
        __import__("ctypes").byref(pkv.make_dims(b.num_seqs, hq, b.k_cache, b.max_blocks_per_seq)),
        b.q.shape[0], mcl, 0)
    outs, pools, slot_sets = [], [], []
    for mode in ("separate", "fused"):
        kc, vc = b.k_cache.clone(), b.v_cache.clone()
        ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
        if mode == "separate":
            slots = _write_separately(b, kc, vc, seq, pos)
            plan = pkv.DecodePlan(bt, cl, hq, kc, max_context_len=mcl, workspace_tensor=ws)
        else:
            slots = torch.full((b.new_seq.shape[0],), -7, dtype=torch.int64, device=dev)
            plan = pkv.DecodePlan(bt, cl, hq, kc, max_context_len=mcl, workspace_tensor=ws,
                                  new_k=b.new_k, new_v=b.new_v, v_cache=vc, token_seq=seq,
                                  token_pos=pos, k_scale=b.k_scale, v_scale=b.v_scale,
                                  slot_mapping_out=slots)
        out = torch.empty_like(b.q)
        if fp8:
            plan.run_multi_fp8(out, b.q, kc, vc, qsl, b.max_query_len, b.scale, b.k_scale,
                               b.v_scale)
        else:
            plan.run_multi(out, b.q, kc, vc, qsl, b.max_query_len, b.scale)
        assert pkv.device_error_bits() == 0
        outs.append(out)
        pools.append((_bits(kc), _bits(vc)))
        slot_sets.append(slots.cpu().numpy())
    np.testing.assert_array_equal(slot_sets[0], slot_sets[1])
    np.testing.assert_array_equal(pools[0][0], pools[1][0])
    np.testing.assert_array_equal(pools[0][1], pools[1][1])
    assert torch.equal(outs[0].view(torch.uint8), outs[1].view(torch.uint8))
    # and the oracle
    k, v = host["k_cache"].copy(), host["v_cache"].copy()
    sl = oracle.slot_mapping(b.block_tables, b.new_seq, b.new_pos)
    if fp8:
        fmt = workloads.fp8_format(dtype)
        oracle.reshape_and_cache_fp8(host["new_k"], host["new_v"], k, v, sl, b.k_scale,
                                     b.v_scale, fmt=fmt)
        ref = oracle.paged_multi_fp8(host["q"], k, v, b.k_scale, b.v_scale, b.block_tables,
                                     b.context_lens, b.query_start_loc, b.scale, fmt=fmt)
    else:
        oracle.reshape_and_cache(host["new_k"], host["new_v"], k, v, sl)
        ref = oracle.paged_multi(host["q"], k, v, b.block_tables, b.context_lens,
                                 b.query_start_loc, b.scale)
    check_close(outs[1], ref, "f32" if dtype == "f32" else "bf16", f"token prologue {dtype}")


def test_token_prologue_with_shared_prefix_plan(cuda_device):
    """The parallel-sampling step: copy-on-write, then one launch writes every sample's
    tail and builds the shared-prefix plan; pools, slots and output bitwise equal to the
    separate calls (slot indexing, reshape_and_cache, the shared plan)."""
    b = workloads.c4_shared_prefix(device=cuda_device, prompts=3, samples=5, prefix=300,
                                   max_tail=60, num_blocks=500)
    dev = cuda_device
    host = b.host()
    bt, cl = dev_i32(b.block_tables, dev), dev_i32(b.context_lens, dev)
    seq, pos = dev_i32(b.new_seq, dev), dev_i32(b.new_pos, dev)
    gs = dev_i32(np.asarray(b.meta["group_start"]), dev)
    sb = dev_i32(np.asarray(b.meta["shared_blocks"]), dev)
    pairs = torch.from_numpy(b.cow_pairs).to(dev)
    outs, pools, slot_sets = [], [], []
    for mode in ("separate", "fused"):
        kc, vc = b.k_cache.clone(), b.v_cache.clone()
        pkv.copy_blocks(kc, vc, pairs)
        if mode == "separate":
            slots = _write_separately(b, kc, vc, seq, pos)
            plan = pkv.SharedDecodePlan(bt, cl, gs, sb, b.num_q_heads, kc,
                                        max_context_len=b.max_context_len)
        else:
            slots = torch.full((b.new_seq.shape[0],), -7, dtype=torch.int64, device=dev)
            plan = pkv.SharedDecodePlan(bt, cl, gs, sb, b.num_q_heads, kc,
                                        max_context_len=b.max_context_len, new_k=b.new_k,
                                        new_v=b.new_v, v_cache=vc, token_seq=seq, token_pos=pos,
                                        slot_mapping_out=slots)
        out = torch.empty_like(b.q)
        plan.run(out, b.q, kc, vc, b.scale)
        assert pkv.device_error_bits() == 0
        outs.append(out)
        pools.append((_bits(kc), _bits(vc)))
        slot_sets.append(slots.cpu().numpy())
    np.testing.assert_array_equal(slot_sets[0], slot_sets[1])
    np.testing.assert_array_equal(pools[0][0], pools[1][0])
    np.testing.assert_array_equal(pools[0][1], pools[1][1])
    assert torch.equal(outs[0].view(torch.uint8), outs[1].view(torch.uint8))
    k, v = oracle_caches_after_step(b, host)
    ref = oracle.paged_decode(host["q"], k, v, b.block_tables, b.context_lens, b.scale)
    check_close(outs[1], ref, "bf16", "shared-prefix step, one-launch prologue")


def test_token_prologue_flags_and_skips_bad_tokens(cuda_device):
    """A token of a sequence out of range, a position past the table and a table entry out
    of range are flagged and skipped (slot -1); the other tokens are written."""
    b = workloads.random_batch(1401, [20, 40, 70], 8, 2, 64, "bf16", device=cuda_device,
                               extra_table=1)
    dev = cuda_device
    bt_np = b.block_tables.copy()
    bt_np[2, 1] = b.num_blocks + 3                     # an entry out of range
    bt, cl = dev_i32(bt_np, dev), dev_i32(b.context_lens, dev)
    T = 6
    seq = dev_i32(np.array([0, 7, 1, 1, 2, -1]), dev)  # 7 and -1: no such sequence
    pos = dev_i32(np.array([3, 0, 39, 16 * bt_np.shape[1], 20, 0]), dev)  # past the table
    gen = torch.Generator(device=dev).manual_seed(3)
    k = torch.randn((T, 2, 64), generator=gen, device=dev).to(torch.bfloat16)
    v = torch.randn((T, 2, 64), generator=gen, device=dev).to(torch.bfloat16)
    kc, vc = b.k_cache.clone(), b.v_cache.clone()
    slots = torch.full((T,), -7, dtype=torch.int64, device=dev)
    pkv.DecodePlan(bt, cl, 8, kc, max_context_len=b.max_context_len, new_k=k, new_v=v,
                   v_cache=vc, token_seq=seq, token_pos=pos, slot_mapping_out=slots)
    bits = pkv.device_error_bits()
    assert bits == pkv.DEVERR_POS | pkv.DEVERR_BLOCK
    got = slots.cpu().numpy()
    want = [int(bt_np[0, 0]) * 16 + 3, -1, int(bt_np[1, 2]) * 16 + 7, -1, -1, -1]
    np.testing.assert_array_equal(got, want)
    # the written tokens landed, the rest of the pools is untouched
    kc2, vc2 = b.k_cache.clone(), b.v_cache.clone()
    keep = torch.tensor([0, 2], device=dev)
    pkv.reshape_and_cache(k[keep], v[keep], kc2, vc2, slots[keep])
    assert torch.equal(kc.view(torch.int16), kc2.view(torch.int16))
    assert torch.equal(vc.view(torch.int16), vc2.view(torch.int16))
