"""GPU parity of paged decode attention (through the C ABI) against the float64
oracle, on the same seeded inputs.

Covers: the tiny fp32 workload, randomised small shapes (head_dim 64/128,
group sizes 1..16, lengths around block boundaries, empty contexts), single-pass
vs split-K vs oracle, the split-K partials against the oracle's merge, the
paging invariants on the GPU (placement permutation and shared-vs-private are
bitwise), poisoned padding, device-side index errors, and every output of the
full-size workloads.
"""
import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_375_b200 as pkv
import workloads
from gpu_util import (check_close, dev_i32, gpu_step, host_bits,
                      oracle_caches_after_step, to_f64)

pytestmark = pytest.mark.gpu


def oracle_out(b, k, v, host):
    return oracle.paged_decode(host["q"], k, v, b.block_tables, b.context_lens, b.scale)


def run_and_check(b, partition_tokens=0, what=""):
    host = b.host()
    out, kc, vc = gpu_step(b, partition_tokens)
    assert pkv.device_error_bits() == 0
    k, v = oracle_caches_after_step(b, host)
    ref = oracle_out(b, k, v, host)
    return check_close(out, ref, b.dtype, what or b.name), out


def test_c1_tiny_fp32(cuda_device):
    b = workloads.c1_tiny_fp32(device=cuda_device)
    err, _ = run_and_check(b)
    assert err <= 1e-5


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("hq,hkv", [(8, 8), (8, 4), (8, 2), (32, 8), (16, 2), (16, 1), (6, 2)])
def test_random_shapes(cuda_device, dtype, d, hq, hkv):
    lens = [1, 2, 15, 16, 17, 31, 32, 33, 47, 64, 100, 255, 256, 257, 300]
    b = workloads.random_batch(100 + d + hq * 7 + hkv, lens, hq, hkv, d, dtype,
                               device=cuda_device, new_token=True, extra_table=2)
    run_and_check(b, what=f"{dtype} d{d} {hq}/{hkv}")


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("partition", [16, 48, 512])
def test_split_k_matches_oracle_and_single_pass(cuda_device, dtype, partition):
    lens = [0, 1, 16, 17, 500, 513, 1024, 1500, 2049]
    b = workloads.random_batch(7 + partition, lens, 16, 2, 128, dtype, device=cuda_device)
    host = b.host()
    ref = oracle_out(b, host["k_cache"], host["v_cache"], host)
    single, _, _ = gpu_step(b, 0)
    split, _, _ = gpu_step(b, partition)
    assert pkv.device_error_bits() == 0
    check_close(single, ref, dtype, "single-pass")
    check_close(split, ref, dtype, f"split {partition}")
    assert torch.all(split[0] == 0)   # empty context gives zeros


def test_split_k_partials_against_oracle_merge(cuda_device):
    """The merge kernel's output equals the oracle's merge of the partials the decode
    kernel wrote (fp32, so the comparison is tight), and each partial matches the
    oracle's own statistics of that partition."""
    lens = [700, 1100, 33, 1600]
    P = 256
    b = workloads.random_batch(21, lens, 4, 1, 64, "f32", device=cuda_device)
    dims = pkv.make_dims(b.num_seqs, b.num_q_heads, b.k_cache, b.max_blocks_per_seq)
    mcl = b.max_context_len
    need = pkv.decode_workspace_bytes(dims, mcl, P)
    ws = torch.zeros(need, dtype=torch.uint8, device=cuda_device)
    out = torch.empty_like(b.q)
    pkv.paged_attention_decode(out, b.q, b.k_cache, b.v_cache, dev_i32(b.block_tables, cuda_device),
                               dev_i32(b.context_lens, cuda_device), b.scale, b.num_kv_heads,
                               max_context_len=mcl, partition_tokens=P, workspace_tensor=ws)
    torch.cuda.synchronize()
    max_parts, po, pm = pkv.decode_workspace_layout(dims, mcl, P)
    B, Hq, D = b.q.shape
    part_o = ws[po:po + B * Hq * max_parts * D * 4].view(torch.float32).reshape(B, Hq, max_parts, D).cpu().numpy()
    part_ml = ws[pm:pm + B * Hq * max_parts * 8].view(torch.float32).reshape(B, Hq, max_parts, 2).cpu().numpy()
    host = b.host()
    got = to_f64(out)
    for s, L in enumerate(lens):
        n = (L + P - 1) // P
        for h in range(Hq):
            if n == 1:
                continue
            merged = oracle.lse_merge(part_ml[s, h, :n, 0], part_ml[s, h, :n, 1], part_o[s, h, :n])
            np.testing.assert_allclose(got[s, h], merged, rtol=0, atol=1e-6)
            for p in range(n):
                m, l, o = oracle.partition_stats(host["q"], host["k_cache"], host["v_cache"],
                                                 b.block_tables, b.context_lens, b.scale, s, h,
                                                 p * P, min(L, (p + 1) * P))
                assert abs(part_ml[s, h, p, 0] - m) <= 1e-5 * max(1.0, abs(m))
                assert abs(part_ml[s, h, p, 1] - l) <= 1e-5 * l
                np.testing.assert_allclose(part_o[s, h, p], o, rtol=0, atol=1e-5)


def test_placement_permutation_is_bitwise_invariant(cuda_device):
    b = workloads.random_batch(31, [5, 16, 130, 611, 1000], 32, 8, 128, "bf16", device=cuda_device)
    p = workloads.permute_placement(b, seed=32)
    o1, _, _ = gpu_step(b)
    o2, _, _ = gpu_step(p)
    assert torch.equal(o1.view(torch.int16), o2.view(torch.int16))


def test_shared_prefix_equals_private_copies_bitwise(cuda_device):
    b = workloads.c4_shared_prefix(device=cuda_device, prompts=4, samples=8, prefix=256,
                                   max_tail=100, num_blocks=2000)
    assert b.cow_pairs.shape[0] > 0
    host = b.host()
    shared, kc, vc = gpu_step(b)
    assert pkv.device_error_bits() == 0
    # the caches after the step are bit-identical to the oracle's
    k, v = oracle_caches_after_step(b, host)
    assert np.array_equal(host_bits(kc), k) and np.array_equal(host_bits(vc), v)
    after = workloads.Batch(b.name, b.seed, b.dtype, b.num_q_heads, b.num_kv_heads, b.head_dim,
                            b.num_blocks, b.context_lens, b.block_tables, b.scale, b.q, kc, vc,
                            b.new_k, b.new_v, b.new_seq, b.new_pos, b.cow_pairs)
    priv = workloads.private_copy(after)
    assert priv.num_blocks > b.num_blocks
    private, _, _ = gpu_step(priv, apply_step=False)
    assert torch.equal(shared.view(torch.int16), private.view(torch.int16))
    ref = oracle.paged_decode(host["q"], k, v, b.block_tables, b.context_lens, b.scale)
    check_close(shared, ref, "bf16", "shared prefix")


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_poisoned_padding_is_never_read(cuda_device, dtype):
    """Unused slots, blocks and table entries hold NaN / -1 / out-of-range values; the
    output is finite and bitwise equal to a run where they hold finite values."""
    b = workloads.random_batch(41, [1, 15, 17, 63, 129], 8, 2, 64, dtype, device=cuda_device,
                               extra_table=4)
    assert torch.isnan(b.k_cache).any()
    bt = b.block_tables.copy()
    bt[bt < 0] = 10 ** 6                       # table padding far out of range
    poisoned_b = workloads.Batch(**{**b.__dict__, "block_tables": bt})
    o1, _, _ = gpu_step(poisoned_b)
    assert pkv.device_error_bits() == 0
    clean_k = torch.nan_to_num(b.k_cache, nan=3.0)
    clean_v = torch.nan_to_num(b.v_cache, nan=-7.0)
    bt2 = b.block_tables.copy()
    bt2[bt2 < 0] = 0
    clean_b = workloads.Batch(**{**b.__dict__, "block_tables": bt2, "k_cache": clean_k,
                                 "v_cache": clean_v})
    o2, _, _ = gpu_step(clean_b)
    assert torch.isfinite(o1).all()
    assert torch.equal(o1, o2)


def test_bad_table_entry_is_flagged_not_read(cuda_device):
    b = workloads.random_batch(51, [40, 20], 4, 4, 64, "bf16", device=cuda_device)
    bt = b.block_tables.copy()
    bt[0, 1] = b.num_blocks + 5
    bad = workloads.Batch(**{**b.__dict__, "block_tables": bt})
    gpu_step(bad)
    bits = pkv.device_error_bits()
    assert bits & pkv.DEVERR_BLOCK
    assert pkv.device_error_bits() == 0       # reading clears the word


def test_context_longer_than_hint_is_flagged(cuda_device):
    b = workloads.random_batch(52, [40, 100], 4, 4, 64, "bf16", device=cuda_device)
    gpu_step(b, max_context_len=64)
    assert pkv.device_error_bits() & pkv.DEVERR_LEN


@pytest.mark.parametrize("name,partition", [
    ("c2_llama2_13b_mha", 0),
    ("c3_llama3_8b_gqa", 0),
    ("c3_llama3_8b_gqa", 512),
    ("c4_shared_prefix", 0),
    ("c5_long_splitk", 0),
    ("c5_long_splitk", 512),
])
def test_full_size_workloads_every_output(cuda_device, name, partition):
    """Full-size workloads in the launch configurations the benchmark uses (the Llama-3-8B
    batch through the fused decode prologue; the long-context batch with the automatic
    partition and with its configured 512-token partitions, about 1,300 partials per
    row): the pools after the step's copies and writes equal the oracle's byte for byte,
    and every output is recomputed by the oracle on all host cores."""
    b = workloads.BUILDERS[name](device=cuda_device)
    host = b.host()                                    # the pools before the step
    k_ref, v_ref = oracle_caches_after_step(b, host)
    if name == "c3_llama3_8b_gqa" and partition == 0:
        dev = b.q.device
        bt, cl = dev_i32(b.block_tables, dev), dev_i32(b.context_lens, dev)
        plan = pkv.DecodePlan(bt, cl, b.num_q_heads, b.k_cache, max_context_len=b.max_context_len,
                              new_k=b.new_k, new_v=b.new_v, v_cache=b.v_cache)
        out = torch.empty_like(b.q)
        plan.run(out, b.q, b.k_cache, b.v_cache, b.scale)
        kc, vc = b.k_cache, b.v_cache
    else:
        out, kc, vc = gpu_step(b, partition)
    if partition:
        assert pkv.decode_partition_tokens(
            pkv.make_dims(b.num_seqs, b.num_q_heads, b.k_cache, b.max_blocks_per_seq),
            b.max_context_len, partition) == partition
    assert pkv.device_error_bits() == 0
    assert np.array_equal(host_bits(kc), k_ref)
    assert np.array_equal(host_bits(vc), v_ref)
    ref = oracle.paged_decode(host["q"], k_ref, v_ref, b.block_tables, b.context_lens, b.scale)
    check_close(out, ref, b.dtype, f"{name} partition {partition}")
