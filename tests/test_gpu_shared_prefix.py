"""GPU parity of the shared-prefix decode (a prefix held by several consecutive sequences
is read once per kv head for the whole group) through the C ABI against the float64
oracle.

The call's definition: member s of a group reads its first P blocks through the group's
first table row and the rest through its own row.  The oracle gets exactly that as a
rewritten block table, so the tests also cover tables that do not share.

Covers: group sizes 1 .. 19 (more members than one item serves), query heads per kv
head 1, 2, 3, 4, 8 and 16, head_dim 64 and 128, bf16 and fp32, contexts ending exactly
at the prefix or one token past it, split-K of the prefix and of the tails, clamped and
invalid groups (flagged), the per-sequence prefix the plan records, plan/run against the
one-shot call, FP8 pools in both formats, and the shared-prefix workload of the
benchmark (CoW + new tokens first) against the oracle.
"""
import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_375_b200 as pkv
import workloads
from gpu_util import check_close, dev_i32, gpu_step, oracle_caches_after_step

pytestmark = pytest.mark.gpu


def substituted_tables(bt, group_start, shared, lens):
    """Block tables as the call defines them: every member's first P blocks taken from its
    group's first row (P lowered to each member's full blocks; groups of one untouched)."""
    bt = bt.copy()
    for i in range(len(shared)):
        a, e = int(group_start[i]), int(group_start[i + 1])
        if e - a < 2:
            continue
        P = min([int(shared[i])] + [int(lens[s]) // 16 for s in range(a, e)])
        for s in range(a + 1, e):
            bt[s, :P] = bt[a, :P]
    return bt


def shared_batch(seed, sizes, prefix_blocks, tails, hq, hkv, d, dtype, share=True):
    """Groups of consecutive sequences: group i has sizes[i] members whose tables begin with
    prefix_blocks[i] common blocks (when `share`) followed by their own tails.  No new
    tokens: a member whose context ends inside the prefix would write into a shared block
    (a serving engine copies such a block first; the benchmark workload test covers that)."""
    rng = np.random.default_rng(seed)
    lens = []
    for n, P in zip(sizes, prefix_blocks):
        for _ in range(n):
            lens.append(P * 16 + int(rng.choice(tails)))
    b = workloads.random_batch(seed, lens, hq, hkv, d, dtype, device="cpu")
    gs = np.concatenate([[0], np.cumsum(sizes)]).astype(np.int32)
    sb = np.asarray(prefix_blocks, dtype=np.int32)
    if share:
        b.block_tables = substituted_tables(b.block_tables, gs, sb, b.context_lens)
    return b, gs, sb


def run_shared(b, gs, sb, partition_tokens=0, plan_run=False):
    dev = b.q.device
    bt = dev_i32(b.block_tables, dev)
    cl = dev_i32(b.context_lens, dev)
    if b.new_seq.shape[0]:
        slots = pkv.slot_mapping(bt, b.num_blocks, token_seq=dev_i32(b.new_seq, dev),
                                 token_pos=dev_i32(b.new_pos, dev))
        if b.dtype in ("fp8", "fp8e5m2"):
            pkv.reshape_and_cache_fp8(b.new_k, b.new_v, b.k_cache, b.v_cache, slots, b.k_scale,
                                      b.v_scale)
        else:
            pkv.reshape_and_cache(b.new_k, b.new_v, b.k_cache, b.v_cache, slots)
    out = torch.empty_like(b.q)
    g, s = dev_i32(gs, dev), dev_i32(sb, dev)
    mcl = max(b.max_context_len, 1)
    fp8 = b.dtype in ("fp8", "fp8e5m2")
    if plan_run:
        plan = pkv.SharedDecodePlan(bt, cl, g, s, b.num_q_heads, b.k_cache, max_context_len=mcl,
                                    partition_tokens=partition_tokens)
        if fp8:
            plan.run_fp8(out, b.q, b.k_cache, b.v_cache, b.scale, b.k_scale, b.v_scale)
        else:
            plan.run(out, b.q, b.k_cache, b.v_cache, b.scale)
        return out, plan
    kw = dict(k_scale=b.k_scale, v_scale=b.v_scale) if fp8 else {}
    pkv.paged_attention_decode_shared(out, b.q, b.k_cache, b.v_cache, bt, cl, g, s, b.scale,
                                      max_context_len=mcl, partition_tokens=partition_tokens,
                                      **kw)
    return out, None


def oracle_ref(b, host, tables):
    """The oracle's decode over `tables` (the batches here write no new tokens)."""
    assert b.new_seq.shape[0] == 0 and b.cow_pairs.shape[0] == 0
    if b.dtype in ("fp8", "fp8e5m2"):
        return oracle.paged_decode_fp8(host["q"], host["k_cache"], host["v_cache"], b.k_scale,
                                       b.v_scale, tables, b.context_lens, b.scale,
                                       fmt=workloads.fp8_format(b.dtype))
    return oracle.paged_decode(host["q"], host["k_cache"], host["v_cache"], tables,
                               b.context_lens, b.scale)


SIZES = [1, 2, 3, 5, 8, 19, 4]
PREFIX = [3, 4, 1, 6, 9, 5, 2]


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("hq,hkv", [(8, 8), (8, 4), (6, 2), (32, 8), (16, 2), (16, 1)])
def test_groups_match_oracle(cuda_device, dtype, d, hq, hkv):
    b, gs, sb = shared_batch(300 + d + 7 * hq + hkv, SIZES, PREFIX, [0, 1, 2, 15, 16, 17, 40],
                             hq, hkv, d, dtype)
    b = b.to(cuda_device)
    host = b.host()
    out, _ = run_shared(b, gs, sb)
    assert pkv.device_error_bits() == 0
    check_close(out, oracle_ref(b, host, b.block_tables), dtype, f"{dtype} d{d} {hq}/{hkv}")


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_tables_that_do_not_share(cuda_device, dtype):
    """Members whose own rows differ still read the first member's prefix blocks."""
    b, gs, sb = shared_batch(11, SIZES, PREFIX, [1, 9, 33], 32, 8, 128, dtype, share=False)
    b = b.to(cuda_device)
    host = b.host()
    out, _ = run_shared(b, gs, sb)
    assert pkv.device_error_bits() == 0
    tables = substituted_tables(b.block_tables, gs, sb, b.context_lens)
    assert (tables != b.block_tables).any()
    check_close(out, oracle_ref(b, host, tables), dtype, "substituted prefix")


@pytest.mark.parametrize("partition", [16, 48, 64, 512])
def test_split_k_of_prefix_and_tails(cuda_device, partition):
    b, gs, sb = shared_batch(23 + partition, [4, 7, 2, 1], [70, 33, 5, 40], [0, 1, 100, 700],
                             32, 8, 128, "bf16")
    b = b.to(cuda_device)
    host = b.host()
    ref = oracle_ref(b, host, b.block_tables)
    out, _ = run_shared(b, gs, sb, partition)
    assert pkv.device_error_bits() == 0
    check_close(out, ref, "bf16", f"partition {partition}")


def test_prefix_recorded_and_clamped(cuda_device):
    """The plan's per-sequence prefix: as given, lowered to a member's full blocks (flagged),
    none for a group of one or a sequence in no group."""
    lens = [16 * 5 + 3, 16 * 5 + 9, 16 * 3 + 2, 40, 16 * 4, 16 * 4 + 1, 99]
    b = workloads.random_batch(5, lens, 16, 4, 128, "f32", device="cpu")
    gs = np.array([0, 3, 4, 6], dtype=np.int32)      # sequence 6 is in no group
    sb = np.array([5, 2, 4], dtype=np.int32)         # group 0: member 2 has 3 full blocks
    b.block_tables = substituted_tables(b.block_tables, gs, sb, b.context_lens)
    b = b.to(cuda_device)
    host = b.host()
    out, plan = run_shared(b, gs, sb, plan_run=True)
    assert pkv.device_error_bits() & pkv.DEVERR_GROUP
    _, _, _, sp_off = pkv.decode_shared_workspace_layout(plan.dims, plan.max_context_len)
    sp = plan.workspace[sp_off:sp_off + 4 * b.num_seqs].view(torch.int32).cpu().numpy()
    np.testing.assert_array_equal(sp, [3, 3, 3, 0, 4, 4, 0])
    check_close(out, oracle_ref(b, host, b.block_tables), "f32", "clamped")


@pytest.mark.parametrize("gs", [[0, 3, 2, 7], [0, 3, 8, 7], [-1, 3, 5, 7]])
def test_invalid_groups_flagged_and_ignored(cuda_device, gs):
    """Bounds that are not nondecreasing in [0, B] are flagged and no group is used: each
    sequence then reads its own table."""
    b, _, _ = shared_batch(9, [3, 2, 2], [4, 4, 4], [1, 20], 16, 4, 128, "f32", share=False)
    b = b.to(cuda_device)
    host = b.host()
    gs = np.array(gs, dtype=np.int32)
    out, _ = run_shared(b, gs, np.array([4, 4, 4], dtype=np.int32))
    assert pkv.device_error_bits() & pkv.DEVERR_GROUP
    check_close(out, oracle_ref(b, host, b.block_tables), "f32", "ignored groups")


def test_plan_run_matches_one_shot_and_reruns(cuda_device):
    b, gs, sb = shared_batch(31, SIZES, PREFIX, [0, 5, 17, 60], 32, 8, 128, "bf16")
    b = b.to(cuda_device)
    one, _ = run_shared(b, gs, sb)
    # the new tokens are already written; write them again (same values) via plan/run
    two, plan = run_shared(b, gs, sb, plan_run=True)
    again = torch.empty_like(two)
    plan.run(again, b.q, b.k_cache, b.v_cache, b.scale)
    assert pkv.device_error_bits() == 0
    assert torch.equal(one, two) and torch.equal(two, again)


def test_empty_and_single_groups(cuda_device):
    """No groups at all, and empty groups between real ones, give plain decode's result."""
    b, _, _ = shared_batch(41, [2, 3], [2, 2], [3, 30], 8, 2, 64, "f32")
    b = b.to(cuda_device)
    host = b.host()
    ref = oracle_ref(b, host, b.block_tables)
    out, _ = run_shared(b, np.array([0], dtype=np.int32), np.zeros(0, dtype=np.int32))
    check_close(out, ref, "f32", "no groups")
    out, _ = run_shared(b, np.array([0, 0, 2, 2, 5], dtype=np.int32),
                        np.array([7, 2, 0, 2], dtype=np.int32))
    assert pkv.device_error_bits() == 0
    check_close(out, ref, "f32", "empty groups")


@pytest.mark.parametrize("dtype", ["fp8", "fp8e5m2"])
def test_fp8_pools(cuda_device, dtype):
    fp8, gs, sb = shared_batch(51, SIZES, PREFIX, [0, 1, 16, 50], 32, 8, 128, dtype)
    fp8 = fp8.to(cuda_device)
    host = fp8.host()
    out, _ = run_shared(fp8, gs, sb)
    assert pkv.device_error_bits() == 0
    check_close(out, oracle_ref(fp8, host, fp8.block_tables), "bf16", dtype)
    out2, _ = run_shared(fp8, gs, sb, plan_run=True)
    assert torch.equal(out, out2)


def test_shared_prefix_workload_small(cuda_device):
    """The benchmark's parallel-sampling batch at a reduced size: copy-on-write and the
    tails' writes first, then the shared-prefix decode, against the oracle."""
    b = workloads.c4_shared_prefix(device=cuda_device, prompts=4, samples=8, prefix=256,
                                   max_tail=100)
    host = b.host()
    gs = np.asarray(b.meta["group_start"], dtype=np.int32)
    sb = np.asarray(b.meta["shared_blocks"], dtype=np.int32)
    # the copies and writes as in the plain step (no decode yet), then the shared decode
    gpu_step(b, apply_step=True)
    dev = b.q.device
    out = torch.empty_like(b.q)
    pkv.paged_attention_decode_shared(out, b.q, b.k_cache, b.v_cache,
                                      dev_i32(b.block_tables, dev), dev_i32(b.context_lens, dev),
                                      dev_i32(gs, dev), dev_i32(sb, dev), b.scale,
                                      max_context_len=b.max_context_len)
    assert pkv.device_error_bits() == 0
    k, v = oracle_caches_after_step(b, host)
    ref = oracle.paged_decode(host["q"], k, v, b.block_tables, b.context_lens, b.scale)
    check_close(out, ref, "bf16", "c4 small")


def test_block_manager_groups_drive_the_shared_decode(cuda_device):
    """Forks and prefix caching in the host block manager, its tables, slots and groups,
    then the KV written through reshape_and_cache (copies first) and the shared decode,
    against the oracle over the manager's own tables."""
    dev = cuda_device
    hq, hkv, d, nb = 32, 8, 128, 600
    rng = np.random.default_rng(77)
    bm = pkv.BlockManager(nb, 16, seed=3, prefix_caching=True)
    ids, prompts = [], {}
    for p, (plen, samples) in enumerate([(70, 4), (200, 8), (33, 1), (160, 3)]):
        root = 100 * p
        prompts[root] = plen
        bm.add_sequence(root, rng.integers(0, 30000, size=plen).tolist())
        ids.append(root)
        for c in range(1, samples):
            bm.fork(root, root + c)
            ids.append(root + c)
    # every sequence decodes a few tokens of its own (copy-on-write of shared partial blocks)
    for _ in range(5):
        bm.append_tokens(ids, rng.integers(0, 30000, size=len(ids)).astype(np.int32))
    pairs = bm.take_copies()
    tables, lens = bm.block_tables(ids, max_blocks=32)
    gs, sb = bm.shared_prefix_groups(ids, 1)
    assert (sb > 0).sum() == 3
    # K/V for every written position, through the manager's slots
    gen = torch.Generator(device=dev).manual_seed(5)
    k_cache = torch.full((nb, hkv, 16, d), float("nan"), dtype=torch.bfloat16, device=dev)
    v_cache = torch.full_like(k_cache, float("nan"))
    slots = np.concatenate([bm.slots(s, 0, int(L)) for s, L in zip(ids, lens)])
    # positions shared by several sequences have one slot: write each slot once
    slots = np.unique(slots)
    T = slots.shape[0]
    k = torch.randn((T, hkv, d), generator=gen, device=dev).to(torch.bfloat16)
    v = torch.randn((T, hkv, d), generator=gen, device=dev).to(torch.bfloat16)
    if pairs.shape[0]:
        pkv.copy_blocks(k_cache, v_cache, torch.from_numpy(pairs))
    pkv.reshape_and_cache(k, v, k_cache, v_cache, torch.from_numpy(slots).to(dev))
    q = torch.randn((len(ids), hq, d), generator=gen, device=dev).to(torch.bfloat16)
    out = torch.empty_like(q)
    scale = float(np.float32(1.0 / np.sqrt(d)))
    pkv.paged_attention_decode_shared(out, q, k_cache, v_cache, dev_i32(tables, dev),
                                      dev_i32(lens, dev), dev_i32(gs, dev), dev_i32(sb, dev),
                                      scale, max_context_len=int(lens.max()))
    assert pkv.device_error_bits() == 0

    def bits(t):
        return t.detach().contiguous().cpu().view(torch.int16).numpy().view(np.uint16)

    ref = oracle.paged_decode(bits(q), bits(k_cache), bits(v_cache), tables, lens, scale)
    check_close(out, ref, "bf16", "block manager groups")
