"""Helpers for the GPU parity tests: run a workload through the C ABI, run the
same workload through the oracle, and compare under the stated tolerances.

Tolerances (fixed for this path): fp32 KV, max |out - ref| <= 1e-5; bf16 KV,
|out - ref| <= 2e-2 + 1e-2 |ref| element-wise; both against the float64
oracle.  Cache maintenance (slots, reshape_and_cache, copy_blocks) is compared
bit for bit.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
import paged_kv_cache_375_b200 as pkv
import workloads

F32_ATOL = 1e-5
BF16_ATOL = 2e-2
BF16_RTOL = 1e-2


def dev_i32(a: np.ndarray, device) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).to(device)


def host_bits(t: torch.Tensor) -> np.ndarray:
    """Host copy: float32 as is, bf16 as its uint16 bit patterns, FP8 as its codes."""
    t = t.detach().contiguous().cpu()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    if t.dtype in (torch.float8_e4m3fn, torch.float8_e5m2):
        return t.view(torch.uint8).numpy()
    return t.numpy()


def to_f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to(torch.float64).cpu().numpy()


def gpu_step(b: workloads.Batch, partition_tokens: int = 0, max_context_len: int | None = None,
             apply_step: bool = True):
    """The hot path on the GPU: copy-on-write copies, slot indexing and writes of the new
    tokens, then decode.  Returns (out, k_cache, v_cache) (the caches are b's, updated)."""
    dev = b.q.device
    k_cache, v_cache = b.k_cache, b.v_cache
    bt = dev_i32(b.block_tables, dev)
    cl = dev_i32(b.context_lens, dev)
    if apply_step:
        if b.cow_pairs.shape[0]:
            pkv.copy_blocks(k_cache, v_cache, torch.from_numpy(b.cow_pairs))
        if b.new_seq.shape[0]:
            slots = pkv.slot_mapping(bt, b.num_blocks, token_seq=dev_i32(b.new_seq, dev),
                                     token_pos=dev_i32(b.new_pos, dev))
            pkv.reshape_and_cache(b.new_k, b.new_v, k_cache, v_cache, slots)
    out = torch.empty_like(b.q)
    pkv.paged_attention_decode(out, b.q, k_cache, v_cache, bt, cl, b.scale, b.num_kv_heads,
                               max_context_len=max_context_len if max_context_len is not None
                               else max(b.max_context_len, 1),
                               partition_tokens=partition_tokens)
    return out, k_cache, v_cache


def oracle_caches_after_step(b: workloads.Batch, host: dict):
    """Host caches after the oracle applies the step's copies and writes."""
    k, v = host["k_cache"].copy(), host["v_cache"].copy()
    if b.cow_pairs.shape[0]:
        oracle.copy_blocks(k, v, b.cow_pairs)
    if b.new_seq.shape[0]:
        slots = oracle.slot_mapping(b.block_tables, b.new_seq, b.new_pos)
        oracle.reshape_and_cache(host["new_k"], host["new_v"], k, v, slots)
    return k, v


def check_close(out_gpu: torch.Tensor, ref: np.ndarray, dtype: str, what: str = ""):
    got = to_f64(out_gpu).reshape(ref.shape)
    assert np.isfinite(got).all(), f"{what}: non-finite output"
    err = np.abs(got - ref)
    if dtype == "f32":
        assert err.max() <= F32_ATOL, f"{what}: max abs err {err.max():.3e} > {F32_ATOL}"
    else:
        bound = BF16_ATOL + BF16_RTOL * np.abs(ref)
        worst = (err / bound).max()
        assert worst <= 1.0, f"{what}: error {worst:.3f} of the bound (max abs {err.max():.3e})"
    return float(err.max())


def compact_all(b: workloads.Batch, k_cache: torch.Tensor, v_cache: torch.Tensor):
    """Host copies of every block some sequence references (each block once, shared
    blocks included) and the block tables renumbered onto them, so the oracle can
    recompute every output of a full-size batch without copying the whole pool back."""
    nblk = (b.context_lens.astype(np.int64) + 15) // 16
    used = np.arange(b.block_tables.shape[1])[None, :] < nblk[:, None]
    uniq, inv = np.unique(b.block_tables[used], return_inverse=True)
    bt = np.full(b.block_tables.shape, -1, dtype=np.int32)
    bt[used] = inv.astype(np.int32)
    idx = torch.from_numpy(uniq if uniq.size else np.zeros(1, np.int64)).long()
    idx = idx.to(k_cache.device)
    return host_bits(k_cache.index_select(0, idx)), host_bits(v_cache.index_select(0, idx)), bt


def sample_tasks(b: workloads.Batch, n: int, seed: int = 0) -> np.ndarray:
    """n (seq, q_head) pairs: the longest and shortest sequences plus random ones."""
    rng = np.random.default_rng(seed)
    order = np.argsort(b.context_lens)
    seqs = list({int(order[0]), int(order[-1])}) + list(rng.integers(0, b.num_seqs, n))
    heads = list(rng.integers(0, b.num_q_heads, len(seqs)))
    heads[0], heads[-1] = 0, b.num_q_heads - 1
    return np.array(list(zip(seqs, heads))[:max(n, 2)], dtype=np.int32)


def compact_for_tasks(b: workloads.Batch, k_cache: torch.Tensor, v_cache: torch.Tensor,
                      tasks: np.ndarray):
    """Host arrays holding only the blocks the sampled sequences reference, with their
    tables renumbered, so the oracle can run on a full-size pool without copying all of it."""
    seqs = sorted(set(int(s) for s in tasks[:, 0]))
    blocks = []
    remap = {}
    for s in seqs:
        L = int(b.context_lens[s])
        for i in range((L + 15) // 16):
            p = int(b.block_tables[s, i])
            if p not in remap:
                remap[p] = len(blocks)
                blocks.append(p)
    idx = torch.tensor(blocks if blocks else [0], dtype=torch.long, device=k_cache.device)
    kh = host_bits(k_cache.index_select(0, idx))
    vh = host_bits(v_cache.index_select(0, idx))
    bt = np.full_like(b.block_tables, -1)
    for s in seqs:
        L = int(b.context_lens[s])
        for i in range((L + 15) // 16):
            bt[s, i] = remap[int(b.block_tables[s, i])]
    return kh, vh, bt
