"""Seeded random configurations through the whole path against the oracle: dtype
(fp32, bf16, FP8 e4m3 and e5m2), head_dim, kv heads and group size, ragged and empty lengths,
one or several query tokens, partition size.  Each case draws its own shapes."""
import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_375_b200 as pkv
import workloads
from gpu_util import check_close, dev_i32, oracle_caches_after_step

pytestmark = pytest.mark.gpu


def _case(seed):
    rng = np.random.default_rng(10_000 + seed)
    dtype = ["f32", "bf16", "fp8", "fp8e5m2"][seed % 4]
    d = 128 if workloads.fp8_format(dtype) else int(rng.choice([64, 128]))
    hkv = int(rng.choice([1, 2, 4, 8]))
    g = int(rng.choice([1, 2, 3, 4, 6, 8, 16]))
    n = int(rng.integers(1, 12))
    lens = np.minimum(np.rint(np.exp(rng.normal(np.log(200), 1.2, size=n))), 3000).astype(int)
    lens[rng.random(n) < 0.1] = 0
    multi = bool(rng.random() < 0.5)
    chunks = np.minimum(rng.integers(1, 25, size=n), lens) if multi else None
    partition = int(rng.choice([0, 16, 48, 256, 1024]))
    return dtype, d, hkv, g, lens, chunks, partition


@pytest.mark.parametrize("seed", range(64))
def test_random_configuration(cuda_device, seed):
    dtype, d, hkv, g, lens, chunks, partition = _case(seed)
    what = f"seed {seed}: {dtype} d{d} {g * hkv}/{hkv} lens {lens.tolist()} chunks " \
           f"{None if chunks is None else chunks.tolist()} p{partition}"
    dev = cuda_device
    if chunks is None:
        b = workloads.random_batch(20_000 + seed, lens, g * hkv, hkv, d, dtype, device=dev,
                                   new_token=True, extra_table=1)
    else:
        b = workloads.chunked_batch(20_000 + seed, lens, chunks, g * hkv, hkv, d, dtype,
                                    device=dev, extra_table=1)
    host = b.host()
    bt, cl = dev_i32(b.block_tables, dev), dev_i32(b.context_lens, dev)
    fmt = workloads.fp8_format(dtype)
    if b.new_seq.shape[0]:
        slots = pkv.slot_mapping(bt, b.num_blocks, token_seq=dev_i32(b.new_seq, dev),
                                 token_pos=dev_i32(b.new_pos, dev))
        if fmt:
            pkv.reshape_and_cache_fp8(b.new_k, b.new_v, b.k_cache, b.v_cache, slots, b.k_scale,
                                      b.v_scale)
        else:
            pkv.reshape_and_cache(b.new_k, b.new_v, b.k_cache, b.v_cache, slots)
    out = torch.empty_like(b.q)
    mcl = max(b.max_context_len, 1)
    if chunks is None:
        if fmt:
            pkv.paged_attention_decode_fp8(out, b.q, b.k_cache, b.v_cache, bt, cl, b.scale,
                                           b.k_scale, b.v_scale, max_context_len=mcl,
                                           partition_tokens=partition)
        else:
            pkv.paged_attention_decode(out, b.q, b.k_cache, b.v_cache, bt, cl, b.scale, hkv,
                                       max_context_len=mcl, partition_tokens=partition)
    else:
        qsl = dev_i32(b.query_start_loc, dev)
        if fmt:
            pkv.paged_attention_multi_fp8(out, b.q, b.k_cache, b.v_cache, bt, cl, qsl, b.scale,
                                          b.k_scale, b.v_scale, b.max_query_len,
                                          max_context_len=mcl, partition_tokens=partition)
        else:
            pkv.paged_attention_multi(out, b.q, b.k_cache, b.v_cache, bt, cl, qsl, b.scale, hkv,
                                      b.max_query_len, max_context_len=mcl,
                                      partition_tokens=partition)
    assert pkv.device_error_bits() == 0, what
    # the oracle: caches after the step's writes, then attention
    k, v = host["k_cache"].copy(), host["v_cache"].copy()
    if b.new_seq.shape[0]:
        sl = oracle.slot_mapping(b.block_tables, b.new_seq, b.new_pos)
        if fmt:
            oracle.reshape_and_cache_fp8(host["new_k"], host["new_v"], k, v, sl, b.k_scale,
                                         b.v_scale, fmt=fmt)
        else:
            oracle.reshape_and_cache(host["new_k"], host["new_v"], k, v, sl)
    if chunks is None:
        ref = (oracle.paged_decode_fp8(host["q"], k, v, b.k_scale, b.v_scale, b.block_tables,
                                       b.context_lens, b.scale, fmt=fmt) if fmt else
               oracle.paged_decode(host["q"], k, v, b.block_tables, b.context_lens, b.scale))
    else:
        ref = (oracle.paged_multi_fp8(host["q"], k, v, b.k_scale, b.v_scale, b.block_tables,
                                      b.context_lens, b.query_start_loc, b.scale, fmt=fmt)
               if fmt else
               oracle.paged_multi(host["q"], k, v, b.block_tables, b.context_lens,
                                  b.query_start_loc, b.scale))
    check_close(out, ref, "bf16" if fmt else dtype, what)


@pytest.mark.parametrize("seed", range(32))
def test_random_shared_prefix_configuration(cuda_device, seed):
    """The shared-prefix decode on random groups: sizes, prefix blocks (sometimes past a
    member's full blocks, then lowered and flagged), tails, tables that share or not, all
    pool dtypes, partitions; the oracle reads the tables as the call defines them."""
    from test_gpu_shared_prefix import substituted_tables
    rng = np.random.default_rng(30_000 + seed)
    dtype = ["f32", "bf16", "fp8", "fp8e5m2"][seed % 4]
    d = 128 if workloads.fp8_format(dtype) else int(rng.choice([64, 128]))
    hkv = int(rng.choice([1, 2, 4, 8]))
    g = int(rng.choice([1, 2, 3, 4, 8, 16]))
    sizes = rng.integers(1, 13, size=int(rng.integers(1, 6)))
    pref = rng.integers(0, 21, size=sizes.shape[0])
    lens = []
    for n, p in zip(sizes, pref):
        lens += (16 * p + rng.integers(0, 300, size=n)).tolist()
    claimed = pref + (rng.random(pref.shape[0]) < 0.2) * rng.integers(1, 4, size=pref.shape[0])
    partition = int(rng.choice([0, 16, 48, 256]))
    share = bool(rng.random() < 0.7)
    b = workloads.random_batch(40_000 + seed, lens, g * hkv, hkv, d, dtype, device="cpu",
                               extra_table=1)
    gs = np.concatenate([[0], np.cumsum(sizes)]).astype(np.int32)
    sb = claimed.astype(np.int32)
    if share:
        b.block_tables = substituted_tables(b.block_tables, gs, sb, b.context_lens)
    b = b.to(cuda_device)
    host = b.host()
    dev = cuda_device
    out = torch.empty_like(b.q)
    fmt = workloads.fp8_format(dtype)
    kw = dict(k_scale=b.k_scale, v_scale=b.v_scale) if fmt else {}
    pkv.paged_attention_decode_shared(out, b.q, b.k_cache, b.v_cache, dev_i32(b.block_tables, dev),
                                      dev_i32(b.context_lens, dev), dev_i32(gs, dev),
                                      dev_i32(sb, dev), b.scale,
                                      max_context_len=max(b.max_context_len, 1),
                                      partition_tokens=partition, **kw)
    bits = pkv.device_error_bits()
    lowered = any(sizes[i] >= 2 and min(lens[gs[i]:gs[i + 1]]) // 16 < sb[i]
                  for i in range(len(sizes)))
    what = f"seed {seed}: {dtype} d{d} {g * hkv}/{hkv} sizes {sizes.tolist()} P {sb.tolist()}"
    assert bits == (pkv.DEVERR_GROUP if lowered else 0), what
    tables = substituted_tables(b.block_tables, gs, sb, b.context_lens)
    if fmt:
        ref = oracle.paged_decode_fp8(host["q"], host["k_cache"], host["v_cache"], b.k_scale,
                                      b.v_scale, tables, b.context_lens, b.scale, fmt=fmt)
    else:
        ref = oracle.paged_decode(host["q"], host["k_cache"], host["v_cache"], tables,
                                  b.context_lens, b.scale)
    check_close(out, ref, "f32" if dtype == "f32" else "bf16", what)
