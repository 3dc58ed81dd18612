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
