"""The native block manager driving the device path, end to end on the GPU.

Prompts (two of them share a system prefix, so the second finds it in the
prefix cache) are added, forked into parallel samples, then decoded for a
few steps: each step appends one token per sequence (slots from the block
manager), applies its copy-on-write pairs with copy_blocks, writes the new
K/V with reshape_and_cache and decodes.  A token's K/V is a fixed function
of (token id, position), so a cached block holds exactly what its reuser
would have written.  The oracle receives the same K/V laid out independently
(each sequence's blocks contiguous in a fresh pool), so a wrong slot, copy,
table entry or write anywhere in the chain shows up as a mismatch.
"""
import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_375_b200 as pkv
from gpu_util import check_close, host_bits

pytestmark = pytest.mark.gpu
BS = 16


def test_block_manager_drives_copy_reshape_and_decode(cuda_device):
    dev = cuda_device
    rng = np.random.default_rng(11)
    hq, hkv, d, nb, vocab, max_pos = 32, 8, 128, 800, 64, 1024
    gen = torch.Generator(device=dev).manual_seed(12)
    emb_k = torch.randn((vocab, hkv, d), generator=gen, device=dev)
    emb_v = torch.randn((vocab, hkv, d), generator=gen, device=dev)
    pos_k = torch.randn((max_pos, hkv, d), generator=gen, device=dev)
    pos_v = torch.randn((max_pos, hkv, d), generator=gen, device=dev)

    def kv(tokens, positions):
        t = torch.as_tensor(np.asarray(tokens), device=dev, dtype=torch.long)
        p = torch.as_tensor(np.asarray(positions), device=dev, dtype=torch.long)
        return ((emb_k[t] + pos_k[p]).to(torch.bfloat16).contiguous(),
                (emb_v[t] + pos_v[p]).to(torch.bfloat16).contiguous())

    k_cache = torch.full((nb, hkv, BS, d), float("nan"), dtype=torch.bfloat16, device=dev)
    v_cache = torch.full_like(k_cache, float("nan"))
    bm = pkv.BlockManager(nb, BS, seed=13, prefix_caching=True)
    system = rng.integers(0, vocab, size=70).tolist()
    prompts = [system + rng.integers(0, vocab, size=40).tolist(),
               system + rng.integers(0, vocab, size=95).tolist(),
               rng.integers(0, vocab, size=150).tolist()]
    seqs = {}
    for i, prompt in enumerate(prompts):
        cached = bm.add_sequence(i * 10, prompt)
        if i == 1:
            assert cached == 64                  # the system prefix's full blocks
        slots = torch.from_numpy(bm.slots(i * 10, cached, len(prompt))).to(dev)
        k, v = kv(prompt[cached:], range(cached, len(prompt)))
        pkv.reshape_and_cache(k, v, k_cache, v_cache, slots)
        seqs[i * 10] = list(prompt)
        for j in range(1, 4):                    # parallel samples share everything
            bm.fork(i * 10, i * 10 + j)
            seqs[i * 10 + j] = list(prompt)
    ids = sorted(seqs)
    scale = float(np.float32(1.0 / np.sqrt(d)))
    for step in range(5):
        toks = rng.integers(0, vocab, size=len(ids)).tolist()
        slots = bm.append_tokens(ids, toks)
        pairs = bm.take_copies()
        if step == 0:
            assert pairs.shape[0] > 0            # forked samples copy their shared tail
        if pairs.shape[0]:
            pkv.copy_blocks(k_cache, v_cache, torch.from_numpy(pairs))
        positions = [len(seqs[s]) for s in ids]
        for s, t in zip(ids, toks):
            seqs[s].append(t)
        k, v = kv(toks, positions)
        pkv.reshape_and_cache(k, v, k_cache, v_cache, torch.from_numpy(slots).to(dev))
        tables, lens = bm.block_tables(ids, max_blocks=32)
        q = torch.randn((len(ids), hq, d), generator=gen, device=dev).to(torch.bfloat16)
        out = torch.empty_like(q)
        pkv.paged_attention_decode(out, q, k_cache, v_cache, torch.from_numpy(tables).to(dev),
                                   torch.from_numpy(lens).to(dev), scale, hkv,
                                   max_context_len=int(lens.max()))
        assert pkv.device_error_bits() == 0
        # independent layout for the oracle: each sequence's blocks contiguous
        nblk = [(len(seqs[s]) + BS - 1) // BS for s in ids]
        ref_tables = np.full((len(ids), max(nblk)), -1, dtype=np.int32)
        parts_k, parts_v, base = [], [], 0
        for i, s in enumerate(ids):
            L = len(seqs[s])
            k, v = kv(seqs[s], range(L))
            pad = nblk[i] * BS - L
            k = torch.cat([k, torch.zeros((pad, hkv, d), dtype=k.dtype, device=dev)])
            v = torch.cat([v, torch.zeros((pad, hkv, d), dtype=v.dtype, device=dev)])
            parts_k.append(k.view(nblk[i], BS, hkv, d).transpose(1, 2))
            parts_v.append(v.view(nblk[i], BS, hkv, d).transpose(1, 2))
            ref_tables[i, :nblk[i]] = np.arange(base, base + nblk[i])
            base += nblk[i]
        ref_k = host_bits(torch.cat(parts_k).contiguous())
        ref_v = host_bits(torch.cat(parts_v).contiguous())
        ref = oracle.paged_decode(host_bits(q), ref_k, ref_v, ref_tables, lens, scale)
        check_close(out, ref, "bf16", f"step {step}")
    st = bm.stats()
    assert st["sequences"] == 12 and st["used"] > 0
