"""GPU parity of the cache-maintenance kernels (through the C ABI) against the
oracle, bit for bit: slot indexing, reshape_and_cache and copy_blocks.  Every
byte of the pools is compared, so a write to a wrong place or a stray write
anywhere fails."""
import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_375_b200 as pkv
import workloads
from gpu_util import dev_i32, host_bits

pytestmark = pytest.mark.gpu


def _tables(rng, lens, nb, width):
    perm = rng.permutation(nb)
    bt = np.full((len(lens), width), -1, dtype=np.int32)
    used = 0
    for s, L in enumerate(lens):
        n = (L + 15) // 16
        bt[s, :n] = perm[used:used + n]
        used += n
    return bt


def test_slot_mapping_matches_oracle(cuda_device):
    rng = np.random.default_rng(1)
    lens = rng.integers(1, 700, size=97)
    nb = 4000
    bt = _tables(rng, lens, nb, 50)
    seq = rng.integers(0, 97, size=3000).astype(np.int32)
    pos = np.array([rng.integers(0, lens[s]) for s in seq], dtype=np.int32)
    got = pkv.slot_mapping(dev_i32(bt, cuda_device), nb, token_seq=dev_i32(seq, cuda_device),
                           token_pos=dev_i32(pos, cuda_device)).cpu().numpy()
    assert np.array_equal(got, oracle.slot_mapping(bt, seq, pos))
    # decode mode: one token per sequence at position context_len - 1
    got = pkv.slot_mapping(dev_i32(bt, cuda_device), nb,
                           context_lens=dev_i32(lens, cuda_device)).cpu().numpy()
    ref = oracle.slot_mapping(bt, np.arange(97, dtype=np.int32), (lens - 1).astype(np.int32))
    assert np.array_equal(got, ref)
    assert pkv.device_error_bits() == 0


def test_slot_mapping_flags_bad_positions_and_entries(cuda_device):
    bt = np.array([[3, -1], [5, 99]], dtype=np.int32)
    seq = np.array([0, 0, 1, 1], dtype=np.int32)
    pos = np.array([2, 40, 20, 17], dtype=np.int32)     # 40 is past the table; entry 99 >= nb
    got = pkv.slot_mapping(dev_i32(bt, cuda_device), 10, token_seq=dev_i32(seq, cuda_device),
                           token_pos=dev_i32(pos, cuda_device)).cpu().numpy()
    assert got.tolist() == [3 * 16 + 2, -1, -1, -1]
    bits = pkv.device_error_bits()
    assert bits & pkv.DEVERR_POS and bits & pkv.DEVERR_BLOCK


@pytest.mark.parametrize("dtype,hkv,d", [("bf16", 8, 128), ("f32", 8, 64), ("bf16", 40, 128),
                                         ("bf16", 1, 64)])
def test_reshape_and_cache_bit_exact(cuda_device, dtype, hkv, d):
    rng = np.random.default_rng(2)
    nb, T = 300, 777
    shape = (nb, hkv, 16, d)
    tdt = workloads.torch_dtype(dtype)
    gen = torch.Generator(device=cuda_device).manual_seed(3)
    kc = torch.randn(shape, generator=gen, device=cuda_device).to(tdt)
    vc = torch.randn(shape, generator=gen, device=cuda_device).to(tdt)
    k = torch.randn((T, hkv, d), generator=gen, device=cuda_device).to(tdt)
    v = torch.randn((T, hkv, d), generator=gen, device=cuda_device).to(tdt)
    slots = rng.choice(nb * 16, size=T, replace=False).astype(np.int64)
    slots[::13] = -1                                   # padding tokens
    kh, vh = host_bits(kc), host_bits(vc)
    pkv.reshape_and_cache(k, v, kc, vc, torch.from_numpy(slots).to(cuda_device))
    assert pkv.device_error_bits() == 0
    oracle.reshape_and_cache(host_bits(k), host_bits(v), kh, vh, slots)
    assert np.array_equal(host_bits(kc), kh)
    assert np.array_equal(host_bits(vc), vh)


def test_reshape_and_cache_flags_slot_beyond_pool(cuda_device):
    kc = torch.zeros((4, 2, 16, 64), dtype=torch.bfloat16, device=cuda_device)
    vc = torch.zeros_like(kc)
    k = torch.ones((2, 2, 64), dtype=torch.bfloat16, device=cuda_device)
    pkv.reshape_and_cache(k, k, kc, vc, torch.tensor([5, 64], dtype=torch.int64, device=cuda_device))
    assert pkv.device_error_bits() & pkv.DEVERR_SLOT
    assert kc.float().sum().item() == 2 * 64          # only slot 5 written
    assert torch.all(kc[0, :, 5] == 1)


@pytest.mark.parametrize("dtype,hkv,d", [("bf16", 8, 128), ("f32", 8, 64), ("bf16", 40, 128)])
def test_copy_blocks_bit_exact(cuda_device, dtype, hkv, d):
    rng = np.random.default_rng(4)
    nb = 500
    tdt = workloads.torch_dtype(dtype)
    gen = torch.Generator(device=cuda_device).manual_seed(5)
    kc = torch.randn((nb, hkv, 16, d), generator=gen, device=cuda_device).to(tdt)
    vc = torch.randn((nb, hkv, 16, d), generator=gen, device=cuda_device).to(tdt)
    perm = rng.permutation(nb)
    pairs = np.stack([perm[:120], perm[120:240]], axis=1).astype(np.int64)
    kh, vh = host_bits(kc), host_bits(vc)
    pkv.copy_blocks(kc, vc, torch.from_numpy(pairs))
    assert pkv.device_error_bits() == 0
    oracle.copy_blocks(kh, vh, pairs)
    assert np.array_equal(host_bits(kc), kh)
    assert np.array_equal(host_bits(vc), vh)


def test_copy_blocks_rejects_and_flags_bad_pairs(cuda_device):
    kc = torch.zeros((8, 1, 16, 64), dtype=torch.bfloat16, device=cuda_device)
    vc = torch.zeros_like(kc)
    with pytest.raises(pkv.PkvError):
        pkv.copy_blocks(kc, vc, torch.tensor([[0, 1], [1, 2]]))       # dst 1 is also a src
    # on the device an out-of-range pair is skipped and flagged
    pkv.copy_blocks(kc, vc, torch.tensor([[0, 9]]), validate=False)
    assert pkv.device_error_bits() & pkv.DEVERR_PAIR


def test_c3_new_token_round_trip(cuda_device):
    """After the decode step's writes, the slot of position L-1 of every sequence holds
    exactly that sequence's new K/V (read back through the block table)."""
    b = workloads.c3_llama3_8b_gqa(device=cuda_device)
    bt = dev_i32(b.block_tables, cuda_device)
    slots = pkv.slot_mapping(bt, b.num_blocks, context_lens=dev_i32(b.context_lens, cuda_device))
    pkv.reshape_and_cache(b.new_k, b.new_v, b.k_cache, b.v_cache, slots)
    assert pkv.device_error_bits() == 0
    pos = b.context_lens - 1
    blk = torch.from_numpy(b.block_tables[np.arange(b.num_seqs), pos // 16].astype(np.int64)).to(cuda_device)
    off = torch.from_numpy((pos % 16).astype(np.int64)).to(cuda_device)
    k_read = b.k_cache[blk, :, off, :]
    v_read = b.v_cache[blk, :, off, :]
    assert torch.equal(k_read.view(torch.int16), b.new_k.view(torch.int16))
    assert torch.equal(v_read.view(torch.int16), b.new_v.view(torch.int16))
