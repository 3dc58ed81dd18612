"""Pools beyond 4 GB (byte offsets past 2^32 and 2^33): the blocks a batch uses sit
at the top of a ~10 GB pool.  Slot indexing, the fused prologue, decode, split-K and
copy_blocks are checked against the oracle, which gets only the referenced blocks
(copied to the host before the step) with the tables renumbered."""
import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_375_b200 as pkv
from gpu_util import check_close, host_bits

pytestmark = pytest.mark.gpu


def _setup(dev, dtype, nb, hkv=8, d=128, seed=1300):
    rng = np.random.default_rng(seed)
    lens = np.array([100, 1000, 5000, 17], dtype=np.int32)
    nblk = (lens + 15) // 16
    top = rng.permutation(np.arange(nb - 4000, nb))
    tables = np.full((len(lens), int(nblk.max())), -1, dtype=np.int32)
    used, at = [], 0
    for s, n in enumerate(nblk):
        tables[s, :n] = top[at:at + n]
        used.extend(top[at:at + n].tolist())
        at += n
    spare = top[at:at + 64]                        # unused blocks, for copy destinations
    tdt = torch.float8_e4m3fn if dtype == "fp8" else torch.bfloat16
    kc = torch.empty((nb, hkv, 16, d), dtype=tdt, device=dev)
    vc = torch.empty_like(kc)
    gen = torch.Generator(device=dev).manual_seed(seed)
    idx = torch.tensor(used + spare.tolist(), dtype=torch.long, device=dev)
    shape = (idx.numel(), hkv, 16, d)
    if dtype == "fp8":
        codes = torch.randint(0, 0x7f, shape, generator=gen, device=dev, dtype=torch.uint8)
        sign = torch.randint(0, 2, shape, generator=gen, device=dev, dtype=torch.uint8) << 7
        kc.view(torch.uint8)[idx] = codes | sign
        vc.view(torch.uint8)[idx] = torch.randint(0, 0x7f, shape, generator=gen, device=dev,
                                                  dtype=torch.uint8)
    else:
        kc[idx] = torch.randn(shape, generator=gen, device=dev).to(tdt)
        vc[idx] = torch.randn(shape, generator=gen, device=dev).to(tdt)
    return lens, tables, used, spare, kc, vc


def _host_blocks(kc, vc, blocks):
    idx = torch.tensor(blocks, dtype=torch.long, device=kc.device)
    return host_bits(kc.index_select(0, idx)), host_bits(vc.index_select(0, idx))


def _u8(t):
    return t.detach().contiguous().cpu().view(torch.uint8).numpy()


@pytest.mark.parametrize("dtype,nb,partition", [("bf16", 300_000, 0), ("bf16", 300_000, 512),
                                                ("fp8", 600_000, 0)])
def test_decode_step_on_a_pool_past_4gb(cuda_device, dtype, nb, partition):
    dev = cuda_device
    hq, hkv, d = 32, 8, 128
    lens, tables, used, _, kc, vc = _setup(dev, dtype, nb, hkv, d)
    B = len(lens)
    assert kc.numel() * kc.element_size() > 2 ** 33
    remap = {b: i for i, b in enumerate(used)}
    rt = np.vectorize(lambda x: remap.get(int(x), -1))(tables).astype(np.int32)
    kh, vh = _host_blocks(kc, vc, used)
    gen = torch.Generator(device=dev).manual_seed(7)
    q = torch.randn((B, hq, d), generator=gen, device=dev).to(torch.bfloat16)
    new_k = torch.randn((B, hkv, d), generator=gen, device=dev).to(torch.bfloat16)
    new_v = torch.randn((B, hkv, d), generator=gen, device=dev).to(torch.bfloat16)
    bt = torch.from_numpy(tables).to(dev)
    cl = torch.from_numpy(lens).to(dev)
    scale = float(np.float32(1 / np.sqrt(d)))
    ks, vs = 1.0 / 64.0, 3.0 / 128.0
    slots = torch.zeros(B, dtype=torch.int64, device=dev)
    plan = pkv.DecodePlan(bt, cl, hq, kc, max_context_len=int(lens.max()),
                          partition_tokens=partition, new_k=new_k, new_v=new_v, v_cache=vc,
                          k_scale=ks, v_scale=vs, slot_mapping_out=slots)
    out = torch.empty_like(q)
    if dtype == "fp8":
        plan.run_fp8(out, q, kc, vc, scale, ks, vs)
    else:
        plan.run(out, q, kc, vc, scale)
    assert pkv.device_error_bits() == 0
    # slots: physical (past 2^32 bytes), as the oracle indexes them
    want = oracle.slot_mapping(tables, np.arange(B), lens - 1)
    assert np.array_equal(slots.cpu().numpy(), want)
    assert (want * hkv * d * kc.element_size() > 2 ** 32).all()   # byte offsets of the blocks
    # the oracle on the renumbered blocks
    rslots = oracle.slot_mapping(rt, np.arange(B), lens - 1)
    nk, nv = host_bits(new_k), host_bits(new_v)
    if dtype == "fp8":
        oracle.reshape_and_cache_fp8(nk, nv, kh, vh, rslots, ks, vs)
        ref = oracle.paged_decode_fp8(host_bits(q), kh, vh, ks, vs, rt, lens, scale)
    else:
        oracle.reshape_and_cache(nk, nv, kh, vh, rslots)
        ref = oracle.paged_decode(host_bits(q), kh, vh, rt, lens, scale)
    gk, gv = _host_blocks(kc, vc, used)
    np.testing.assert_array_equal(gk, kh)
    np.testing.assert_array_equal(gv, vh)
    check_close(out, ref, "bf16", f"{dtype} pool past 4 GB p{partition}")


def test_copy_blocks_past_4gb(cuda_device):
    dev = cuda_device
    lens, tables, used, spare, kc, vc = _setup(dev, "bf16", 300_000)
    pairs = np.stack([np.array(used[:32]), spare[:32]], axis=1).astype(np.int64)
    before_k, before_v = _host_blocks(kc, vc, used[:32])
    pkv.copy_blocks(kc, vc, torch.from_numpy(pairs))
    assert pkv.device_error_bits() == 0
    after_k, after_v = _host_blocks(kc, vc, spare[:32].tolist())
    np.testing.assert_array_equal(after_k, before_k)
    np.testing.assert_array_equal(after_v, before_v)
