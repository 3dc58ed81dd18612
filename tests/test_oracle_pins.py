"""Pins of the float64 oracle against what the pages and the mathematics fix.

No test here compares the oracle with itself: each checks it against an
independent statement -- a hand-derived fixture, numpy dense attention over
contiguous K/V, a closed form, or a paging invariant (the block table changes
where K/V live, never what attention computes: ipipp.com vLLM article, section
"二、PagedAttention分页原理深度剖析"; shared prefix blocks with copy-on-write:
"vLLM 深读", section "先看浪费在哪里").
"""
import glob
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
import workloads

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
BS = 16


# ---------------------------------------------------------------- helpers ----
def to_bf16_bits(x: np.ndarray) -> np.ndarray:
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def bf16_bits_to_f64(b: np.ndarray) -> np.ndarray:
    return (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def place_blocks(K: np.ndarray, table, num_blocks: int, fill=np.nan) -> np.ndarray:
    """Put contiguous rows K[L][Hkv][D] into a pool [NB][Hkv][16][D] block by block:
    logical block i (rows 16i..16i+15) becomes physical block table[i]."""
    L, hkv, d = K.shape
    nblk = (L + BS - 1) // BS
    padded = np.full((nblk * BS, hkv, d), fill, dtype=K.dtype)
    padded[:L] = K
    blocks = padded.reshape(nblk, BS, hkv, d).transpose(0, 2, 1, 3)
    pool = np.full((num_blocks, hkv, BS, d), fill, dtype=K.dtype)
    for i in range(nblk):
        pool[table[i]] = blocks[i]
    return pool


def dense_attention(q: np.ndarray, K: np.ndarray, V: np.ndarray, scale: float) -> np.ndarray:
    """numpy float64 softmax(scale q K^T) V for one sequence.
    q [Hq][D]; K, V [L][Hkv][D]; query head h reads kv head h // (Hq/Hkv)."""
    hq = q.shape[0]
    hkv = K.shape[1]
    g = hq // hkv
    out = np.zeros(q.shape, dtype=np.float64)
    for h in range(hq):
        Kh = K[:, h // g, :].astype(np.float64)
        Vh = V[:, h // g, :].astype(np.float64)
        z = float(np.float32(scale)) * (Kh @ q[h].astype(np.float64))
        w = np.exp(z - z.max())
        out[h] = (w[:, None] * Vh).sum(0) / w.sum()
    return out


def random_paged(rng, lens, hq, hkv, d, num_blocks=None, dtype="f32"):
    """Contiguous per-sequence K/V plus the same data paged into a scattered pool."""
    nblk = [(L + BS - 1) // BS for L in lens]
    nb = num_blocks or sum(nblk) + 5
    perm = rng.permutation(nb)
    tables, used = [], 0
    for n in nblk:
        tables.append(perm[used:used + n].tolist())
        used += n
    mb = max(nblk + [1])
    bt = np.full((len(lens), mb), -1, dtype=np.int32)
    for s, t in enumerate(tables):
        bt[s, :len(t)] = t
    Ks = [rng.standard_normal((L, hkv, d)).astype(np.float32) for L in lens]
    Vs = [rng.standard_normal((L, hkv, d)).astype(np.float32) for L in lens]
    q = rng.standard_normal((len(lens), hq, d)).astype(np.float32)
    kpool = np.full((nb, hkv, BS, d), np.nan, dtype=np.float32)
    vpool = np.full((nb, hkv, BS, d), np.nan, dtype=np.float32)
    for s in range(len(lens)):
        kp = place_blocks(Ks[s], tables[s], nb)
        vp = place_blocks(Vs[s], tables[s], nb)
        for b in tables[s]:
            kpool[b] = kp[b]
            vpool[b] = vp[b]
    if dtype == "bf16":
        Ks = [bf16_bits_to_f64(to_bf16_bits(K)) for K in Ks]
        Vs = [bf16_bits_to_f64(to_bf16_bits(V)) for V in Vs]
        return (to_bf16_bits(q), to_bf16_bits(kpool), to_bf16_bits(vpool), bt,
                np.array(lens, dtype=np.int32), Ks, Vs, bf16_bits_to_f64(to_bf16_bits(q)))
    return q, kpool, vpool, bt, np.array(lens, dtype=np.int32), Ks, Vs, q


# --------------------------------------------------------- golden fixtures ----
def _golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def test_golden_fixture_files_have_citations():
    files = sorted(glob.glob(os.path.join(GOLDEN, "*.json")))
    assert len(files) >= 7
    for f in files:
        data = json.load(open(f))
        assert data.get("citation") and data.get("derivation"), f


def test_golden_slot_mapping():
    g = _golden("slot_mapping_example.json")
    pos = np.array(g["positions"], dtype=np.int32)
    seq = np.zeros_like(pos)
    slots = oracle.slot_mapping(np.array(g["block_tables"], dtype=np.int32), seq, pos,
                                g["block_size"])
    assert slots.tolist() == g["expected_slots"]


@pytest.mark.parametrize("name", ["attention_two_tokens.json", "attention_uniform_keys.json",
                                  "attention_gqa_two_heads.json",
                                  "paged_gather_twenty_tokens.json"])
def test_golden_attention(name):
    g = _golden(name)
    L, d = g["context_len"], g["head_dim"]
    hq, hkv = g["num_q_heads"], g["num_kv_heads"]
    if g["k_tokens"] == "j":
        K = np.arange(L, dtype=np.float32).reshape(L, 1, 1)
        V = (np.arange(L, dtype=np.float32) + 1).reshape(L, 1, 1)
    else:
        K = np.array(g["k_tokens"], dtype=np.float32)
        V = np.array(g["v_tokens"], dtype=np.float32)
    kpool = place_blocks(K, g["block_table"], g["num_blocks"])
    vpool = place_blocks(V, g["block_table"], g["num_blocks"])
    q = np.array(g["q"], dtype=np.float32).reshape(1, hq, d)
    out = oracle.paged_decode(q, kpool, vpool, np.array([g["block_table"]], dtype=np.int32),
                              np.array([L], dtype=np.int32), g["scale"])
    np.testing.assert_allclose(out[0], np.array(g["expected"]), rtol=0, atol=g["atol"])


def test_golden_lse_merge():
    g = _golden("lse_merge_two_parts.json")
    out = oracle.lse_merge(np.array(g["m"]), np.array(g["l"]), np.array(g["o"]))
    np.testing.assert_allclose(out, g["expected"], rtol=0, atol=g["atol"])


def test_golden_copy_blocks():
    g = _golden("copy_blocks_example.json")
    nb = g["num_blocks"]
    base = (100.0 * np.arange(nb)).reshape(nb, 1, 1, 1)
    k = (base + np.arange(BS).reshape(1, 1, BS, 1)).astype(np.float32)
    v = -k
    oracle.copy_blocks(k, v, np.array(g["pairs"]))
    for b, b0 in enumerate(g["expected_block_base"]):
        assert np.array_equal(k[b, 0, :, 0], b0 + np.arange(BS, dtype=np.float32))
        assert np.array_equal(v[b, 0, :, 0], -(b0 + np.arange(BS, dtype=np.float32)))


# ------------------------------------------------------- dense reduction ----
@pytest.mark.parametrize("d", [4, 8, 64])
@pytest.mark.parametrize("hq,hkv", [(1, 1), (4, 1), (8, 2), (6, 3)])
def test_dense_reduction_fp32(d, hq, hkv):
    rng = np.random.default_rng(1000 * d + 10 * hq + hkv)
    lens = [1, 15, 16, 17, 33, 64]
    q, kp, vp, bt, cl, Ks, Vs, qf = random_paged(rng, lens, hq, hkv, d)
    scale = 1.0 / math.sqrt(d)
    out = oracle.paged_decode(q, kp, vp, bt, cl, scale)
    for s in range(len(lens)):
        ref = dense_attention(qf[s], Ks[s], Vs[s], scale)
        np.testing.assert_allclose(out[s], ref, rtol=0, atol=1e-12)


def test_dense_reduction_bf16():
    rng = np.random.default_rng(7)
    lens = [3, 16, 40, 64]
    q, kp, vp, bt, cl, Ks, Vs, qf = random_paged(rng, lens, 8, 2, 64, dtype="bf16")
    out = oracle.paged_decode(q, kp, vp, bt, cl, 0.125)
    for s in range(len(lens)):
        ref = dense_attention(qf[s], Ks[s], Vs[s], 0.125)
        np.testing.assert_allclose(out[s], ref, rtol=0, atol=1e-12)


def test_dense_reduction_c1_config():
    """The tiny fp32 configuration against numpy dense attention over the contiguous K/V
    read back block by block from the generator's pool."""
    b = workloads.c1_tiny_fp32()
    h = b.host()
    out = oracle.paged_decode(h["q"], h["k_cache"], h["v_cache"], b.block_tables,
                              b.context_lens, b.scale)
    for s in range(b.num_seqs):
        L = int(b.context_lens[s])
        nblk = (L + BS - 1) // BS
        blocks = h["k_cache"][b.block_tables[s, :nblk]]          # [nblk][Hkv][16][D]
        K = blocks.transpose(0, 2, 1, 3).reshape(nblk * BS, b.num_kv_heads, b.head_dim)[:L]
        blocks = h["v_cache"][b.block_tables[s, :nblk]]
        V = blocks.transpose(0, 2, 1, 3).reshape(nblk * BS, b.num_kv_heads, b.head_dim)[:L]
        assert np.isfinite(K).all() and np.isfinite(V).all()
        ref = dense_attention(h["q"][s], K, V, b.scale)
        np.testing.assert_allclose(out[s], ref, rtol=0, atol=1e-12)


# ------------------------------------------------------------ closed forms ----
def test_single_token_returns_its_value_exactly():
    rng = np.random.default_rng(3)
    q, kp, vp, bt, cl, Ks, Vs, _ = random_paged(rng, [1, 1], 4, 2, 64)
    out = oracle.paged_decode(q, kp, vp, bt, cl, 0.125)
    for s in range(2):
        for h in range(4):
            assert np.array_equal(out[s, h], Vs[s][0, h // 2].astype(np.float64))


def test_zero_scale_gives_mean_of_values():
    rng = np.random.default_rng(4)
    lens = [5, 31, 48]
    q, kp, vp, bt, cl, Ks, Vs, _ = random_paged(rng, lens, 2, 2, 8)
    out = oracle.paged_decode(q, kp, vp, bt, cl, 0.0)
    for s, L in enumerate(lens):
        np.testing.assert_allclose(out[s], Vs[s].astype(np.float64).mean(0), rtol=0, atol=1e-12)


def test_equal_keys_give_mean_of_values():
    rng = np.random.default_rng(5)
    L, d = 37, 8
    K = np.repeat(rng.standard_normal((1, 1, d)).astype(np.float32), L, axis=0)
    V = rng.standard_normal((L, 1, d)).astype(np.float32)
    table = [4, 0, 2]
    q = rng.standard_normal((1, 1, d)).astype(np.float32)
    out = oracle.paged_decode(q, place_blocks(K, table, 5), place_blocks(V, table, 5),
                              np.array([table], dtype=np.int32), np.array([L], dtype=np.int32),
                              0.7)
    np.testing.assert_allclose(out[0, 0], V[:, 0].astype(np.float64).mean(0), rtol=0, atol=1e-12)


def test_dominant_key_selects_its_value():
    rng = np.random.default_rng(6)
    L, d, j_star = 45, 16, 29
    K = rng.standard_normal((L, 1, d)).astype(np.float32)
    q = rng.standard_normal((1, 1, d)).astype(np.float32)
    K[j_star, 0] = 64.0 * q[0, 0]            # its score exceeds all others by far more than 60
    V = rng.standard_normal((L, 1, d)).astype(np.float32)
    table = [2, 0, 1]
    scale = 1.0
    z = (K[:, 0].astype(np.float64) @ q[0, 0].astype(np.float64)) * scale
    assert z[j_star] - np.delete(z, j_star).max() > 60
    out = oracle.paged_decode(q, place_blocks(K, table, 3), place_blocks(V, table, 3),
                              np.array([table], dtype=np.int32), np.array([L], dtype=np.int32),
                              scale)
    np.testing.assert_allclose(out[0, 0], V[j_star, 0].astype(np.float64), rtol=0, atol=1e-12)


def test_empty_context_gives_zero():
    rng = np.random.default_rng(8)
    q, kp, vp, bt, cl, _, _, _ = random_paged(rng, [0, 20], 2, 1, 8)
    out = oracle.paged_decode(q, kp, vp, bt, cl, 0.3)
    assert np.array_equal(out[0], np.zeros((2, 8)))
    assert np.isfinite(out[1]).all()


# --------------------------------------------------------------- GQA ----
def test_gqa_equals_mha_with_repeated_kv_heads():
    rng = np.random.default_rng(9)
    lens = [7, 40, 65]
    q, kp, vp, bt, cl, _, _, _ = random_paged(rng, lens, 8, 2, 16)
    gqa = oracle.paged_decode(q, kp, vp, bt, cl, 0.25)
    kp_mha = np.repeat(kp, 4, axis=1)     # kv head k serves query heads 4k..4k+3
    vp_mha = np.repeat(vp, 4, axis=1)
    mha = oracle.paged_decode(q, np.ascontiguousarray(kp_mha), np.ascontiguousarray(vp_mha),
                              bt, cl, 0.25)
    assert np.array_equal(gqa, mha)


def test_gqa_head_mapping_is_not_interleaved():
    """Query heads 0..g-1 read kv head 0 (a reading; an interleaved h % Hkv mapping would fail)."""
    rng = np.random.default_rng(10)
    q, kp, vp, bt, cl, Ks, Vs, qf = random_paged(rng, [1], 4, 2, 8)
    out = oracle.paged_decode(q, kp, vp, bt, cl, 1.0)
    assert np.array_equal(out[0, 1], Vs[0][0, 0].astype(np.float64))
    assert np.array_equal(out[0, 2], Vs[0][0, 1].astype(np.float64))


# ------------------------------------------------------- paging invariants ----
def test_block_placement_permutation_is_bitwise_invariant():
    b = workloads.random_batch(11, [3, 16, 17, 100, 250], 8, 2, 32, "bf16", device="cpu")
    p = workloads.permute_placement(b, seed=12)
    assert not np.array_equal(b.block_tables, p.block_tables)
    hb, hp = b.host(), p.host()
    ob = oracle.paged_decode(hb["q"], hb["k_cache"], hb["v_cache"], b.block_tables,
                             b.context_lens, b.scale)
    op = oracle.paged_decode(hp["q"], hp["k_cache"], hp["v_cache"], p.block_tables,
                             p.context_lens, p.scale)
    assert np.array_equal(ob, op)


def _apply_step_oracle(b: workloads.Batch):
    """Copy-on-write copies, then the new tokens' writes, on host copies of the pool."""
    h = b.host()
    k, v = h["k_cache"].copy(), h["v_cache"].copy()
    oracle.copy_blocks(k, v, b.cow_pairs)
    slots = oracle.slot_mapping(b.block_tables, b.new_seq, b.new_pos)
    oracle.reshape_and_cache(h["new_k"], h["new_v"], k, v, slots)
    return h, k, v


def test_shared_prefix_equals_private_copies():
    b = workloads.c4_shared_prefix(prompts=3, samples=4, prefix=64, max_tail=40, num_blocks=200)
    assert b.cow_pairs.shape[0] > 0
    h, k, v = _apply_step_oracle(b)
    shared = oracle.paged_decode(h["q"], k, v, b.block_tables, b.context_lens, b.scale)
    assert np.isfinite(shared).all()
    after = workloads.Batch(b.name, b.seed, b.dtype, b.num_q_heads, b.num_kv_heads, b.head_dim,
                            b.num_blocks, b.context_lens, b.block_tables, b.scale, b.q,
                            torch.from_numpy(k.view(np.int16)).view(torch.bfloat16),
                            torch.from_numpy(v.view(np.int16)).view(torch.bfloat16),
                            b.new_k, b.new_v, b.new_seq, b.new_pos, b.cow_pairs)
    priv = workloads.private_copy(after)
    assert priv.num_blocks > b.num_blocks          # some blocks really were shared
    hp = priv.host()
    private = oracle.paged_decode(hp["q"], hp["k_cache"], hp["v_cache"], priv.block_tables,
                                  priv.context_lens, priv.scale)
    assert np.array_equal(shared, private)


def test_padding_is_never_read():
    """NaN in every slot past the context, in unreferenced blocks and -1 table padding:
    the result is finite and equal to the run with finite values there."""
    b = workloads.random_batch(13, [1, 15, 17, 47, 64], 4, 2, 16, "f32", device="cpu",
                               extra_table=3)
    h = b.host()
    assert np.isnan(h["k_cache"]).any()
    poisoned = oracle.paged_decode(h["q"], h["k_cache"], h["v_cache"], b.block_tables,
                                   b.context_lens, b.scale)
    assert np.isfinite(poisoned).all()
    k = np.where(np.isnan(h["k_cache"]), np.float32(3.0), h["k_cache"])
    v = np.where(np.isnan(h["v_cache"]), np.float32(-7.0), h["v_cache"])
    bt = np.where(b.block_tables < 0, 0, b.block_tables).astype(np.int32)
    clean = oracle.paged_decode(h["q"], k, v, bt, b.context_lens, b.scale)
    assert np.array_equal(poisoned, clean)


# --------------------------------------------------- partition and merge ----
@pytest.mark.parametrize("part", [16, 48, 512, None])
def test_partition_merge_equals_single_pass(part):
    rng = np.random.default_rng(14)
    lens = [1, 16, 47, 600, 1100]
    q, kp, vp, bt, cl, _, _, _ = random_paged(rng, lens, 4, 2, 8)
    full = oracle.paged_decode(q, kp, vp, bt, cl, 0.3)
    for s, L in enumerate(lens):
        P = part or L
        for h in range(4):
            ms, ls, os_ = [], [], []
            for t0 in range(0, max(L, 1), P):
                m, l, o = oracle.partition_stats(q, kp, vp, bt, cl, 0.3, s, h, t0, min(L, t0 + P))
                ms.append(m)
                ls.append(l)
                os_.append(o)
            merged = oracle.lse_merge(np.array(ms), np.array(ls), np.array(os_))
            np.testing.assert_allclose(merged, full[s, h], rtol=0, atol=1e-12)


def test_merge_ignores_empty_parts():
    m = np.array([-np.inf, 0.5, -np.inf])
    l = np.array([0.0, 2.0, 0.0])
    o = np.array([[np.nan, np.nan], [1.0, -2.0], [0.0, 0.0]])
    assert np.array_equal(oracle.lse_merge(m, l, o), np.array([1.0, -2.0]))
    assert np.array_equal(oracle.lse_merge(m[[0]], l[[0]], o[[0]]), np.zeros(2))


def test_golden_lse_merge_from_float32_partials():
    """The hand-derived two-part merge, entered as single-precision partials (the
    form a GPU writes them in): only the rounding of ln 3 to float32 remains."""
    g = _golden("lse_merge_two_parts.json")
    out = oracle.lse_merge(np.array(g["m"], dtype=np.float32), np.array(g["l"], dtype=np.float32),
                           np.array(g["o"], dtype=np.float32))
    np.testing.assert_allclose(out, g["expected"], rtol=0, atol=1e-6)


def test_float32_merge_is_the_merge_of_the_widened_partials():
    """Single-precision partials (with empty parts and rows whose every part is
    empty) merge exactly as their values widened to float64 by numpy do; the
    float64 merge is pinned on its own above (fixture, associativity)."""
    rng = np.random.default_rng(31)
    for trial in range(40):
        P = int(rng.integers(1, 12))
        D = int(rng.choice([1, 3, 64, 128]))
        m = (rng.standard_normal(P) * 6).astype(np.float32)
        l = (rng.random(P) * 50 + 0.5).astype(np.float32)
        o = rng.standard_normal((P, D)).astype(np.float32)
        empty = rng.random(P) < (1.0 if trial % 10 == 9 else 0.3)
        m[empty] = -np.inf
        l[empty] = 0.0
        o[empty] = np.nan
        got = oracle.lse_merge(m, l, o)
        want = oracle.lse_merge(m.astype(np.float64), l.astype(np.float64), o.astype(np.float64))
        assert np.array_equal(got, want, equal_nan=False), trial
        if empty.all():
            assert np.array_equal(got, np.zeros(D))


def test_float32_merge_of_rounded_partitions_matches_single_pass():
    """Partition statistics rounded to float32 and merged through the
    single-precision entry stay within float32 rounding of the single pass."""
    rng = np.random.default_rng(32)
    lens = [5, 33, 700]
    q, kp, vp, bt, cl, _, _, _ = random_paged(rng, lens, 4, 2, 16)
    full = oracle.paged_decode(q, kp, vp, bt, cl, 0.25)
    for s, L in enumerate(lens):
        for h in range(4):
            parts = [oracle.partition_stats(q, kp, vp, bt, cl, 0.25, s, h, t0, min(L, t0 + 64))
                     for t0 in range(0, L, 64)]
            m = np.array([p[0] for p in parts], dtype=np.float32)
            l = np.array([p[1] for p in parts], dtype=np.float32)
            o = np.array([p[2] for p in parts], dtype=np.float32)
            merged = oracle.lse_merge(m, l, o)
            np.testing.assert_allclose(merged, full[s, h], rtol=0, atol=2e-6)


# ------------------------------------------------- reshape_and_cache, slots ----
def test_reshape_then_decode_equals_dense():
    """Write a whole context token by token through slot_mapping + reshape_and_cache into a
    NaN pool, then decode: the result is dense attention over the tokens written."""
    rng = np.random.default_rng(15)
    lens = [5, 16, 33]
    hq, hkv, d = 4, 2, 8
    nb = 12
    perm = rng.permutation(nb)
    tables, used = [], 0
    for L in lens:
        n = (L + BS - 1) // BS
        tables.append(perm[used:used + n].tolist())
        used += n
    bt = np.full((len(lens), 3), -1, dtype=np.int32)
    for s, t in enumerate(tables):
        bt[s, :len(t)] = t
    kpool = np.full((nb, hkv, BS, d), np.nan, dtype=np.float32)
    vpool = np.full((nb, hkv, BS, d), np.nan, dtype=np.float32)
    seq = np.concatenate([np.full(L, s) for s, L in enumerate(lens)]).astype(np.int32)
    pos = np.concatenate([np.arange(L) for L in lens]).astype(np.int32)
    order = rng.permutation(seq.shape[0])           # write order does not matter
    seq, pos = seq[order], pos[order]
    knew = rng.standard_normal((seq.shape[0], hkv, d)).astype(np.float32)
    vnew = rng.standard_normal((seq.shape[0], hkv, d)).astype(np.float32)
    slots = oracle.slot_mapping(bt, seq, pos)
    assert len(set(slots.tolist())) == len(slots)
    oracle.reshape_and_cache(knew, vnew, kpool, vpool, slots)
    q = rng.standard_normal((len(lens), hq, d)).astype(np.float32)
    cl = np.array(lens, dtype=np.int32)
    out = oracle.paged_decode(q, kpool, vpool, bt, cl, 0.4)
    for s, L in enumerate(lens):
        K = np.zeros((L, hkv, d), dtype=np.float32)
        V = np.zeros((L, hkv, d), dtype=np.float32)
        for t in np.nonzero(seq == s)[0]:
            K[pos[t]] = knew[t]
            V[pos[t]] = vnew[t]
        np.testing.assert_allclose(out[s], dense_attention(q[s], K, V, 0.4), rtol=0, atol=1e-12)
    # exactly the written rows changed: T tokens x Hkv heads rows of D values
    assert np.isfinite(kpool).all(axis=-1).sum() == seq.shape[0] * hkv


def test_reshape_skips_negative_slots_and_rejects_out_of_range():
    k = np.ones((2, 1, 4), dtype=np.float32)
    kc = np.zeros((2, 1, BS, 4), dtype=np.float32)
    vc = np.zeros_like(kc)
    oracle.reshape_and_cache(k, k, kc, vc, np.array([-1, 17]))
    assert kc[1, 0, 1].tolist() == [1, 1, 1, 1] and kc.sum() == 4
    with pytest.raises(oracle.OracleError):
        oracle.reshape_and_cache(k, k, kc, vc, np.array([0, 32]))


def test_copy_blocks_snapshot_semantics():
    nb = 3
    k = np.arange(nb * BS * 2, dtype=np.float32).reshape(nb, 1, BS, 2)
    v = k + 0.5
    k0, v0 = k.copy(), v.copy()
    oracle.copy_blocks(k, v, np.array([[0, 1], [1, 2]]))   # a chain: reads happen first
    assert np.array_equal(k[1], k0[0]) and np.array_equal(k[2], k0[1])
    assert np.array_equal(v[1], v0[0]) and np.array_equal(v[2], v0[1])
    assert np.array_equal(k[0], k0[0])
    with pytest.raises(oracle.OracleError):
        oracle.copy_blocks(k, v, np.array([[0, 3]]))


def test_bad_table_entry_and_length_are_errors():
    rng = np.random.default_rng(16)
    q, kp, vp, bt, cl, _, _, _ = random_paged(rng, [20], 1, 1, 4)
    bad = bt.copy()
    bad[0, 1] = kp.shape[0]
    with pytest.raises(oracle.OracleError):
        oracle.paged_decode(q, kp, vp, bad, cl, 1.0)
    with pytest.raises(oracle.OracleError):
        oracle.paged_decode(q, kp, vp, bt, np.array([33], dtype=np.int32), 1.0)


# -------------------------------------------------------- tolerance sanity ----
def test_bf16_rounding_of_exact_output_meets_the_tolerance():
    """The bf16 tolerance (|e| <= 2e-2 + 1e-2 |ref|) is attainable: rounding the exact
    output to bf16 alone stays far inside it."""
    b = workloads.random_batch(17, [100, 1000, 2000], 32, 8, 128, "bf16", device="cpu")
    h = b.host()
    ref = oracle.paged_decode(h["q"], h["k_cache"], h["v_cache"], b.block_tables,
                              b.context_lens, b.scale)
    rounded = torch.from_numpy(ref).to(torch.bfloat16).double().numpy()
    err = np.abs(rounded - ref)
    assert (err <= 2e-2 + 1e-2 * np.abs(ref)).all()
    assert err.max() <= 2.0 ** -8 * np.abs(ref).max()


# ------------------------------------------------------- several query tokens ----
def _multi_case(rng, lens, chunks, hq, hkv, d):
    q1, kp, vp, bt, cl, Ks, Vs, _ = random_paged(rng, lens, hq, hkv, d)
    qsl = np.concatenate([[0], np.cumsum(chunks)]).astype(np.int32)
    q = rng.standard_normal((int(qsl[-1]), hq, d)).astype(np.float32)
    return q, kp, vp, bt, cl, Ks, Vs, qsl


def test_multi_with_one_token_per_sequence_is_decode():
    rng = np.random.default_rng(20)
    lens = [1, 16, 37, 90]
    q, kp, vp, bt, cl, _, _, _ = random_paged(rng, lens, 8, 2, 16)
    qsl = np.arange(len(lens) + 1, dtype=np.int32)
    assert np.array_equal(oracle.paged_multi(q, kp, vp, bt, cl, qsl, 0.3),
                          oracle.paged_decode(q, kp, vp, bt, cl, 0.3))


def test_multi_matches_dense_causal_attention():
    rng = np.random.default_rng(21)
    lens, chunks = [5, 33, 64, 70], [5, 4, 1, 16]
    q, kp, vp, bt, cl, Ks, Vs, qsl = _multi_case(rng, lens, chunks, 8, 2, 16)
    out = oracle.paged_multi(q, kp, vp, bt, cl, qsl, 0.25)
    for s, (L, n) in enumerate(zip(lens, chunks)):
        for i in range(n):
            p = L - n + i                                  # this token's position
            row = qsl[s] + i
            ref = dense_attention(q[row], Ks[s][:p + 1], Vs[s][:p + 1], 0.25)
            np.testing.assert_allclose(out[row], ref, rtol=0, atol=1e-12)


def test_multi_last_token_sees_the_whole_context_and_first_prompt_token_only_itself():
    rng = np.random.default_rng(22)
    lens, chunks = [20, 48], [20, 3]               # the first chunk is a whole prompt
    q, kp, vp, bt, cl, Ks, Vs, qsl = _multi_case(rng, lens, chunks, 4, 4, 8)
    out = oracle.paged_multi(q, kp, vp, bt, cl, qsl, 0.5)
    last = qsl[1:] - 1
    assert np.array_equal(out[last], oracle.paged_decode(np.ascontiguousarray(q[last]), kp, vp,
                                                         bt, cl, 0.5))
    for h in range(4):                             # position 0 attends to key 0 alone
        assert np.array_equal(out[0, h], Vs[0][0, h].astype(np.float64))


def test_multi_rejects_chunks_longer_than_the_context():
    rng = np.random.default_rng(23)
    q, kp, vp, bt, cl, _, _, qsl = _multi_case(rng, [4], [5], 1, 1, 8)
    with pytest.raises(oracle.OracleError):
        oracle.paged_multi(q, kp, vp, bt, cl, qsl, 1.0)


# ------------------------------------------------------------- FP8 (e4m3) ----
def test_golden_e4m3_examples():
    g = _golden("e4m3_examples.json")
    codes = oracle.e4m3_quantize(np.array(g["values"], dtype=np.float32))
    assert codes.tolist() == g["codes"]


def test_e4m3_every_finite_code_round_trips():
    codes = np.array([c for c in range(256) if c & 0x7f != 0x7f], dtype=np.uint8)
    vals = oracle.e4m3_values(codes)
    assert np.isfinite(vals).all() and np.abs(vals).max() == 448.0
    assert np.array_equal(oracle.e4m3_quantize(vals.astype(np.float32)), codes)
    assert np.isnan(oracle.e4m3_values(np.array([0x7f, 0xff], dtype=np.uint8))).all()


def test_e4m3_rounds_to_the_nearest_value_ties_to_even():
    rng = np.random.default_rng(30)
    x = np.concatenate([rng.standard_normal(4000) * 10.0 ** rng.uniform(-4, 2.5, 4000),
                        rng.uniform(-500, 500, 200)]).astype(np.float32)
    codes = oracle.e4m3_quantize(x)
    grid_codes = np.array([c for c in range(256) if c & 0x7f != 0x7f], dtype=np.uint8)
    grid = oracle.e4m3_values(grid_codes)
    for xi, ci in zip(x.astype(np.float64), codes):
        if abs(xi) >= 448.0:
            assert oracle.e4m3_values(np.array([ci]))[0] == np.copysign(448.0, xi)
            continue
        d = np.abs(grid - xi)
        best = grid_codes[d == d.min()]
        if len(best) > 1:                                   # a tie: the even mantissa wins
            best = [c for c in best if (c & 1) == 0 and (c & 0x80) == (ci & 0x80)] or best
        assert ci in best, (xi, ci, best)


def test_two_term_e4m3_keeps_eight_bits():
    """The reading of the FP8 tensor-core arithmetic: q (scaled by a power of two so that
    |c q| < 128) and the weights (at most 2^8 under the lazy maximum) enter as
    high = e4m3(x) and low = e4m3(16 (x - high)), x ~ high + low / 16.  From e4m3's
    definition: 3 stored mantissa bits per term, the low term 4 binades finer, so for
    |x| in [2^-6, 2^8) the pair is within 2^-8 relative (about 8 significant bits, as
    bf16); below 2^-6 the low term reaches e4m3's subnormals and the error stays under
    2^-14 absolute.  The weights are first rounded to f16 (11 bits), which adds at most
    2^-11 relative."""
    rng = np.random.default_rng(31)
    n = 200000
    sign = rng.choice([-1.0, 1.0], n)

    def pair(x):
        hi = oracle.e4m3_values(oracle.e4m3_quantize(x))
        lo = oracle.e4m3_values(oracle.e4m3_quantize(16.0 * (x - hi)))
        return hi + lo / 16.0

    x = np.exp2(rng.uniform(-6, 8, n)) * sign
    rel = np.abs(pair(x) - x) / np.abs(x)
    assert rel.max() <= 2.0 ** -8
    x16 = x.astype(np.float16).astype(np.float64)          # the weights' f16 step
    rel16 = np.abs(pair(x16) - x) / np.abs(x)
    assert rel16.max() <= 2.0 ** -8 + 2.0 ** -11
    small = np.exp2(rng.uniform(-24, -6, n)) * sign
    assert np.abs(pair(small) - small).max() <= 2.0 ** -14
    # one term alone is only 4 bits: the pair is what makes the tolerance hold
    one = oracle.e4m3_values(oracle.e4m3_quantize(x))
    assert (np.abs(one - x) / np.abs(x)).max() > 2.0 ** -5


def test_e4m3_divides_by_the_scale_in_float():
    x = np.array([1.0, 3.0, -7.5], dtype=np.float32)
    assert np.array_equal(oracle.e4m3_quantize(x, 0.5), oracle.e4m3_quantize(x / np.float32(0.5)))


# ------------------------------------------------------------- FP8 (e5m2) ----
def test_golden_e5m2_examples():
    g = _golden("e5m2_examples.json")
    codes = oracle.e5m2_quantize(np.array(g["values"], dtype=np.float32))
    assert codes.tolist() == g["codes"]


def test_e5m2_every_finite_code_round_trips_and_specials():
    codes = np.array([c for c in range(256) if (c >> 2) & 31 != 31], dtype=np.uint8)
    vals = oracle.e5m2_values(codes)
    assert np.isfinite(vals).all() and np.abs(vals).max() == 57344.0
    assert np.array_equal(oracle.e5m2_quantize(vals.astype(np.float32)), codes)
    assert np.isinf(oracle.e5m2_values(np.array([0x7c, 0xfc], dtype=np.uint8))).all()
    assert np.isnan(oracle.e5m2_values(np.array([0x7d, 0x7e, 0x7f, 0xff], dtype=np.uint8))).all()


def test_e5m2_values_are_the_upper_byte_of_binary16():
    """An e5m2 code is the upper byte of an IEEE binary16 with the lower byte zero."""
    codes = np.arange(256, dtype=np.uint8)
    f16 = (codes.astype(np.uint16) << 8).view(np.float16).astype(np.float64)
    vals = oracle.e5m2_values(codes)
    same = np.isnan(f16) == np.isnan(vals)
    assert same.all()
    ok = ~np.isnan(f16)
    assert np.array_equal(f16[ok], vals[ok])


def test_e5m2_rounds_to_the_nearest_value_ties_to_even():
    rng = np.random.default_rng(33)
    x = np.concatenate([rng.standard_normal(3000) * 10.0 ** rng.uniform(-6, 4.5, 3000),
                        rng.uniform(-60000, 60000, 200)]).astype(np.float32)
    codes = oracle.e5m2_quantize(x)
    grid_codes = np.array([c for c in range(256) if (c >> 2) & 31 != 31], dtype=np.uint8)
    grid = oracle.e5m2_values(grid_codes)
    for xi, ci in zip(x.astype(np.float64), codes):
        if abs(xi) >= 57344.0:
            assert oracle.e5m2_values(np.array([ci]))[0] == np.copysign(57344.0, xi)
            continue
        d = np.abs(grid - xi)
        best = grid_codes[d == d.min()]
        if len(best) > 1:                                   # a tie: the even mantissa wins
            best = [c for c in best if (c & 1) == 0 and (c & 0x80) == (ci & 0x80)] or best
        assert ci in best, (xi, ci, best)


def test_e5m2_agrees_with_torch_in_range():
    """Inside the finite range torch's float32 -> float8_e5m2 cast rounds to nearest even
    as well (outside it torch overflows to infinity where the KV cache saturates)."""
    rng = np.random.default_rng(34)
    x = (rng.standard_normal(5000) * 10.0 ** rng.uniform(-5, 4, 5000)).astype(np.float32)
    x = x[np.abs(x) < 57344.0]
    want = torch.from_numpy(x).to(torch.float8_e5m2).view(torch.uint8).numpy()
    assert np.array_equal(oracle.e5m2_quantize(x), want)


def test_e5m2_decode_and_multi_match_dense_attention():
    rng = np.random.default_rng(35)
    lens, chunks = [1, 16, 33, 70], [1, 3, 5, 16]
    hq, hkv, d = 8, 2, 32
    q32, kp32, vp32, bt, cl, _, _, _ = random_paged(rng, lens, hq, hkv, d)
    k_scale, v_scale = np.float32(0.05), np.float32(0.02)
    kc = oracle.e5m2_quantize(np.nan_to_num(kp32), k_scale)
    vc = oracle.e5m2_quantize(np.nan_to_num(vp32), v_scale)
    kd = oracle.e5m2_values(kc) * float(k_scale)
    vd = oracle.e5m2_values(vc) * float(v_scale)
    qb = to_bf16_bits(q32)
    out = oracle.paged_decode_fp8(qb, kc, vc, k_scale, v_scale, bt, cl, 0.125, fmt="e5m2")
    qf = bf16_bits_to_f64(qb)
    ctx = []
    for s, L in enumerate(lens):
        nb = (L + BS - 1) // BS
        K = kd[bt[s, :nb]].transpose(0, 2, 1, 3).reshape(nb * BS, hkv, d)[:L]
        V = vd[bt[s, :nb]].transpose(0, 2, 1, 3).reshape(nb * BS, hkv, d)[:L]
        ctx.append((K, V))
        np.testing.assert_allclose(out[s], dense_attention(qf[s], K, V, 0.125), rtol=0,
                                   atol=1e-12)
    qsl = np.concatenate([[0], np.cumsum(chunks)]).astype(np.int32)
    qm = to_bf16_bits(rng.standard_normal((int(qsl[-1]), hq, d)).astype(np.float32))
    outm = oracle.paged_multi_fp8(qm, kc, vc, k_scale, v_scale, bt, cl, qsl, 0.2, fmt="e5m2")
    qmf = bf16_bits_to_f64(qm)
    for s, (L, n) in enumerate(zip(lens, chunks)):
        K, V = ctx[s]
        for i in range(n):
            p = L - n + i
            np.testing.assert_allclose(outm[qsl[s] + i], dense_attention(
                qmf[qsl[s] + i], K[:p + 1], V[:p + 1], 0.2), rtol=0, atol=1e-12)


def test_e5m2_reshape_quantises_into_the_slot():
    rng = np.random.default_rng(36)
    kf = (rng.standard_normal((3, 2, 16)) * 30).astype(np.float32)
    vf = (rng.standard_normal((3, 2, 16)) * 30).astype(np.float32)
    k, v = to_bf16_bits(kf), to_bf16_bits(vf)
    kf, vf = bf16_bits_to_f64(k).astype(np.float32), bf16_bits_to_f64(v).astype(np.float32)
    kc = np.zeros((4, 2, 16, 16), dtype=np.uint8)
    vc = np.zeros_like(kc)
    oracle.reshape_and_cache_fp8(k, v, kc, vc, np.array([5, -1, 50], dtype=np.int64), 0.5,
                                 0.25, fmt="e5m2")
    assert np.array_equal(kc[0, :, 5], oracle.e5m2_quantize(kf[0], 0.5))
    assert np.array_equal(vc[3, :, 2], oracle.e5m2_quantize(vf[2], 0.25))
    assert kc.astype(np.int64).sum() == oracle.e5m2_quantize(kf[[0, 2]], 0.5).astype(np.int64).sum()


def test_fp8_decode_matches_dense_attention_on_dequantised_values():
    rng = np.random.default_rng(31)
    lens = [1, 16, 33, 70]
    hq, hkv, d = 8, 2, 64
    q32, kp32, vp32, bt, cl, Ks, Vs, _ = random_paged(rng, lens, hq, hkv, d)
    k_scale, v_scale = np.float32(0.05), np.float32(0.02)
    kc = oracle.e4m3_quantize(np.nan_to_num(kp32), k_scale)
    vc = oracle.e4m3_quantize(np.nan_to_num(vp32), v_scale)
    qb = to_bf16_bits(q32)
    out = oracle.paged_decode_fp8(qb, kc, vc, k_scale, v_scale, bt, cl, 0.125)
    qf = bf16_bits_to_f64(qb)
    kd = oracle.e4m3_values(kc) * float(k_scale)
    vd = oracle.e4m3_values(vc) * float(v_scale)
    for s, L in enumerate(lens):
        n = (L + BS - 1) // BS
        K = kd[bt[s, :n]].transpose(0, 2, 1, 3).reshape(n * BS, hkv, d)[:L]
        V = vd[bt[s, :n]].transpose(0, 2, 1, 3).reshape(n * BS, hkv, d)[:L]
        np.testing.assert_allclose(out[s], dense_attention(qf[s], K, V, 0.125), rtol=0,
                                   atol=1e-12)


def test_fp8_multi_matches_dense_causal_attention_on_dequantised_values():
    """Several causal query tokens over FP8 pools: dense fp64 attention over the widened,
    scaled codes, each chunk token seeing keys up to its own position; one-token chunks
    equal FP8 decode."""
    rng = np.random.default_rng(32)
    lens, chunks = [4, 16, 33, 70], [4, 1, 5, 16]
    hq, hkv, d = 8, 2, 32
    _, kp32, vp32, bt, cl, _, _, _ = random_paged(rng, lens, hq, hkv, d)
    k_scale, v_scale = np.float32(0.04), np.float32(0.03)
    kc = oracle.e4m3_quantize(np.nan_to_num(kp32), k_scale)
    vc = oracle.e4m3_quantize(np.nan_to_num(vp32), v_scale)
    qsl = np.concatenate([[0], np.cumsum(chunks)]).astype(np.int32)
    qb = to_bf16_bits(rng.standard_normal((int(qsl[-1]), hq, d)).astype(np.float32))
    out = oracle.paged_multi_fp8(qb, kc, vc, k_scale, v_scale, bt, cl, qsl, 0.2)
    qf = bf16_bits_to_f64(qb)
    kd = oracle.e4m3_values(kc) * float(k_scale)
    vd = oracle.e4m3_values(vc) * float(v_scale)
    for s, (L, n) in enumerate(zip(lens, chunks)):
        nb = (L + BS - 1) // BS
        K = kd[bt[s, :nb]].transpose(0, 2, 1, 3).reshape(nb * BS, hkv, d)[:L]
        V = vd[bt[s, :nb]].transpose(0, 2, 1, 3).reshape(nb * BS, hkv, d)[:L]
        for i in range(n):
            p = L - n + i
            row = qsl[s] + i
            np.testing.assert_allclose(out[row], dense_attention(qf[row], K[:p + 1], V[:p + 1],
                                                                 0.2), rtol=0, atol=1e-12)
    one = np.arange(len(lens) + 1, dtype=np.int32)
    qd = np.ascontiguousarray(qb[:len(lens)])
    assert np.array_equal(oracle.paged_multi_fp8(qd, kc, vc, k_scale, v_scale, bt, cl, one, 0.2),
                          oracle.paged_decode_fp8(qd, kc, vc, k_scale, v_scale, bt, cl, 0.2))


def test_fp8_reshape_quantises_into_the_slot():
    rng = np.random.default_rng(32)
    hkv, d, nb = 2, 64, 4
    k = to_bf16_bits(rng.standard_normal((3, hkv, d)).astype(np.float32))
    v = to_bf16_bits(rng.standard_normal((3, hkv, d)).astype(np.float32))
    kc = np.zeros((nb, hkv, BS, d), dtype=np.uint8)
    vc = np.zeros_like(kc)
    slots = np.array([5, -1, 50])
    oracle.reshape_and_cache_fp8(k, v, kc, vc, slots, 0.1, 0.3)
    kf = bf16_bits_to_f64(k).astype(np.float32)
    vf = bf16_bits_to_f64(v).astype(np.float32)
    assert np.array_equal(kc[0, :, 5], oracle.e4m3_quantize(kf[0], 0.1))
    assert np.array_equal(vc[3, :, 2], oracle.e4m3_quantize(vf[2], 0.3))
    assert kc.astype(np.int64).sum() == oracle.e4m3_quantize(kf[[0, 2]], 0.1).astype(np.int64).sum()
