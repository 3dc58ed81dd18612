"""The native host block manager (include/pkv_block_manager.h), on the CPU.

The main check simulates the KV pool: every token is written to the slot the
manager hands out, every copy-on-write pair copies a whole block, and then
every live sequence, read back through its block table, must return exactly
its own tokens -- paging changes where K/V live, never what a sequence sees
(ipipp.com vLLM article, "二、PagedAttention分页原理深度剖析").  Reference counts
must equal the number of table entries pointing at each block, and the pool
must account for every block.  Prefix caching is checked against what the
wiki entry's "Automatic Prefix Caching" section fixes: chained hashes of full
blocks, exact block-by-block matching, full blocks only, LRU eviction.
"""
import numpy as np
import pytest

import paged_kv_cache_375_b200 as pkv

BS = 16


class SimPool:
    """Token ids stored per physical slot, updated exactly as the device would be."""

    def __init__(self, num_blocks):
        self.slots = np.full(num_blocks * BS, -1, dtype=np.int64)

    def write(self, slots, tokens):
        self.slots[np.asarray(slots)] = np.asarray(tokens)

    def copy(self, pairs):
        snap = self.slots.copy()
        for src, dst in pairs:
            self.slots[dst * BS:(dst + 1) * BS] = snap[src * BS:(src + 1) * BS]

    def read(self, table, length):
        pos = np.arange(length)
        return self.slots[table[pos // BS] * BS + pos % BS]


def check_invariants(bm, pool, seqs, num_blocks):
    ids = sorted(seqs)
    if ids:
        tables, lens = bm.block_tables(ids, max_blocks=256)
        refs = np.zeros(num_blocks, dtype=np.int64)
        for i, s in enumerate(ids):
            assert lens[i] == len(seqs[s])
            n = (lens[i] + BS - 1) // BS
            assert (tables[i, n:] == -1).all()
            row = tables[i, :n]
            assert len(set(row.tolist())) == n            # a sequence never repeats a block
            refs[row] += 1
            got = pool.read(row, lens[i])
            assert np.array_equal(got, np.array(seqs[s])), f"sequence {s} reads wrong tokens"
        for b in range(num_blocks):
            assert bm.refcount(b) == refs[b]
    st = bm.stats()
    assert st["free"] + st["evictable"] + st["used"] == num_blocks
    assert st["sequences"] == len(seqs)


@pytest.mark.parametrize("prefix_caching", [False, True])
@pytest.mark.parametrize("seed", [1, 2, 3])
def test_random_operations_keep_every_sequence_intact(prefix_caching, seed):
    rng = np.random.default_rng(seed)
    num_blocks = 400
    bm = pkv.BlockManager(num_blocks, BS, seed=seed, prefix_caching=prefix_caching)
    pool = SimPool(num_blocks)
    seqs = {}
    prompts = [rng.integers(0, 50, size=int(rng.integers(1, 90))).tolist() for _ in range(6)]
    next_id = 0
    for it in range(600):
        op = rng.random()
        if op < 0.2 or not seqs:
            prompt = list(prompts[rng.integers(len(prompts))])
            if rng.random() < 0.5:
                prompt += rng.integers(0, 50, size=int(rng.integers(0, 40))).tolist()
            try:
                cached = bm.add_sequence(next_id, prompt)
            except pkv.PkvError as e:
                assert e.status == 10
                continue
            assert cached % BS == 0 and cached <= len(prompt)
            if not prefix_caching:
                assert cached == 0
            # the caller writes the K/V of the prompt tokens that were not cached
            pool.write(bm.slots(next_id, cached, len(prompt)), prompt[cached:])
            seqs[next_id] = prompt
            next_id += 1
        elif op < 0.35:
            parent = int(rng.choice(list(seqs)))
            bm.fork(parent, next_id)
            seqs[next_id] = list(seqs[parent])
            next_id += 1
        elif op < 0.85:
            ids = rng.choice(list(seqs), size=min(len(seqs), int(rng.integers(1, 6))),
                             replace=False).tolist()
            toks = rng.integers(0, 50, size=len(ids)).tolist()
            try:
                slots = bm.append_tokens(ids, toks)
            except pkv.PkvError as e:
                assert e.status == 10
                check_invariants(bm, pool, seqs, num_blocks)   # nothing changed
                continue
            pool.copy(bm.take_copies())                          # copies before writes
            pool.write(slots, toks)
            for s, t in zip(ids, toks):
                seqs[s].append(t)
        else:
            s = int(rng.choice(list(seqs)))
            bm.free_sequence(s)
            del seqs[s]
        if it % 25 == 0:
            check_invariants(bm, pool, seqs, num_blocks)
    check_invariants(bm, pool, seqs, num_blocks)
    for s in list(seqs):
        bm.free_sequence(s)
    st = bm.stats()
    assert st["used"] == 0 and st["sequences"] == 0


def test_fork_then_append_copies_the_shared_partial_block_once():
    bm = pkv.BlockManager(50, BS, seed=4)
    bm.add_sequence(0, list(range(20)))          # 2 blocks, the second partial
    for c in range(1, 4):
        bm.fork(0, c)
    tables, _ = bm.block_tables([0], 8)
    shared_tail = int(tables[0, 1])
    assert bm.refcount(shared_tail) == 4
    bm.append_tokens([1, 2, 3, 0], [7, 7, 7, 7])
    pairs = bm.take_copies()
    assert pairs.shape == (3, 2) and (pairs[:, 0] == shared_tail).all()
    assert bm.refcount(shared_tail) == 1         # the last holder writes in place
    # full shared blocks are never copied: appending into a fresh block needs no copy
    bm2 = pkv.BlockManager(50, BS, seed=5)
    bm2.add_sequence(0, list(range(32)))
    bm2.fork(0, 1)
    bm2.append_tokens([0, 1], [1, 2])
    assert bm2.take_copies().shape == (0, 2)


def test_prefix_cache_reuses_full_blocks_only_and_matches_exactly():
    bm = pkv.BlockManager(100, BS, seed=6, prefix_caching=True)
    prompt = list(range(100, 150))               # 3 full blocks + 2 tokens
    assert bm.add_sequence(0, prompt) == 0
    assert bm.add_sequence(1, prompt) == 48      # full blocks reused, not the partial one
    t, _ = bm.block_tables([0, 1], 8)
    assert (t[0, :3] == t[1, :3]).all() and t[0, 3] != t[1, 3]
    # a difference inside block 1 stops the match after block 0
    other = list(prompt)
    other[20] = -5
    assert bm.add_sequence(2, other) == 16
    # same tokens, different prefix: the chained hash does not match
    shifted = [7] * 16 + prompt[16:]
    assert bm.add_sequence(3, shifted) == 0


def test_prefix_cache_survives_free_and_evicts_least_recently_used():
    nb = 8
    bm = pkv.BlockManager(nb, BS, seed=7, prefix_caching=True)
    a = list(range(32))                          # 2 full blocks
    b = list(range(1000, 1032))
    bm.add_sequence(0, a)
    bm.free_sequence(0)
    bm.add_sequence(1, b)
    bm.free_sequence(1)
    st = bm.stats()
    assert st["evictable"] == 4 and st["used"] == 0
    assert bm.add_sequence(2, a) == 32           # still cached after its owner ended
    bm.free_sequence(2)                          # a is now more recently used than b
    # use up the pool: 4 free blocks, then the oldest cached blocks (b's) go first
    bm.add_sequence(3, list(range(5000, 5000 + 16 * 6)))
    assert bm.stats()["evictable"] == 2
    bm.free_sequence(3)
    assert bm.add_sequence(4, a) == 32           # a survived
    assert bm.add_sequence(5, b) == 0            # b was evicted


def test_exhaustion_is_reported_and_changes_nothing():
    bm = pkv.BlockManager(3, BS, seed=8)
    bm.add_sequence(0, list(range(40)))          # all 3 blocks
    before = bm.stats()
    with pytest.raises(pkv.PkvError) as e:
        bm.add_sequence(1, [1])
    assert e.value.status == 10
    with pytest.raises(pkv.PkvError):
        bm.append_tokens([0] * 9, [1] * 9)       # 8 fit in the last block, the 9th needs a new one
    assert bm.stats() == before
    with pytest.raises(pkv.PkvError) as e:
        bm.fork(5, 6)
    assert e.value.status == 11
    with pytest.raises(pkv.PkvError):
        bm.add_sequence(0, [1])                  # id already in use


def _lcp_full(tables, lens, a, b):
    full = min(lens[a], lens[b]) // BS
    c = 0
    while c < full and tables[a, c] == tables[b, c]:
        c += 1
    return c


def check_groups(bm, ids, min_shared):
    """Runs of consecutive sequences with common leading blocks, checked by brute force:
    they tile the list in order, every member holds the run's first P table entries, P is
    the exact minimum over members of the blocks common with the first member (full ones
    only), and no run could take its next sequence."""
    gs, sb = bm.shared_prefix_groups(ids, min_shared)
    tables, lens = bm.block_tables(ids, max_blocks=256)
    n = len(ids)
    assert gs[0] == 0 and gs[-1] == n and (np.diff(gs) >= 1).all() and len(sb) == len(gs) - 1
    for r in range(len(sb)):
        a, e = int(gs[r]), int(gs[r + 1])
        if e - a == 1:
            assert sb[r] == 0
        else:
            p = min(_lcp_full(tables, lens, a, m) for m in range(a + 1, e))
            assert sb[r] == p >= min_shared
            for m in range(a, e):
                assert (tables[m, :p] == tables[a, :p]).all() and p <= lens[m] // BS
        if e < n:
            ext = _lcp_full(tables, lens, a, e)
            if e - a >= 2:
                ext = min(ext, int(sb[r]))
            assert ext < min_shared
    return gs, sb


def test_shared_prefix_groups_of_forks_and_cached_prompts():
    bm = pkv.BlockManager(400, BS, seed=9, prefix_caching=True)
    bm.add_sequence(0, list(range(40)))            # 2 full blocks + a partial one
    for c in (1, 2, 3):
        bm.fork(0, c)
    bm.add_sequence(10, list(range(1000, 1100)))   # 6 full blocks + a partial one
    bm.fork(10, 11)
    bm.add_sequence(20, list(range(5000, 5010)))   # shares nothing
    prompt = list(range(7000, 7048))               # 3 full blocks, cached on first use
    bm.add_sequence(30, prompt + [1])
    bm.add_sequence(31, prompt + [2, 3])           # prefix caching shares the 3 full blocks
    ids = [0, 1, 2, 3, 10, 11, 20, 30, 31]
    bm.append_tokens(ids, [5] * len(ids))          # copies the shared partial blocks
    bm.take_copies()
    gs, sb = check_groups(bm, ids, 1)
    assert gs.tolist() == [0, 4, 6, 7, 9] and sb.tolist() == [2, 6, 0, 3]
    gs, sb = check_groups(bm, ids, 3)
    assert gs.tolist() == [0, 1, 2, 3, 4, 6, 7, 9] and sb.tolist() == [0, 0, 0, 0, 6, 0, 3]
    # another order splits the runs
    check_groups(bm, [0, 10, 1, 11, 2, 3], 1)
    with pytest.raises(pkv.PkvError):
        bm.shared_prefix_groups([0, 99], 1)
    with pytest.raises(pkv.PkvError):
        bm.shared_prefix_groups([0, 1], 0)


@pytest.mark.parametrize("seed", [1, 2, 3, 4])
def test_shared_prefix_groups_random_forest(seed):
    rng = np.random.default_rng(seed)
    bm = pkv.BlockManager(3000, BS, seed=seed)
    ids = []
    for p in range(12):
        root = 100 * p
        bm.add_sequence(root, rng.integers(0, 1000, size=int(rng.integers(1, 120))).tolist())
        fam = [root]
        for c in range(int(rng.integers(0, 6))):
            parent = int(rng.choice(fam))
            bm.fork(parent, root + c + 1)
            fam.append(root + c + 1)
            steps = int(rng.integers(0, 40))
            for _ in range(steps):
                bm.append_tokens([root + c + 1], [int(rng.integers(0, 1000))])
        ids += fam
    bm.take_copies()
    for m in (1, 2, 4):
        check_groups(bm, ids, m)
        check_groups(bm, list(rng.permutation(ids)), m)


@pytest.mark.parametrize("seed", [5, 6, 7])
def test_prefix_order_puts_sharers_together(seed):
    """In the prefix order every family of forks (sharing at least one full block) forms
    one run, whatever order the step's rows came in; the order is a permutation."""
    rng = np.random.default_rng(seed)
    bm = pkv.BlockManager(4000, BS, seed=seed)
    fams = []
    for p in range(10):
        root = 100 * p
        bm.add_sequence(root, rng.integers(0, 1000, size=int(rng.integers(16, 200))).tolist())
        fam = [root]
        for c in range(int(rng.integers(1, 6))):
            bm.fork(root, root + c + 1)
            fam.append(root + c + 1)
        for s in fam:
            for _ in range(int(rng.integers(0, 30))):
                bm.append_tokens([s], [int(rng.integers(0, 1000))])
        fams.append(fam)
    bm.take_copies()
    ids = [s for f in fams for s in f]
    shuffled = list(rng.permutation(ids))
    order = bm.prefix_order(shuffled)
    assert sorted(order.tolist()) == list(range(len(ids)))
    ordered = [int(shuffled[i]) for i in order]
    gs, sb = check_groups(bm, ordered, 1)
    runs = [set(ordered[gs[r]:gs[r + 1]]) for r in range(len(sb))]
    for f in fams:
        assert set(f) in runs, f"family {f} split over runs"
    with pytest.raises(pkv.PkvError):
        bm.prefix_order([0, 12345])
