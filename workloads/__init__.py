"""Seeded synthetic inputs for paged KV-cache decode.

This module only draws inputs: context lengths, block tables (from a host block
manager with a shuffled free list, reference counts and copy-on-write pair
emission), the pool contents, the query rows and the new tokens' K/V.  It holds
none of the attention arithmetic and does not compute slots; the CUDA path and
the oracle each do that themselves from what is drawn here.

Shapes follow the serving scenarios the pages describe:
  * 16-token blocks and a per-sequence block table (ipipp.com vLLM article,
    "二、PagedAttention分页原理深度剖析");
  * blocks taken on demand from one shared pool, any free block serving any
    request ("vLLM 深读", "先看浪费在哪里");
  * parallel samples pointing at the same prefix blocks, reference counted,
    with copy-on-write on the first write to a shared block (same sections);
  * LLaMA-2-13B on one 80 GB card and up to 256 concurrent sequences (the
    ipipp.com article's sections one and four).

Every tensor is seeded: lengths, the free-list shuffle and the tables come from
numpy's PCG64 (``default_rng(seed)``), values from ``torch.randn`` with a
generator seeded the same way on the device the batch is built on, drawn in
float32 and rounded to bf16 where the configuration is bf16.  Slots that hold
no token (past a sequence's length, unreferenced blocks) are filled with NaN so
that any read of them shows up in the result; unused block-table entries are -1.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np
import torch

BLOCK_SIZE = 16

CONFIGS = {
    "c1_tiny_fp32": "tiny fp32: 4 seqs, lens {17,50,100,128}, 8q=8kv heads, d64, 64-block pool",
    "c2_llama2_13b_mha": "LLaMA-2-13B-shaped MHA bf16: batch 64, 40 heads, d128, lens U[128,2048], 20k-block pool",
    "c3_llama3_8b_gqa": "Llama-3-8B-shaped GQA bf16: batch 256, 32q/8kv, d128, lognormal lens (median 1000) clipped "
                        "[16,8192], reshape_and_cache of the new token before attention",
    "c4_shared_prefix": "parallel sampling bf16 GQA 32q/8kv d128: 32 prompts x 8 samples sharing 1024+r prefix "
                        "tokens, tails U[0,512], copy-on-write via copy_blocks, then decode",
    "c5_long_splitk": "long context bf16 GQA 64q/8kv d128: batch 8, lens U[32768,131072], split-K partitions "
                      "merged by log-sum-exp (512 tokens as configured; the automatic size is 4096)",
}
CONFIG_SEEDS = {name: i + 1 for i, name in enumerate(CONFIGS)}

# Spread of the lognormal context lengths of the Llama-3-8B-shaped batch: only
# the median (1000) is given, sigma is a reading (about 0.3 % clipped at 8192).
C3_LOGNORMAL_SIGMA = 0.75


class BlockManager:
    """Host-side block bookkeeping: a shuffled free list and reference counts.

    Blocks are popped from a seeded permutation of the pool, so physical
    placement is scattered.  ``fork`` shares a table's blocks (reference count
    +1 each); ``prepare_write`` gives a sequence a private block before it
    writes into a shared one and records the (src, dst) copy-on-write pair.
    """

    def __init__(self, num_blocks: int, rng: np.random.Generator):
        self.num_blocks = num_blocks
        self.free = list(rng.permutation(num_blocks).astype(np.int64))
        self.refcount = np.zeros(num_blocks, dtype=np.int64)
        self.cow_pairs: list[tuple[int, int]] = []

    def allocate(self, n: int) -> list[int]:
        if n > len(self.free):
            raise MemoryError(f"pool exhausted: need {n} blocks, {len(self.free)} free")
        out = [int(self.free.pop()) for _ in range(n)]
        for b in out:
            self.refcount[b] = 1
        return out

    def fork(self, table: list[int]) -> list[int]:
        for b in table:
            self.refcount[b] += 1
        return list(table)

    def prepare_write(self, table: list[int], logical_block: int) -> None:
        """Make ``table[logical_block]`` private before a write (copy-on-write)."""
        b = table[logical_block]
        if self.refcount[b] > 1:
            (new,) = self.allocate(1)
            self.refcount[b] -= 1
            table[logical_block] = new
            self.cow_pairs.append((b, new))

    def blocks_in_use(self) -> int:
        return int((self.refcount > 0).sum())


@dataclass
class Batch:
    """One decode step's inputs.  Tensors live on ``device``."""

    name: str
    seed: int
    dtype: str                      # "f32", "bf16", "fp8" (e4m3 caches, bf16 q and new K/V)
                                    # or "fp8e5m2" (e5m2 caches)
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    num_blocks: int
    context_lens: np.ndarray        # int32 [B], including the token being decoded
    block_tables: np.ndarray        # int32 [B][MB], -1 past each sequence's blocks
    scale: float                    # a float32 value
    q: torch.Tensor                 # [B][Hq][D]
    k_cache: torch.Tensor           # [NB][Hkv][BS][D]
    v_cache: torch.Tensor
    new_k: torch.Tensor             # [T][Hkv][D] tokens to write before attention
    new_v: torch.Tensor
    new_seq: np.ndarray             # int32 [T] sequence of each new token
    new_pos: np.ndarray             # int32 [T] position of each new token
    cow_pairs: np.ndarray           # int64 [P][2] (src, dst), applied before the writes
    meta: dict = field(default_factory=dict)
    # several query tokens per sequence: rows query_start_loc[s] .. [s+1]-1 of q
    query_start_loc: np.ndarray | None = None
    # FP8 caches: a cached code c stands for c * k_scale (K) or c * v_scale (V)
    k_scale: float = 1.0
    v_scale: float = 1.0

    @property
    def num_seqs(self) -> int:
        return int(self.context_lens.shape[0])

    @property
    def block_size(self) -> int:
        return BLOCK_SIZE

    @property
    def max_blocks_per_seq(self) -> int:
        return int(self.block_tables.shape[1])

    @property
    def max_query_len(self) -> int:
        if self.query_start_loc is None:
            return 1
        return int(np.diff(self.query_start_loc).max()) if self.num_seqs else 1

    @property
    def max_context_len(self) -> int:
        return int(self.context_lens.max()) if self.num_seqs else 0

    @property
    def elem_bytes(self) -> int:
        """Bytes of one cache element."""
        return {"f32": 4, "bf16": 2, "fp8": 1, "fp8e5m2": 1}[self.dtype]

    @property
    def q_elem_bytes(self) -> int:
        """Bytes of one q / out / new K/V element."""
        return 4 if self.dtype == "f32" else 2

    def kv_bytes(self) -> int:
        """Algorithmic K+V bytes one decode step reads: every context token once per kv head."""
        return int(self.context_lens.astype(np.int64).sum()) * self.num_kv_heads * self.head_dim \
            * self.elem_bytes * 2

    def unique_kv_bytes(self) -> int:
        """K+V bytes of distinct physical slots read (shared prefix blocks counted once)."""
        used: dict[int, int] = {}
        for s in range(self.num_seqs):
            L = int(self.context_lens[s])
            for i in range((L + BLOCK_SIZE - 1) // BLOCK_SIZE):
                b = int(self.block_tables[s, i])
                used[b] = max(used.get(b, 0), min(BLOCK_SIZE, L - i * BLOCK_SIZE))
        return sum(used.values()) * self.num_kv_heads * self.head_dim * self.elem_bytes * 2

    def io_bytes(self) -> int:
        """q + out + block-table + context-length bytes of one decode step."""
        T, Hq, D = self.q.shape[0], self.num_q_heads, self.head_dim
        return 2 * T * Hq * D * self.q_elem_bytes + self.block_tables.nbytes + self.context_lens.nbytes

    def host(self) -> dict:
        """Host numpy copies: float32 arrays, uint16 arrays holding bf16 bits, or uint8
        arrays holding e4m3 codes."""
        def h(t):
            t = t.detach().contiguous().cpu()
            if t.dtype == torch.bfloat16:
                return t.view(torch.int16).numpy().view(np.uint16)
            if t.dtype in (torch.float8_e4m3fn, torch.float8_e5m2):
                return t.view(torch.uint8).numpy()
            return t.numpy()
        return {"q": h(self.q), "k_cache": h(self.k_cache), "v_cache": h(self.v_cache),
                "new_k": h(self.new_k), "new_v": h(self.new_v)}

    def to(self, device) -> "Batch":
        return Batch(self.name, self.seed, self.dtype, self.num_q_heads, self.num_kv_heads,
                     self.head_dim, self.num_blocks, self.context_lens.copy(),
                     self.block_tables.copy(), self.scale, self.q.to(device),
                     self.k_cache.to(device), self.v_cache.to(device), self.new_k.to(device),
                     self.new_v.to(device), self.new_seq.copy(), self.new_pos.copy(),
                     self.cow_pairs.copy(), dict(self.meta),
                     None if self.query_start_loc is None else self.query_start_loc.copy(),
                     self.k_scale, self.v_scale)


def torch_dtype(dtype: str) -> torch.dtype:
    """Element type of q / out / new K/V (an FP8 configuration's caches are e4m3)."""
    return {"f32": torch.float32, "bf16": torch.bfloat16, "fp8": torch.bfloat16,
            "fp8e5m2": torch.bfloat16}[dtype]


def fp8_format(dtype: str) -> str | None:
    """The FP8 code format of a configuration's pools ("e4m3", "e5m2"), None if not FP8."""
    return {"fp8": "e4m3", "fp8e5m2": "e5m2"}.get(dtype)


# Scales of the FP8 configurations' pools (exact in float32, different so that
# a swapped pair shows).
FP8_K_SCALE = 1.0 / 64.0
FP8_V_SCALE = 3.0 / 128.0
E4M3_NAN_CODE = 0x7F


def _random_codes(shape, gen, device, chunk_rows: int | None = None) -> torch.Tensor:
    """Random e4m3 bit patterns: sign, exponent field 1..15 and mantissa drawn uniformly
    (magnitudes log-uniform over 2^-6 .. 448); the NaN pattern is replaced by its
    neighbour 0x7e.  A drawing of codes, not a quantisation."""
    out = torch.empty(shape, dtype=torch.uint8, device=device)
    rows = shape[0]
    step = chunk_rows or rows
    for r0 in range(0, rows, step):
        r1 = min(rows, r0 + step)
        sub = (r1 - r0,) + tuple(shape[1:])
        sign = torch.randint(0, 2, sub, generator=gen, device=device, dtype=torch.uint8)
        expo = torch.randint(1, 16, sub, generator=gen, device=device, dtype=torch.uint8)
        mant = torch.randint(0, 8, sub, generator=gen, device=device, dtype=torch.uint8)
        c = (sign << 7) | (expo << 3) | mant
        out[r0:r1] = torch.where((c & 0x7F) == E4M3_NAN_CODE, c - 1, c)
    return out.view(torch.float8_e4m3fn)


def _random_codes_e5m2(shape, gen, device, chunk_rows: int | None = None) -> torch.Tensor:
    """Random e5m2 bit patterns: sign, exponent field 8..22 and mantissa drawn uniformly
    (magnitudes log-uniform over 2^-7 .. 2^7 x 1.75).  A drawing of codes."""
    out = torch.empty(shape, dtype=torch.uint8, device=device)
    rows = shape[0]
    step = chunk_rows or rows
    for r0 in range(0, rows, step):
        r1 = min(rows, r0 + step)
        sub = (r1 - r0,) + tuple(shape[1:])
        sign = torch.randint(0, 2, sub, generator=gen, device=device, dtype=torch.uint8)
        expo = torch.randint(8, 23, sub, generator=gen, device=device, dtype=torch.uint8)
        mant = torch.randint(0, 4, sub, generator=gen, device=device, dtype=torch.uint8)
        out[r0:r1] = (sign << 7) | (expo << 2) | mant
    return out.view(torch.float8_e5m2)


def default_scale(head_dim: int) -> float:
    """1/sqrt(head_dim), rounded to float32 (the value both sides receive)."""
    return float(np.float32(1.0 / math.sqrt(head_dim)))


def _randn(shape, gen, device, dtype: str, chunk_rows: int | None = None) -> torch.Tensor:
    out = torch.empty(shape, dtype=torch_dtype(dtype), device=device)
    rows = shape[0]
    step = chunk_rows or rows or 1
    for r0 in range(0, rows, step):
        r1 = min(rows, r0 + step)
        out[r0:r1] = torch.randn((r1 - r0,) + tuple(shape[1:]), generator=gen, device=device,
                                 dtype=torch.float32).to(out.dtype)
    return out


def _assemble(name: str, seed: int, dtype: str, hq: int, hkv: int, d: int, num_blocks: int,
              lens: np.ndarray, tables: list[list[int]], initial_tables: list[list[int]],
              prefill_lens: np.ndarray, new_seq: np.ndarray, new_pos: np.ndarray,
              cow_pairs: list[tuple[int, int]], device, meta: dict,
              scale: float | None = None) -> Batch:
    """Draw values and poison every slot that holds no token.

    ``initial_tables`` / ``prefill_lens`` describe the pool before this step's
    copy-on-write copies and new-token writes: exactly positions
    [0, prefill_len) of each sequence hold finite values then.
    """
    B = len(tables)
    mb = max([len(t) for t in tables] + [len(t) for t in initial_tables] + [1])
    bt = np.full((B, mb), -1, dtype=np.int32)
    for s, t in enumerate(tables):
        bt[s, :len(t)] = t
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    shape = (num_blocks, hkv, BLOCK_SIZE, d)
    chunk = max(1, (1 << 26) // (hkv * BLOCK_SIZE * d))
    fp8 = fp8_format(dtype) is not None
    vdt = "bf16" if fp8 else dtype
    if fp8:
        draw = _random_codes if dtype == "fp8" else _random_codes_e5m2
        k_cache = draw(shape, gen, device, chunk)
        v_cache = draw(shape, gen, device, chunk)
    else:
        k_cache = _randn(shape, gen, device, dtype, chunk)
        v_cache = _randn(shape, gen, device, dtype, chunk)
    q = _randn((B, hq, d), gen, device, vdt)
    T = int(new_seq.shape[0])
    new_k = _randn((T, hkv, d), gen, device, vdt)
    new_v = _randn((T, hkv, d), gen, device, vdt)

    # Poison: unreferenced blocks, and slots at or past the prefill length.
    referenced = np.zeros(num_blocks, dtype=bool)
    partial: dict[int, int] = {}
    for s, t in enumerate(initial_tables):
        n_full, rem = divmod(int(prefill_lens[s]), BLOCK_SIZE)
        for b in t[:n_full]:
            referenced[b] = True
        if rem:
            b = t[n_full]
            # a block shared by several sequences is valid up to its largest use
            partial[b] = max(partial.get(b, 0), rem)
    for b in list(partial):
        if referenced[b]:          # full for some sharer: nothing to poison
            del partial[b]
        else:
            referenced[b] = True
    unref = torch.from_numpy(np.nonzero(~referenced)[0]).to(device)
    # NaN for float pools; the NaN code through a byte view for e4m3 pools
    kp, vp = (k_cache.view(torch.uint8), v_cache.view(torch.uint8)) if fp8 else (k_cache, v_cache)
    nan = E4M3_NAN_CODE if fp8 else float("nan")
    if unref.numel():
        kp.index_fill_(0, unref, nan)
        vp.index_fill_(0, unref, nan)
    for b, rem in partial.items():
        kp[b, :, rem:, :] = nan
        vp[b, :, rem:, :] = nan

    pairs = np.array(cow_pairs, dtype=np.int64).reshape(-1, 2)
    b = Batch(name, seed, dtype, hq, hkv, d, num_blocks, lens.astype(np.int32), bt,
              default_scale(d) if scale is None else scale, q, k_cache, v_cache, new_k, new_v,
              new_seq.astype(np.int32), new_pos.astype(np.int32), pairs, meta)
    if fp8:
        b.k_scale, b.v_scale = FP8_K_SCALE, FP8_V_SCALE
    return b


def random_batch(seed: int, lens, hq: int, hkv: int, d: int, dtype: str = "bf16",
                 num_blocks: int | None = None, device="cpu", new_token: bool = False,
                 scale: float | None = None, name: str = "random", extra_table: int = 0) -> Batch:
    """A decode batch with the given context lengths and blocks from a shuffled free list.

    With ``new_token`` the last position of every sequence is left poisoned and
    its K/V is returned as a new token to write before attention.
    ``extra_table`` adds that many unused (-1) columns to the block table.
    """
    lens = np.asarray(lens, dtype=np.int64)
    rng = np.random.default_rng(seed)
    need = int(sum((int(L) + BLOCK_SIZE - 1) // BLOCK_SIZE for L in lens))
    nb = num_blocks if num_blocks is not None else max(need + 8, 16)
    bm = BlockManager(nb, rng)
    tables = [bm.allocate((int(L) + BLOCK_SIZE - 1) // BLOCK_SIZE) for L in lens]
    width = max([len(t) for t in tables] + [1]) + extra_table
    if new_token:
        prefill = np.maximum(lens - 1, 0)
        ns = np.nonzero(lens > 0)[0]
        new_seq, new_pos = ns, lens[ns] - 1
    else:
        prefill = lens.copy()
        new_seq = new_pos = np.zeros(0, dtype=np.int64)
    b = _assemble(name, seed, dtype, hq, hkv, d, nb, lens, tables, tables, prefill,
                  new_seq, new_pos, [], device, {"blocks_in_use": bm.blocks_in_use()}, scale)
    if b.block_tables.shape[1] < width:
        bt = np.full((b.num_seqs, width), -1, dtype=np.int32)
        bt[:, :b.block_tables.shape[1]] = b.block_tables
        b.block_tables = bt
    return b


def c1_tiny_fp32(device="cpu") -> Batch:
    """4 seqs, lens {17,50,100,128}, 8 q heads = 8 kv heads, d64, fp32, 64-block pool whose
    blocks are handed out by a seeded permutation, scale 1/sqrt(64)."""
    return random_batch(CONFIG_SEEDS["c1_tiny_fp32"], [17, 50, 100, 128], 8, 8, 64, "f32",
                        num_blocks=64, device=device, scale=0.125, name="c1_tiny_fp32")


def c2_llama2_13b_mha(device="cpu", num_seqs: int = 64) -> Batch:
    """LLaMA-2-13B-shaped MHA decode: 40 heads, d128, lens uniform in [128, 2048], 20k pool."""
    seed = CONFIG_SEEDS["c2_llama2_13b_mha"]
    rng = np.random.default_rng(seed)
    lens = rng.integers(128, 2048, size=num_seqs, endpoint=True)
    return random_batch(seed, lens, 40, 40, 128, "bf16", num_blocks=20000, device=device,
                        name="c2_llama2_13b_mha")


def c3_lens(num_seqs: int = 256, seed: int | None = None) -> np.ndarray:
    rng = np.random.default_rng(CONFIG_SEEDS["c3_llama3_8b_gqa"] if seed is None else seed)
    raw = rng.lognormal(mean=math.log(1000.0), sigma=C3_LOGNORMAL_SIGMA, size=num_seqs)
    return np.clip(np.rint(raw), 16, 8192).astype(np.int64)


def c3_llama3_8b_gqa(device="cpu", num_seqs: int = 256) -> Batch:
    """Llama-3-8B-shaped GQA decode: 32 q / 8 kv heads, d128, lognormal lens (median 1000,
    sigma 0.75) clipped to [16, 8192]; the new token of each sequence (position L-1) is
    written by reshape_and_cache before attention."""
    seed = CONFIG_SEEDS["c3_llama3_8b_gqa"]
    lens = c3_lens(num_seqs)
    need = int(sum((int(L) + BLOCK_SIZE - 1) // BLOCK_SIZE for L in lens))
    nb = max(32768, int(math.ceil(1.25 * need)))
    b = random_batch(seed, lens, 32, 8, 128, "bf16", num_blocks=nb, device=device,
                     new_token=True, name="c3_llama3_8b_gqa")
    b.meta["lognormal_sigma"] = C3_LOGNORMAL_SIGMA
    return b


def c3_fp8(device="cpu", num_seqs: int = 256) -> Batch:
    """The Llama-3-8B-shaped GQA decode batch (same lengths and tables) over FP8 e4m3
    pools with one scale per pool; q and the new tokens' K/V are bf16."""
    seed = CONFIG_SEEDS["c3_llama3_8b_gqa"]
    lens = c3_lens(num_seqs)
    need = int(sum((int(L) + BLOCK_SIZE - 1) // BLOCK_SIZE for L in lens))
    nb = max(32768, int(math.ceil(1.25 * need)))
    b = random_batch(seed, lens, 32, 8, 128, "fp8", num_blocks=nb, device=device,
                     new_token=True, name="c3_fp8_llama3_8b_gqa")
    b.meta["lognormal_sigma"] = C3_LOGNORMAL_SIGMA
    return b


def c3_fp8e5m2(device="cpu", num_seqs: int = 256) -> Batch:
    """The Llama-3-8B-shaped GQA decode batch over FP8 e5m2 pools (one scale per pool)."""
    seed = CONFIG_SEEDS["c3_llama3_8b_gqa"]
    lens = c3_lens(num_seqs)
    need = int(sum((int(L) + BLOCK_SIZE - 1) // BLOCK_SIZE for L in lens))
    nb = max(32768, int(math.ceil(1.25 * need)))
    b = random_batch(seed, lens, 32, 8, 128, "fp8e5m2", num_blocks=nb, device=device,
                     new_token=True, name="c3_fp8e5m2_llama3_8b_gqa")
    b.meta["lognormal_sigma"] = C3_LOGNORMAL_SIGMA
    return b


def chunked_batch(seed: int, lens, chunks, hq: int, hkv: int, d: int, dtype: str = "bf16",
                  num_blocks: int | None = None, device="cpu", name: str = "chunked",
                  extra_table: int = 0) -> Batch:
    """Each sequence ends with a chunk of new tokens (chunks[s] of them, its last
    positions): their K/V are the new tokens to write before attention and each gets a
    query row; query_start_loc separates the chunks."""
    lens = np.asarray(lens, dtype=np.int64)
    chunks = np.asarray(chunks, dtype=np.int64)
    assert (chunks <= lens).all()
    rng = np.random.default_rng(seed)
    need = int(sum((int(L) + BLOCK_SIZE - 1) // BLOCK_SIZE for L in lens))
    nb = num_blocks if num_blocks is not None else max(need + 8, 16)
    bm = BlockManager(nb, rng)
    tables = [bm.allocate((int(L) + BLOCK_SIZE - 1) // BLOCK_SIZE) for L in lens]
    new_seq = np.concatenate([np.full(int(c), s) for s, c in enumerate(chunks)] + [np.zeros(0)])
    new_pos = np.concatenate([np.arange(int(L - c), int(L)) for L, c in zip(lens, chunks)]
                             + [np.zeros(0)])
    b = _assemble(name, seed, dtype, hq, hkv, d, nb, lens, tables, tables, lens - chunks,
                  new_seq.astype(np.int64), new_pos.astype(np.int64), [], device,
                  {"blocks_in_use": bm.blocks_in_use()})
    T = int(chunks.sum())
    gen = torch.Generator(device=device)
    gen.manual_seed(seed + 7919)
    b.q = _randn((T, hq, d), gen, device, dtype)
    b.query_start_loc = np.concatenate([[0], np.cumsum(chunks)]).astype(np.int32)
    width = max(b.block_tables.shape[1], 1) + extra_table
    if b.block_tables.shape[1] < width:
        bt = np.full((b.num_seqs, width), -1, dtype=np.int32)
        bt[:, :b.block_tables.shape[1]] = b.block_tables
        b.block_tables = bt
    return b


def c3_spec_decode(device="cpu", num_seqs: int = 256, draft: int = 4,
                   dtype: str = "bf16") -> Batch:
    """The Llama-3-8B-shaped GQA batch verifying `draft` speculative tokens per sequence:
    the draft tokens are the last positions of each context (lognormal lengths as in the
    decode batch, at least `draft`), written by reshape_and_cache, each with its query
    row, attending causally."""
    lens = np.maximum(c3_lens(num_seqs), draft)
    need = int(sum((int(L) + BLOCK_SIZE - 1) // BLOCK_SIZE for L in lens))
    b = chunked_batch(CONFIG_SEEDS["c3_llama3_8b_gqa"] + 100, lens, np.full(num_seqs, draft),
                      32, 8, 128, dtype, num_blocks=max(32768, int(math.ceil(1.25 * need))),
                      device=device, name="c3_spec_decode" if dtype == "bf16" else
                      f"c3_spec_decode_{dtype}")
    b.meta["draft_tokens"] = draft
    return b


def c3_spec_fp8(device="cpu", num_seqs: int = 256, draft: int = 4) -> Batch:
    """The speculative-verification batch over FP8 e4m3 pools (bf16 q and new K/V)."""
    return c3_spec_decode(device, num_seqs, draft, "fp8")


def c3_prefill(device="cpu", num_seqs: int = 16, chunk: int = 1024,
               max_cached: int = 3072) -> Batch:
    """A chunked-prefill step of the Llama-3-8B-shaped model (32 q / 8 kv heads, d128,
    bf16): each of `num_seqs` prompts processes its next `chunk` tokens over a cached
    prefix of U[0, max_cached] tokens (multiples of 16 tokens: earlier chunks filled
    whole blocks), so the chunk is the last `chunk` positions of a context of
    prefix + chunk tokens; the chunk's K/V are written by reshape_and_cache, then every
    chunk token attends causally."""
    seed = CONFIG_SEEDS["c3_llama3_8b_gqa"] + 200
    rng = np.random.default_rng(seed)
    cached = rng.integers(0, max_cached // BLOCK_SIZE, size=num_seqs, endpoint=True) * BLOCK_SIZE
    lens = cached + chunk
    need = int(sum((int(L) + BLOCK_SIZE - 1) // BLOCK_SIZE for L in lens))
    b = chunked_batch(seed, lens, np.full(num_seqs, chunk), 32, 8, 128, "bf16",
                      num_blocks=max(4096, int(math.ceil(1.25 * need))), device=device,
                      name="c3_prefill")
    b.meta["chunk"] = chunk
    return b


def c4_shared_prefix(device="cpu", prompts: int = 32, samples: int = 8, prefix: int = 1024,
                     max_tail: int = 512, num_blocks: int | None = None) -> Batch:
    """Parallel sampling with a shared prefix.

    Each prompt has ``prefix + r`` tokens (r uniform in [1, 15], so the last prefix block is
    shared and partially filled); its ``samples`` sequences share all prefix blocks with
    reference count ``samples``.  Each sample then appends a tail of U[0, max_tail] tokens:
    the first write into the shared partial block takes a private copy (copy-on-write, the
    copy done by copy_blocks) while the block is still shared; a sample with an empty tail
    writes nothing.  The tails are written by reshape_and_cache, then every sequence decodes
    with context = prefix + r + tail.
    """
    seed = CONFIG_SEEDS["c4_shared_prefix"]
    rng = np.random.default_rng(seed)
    r = rng.integers(1, 15, size=prompts, endpoint=True)
    tails = rng.integers(0, max_tail, size=(prompts, samples), endpoint=True)
    prefix_lens = prefix + r
    need = int(sum((int(p) + BLOCK_SIZE - 1) // BLOCK_SIZE for p in prefix_lens)) \
        + prompts * samples * (1 + (max_tail + BLOCK_SIZE - 1) // BLOCK_SIZE)
    nb = num_blocks if num_blocks is not None else max(32768, int(math.ceil(1.25 * need)))
    bm = BlockManager(nb, rng)
    tables, initial, prefill, lens = [], [], [], []
    seq_ids, positions = [], []
    for i in range(prompts):
        n_prefix_blocks = (int(prefix_lens[i]) + BLOCK_SIZE - 1) // BLOCK_SIZE
        base = bm.allocate(n_prefix_blocks)
        group = [base] + [bm.fork(base) for _ in range(samples - 1)]
        for j in range(samples):
            t = group[j]
            initial.append(list(t))
            P0 = int(prefix_lens[i])
            L = P0 + int(tails[i, j])
            for pos in range(P0, L):
                li = pos // BLOCK_SIZE
                if li < len(t):
                    bm.prepare_write(t, li)
                else:
                    t.extend(bm.allocate(1))
            s = len(tables)
            tables.append(t)
            prefill.append(P0)
            lens.append(L)
            seq_ids.extend([s] * (L - P0))
            positions.extend(range(P0, L))
    # the samples of prompt i are sequences i*samples .. (i+1)*samples - 1; all of them
    # keep the prompt's full blocks (the partial last one is copied on a sample's first write)
    meta = {"prompts": prompts, "samples": samples, "prefix_lens": prefix_lens.tolist(),
            "tails": tails.reshape(-1).tolist(), "blocks_in_use": bm.blocks_in_use(),
            "group_start": [i * samples for i in range(prompts + 1)],
            "shared_blocks": [int(p) // BLOCK_SIZE for p in prefix_lens]}
    return _assemble("c4_shared_prefix", seed, "bf16", 32, 8, 128, nb, np.array(lens),
                     tables, initial, np.array(prefill), np.array(seq_ids, dtype=np.int64),
                     np.array(positions, dtype=np.int64), bm.cow_pairs, device, meta)


def c5_long_splitk(device="cpu", num_seqs: int = 8) -> Batch:
    """Long-context GQA decode: 64 q / 8 kv heads, d128, lens uniform in [32768, 131072],
    blocks scattered over an 81,920-block pool (10,240 per sequence for other batch
    sizes); meant for 512-token split-K partitions."""
    seed = CONFIG_SEEDS["c5_long_splitk"]
    rng = np.random.default_rng(seed)
    lens = rng.integers(32768, 131072, size=num_seqs, endpoint=True)
    return random_batch(seed, lens, 64, 8, 128, "bf16", num_blocks=10240 * num_seqs,
                        device=device, name="c5_long_splitk")


CONFIGS["c3_prefill"] = ("chunked prefill, Llama-3-8B-shaped GQA bf16 (32q/8kv, d128): 16 prompts x "
                          "1024-token chunks over cached prefixes U[0, 3072] (causal)")
CONFIGS["c3_spec_decode"] = ("Llama-3-8B-shaped GQA bf16, batch 256, verifying 4 speculative tokens "
                              "per sequence (causal, 16 query rows per kv head)")
CONFIGS["c3_spec_fp8"] = ("the speculative-verification batch (256 x 4 draft tokens, causal) over FP8 "
                          "e4m3 pools, bf16 q/out")
CONFIGS["c3_fp8e5m2"] = ("Llama-3-8B-shaped GQA over FP8 e5m2 pools (one scale per pool), bf16 q/out: "
                         "batch 256, 32q/8kv, d128, the same lognormal lens")
CONFIGS["c3_fp8"] = ("Llama-3-8B-shaped GQA over FP8 e4m3 pools (one scale per pool), bf16 q/out: "
                     "batch 256, 32q/8kv, d128, the same lognormal lens, reshape_and_cache_fp8 "
                     "of the new token before attention")

BUILDERS = {
    "c1_tiny_fp32": c1_tiny_fp32,
    "c3_spec_decode": c3_spec_decode,
    "c3_prefill": c3_prefill,
    "c3_fp8": c3_fp8,
    "c3_spec_fp8": c3_spec_fp8,
    "c3_fp8e5m2": c3_fp8e5m2,
    "c2_llama2_13b_mha": c2_llama2_13b_mha,
    "c3_llama3_8b_gqa": c3_llama3_8b_gqa,
    "c4_shared_prefix": c4_shared_prefix,
    "c5_long_splitk": c5_long_splitk,
}


def private_copy(batch: Batch, device=None) -> Batch:
    """The same batch with every sequence holding private copies of all its blocks.

    Shared physical blocks are duplicated into fresh blocks appended to the pool, so each
    sequence reads the same values from blocks nobody else references.  Used to check that
    sharing a prefix changes nothing in the result.
    """
    device = device or batch.k_cache.device
    owners: dict[int, int] = {}
    tables = batch.block_tables.copy()
    extra_src = []
    nb = batch.num_blocks
    for s in range(batch.num_seqs):
        L = int(batch.context_lens[s])
        for i in range((L + BLOCK_SIZE - 1) // BLOCK_SIZE):
            b = int(tables[s, i])
            if b in owners and owners[b] != s:
                tables[s, i] = nb + len(extra_src)
                extra_src.append(b)
            else:
                owners[b] = s
    idx = torch.tensor(extra_src, dtype=torch.long, device=batch.k_cache.device)
    k = torch.cat([batch.k_cache, batch.k_cache.index_select(0, idx)]) if extra_src else batch.k_cache.clone()
    v = torch.cat([batch.v_cache, batch.v_cache.index_select(0, idx)]) if extra_src else batch.v_cache.clone()
    out = Batch(batch.name + "_private", batch.seed, batch.dtype, batch.num_q_heads,
                batch.num_kv_heads, batch.head_dim, nb + len(extra_src), batch.context_lens.copy(),
                tables, batch.scale, batch.q, k.to(device), v.to(device), batch.new_k, batch.new_v,
                batch.new_seq.copy(), batch.new_pos.copy(), np.zeros((0, 2), dtype=np.int64),
                dict(batch.meta))
    return out


def permute_placement(batch: Batch, seed: int) -> Batch:
    """The same batch with every physical block moved to a new random place (data moves too)."""
    rng = np.random.default_rng(seed)
    perm = rng.permutation(batch.num_blocks)          # old block b goes to perm[b]
    inv = np.argsort(perm)                            # new block n holds old block inv[n]
    idx = torch.from_numpy(inv).to(batch.k_cache.device)
    tables = batch.block_tables.copy()
    valid = tables >= 0
    tables[valid] = perm[tables[valid]]
    pairs = batch.cow_pairs.copy()
    if pairs.size:
        pairs = perm[pairs]
    return Batch(batch.name + "_permuted", batch.seed, batch.dtype, batch.num_q_heads,
                 batch.num_kv_heads, batch.head_dim, batch.num_blocks, batch.context_lens.copy(),
                 tables.astype(np.int32), batch.scale, batch.q,
                 batch.k_cache.index_select(0, idx), batch.v_cache.index_select(0, idx),
                 batch.new_k, batch.new_v, batch.new_seq.copy(), batch.new_pos.copy(),
                 pairs.astype(np.int64), dict(batch.meta))
