// pkv_decode.cuh -- paged decode attention for sm_100a.
//
// What is computed (ipipp.com vLLM article, section
// "二、PagedAttention分页原理深度剖析"): for every sequence and query head,
// softmax(scale * q . K^T) V over the sequence's context, where the context is
// stored in 16-token blocks scattered over one pool and found block by block
// through the sequence's block table.
//
// How it runs on a B200:
//  * A planning step turns context_lens into a work list of items
//    (sequence, partition), longest first.  A partition is at most
//    `part_blocks` blocks; a sequence longer than one partition is split
//    (split-K) and its partial results are merged by log-sum-exp afterwards.
//    A second planner serves batches whose consecutive sequences share their
//    leading blocks: a shared-prefix item reads those blocks once for one
//    query token of each of several sequences, and their partial results
//    are merged with those of each sequence's own blocks.
//  * The decode kernel is persistent (one CTA per SM).  Work units (item x kv
//    head x row group) are handed out through an atomic counter by a
//    scheduler warp, which publishes each into a ring in shared memory: its
//    metadata, its q rows (bulk copies) and its slice of the block table.
//  * The decode warps take the blocks of an item round-robin.  Each warp (or
//    the lead warp of a pair) owns a few tile stages and issues its own TMA
//    tensor loads -- one per 128-byte column chunk of the 16-token K and V
//    tiles, contiguous per (block, kv head) in the HND pool -- into
//    128B-swizzled shared memory, running ahead across item boundaries.  At
//    the end of an item the warps merge their online-softmax states.
//  * bf16 and FP8: per pair of 16-token tiles, S^T = K Q^T on mma.sync
//    (tile tokens = M, the item's query rows = N, up to 16), online softmax in
//    log2 units with a lazily moved maximum, P^T through movmatrix, O^T +=
//    V^T P^T, and the row sums by one more MMA.  Every KV tile is read from
//    HBM once per GQA group.  FP8 codes are widened to f16 in registers.
//  * fp32: the same pipeline with a CUDA-core consumer (fp32 has no exact
//    tensor-core path; TF32 would break the fp32 tolerance).
//  * Padding slots of the last block are never used: their scores are set
//    to -inf and their V values are masked to zero before the MMA
//    (0 * NaN would otherwise poison the output).
#pragma once

#include <type_traits>

#include "pkv_device.cuh"

namespace pkv {

constexpr int kRing = 4;          // items in flight between producer and consumers
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

// One unit of planned work.  An ordinary item covers blocks blk0 .. of
// sequence `seq` (at most part_blocks of them) for that sequence's own query
// rows.  A shared-prefix item (q_start >= 0) covers blocks blk0 .. of a
// prefix that the q_len consecutive sequences q_start .. q_start + q_len - 1
// share, read through the table of `seq` (the first of them), for one query
// token of each of those sequences at once.
struct PlanItem {
  int32_t seq;      // sequence whose block table is read
  int32_t part;     // partial-result slot of the rows (used when nparts > 1)
  int32_t len;      // keys at positions < len belong to the item's context
  int32_t nparts;   // 1: the item is its rows' whole context (output written directly)
  int32_t blk0;     // first block
  int32_t q_start;  // shared-prefix items: first query row; -1: the rows of `seq`
  int32_t q_len;    // shared-prefix items: sequences served
  int32_t pad;
};

// Context length after validation against the table width and the host's
// max_context_len hint; out-of-range values are clamped and flagged.
__device__ __forceinline__ int32_t checked_len(int32_t L, int32_t max_len) {
  if (L < 0 || L > max_len) {
    raise_error(PKV_DEVERR_LEN);
    L = L < 0 ? 0 : max_len;
  }
  return L;
}

__device__ __forceinline__ int32_t num_parts(int32_t L, int32_t part_tokens) {
  int32_t n = (L + part_tokens - 1) / part_tokens;
  return n < 1 ? 1 : n;
}

// ----------------------------------------------------------------- planning
constexpr int kPlanThreads = 1024;
constexpr int kPlanBuckets = 1024;  // item sizes in blocks; larger sizes share the top bucket

__device__ __forceinline__ int plan_bucket(int32_t blocks) {
  return blocks < kPlanBuckets - 1 ? blocks : kPlanBuckets - 1;
}

__device__ __forceinline__ int32_t part_size_blocks(int32_t L, int32_t p, int32_t part_blocks) {
  int32_t total = (L + kBlock - 1) / kBlock;
  int32_t rest = total - p * part_blocks;
  return rest < part_blocks ? rest : part_blocks;
}

// Exclusive scan of the item-size histogram in descending bucket order (one
// CTA of kPlanThreads threads, thread i owning bucket kPlanBuckets-1-i):
// afterwards hist[b] is the position of bucket b's first item.  Also sets
// counters[1] = number of items and zeroes the work and finish counters.
__device__ __forceinline__ void plan_scan(uint32_t* hist, uint32_t* warp_sums,
                                          uint32_t* __restrict__ counters) {
  const int tid = threadIdx.x;
  const int bucket = kPlanBuckets - 1 - tid;
  uint32_t v = hist[bucket];
  uint32_t incl = v;
  const int lane = tid & 31, warp = tid >> 5;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    uint32_t n = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += n;
  }
  if (lane == 31) warp_sums[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    uint32_t w = warp_sums[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      uint32_t n = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += n;
    }
    warp_sums[lane] = w;  // inclusive over warps
  }
  __syncthreads();
  const uint32_t base = (warp > 0 ? warp_sums[warp - 1] : 0u) + incl - v;
  __syncthreads();
  hist[bucket] = base;  // becomes the write cursor of the bucket
  if (tid == kPlanThreads - 1) {
    counters[1] = warp_sums[kPlanThreads / 32 - 1];
    counters[0] = 0u;
    counters[2] = 0u;
  }
  __syncthreads();
}

// The plan, run by one CTA of kPlanThreads threads: counts the work items per
// size, scans, and writes them sorted by size (largest first).  counters[0] =
// work counter, counters[1] = items, counters[2] = CTAs finished; the work and
// finish counters are zeroed here, and the decode kernel's last CTA zeroes
// them again, so one plan serves any number of runs.  The caller has already
// passed griddepcontrol.wait.
__device__ __forceinline__ void plan_body(const int32_t* __restrict__ context_lens,
                                          int32_t num_seqs, int32_t max_len, int32_t part_blocks,
                                          PlanItem* __restrict__ items,
                                          uint32_t* __restrict__ counters, uint32_t* hist,
                                          uint32_t* warp_sums) {
  const int tid = threadIdx.x;
  const int32_t part_tokens = part_blocks * kBlock;
  for (int b = tid; b < kPlanBuckets; b += kPlanThreads) hist[b] = 0;
  __syncthreads();
  for (int32_t s = tid; s < num_seqs; s += kPlanThreads) {
    int32_t L = checked_len(context_lens[s], max_len);
    int32_t n = num_parts(L, part_tokens);
    for (int32_t p = 0; p < n; ++p) atomicAdd(&hist[plan_bucket(part_size_blocks(L, p, part_blocks))], 1u);
  }
  __syncthreads();
  plan_scan(hist, warp_sums, counters);
  for (int32_t s = tid; s < num_seqs; s += kPlanThreads) {
    int32_t L = context_lens[s];
    L = L < 0 ? 0 : (L > max_len ? max_len : L);
    int32_t n = num_parts(L, part_tokens);
    for (int32_t p = 0; p < n; ++p) {
      uint32_t pos = atomicAdd(&hist[plan_bucket(part_size_blocks(L, p, part_blocks))], 1u);
      items[pos] = PlanItem{s, p, L, n, p * part_blocks, -1, 0, 0};
    }
  }
}

// Single CTA: the plan alone.
__global__ void __launch_bounds__(kPlanThreads)
    plan_kernel(const int32_t* __restrict__ context_lens, int32_t num_seqs, int32_t max_len,
                int32_t part_blocks, PlanItem* __restrict__ items,
                uint32_t* __restrict__ counters) {
  __shared__ uint32_t hist[kPlanBuckets];
  __shared__ uint32_t warp_sums[kPlanThreads / 32];
  pdl_wait();
  pdl_trigger();
  plan_body(context_lens, num_seqs, max_len, part_blocks, items, counters, hist, warp_sums);
}

// ------------------------------------------------------- shared-prefix plan
// Parallel samples of one prompt (or requests behind one system prompt) hold
// the same physical blocks at the start of their tables: the pages' prefix
// sharing with reference counts ("vLLM 深读：用 PagedAttention 撑起高并发 LLM
// 推理", section "先看浪费在哪里").  This plan reads such a prefix once per kv
// head for a whole group of sequences: a shared-prefix item multiplies its
// tiles against one query token of each of up to `members_per_item`
// sequences, and each sequence's own blocks after the prefix become ordinary
// items; the two partial results meet in the log-sum-exp merge.
//
// Group i covers sequences group_start[i] .. group_start[i+1] - 1 (bounds
// nondecreasing within [0, num_seqs]; a sequence in no group has no shared
// prefix).  Every member's first shared_blocks[i] blocks are read through the
// FIRST member's table.  A group of fewer than two members, or bounds that
// are not nondecreasing in [0, num_seqs] (flagged PKV_DEVERR_GROUP, then no
// group is used), give no shared prefix; a negative count, or one beyond a
// member's full blocks, is raised to 0 or lowered to them and flagged
// PKV_DEVERR_GROUP.
//
// Outputs besides the work list: seq_prefix[s] = shared blocks of sequence s
// (what the merge needs to count its partials), group_pref[i] scratch.  The
// partials of a sequence with P shared blocks are slots 0 .. np(P*16) - 1
// for the prefix and np(P*16) .. for its own tokens, np = num_parts.

// The group holding sequence s (groups 0 .. G-1 with nondecreasing bounds), or -1.
constexpr int kPlanGroupCache = 2048;

__device__ __forceinline__ int32_t group_of(const int32_t* group_start, int32_t G, int32_t s) {
  if (G <= 0 || s < group_start[0] || s >= group_start[G]) return -1;
  int32_t lo = 0, hi = G - 1;
  while (lo < hi) {
    const int32_t mid = (lo + hi + 1) / 2;
    if (group_start[mid] <= s) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// The shared-prefix plan, run by one CTA of kPlanThreads threads (the caller
// has passed griddepcontrol.wait); gs_cache holds kPlanGroupCache ints of
// shared memory.
__device__ __forceinline__ void plan_shared_body(
    const int32_t* __restrict__ context_lens, const int32_t* __restrict__ group_start,
    const int32_t* __restrict__ shared_blocks, int32_t num_groups, int32_t num_seqs,
    int32_t max_len, int32_t part_blocks, int32_t members_per_item, PlanItem* __restrict__ items,
    uint32_t* __restrict__ counters, int32_t* __restrict__ seq_prefix, int32_t* group_pref,
    uint32_t* hist, uint32_t* warp_sums, int32_t* gs_cache) {
  const int tid = threadIdx.x;
  const int32_t part_tokens = part_blocks * kBlock;
  for (int b = tid; b < kPlanBuckets; b += kPlanThreads) hist[b] = 0;
  // the group bounds (kept in shared memory for the searches below if they fit)
  const bool cached = num_groups < kPlanGroupCache;
  int bad = 0;
  for (int32_t i = tid; i <= num_groups; i += kPlanThreads) {
    const int32_t a = group_start[i];
    if (a < 0 || a > num_seqs || (i < num_groups && a > group_start[i + 1])) bad = 1;
    if (cached) gs_cache[i] = a;
  }
  const bool groups_ok = __syncthreads_or(bad) == 0;
  if (!groups_ok && tid == 0) raise_error(PKV_DEVERR_GROUP);
  const int32_t G = groups_ok ? num_groups : 0;
  const int32_t* gsp = cached ? gs_cache : group_start;
  // each group's prefix as given, within the table width; none (and no check)
  // for a group of fewer than two members
  for (int32_t i = tid; i < G; i += kPlanThreads) {
    int32_t p = 0;
    if (gsp[i + 1] - gsp[i] >= 2) {
      p = shared_blocks[i];
      const int32_t cap = max_len / kBlock;
      if (p < 0 || p > cap) {
        raise_error(PKV_DEVERR_GROUP);
        p = p < 0 ? 0 : cap;
      }
    }
    group_pref[i] = p;
  }
  __syncthreads();
  // ... and never past a member's own full blocks
  for (int32_t s = tid; s < num_seqs; s += kPlanThreads) {
    const int32_t gi = group_of(gsp, G, s);
    if (gi < 0) continue;
    const int32_t full = checked_len(context_lens[s], max_len) / kBlock;
    if (full < group_pref[gi]) {
      raise_error(PKV_DEVERR_GROUP);
      atomicMin(&group_pref[gi], full);
    }
  }
  __syncthreads();
  // sizes: each sequence's own partitions, each group's prefix partitions
  // (one item per members_per_item sequences)
  for (int32_t s = tid; s < num_seqs; s += kPlanThreads) {
    const int32_t gi = group_of(gsp, G, s);
    const int32_t pref = gi >= 0 ? group_pref[gi] : 0;
    seq_prefix[s] = pref;
    const int32_t tail = checked_len(context_lens[s], max_len) - pref * kBlock;
    const int32_t n = num_parts(tail, part_tokens);
    for (int32_t p = 0; p < n; ++p)
      atomicAdd(&hist[plan_bucket(part_size_blocks(tail, p, part_blocks))], 1u);
  }
  for (int32_t i = tid; i < G; i += kPlanThreads) {
    const int32_t pref = group_pref[i];
    if (pref == 0) continue;
    const int32_t members = gsp[i + 1] - gsp[i];
    const uint32_t per = static_cast<uint32_t>((members + members_per_item - 1) / members_per_item);
    const int32_t n = num_parts(pref * kBlock, part_tokens);
    for (int32_t p = 0; p < n; ++p)
      atomicAdd(&hist[plan_bucket(part_size_blocks(pref * kBlock, p, part_blocks))], per);
  }
  __syncthreads();
  plan_scan(hist, warp_sums, counters);
  for (int32_t s = tid; s < num_seqs; s += kPlanThreads) {
    const int32_t pref = seq_prefix[s];
    int32_t L = context_lens[s];
    L = L < 0 ? 0 : (L > max_len ? max_len : L);
    const int32_t tail = L - pref * kBlock;
    const int32_t np = pref > 0 ? num_parts(pref * kBlock, part_tokens) : 0;
    const int32_t n = num_parts(tail, part_tokens);
    for (int32_t p = 0; p < n; ++p) {
      const uint32_t pos = atomicAdd(&hist[plan_bucket(part_size_blocks(tail, p, part_blocks))], 1u);
      items[pos] = PlanItem{s, np + p, L, np + n, pref + p * part_blocks, -1, 0, 0};
    }
  }
  for (int32_t i = tid; i < G; i += kPlanThreads) {
    const int32_t pref = group_pref[i];
    if (pref == 0) continue;
    const int32_t first = gsp[i], members = gsp[i + 1] - first;
    const int32_t per = (members + members_per_item - 1) / members_per_item;
    const int32_t n = num_parts(pref * kBlock, part_tokens);
    for (int32_t p = 0; p < n; ++p) {
      // the items of one partition sit next to each other: their tiles are
      // read close in time and mostly served once from HBM
      const uint32_t pos = atomicAdd(
          &hist[plan_bucket(part_size_blocks(pref * kBlock, p, part_blocks))], static_cast<uint32_t>(per));
      for (int32_t j = 0; j < per; ++j) {
        const int32_t q0 = first + j * members_per_item;
        const int32_t qn = members - j * members_per_item < members_per_item
                               ? members - j * members_per_item
                               : members_per_item;
        items[pos + j] = PlanItem{first, p, pref * kBlock, 2, p * part_blocks, q0, qn, 0};
      }
    }
  }
}

__global__ void __launch_bounds__(kPlanThreads)
    plan_shared_kernel(const int32_t* __restrict__ context_lens,
                       const int32_t* __restrict__ group_start,
                       const int32_t* __restrict__ shared_blocks, int32_t num_groups,
                       int32_t num_seqs, int32_t max_len, int32_t part_blocks,
                       int32_t members_per_item, PlanItem* __restrict__ items,
                       uint32_t* __restrict__ counters, int32_t* __restrict__ seq_prefix,
                       int32_t* group_pref) {
  __shared__ uint32_t hist[kPlanBuckets];
  __shared__ uint32_t warp_sums[kPlanThreads / 32];
  __shared__ int32_t gs_cache[kPlanGroupCache];  // the group bounds, when they fit
  pdl_wait();
  pdl_trigger();
  plan_shared_body(context_lens, group_start, shared_blocks, num_groups, num_seqs, max_len,
                   part_blocks, members_per_item, items, counters, seq_prefix, group_pref, hist,
                   warp_sums, gs_cache);
}

// ------------------------------------------------------------ decode kernel
struct DecodeParams {
  void* out;                     // [T][Hq][D], dtype of the cache (T query tokens)
  const void* q;                 // [T][Hq][D]
  const int32_t* block_tables;   // [B][MB]
  const PlanItem* items;         // planned work, longest first
  uint32_t* counters;            // [0] work counter, [1] number of items, [2] CTAs done
  float* part_o;                 // [T][Hq][max_parts][D]
  float* part_ml;                // [T][Hq][max_parts][2]
  // Query tokens of sequence s: rows query_start_loc[s] .. query_start_loc[s+1]-1
  // at positions L-n .. L-1 (causal); NULL means one token per sequence, row s.
  const int32_t* query_start_loc;
  int32_t max_query_len;         // longest chunk (tokens); longer chunks are flagged
  int32_t group_tokens;          // chunk tokens per item (row group): group_tokens x group <= GMAX
  int32_t row_groups;            // items per (sequence, partition, kv head)
  int32_t num_q_tokens;          // rows of q and out
  int32_t num_q_heads;
  int32_t num_kv_heads;
  int32_t group;                 // Hq / Hkv
  int32_t max_blocks_per_seq;
  int32_t num_blocks;
  int32_t max_parts;
  int32_t part_blocks;
  float qk_scale_log2;           // scale * log2(e) (times the K scale for FP8 caches)
  float out_scale;               // 1, or the V scale for FP8 caches
};

// Tag type of an FP8 (e4m3) cache: one-byte codes, bf16 q and out.
struct Fp8Kv {};
// Tag type of an FP8 (e5m2) cache.
struct Fp8E5m2Kv {};

// Bytes per q / out element for a cache element type.
template <typename T>
constexpr int q_elem_bytes() {
  return sizeof(T) == 4 ? 4 : 2;
}

// Largest partition (in blocks) the decode kernel handles; the block-table
// slice of every item in flight is staged in shared memory.
constexpr int kMaxItemBlocks = 512;

// Shared-memory map of the decode kernel (offsets from a 1024-aligned base).
// MB merge buffers: with two, consecutive items alternate buffers and one
// barrier per item suffices; with one (when two do not fit), a second
// barrier keeps the next item's states out until the current one is combined.
// SPLIT warps share one set of tile stages, each taking GMAX / SPLIT of an
// item's query rows; W / SPLIT "lead" warps own the stages and issue the loads.
template <int ELEM, int D, int GMAX, int W, int S, int MB = 2, int QELEM = ELEM, int SPLIT = 1>
struct DecodeLayout {
  static constexpr int kLead = W / SPLIT;                     // warps owning stages
  static constexpr int kRowsPerWarp = GMAX / SPLIT;           // query rows one warp holds
  static constexpr int kTileBytes = kBlock * D * ELEM;       // one K (or V) tile
  static constexpr int kChunks = D * ELEM / 128;             // 128-byte column chunks
  static constexpr int kStageBytes = 2 * kTileBytes;
  static constexpr int kQBytes = ((GMAX * D * QELEM) + 127) / 128 * 128;
  static constexpr int kStagesOff = 0;
  static constexpr int kRingOff = kStagesOff + kLead * S * kStageBytes;
  static constexpr int kTablesOff = kRingOff + kRing * kQBytes;
  static constexpr int kMergeOff = kTablesOff + kRing * kMaxItemBlocks * 4;
  // Rows of a warp's merge slot when the largest item has rows_max rows.
  __host__ __device__ static int slot_rows(int rows_max) {
    return rows_max < kRowsPerWarp ? rows_max : kRowsPerWarp;
  }
  // merge area: MB buffers x W warps x (r*D + 2r rounded up to 4) floats for
  // r slot rows; every warp's slot starts 16-byte aligned.
  __host__ __device__ static int merge_floats_per_warp(int r) { return r * D + (2 * r + 3) / 4 * 4; }
  __host__ __device__ static int meta_off(int rows_max) {
    return kMergeOff + MB * W * merge_floats_per_warp(slot_rows(rows_max)) * 4;
  }
  static constexpr int kMetaBytes = kRing * 64;
  __host__ __device__ static int bars_off(int rows_max) {
    return (meta_off(rows_max) + kMetaBytes + 7) / 8 * 8;
  }
  // full[kLead][S], empty[kLead][S], item_full[kRing], item_empty[kRing], merge[2]
  static constexpr int kNumBars = 2 * kLead * S + 2 * kRing + 2;
  __host__ __device__ static int flags_off(int rows_max) { return bars_off(rows_max) + kNumBars * 8; }
  __host__ __device__ static int total_bytes(int rows_max) {
    return flags_off(rows_max) + (kLead * S + 4) * 4 + 1024;  // + slack for 1024-byte alignment
  }
};

struct ItemMeta {
  int32_t seq, kv_head, part, len, nparts, blk_begin, nblk;
  int32_t q_start, q_len;        // query rows of the chunk and its length
  // rows of token i see keys up to len - q_causal + i: q_causal = q_len for a
  // causal chunk, 1 for a shared prefix (every row sees every key of it)
  int32_t q_causal;
};
static_assert(sizeof(ItemMeta) <= 64, "a ring slot's metadata area is 64 bytes");

// ---- consumer state for bf16 (tensor cores) ----
//
// Per 16-token tile the scores are computed transposed, S^T = K Q^T, with the
// tile's tokens as the MMA's M (16) and the item's query rows (the GQA group's
// heads, times the chunk's tokens) as N (8 per n-tile), so one m16n8k16 covers
// a k-step of all of them.  The output is kept transposed too, O^T += V^T P^T
// (M = head_dim in tiles of 16, N = the rows, K = the tile's tokens); P^T reaches the B-fragment layout through
// movmatrix.  Two tiles are processed per step for instruction-level
// parallelism.  The running max only moves when it grows by more than
// kRescaleSlack (log2 units): weights then stay below 2^kRescaleSlack and the
// accumulators are rescaled rarely (a warp vote decides).
constexpr float kRescaleSlack = 8.f;

template <int D, int GMAX>
struct Bf16State {
  static constexpr int KS = D / 16;    // k-steps of S^T = K Q^T
  static constexpr int MT = D / 16;    // m-tiles of O^T
  static constexpr int NH = GMAX / 8;  // n-tiles of query heads
  uint32_t qb[NH][KS][2];              // B fragments of Q^T
  float o[NH][MT][4];                  // O^T accumulators
  float m[NH][2];                      // running max of rows 8nh + 2(lane%4) + {0,1}
  float lsum[NH][4];                   // softmax denominators, summed by a tensor-core MMA
  int32_t lim[NH][2];                  // last key position those rows may see (causal)
  int32_t lim_min;                     // smallest limit over the item's rows
};

// Query rows of an item: row n = i*g + h is chunk token i (at position
// len - q_len + i) and query head h of the group; `rows` = q_len * g.
// A warp holding rows row0 .. row0 + rows - 1 of the item gets qs pointing at
// row row0.
template <int D, int GMAX>
__device__ __forceinline__ void bf16_begin_item(Bf16State<D, GMAX>& st, const uint8_t* qs,
                                                int rows, int g, int len, int q_len, int lane,
                                                int row0 = 0) {
  using St = Bf16State<D, GMAX>;
  const int r = lane >> 2, qd = (lane & 3) * 2;
  const uint16_t* q16 = reinterpret_cast<const uint16_t*>(qs);
#pragma unroll
  for (int nh = 0; nh < St::NH; ++nh) {
    const int head = nh * 8 + r;
#pragma unroll
    for (int ks = 0; ks < St::KS; ++ks) {
      const int c = ks * 16 + qd;
      st.qb[nh][ks][0] = head < rows ? *reinterpret_cast<const uint32_t*>(q16 + head * D + c) : 0u;
      st.qb[nh][ks][1] = head < rows ? *reinterpret_cast<const uint32_t*>(q16 + head * D + c + 8) : 0u;
    }
#pragma unroll
    for (int hc = 0; hc < 2; ++hc) {
      const int n = nh * 8 + qd + hc;
      st.lim[nh][hc] = n < rows ? len - q_len + (row0 + n) / g : -1;
    }
#pragma unroll
    for (int mt = 0; mt < St::MT; ++mt) {
      st.o[nh][mt][0] = st.o[nh][mt][1] = st.o[nh][mt][2] = st.o[nh][mt][3] = 0.f;
    }
    st.m[nh][0] = st.m[nh][1] = -INFINITY;
    st.lsum[nh][0] = st.lsum[nh][1] = st.lsum[nh][2] = st.lsum[nh][3] = 0.f;
  }
  st.lim_min = len - q_len + row0 / g;
}

// Two 16-token tiles (the second may be absent: valid1 = 0 and its pointers
// equal the first's).  validX tokens of tile X belong to the context; its
// first token sits at position posX.
template <int D, int GMAX>
__device__ __forceinline__ void bf16_step(Bf16State<D, GMAX>& st, const uint8_t* k0,
                                          const uint8_t* v0, int valid0, int pos0,
                                          const uint8_t* k1, const uint8_t* v1, int valid1,
                                          int pos1, float sc, int lane) {
  using St = Bf16State<D, GMAX>;
  constexpr int NH = St::NH;
  const int r = lane >> 2, qd = (lane & 3) * 2;
  // ---- S^T = K Q^T for both tiles (two accumulation chains each) ----
  float s[2][2][NH][4];
#pragma unroll
  for (int t = 0; t < 2; ++t)
#pragma unroll
    for (int c = 0; c < 2; ++c)
#pragma unroll
      for (int nh = 0; nh < NH; ++nh) s[t][c][nh][0] = s[t][c][nh][1] = s[t][c][nh][2] = s[t][c][nh][3] = 0.f;
  {
    // ldmatrix.x4 rows: lanes 0-7 tokens 0-7 / low 8 columns, 8-15 tokens 8-15 / low,
    // 16-23 tokens 0-7 / high, 24-31 tokens 8-15 / high -> A fragments a0..a3.
    const uint32_t tok = ((lane >> 3) & 1) * 8 + (lane & 7);
    const uint32_t gsel = lane >> 4;
    const uint32_t base0 = smem_addr(k0) + tok * 128u, base1 = smem_addr(k1) + tok * 128u;
#pragma unroll
    for (int ks = 0; ks < St::KS; ++ks) {
      const uint32_t off = (ks >> 2) * (kBlock * 128u) + (((((ks & 3) * 2) + gsel) ^ (tok & 7u)) << 4);
      uint32_t a[4], b[4];
      ldmatrix_x4(base0 + off, a[0], a[1], a[2], a[3]);
      ldmatrix_x4(base1 + off, b[0], b[1], b[2], b[3]);
#pragma unroll
      for (int nh = 0; nh < NH; ++nh) {
        mma_bf16_16816(s[0][ks & 1][nh], a, st.qb[nh][ks][0], st.qb[nh][ks][1]);
        mma_bf16_16816(s[1][ks & 1][nh], b, st.qb[nh][ks][0], st.qb[nh][ks][1]);
      }
    }
  }
  // ---- mask (raw scores; element i of a C fragment is token r + 8(i>>1), head 2q + (i&1)).
  // Tiles that are full and wholly inside every row's causal window need no mask.
  float z[2][NH][4];
#pragma unroll
  for (int t = 0; t < 2; ++t)
#pragma unroll
    for (int nh = 0; nh < NH; ++nh)
#pragma unroll
      for (int i = 0; i < 4; ++i) z[t][nh][i] = s[t][0][nh][i] + s[t][1][nh][i];
  if (!(valid0 == kBlock && valid1 == kBlock && pos1 + kBlock - 1 <= st.lim_min)) {
#pragma unroll
    for (int t = 0; t < 2; ++t) {
      const int valid = t ? valid1 : valid0;
      const int pos = t ? pos1 : pos0;
#pragma unroll
      for (int nh = 0; nh < NH; ++nh)
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int tok = r + 8 * (i >> 1);
          if (!(tok < valid && pos + tok <= st.lim[nh][i & 1])) z[t][nh][i] = -INFINITY;
        }
    }
  }
  // ---- running max per head column (scaled by sc > 0 after the reduction), lazy rescale ----
  bool grow = false;
  float m_new[NH][2];
#pragma unroll
  for (int nh = 0; nh < NH; ++nh)
#pragma unroll
    for (int hc = 0; hc < 2; ++hc) {
      float mx = fmaxf(fmaxf(z[0][nh][hc], z[0][nh][hc + 2]), fmaxf(z[1][nh][hc], z[1][nh][hc + 2]));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
      m_new[nh][hc] = mx * sc;
      grow |= m_new[nh][hc] > st.m[nh][hc] + kRescaleSlack;
    }
  if (__any_sync(0xffffffffu, grow)) {
#pragma unroll
    for (int nh = 0; nh < NH; ++nh)
#pragma unroll
      for (int hc = 0; hc < 2; ++hc) {
        const bool up = m_new[nh][hc] > st.m[nh][hc] + kRescaleSlack;
        const float alpha = up ? fast_exp2(st.m[nh][hc] - m_new[nh][hc]) : 1.f;  // 0 from -inf
        st.m[nh][hc] = up ? m_new[nh][hc] : st.m[nh][hc];
        st.lsum[nh][hc] *= alpha;
        st.lsum[nh][hc + 2] *= alpha;
#pragma unroll
        for (int mt = 0; mt < St::MT; ++mt) {
          st.o[nh][mt][hc] *= alpha;
          st.o[nh][mt][hc + 2] *= alpha;
        }
      }
  }
  // ---- P = exp2(z sc - m) in bf16, transposed into B fragments; l += ones . P^T ----
  constexpr uint32_t kOnes = 0x3f803f80u;  // bf16x2 (1, 1)
  const uint32_t ones[4] = {kOnes, kOnes, kOnes, kOnes};
  uint32_t pb[2][NH][2];
#pragma unroll
  for (int nh = 0; nh < NH; ++nh) {
    const float mu0 = st.m[nh][0] == -INFINITY ? 0.f : st.m[nh][0];
    const float mu1 = st.m[nh][1] == -INFINITY ? 0.f : st.m[nh][1];
#pragma unroll
    for (int t = 0; t < 2; ++t) {
      const uint32_t lo = pack_bf16x2(fast_exp2(fmaf(z[t][nh][0], sc, -mu0)),
                                      fast_exp2(fmaf(z[t][nh][1], sc, -mu1)));
      const uint32_t hi = pack_bf16x2(fast_exp2(fmaf(z[t][nh][2], sc, -mu0)),
                                      fast_exp2(fmaf(z[t][nh][3], sc, -mu1)));
      pb[t][nh][0] = movmatrix_trans(lo);
      pb[t][nh][1] = movmatrix_trans(hi);
      mma_bf16_16816(st.lsum[nh], ones, pb[t][nh][0], pb[t][nh][1]);
    }
  }
  // ---- O^T += V^T P^T ----
  {
    // ldmatrix.x4.trans rows: lanes 0-7 tokens 0-7 / low 8 d, 8-15 tokens 0-7 / high,
    // 16-23 tokens 8-15 / low, 24-31 tokens 8-15 / high -> A fragments a0..a3 of V^T.
    const uint32_t tok = (lane >> 4) * 8 + (lane & 7);
    const uint32_t gsel = (lane >> 3) & 1;
#pragma unroll
    for (int t = 0; t < 2; ++t) {
      const int valid = t ? valid1 : valid0;
      const uint32_t base = smem_addr(t ? v1 : v0) + tok * 128u;
      uint32_t mk0 = 0xffffffffu, mk1 = 0xffffffffu;
      const bool partial = valid < kBlock;
      if (partial) {
        mk0 = (qd < valid ? 0x0000ffffu : 0u) | (qd + 1 < valid ? 0xffff0000u : 0u);
        mk1 = (qd + 8 < valid ? 0x0000ffffu : 0u) | (qd + 9 < valid ? 0xffff0000u : 0u);
      }
#pragma unroll
      for (int mt = 0; mt < St::MT; ++mt) {
        const uint32_t off = (mt >> 2) * (kBlock * 128u) + (((((mt & 3) * 2) + gsel) ^ (tok & 7u)) << 4);
        uint32_t a[4];
        ldmatrix_x4_trans(base + off, a[0], a[1], a[2], a[3]);
        if (partial) {
          a[0] &= mk0;
          a[1] &= mk0;
          a[2] &= mk1;
          a[3] &= mk1;
        }
#pragma unroll
        for (int nh = 0; nh < NH; ++nh) mma_bf16_16816(st.o[nh][mt], a, pb[t][nh][0], pb[t][nh][1]);
      }
    }
  }
}

// Write this warp's (m, l, O) rows into its slot of the merge area.
template <int D, int GMAX>
__device__ __forceinline__ void bf16_publish(Bf16State<D, GMAX>& st, float* slot, int rows,
                                             int lane) {
  const int g = rows;  // the slot holds `rows` rows
  using St = Bf16State<D, GMAX>;
  const int r = lane >> 2, qd = (lane & 3) * 2;
  float* O = slot;
  float* M = slot + g * D;
  float* L = M + g;
#pragma unroll
  for (int nh = 0; nh < St::NH; ++nh)
#pragma unroll
    for (int hc = 0; hc < 2; ++hc) {
      const float l = st.lsum[nh][hc];  // every row of the ones-MMA holds the full sum
      const int head = nh * 8 + qd + hc;
      if (head < g) {
#pragma unroll
        for (int mt = 0; mt < St::MT; ++mt) {
          O[head * D + mt * 16 + r] = st.o[nh][mt][hc];
          O[head * D + mt * 16 + r + 8] = st.o[nh][mt][hc + 2];
        }
        if (r == 0) {
          M[head] = st.m[nh][hc];
          L[head] = l;
        }
      }
    }
}

// ---- consumer state for an FP8 (e4m3) cache (f16 tensor cores) ----
//
// Tiles hold one-byte codes [16 tokens][128 d].  K fragments come from
// ldmatrix on 16-bit units, so a lane holds four consecutive d-values of a
// token; the k-order of S^T = K Q^T is permuted to match (k-slots 2q, 2q+1,
// 2q+8, 2q+9 of a 16-wide step are d 4q, 4q+1, 4q+2, 4q+3 of that step) and
// Q's fragments are built in the same order.  V fragments come from
// ldmatrix.trans on 16-bit units (pairs of d-values); a byte permute splits
// the pairs, so row r of an output m-tile is d = 16mt + 2r and row r+8 is
// d = 16mt + 2r + 1.  Codes become f16 exactly: e4m3 by cvt.f16x2.e4m3x2,
// e5m2 (the upper byte of a binary16) by the byte permute alone; the K scale
// is folded into the score scale and the V scale into the output.
// (The e4m3 m16n8k32 MMA straight on the codes, with q split into two e4m3
// terms, was measured slower here: more issued instructions per tile.)
template <int GMAX>
struct Fp8State {
  static constexpr int D = 128;
  static constexpr int KS = 8, MT = 8, NH = GMAX / 8;
  uint32_t qb[NH][KS][2];  // f16 B fragments of Q^T in the permuted k-order
  float o[NH][MT][4];
  float m[NH][2];          // running max of the scaled scores (log2 units)
  float lsum[NH][4];       // running sums of P, accumulated by a tensor-core MMA
  int32_t lim[NH][2];
  int32_t lim_min;         // smallest limit over the item's rows
};

template <int GMAX>
__device__ __forceinline__ void fp8_begin_item(Fp8State<GMAX>& st, const uint8_t* qs, int rows,
                                               int g, int len, int q_len, int lane,
                                               int row0 = 0) {
  using St = Fp8State<GMAX>;
  const int r = lane >> 2, q4 = (lane & 3) * 4, qd = (lane & 3) * 2;
  const uint16_t* q16 = reinterpret_cast<const uint16_t*>(qs);  // bf16 rows of 128
#pragma unroll
  for (int nh = 0; nh < St::NH; ++nh) {
    const int row = nh * 8 + r;
#pragma unroll
    for (int ks = 0; ks < St::KS; ++ks) {
      if (row < rows) {
        const uint2 w = *reinterpret_cast<const uint2*>(q16 + row * 128 + ks * 16 + q4);
        st.qb[nh][ks][0] = pack_f16x2(bf16lo_to_f32(w.x), bf16hi_to_f32(w.x));
        st.qb[nh][ks][1] = pack_f16x2(bf16lo_to_f32(w.y), bf16hi_to_f32(w.y));
      } else {
        st.qb[nh][ks][0] = st.qb[nh][ks][1] = 0u;
      }
    }
#pragma unroll
    for (int hc = 0; hc < 2; ++hc) {
      const int n = nh * 8 + qd + hc;
      st.lim[nh][hc] = n < rows ? len - q_len + (row0 + n) / g : -1;
    }
#pragma unroll
    for (int mt = 0; mt < St::MT; ++mt) {
      st.o[nh][mt][0] = st.o[nh][mt][1] = st.o[nh][mt][2] = st.o[nh][mt][3] = 0.f;
    }
    st.m[nh][0] = st.m[nh][1] = -INFINITY;
    st.lsum[nh][0] = st.lsum[nh][1] = st.lsum[nh][2] = st.lsum[nh][3] = 0.f;
  }
  st.lim_min = len - q_len + row0 / g;
}

// Four FP8 codes (one 32-bit word, bytes b0..b3) to two f16x2: (b0, b1) to `lo`,
// (b2, b3) to `hi`.  e4m3 codes are converted (exactly); e5m2 codes are the
// upper bytes of binary16 values, so a byte permute places them.
template <bool kE5m2>
__device__ __forceinline__ void fp8x4_to_f16x2x2(uint32_t x, uint32_t& lo, uint32_t& hi) {
  if constexpr (kE5m2) {
    lo = __byte_perm(x, 0u, 0x1404u);
    hi = __byte_perm(x, 0u, 0x3424u);
  } else {
    e4m3x4_to_f16x2x2(x, lo, hi);
  }
}

// The same with the pairs (b0, b2) to `lo` and (b1, b3) to `hi` (the V layout
// after ldmatrix.trans on 16-bit units).
template <bool kE5m2>
__device__ __forceinline__ void fp8x4_to_f16x2x2_interleaved(uint32_t x, uint32_t& lo,
                                                             uint32_t& hi) {
  if constexpr (kE5m2) {
    lo = __byte_perm(x, 0u, 0x2404u);
    hi = __byte_perm(x, 0u, 0x3414u);
  } else {
    e4m3x4_to_f16x2x2(__byte_perm(x, 0u, 0x3120u), lo, hi);
  }
}

template <int GMAX, bool kE5m2 = false>
__device__ __forceinline__ void fp8_step(Fp8State<GMAX>& st, const uint8_t* k0,
                                         const uint8_t* v0, int valid0, int pos0,
                                         const uint8_t* k1, const uint8_t* v1, int valid1,
                                         int pos1, float sc, int lane) {
  using St = Fp8State<GMAX>;
  constexpr int NH = St::NH;
  const int r = lane >> 2, qd = (lane & 3) * 2;
  // ldmatrix.x4 rows: lanes 0-7 tokens 0-7 / granule 2p, 8-15 tokens 8-15 / 2p,
  // 16-23 tokens 0-7 / 2p+1, 24-31 tokens 8-15 / 2p+1 (a granule = 16 codes).
  const uint32_t tok = ((lane >> 3) & 1) * 8 + (lane & 7);
  const uint32_t gsel = lane >> 4;
  // ---- S^T = K Q^T, one accumulation chain per tile ----
  float s[2][NH][4];
#pragma unroll
  for (int t = 0; t < 2; ++t)
#pragma unroll
    for (int nh = 0; nh < NH; ++nh) s[t][nh][0] = s[t][nh][1] = s[t][nh][2] = s[t][nh][3] = 0.f;
#pragma unroll
  for (int kp = 0; kp < St::KS / 2; ++kp) {
    const uint32_t off = ((((kp * 2) + gsel) ^ (tok & 7u)) << 4);
#pragma unroll
    for (int t = 0; t < 2; ++t) {
      uint32_t m0, m1, m2, m3;
      ldmatrix_x4(smem_addr(t ? k1 : k0) + tok * 128u + off, m0, m1, m2, m3);
      uint32_t a_lo[4], a_hi[4];
      fp8x4_to_f16x2x2<kE5m2>(m0, a_lo[0], a_lo[2]);
      fp8x4_to_f16x2x2<kE5m2>(m1, a_lo[1], a_lo[3]);
      fp8x4_to_f16x2x2<kE5m2>(m2, a_hi[0], a_hi[2]);
      fp8x4_to_f16x2x2<kE5m2>(m3, a_hi[1], a_hi[3]);
#pragma unroll
      for (int nh = 0; nh < NH; ++nh) {
        mma_f16_16816(s[t][nh], a_lo, st.qb[nh][2 * kp][0], st.qb[nh][2 * kp][1]);
        mma_f16_16816(s[t][nh], a_hi, st.qb[nh][2 * kp + 1][0], st.qb[nh][2 * kp + 1][1]);
      }
    }
  }
  // ---- mask (raw scores; element i of a C fragment is token r + 8(i>>1), row 2q + (i&1)).
  // Tiles that are full and wholly inside every row's causal window need no mask.
  if (!(valid0 == kBlock && valid1 == kBlock && pos1 + kBlock - 1 <= st.lim_min)) {
#pragma unroll
    for (int t = 0; t < 2; ++t) {
      const int valid = t ? valid1 : valid0;
      const int pos = t ? pos1 : pos0;
#pragma unroll
      for (int nh = 0; nh < NH; ++nh)
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int tk = r + 8 * (i >> 1);
          if (!(tk < valid && pos + tk <= st.lim[nh][i & 1])) s[t][nh][i] = -INFINITY;
        }
    }
  }
  // ---- running max (scaled by sc > 0 after the reduction), lazy rescale ----
  bool grow = false;
  float m_new[NH][2];
#pragma unroll
  for (int nh = 0; nh < NH; ++nh)
#pragma unroll
    for (int hc = 0; hc < 2; ++hc) {
      float mx = fmaxf(fmaxf(s[0][nh][hc], s[0][nh][hc + 2]), fmaxf(s[1][nh][hc], s[1][nh][hc + 2]));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
      m_new[nh][hc] = mx * sc;
      grow |= m_new[nh][hc] > st.m[nh][hc] + kRescaleSlack;
    }
  if (__any_sync(0xffffffffu, grow)) {
#pragma unroll
    for (int nh = 0; nh < NH; ++nh)
#pragma unroll
      for (int hc = 0; hc < 2; ++hc) {
        const bool up = m_new[nh][hc] > st.m[nh][hc] + kRescaleSlack;
        const float alpha = up ? fast_exp2(st.m[nh][hc] - m_new[nh][hc]) : 1.f;  // 0 from -inf
        st.m[nh][hc] = up ? m_new[nh][hc] : st.m[nh][hc];
        st.lsum[nh][hc] *= alpha;
        st.lsum[nh][hc + 2] *= alpha;
#pragma unroll
        for (int mt = 0; mt < St::MT; ++mt) {
          st.o[nh][mt][hc] *= alpha;
          st.o[nh][mt][hc + 2] *= alpha;
        }
      }
  }
  // ---- P = exp2(s sc - m) in f16, transposed into B fragments; l += ones . P^T ----
  constexpr uint32_t kOnes = 0x3c003c00u;  // f16x2 (1, 1)
  const uint32_t ones[4] = {kOnes, kOnes, kOnes, kOnes};
  uint32_t pb[2][NH][2];
#pragma unroll
  for (int nh = 0; nh < NH; ++nh) {
    const float mu0 = st.m[nh][0] == -INFINITY ? 0.f : st.m[nh][0];
    const float mu1 = st.m[nh][1] == -INFINITY ? 0.f : st.m[nh][1];
#pragma unroll
    for (int t = 0; t < 2; ++t) {
      const uint32_t lo = pack_f16x2(fast_exp2(fmaf(s[t][nh][0], sc, -mu0)),
                                     fast_exp2(fmaf(s[t][nh][1], sc, -mu1)));
      const uint32_t hi = pack_f16x2(fast_exp2(fmaf(s[t][nh][2], sc, -mu0)),
                                     fast_exp2(fmaf(s[t][nh][3], sc, -mu1)));
      pb[t][nh][0] = movmatrix_trans(lo);
      pb[t][nh][1] = movmatrix_trans(hi);
      mma_f16_16816(st.lsum[nh], ones, pb[t][nh][0], pb[t][nh][1]);
    }
  }
  // ---- O^T += V^T P^T (m-tile rows interleave d: r -> 2r, r+8 -> 2r+1) ----
#pragma unroll
  for (int t = 0; t < 2; ++t) {
    const int valid = t ? valid1 : valid0;
    const uint32_t base = smem_addr(t ? v1 : v0) + tok * 128u;
    uint32_t mk0 = 0xffffffffu, mk1 = 0xffffffffu;
    const bool partial = valid < kBlock;
    if (partial) {
      mk0 = (qd < valid ? 0x0000ffffu : 0u) | (qd + 1 < valid ? 0xffff0000u : 0u);
      mk1 = (qd + 8 < valid ? 0x0000ffffu : 0u) | (qd + 9 < valid ? 0xffff0000u : 0u);
    }
#pragma unroll
    for (int mp = 0; mp < St::MT / 2; ++mp) {
      const uint32_t off = ((((mp * 2) + gsel) ^ (tok & 7u)) << 4);
      uint32_t m0, m1, m2, m3;
      ldmatrix_x4_trans(base + off, m0, m1, m2, m3);
      // m0 / m1: tokens 0-7 / 8-15 of granule 2mp; m2 / m3: of granule 2mp+1
#pragma unroll
      for (int hlf = 0; hlf < 2; ++hlf) {
        uint32_t a[4];
        fp8x4_to_f16x2x2_interleaved<kE5m2>(hlf ? m2 : m0, a[0], a[1]);
        fp8x4_to_f16x2x2_interleaved<kE5m2>(hlf ? m3 : m1, a[2], a[3]);
        if (partial) {
          a[0] &= mk0;
          a[1] &= mk0;
          a[2] &= mk1;
          a[3] &= mk1;
        }
#pragma unroll
        for (int nh = 0; nh < NH; ++nh) mma_f16_16816(st.o[nh][2 * mp + hlf], a, pb[t][nh][0], pb[t][nh][1]);
      }
    }
  }
}

template <int GMAX>
__device__ __forceinline__ void fp8_publish(Fp8State<GMAX>& st, float* slot, int rows, int lane) {
  using St = Fp8State<GMAX>;
  constexpr int D = 128;
  const int r = lane >> 2, qd = (lane & 3) * 2;
  float* O = slot;
  float* M = slot + rows * D;
  float* L = M + rows;
#pragma unroll
  for (int nh = 0; nh < St::NH; ++nh)
#pragma unroll
    for (int hc = 0; hc < 2; ++hc) {
      const int row = nh * 8 + qd + hc;
      if (row < rows) {
#pragma unroll
        for (int mt = 0; mt < St::MT; ++mt) {
          O[row * D + mt * 16 + 2 * r] = st.o[nh][mt][hc];
          O[row * D + mt * 16 + 2 * r + 1] = st.o[nh][mt][hc + 2];
        }
        if (r == 0) {
          M[row] = st.m[nh][hc];
          L[row] = st.lsum[nh][hc];  // every row of the ones-MMA holds the full sum
        }
      }
    }
}

// ---- consumer state for fp32 (CUDA cores) ----
template <int D, int GMAX>
struct F32State {
  static constexpr int NV = D / 32;  // output columns per lane
  float o[GMAX][NV];
  float m[GMAX], l[GMAX];
  int32_t lim[GMAX];                 // last key position each row may see (causal)
};

template <int D, int GMAX>
__device__ __forceinline__ void f32_begin_item(F32State<D, GMAX>& st, int rows, int g, int len,
                                               int q_len) {
#pragma unroll
  for (int h = 0; h < GMAX; ++h) {
    st.lim[h] = h < rows ? len - q_len + h / g : -1;
    st.m[h] = -INFINITY;
    st.l[h] = 0.f;
#pragma unroll
    for (int i = 0; i < F32State<D, GMAX>::NV; ++i) st.o[h][i] = 0.f;
  }
}

template <int D, int GMAX>
__device__ __forceinline__ void f32_block(F32State<D, GMAX>& st, const float* qs,
                                          const uint8_t* ktile, const uint8_t* vtile, int valid,
                                          int pos, float sc, int g, int lane) {
  constexpr int NV = F32State<D, GMAX>::NV;
  const int t = lane & 15, hf = lane >> 4;
  float acc[GMAX];
#pragma unroll
  for (int h = 0; h < GMAX; ++h) acc[h] = 0.f;
#pragma unroll
  for (int dd = 0; dd < D / 8; ++dd) {
    const int d0 = hf * (D / 2) + dd * 4;
    const uint32_t byte = d0 * 4;
    const float4 kv = *reinterpret_cast<const float4*>(
        ktile + (byte >> 7) * (kBlock * 128) + swz128(t, byte & 127));
#pragma unroll
    for (int h = 0; h < GMAX; ++h) {
      if (h < g) {
        const float4 qv = *reinterpret_cast<const float4*>(qs + h * D + d0);
        acc[h] = fmaf(qv.x, kv.x, fmaf(qv.y, kv.y, fmaf(qv.z, kv.z, fmaf(qv.w, kv.w, acc[h]))));
      }
    }
  }
  float pr[GMAX];
#pragma unroll
  for (int h = 0; h < GMAX; ++h) {
    if (h < g) {
      float a = acc[h] + __shfl_xor_sync(0xffffffffu, acc[h], 16);
      const float z = (t < valid && pos + t <= st.lim[h]) ? a * sc : -INFINITY;
      float mx = z;
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
      const float m_new = fmaxf(st.m[h], mx);
      const float m_use = m_new == -INFINITY ? 0.f : m_new;
      const float alpha = exp2f(st.m[h] - m_use);
      const float pz = exp2f(z - m_use);
      float ps = pz;
      ps += __shfl_xor_sync(0xffffffffu, ps, 1);
      ps += __shfl_xor_sync(0xffffffffu, ps, 2);
      ps += __shfl_xor_sync(0xffffffffu, ps, 4);
      ps += __shfl_xor_sync(0xffffffffu, ps, 8);
      st.m[h] = m_new;
      st.l[h] = st.l[h] * alpha + ps;
#pragma unroll
      for (int i = 0; i < NV; ++i) st.o[h][i] *= alpha;
      pr[h] = pz;
    }
  }
  for (int tt = 0; tt < valid; ++tt) {
    float v[NV];
#pragma unroll
    for (int i = 0; i < NV; ++i) {
      v[i] = *reinterpret_cast<const float*>(vtile + i * (kBlock * 128) +
                                             swz128(tt, (lane * 4) & 127));
    }
#pragma unroll
    for (int h = 0; h < GMAX; ++h) {
      if (h < g) {
        const float pt = __shfl_sync(0xffffffffu, pr[h], tt);
#pragma unroll
        for (int i = 0; i < NV; ++i) st.o[h][i] = fmaf(pt, v[i], st.o[h][i]);
      }
    }
  }
}

template <int D, int GMAX>
__device__ __forceinline__ void f32_publish(F32State<D, GMAX>& st, float* slot, int g,
                                            int lane) {
  float* O = slot;
  float* M = slot + g * D;
  float* L = M + g;
#pragma unroll
  for (int h = 0; h < GMAX; ++h) {
    if (h < g) {
#pragma unroll
      for (int i = 0; i < F32State<D, GMAX>::NV; ++i) O[h * D + lane + 32 * i] = st.o[h][i];
      if (lane == 0) {
        M[h] = st.m[h];
        L[h] = st.l[h];
      }
    }
  }
}

// ---- combine the warps' states of one item and store the result ----
// The item's `rows` rows are chunk token i = n / group, head n % group.  Row
// n's states sit in the slots of the L = W / SPLIT warps holding it (row
// n - RPW*half of the warps half*L .. half*L + L - 1, half = n / RPW), each
// slot laid out as [rh rows x D outputs][rh maxima][rh sums], rh = the rows
// that half holds.
template <typename T, int D, int W, int SPLIT, int RPW>
__device__ __forceinline__ void combine_and_store(const DecodeParams& prm, const ItemMeta& it,
                                                  const float* merge, int per_warp, int rows,
                                                  int warp, int lane) {
  constexpr int L = W / SPLIT;
  const int tid = warp * 32 + lane;
  for (int e = tid * 4; e < rows * D; e += W * 32 * 4) {
    const int h = e / D, d = e % D;
    const int half = SPLIT == 1 ? 0 : h / RPW;
    const int local = h - half * RPW;
    const int rh = SPLIT == 1 ? rows : (rows - half * RPW < RPW ? rows - half * RPW : RPW);
    const float* base = merge + half * L * per_warp;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < L; ++w) M = fmaxf(M, base[w * per_warp + rh * D + local]);
    float lsum = 0.f;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    if (M != -INFINITY) {
#pragma unroll
      for (int w = 0; w < L; ++w) {
        const float* slot = base + w * per_warp;
        const float f = exp2f(slot[rh * D + local] - M);
        lsum = fmaf(slot[rh * D + rh + local], f, lsum);
        const float4 ov = *reinterpret_cast<const float4*>(slot + local * D + d);
        acc.x = fmaf(ov.x, f, acc.x);
        acc.y = fmaf(ov.y, f, acc.y);
        acc.z = fmaf(ov.z, f, acc.z);
        acc.w = fmaf(ov.w, f, acc.w);
      }
      const float inv = prm.out_scale / lsum;
      acc.x *= inv;
      acc.y *= inv;
      acc.z *= inv;
      acc.w *= inv;
    }
    const int group = prm.group;
    const size_t row = static_cast<size_t>(it.q_start + h / group) * prm.num_q_heads +
                       it.kv_head * group + h % group;
    if (it.nparts == 1) {
      if constexpr (sizeof(T) != 4) {  // bf16 output (bf16 and FP8 caches)
        uint2 packed = make_uint2(pack_bf16x2(acc.x, acc.y), pack_bf16x2(acc.z, acc.w));
        *reinterpret_cast<uint2*>(reinterpret_cast<__nv_bfloat16*>(prm.out) + row * D + d) = packed;
      } else {
        *reinterpret_cast<float4*>(reinterpret_cast<float*>(prm.out) + row * D + d) = acc;
      }
    } else {
      const size_t prow = row * prm.max_parts + it.part;
      *reinterpret_cast<float4*>(prm.part_o + prow * D + d) = acc;
      if (d == 0) {
        prm.part_ml[prow * 2 + 0] = M == -INFINITY ? -INFINITY : M * kLn2;
        prm.part_ml[prow * 2 + 1] = lsum;
      }
    }
  }
}

// The persistent decode kernel.  Warps 0..W-1 decode; warp W schedules.
//
// The scheduler warp fetches work units (item x kv head x row group) from the
// global work counter and publishes each into a ring slot: its metadata, its
// q rows (one bulk copy per chunk token) and the slice of the block table it
// covers.  Every lead decode warp (the
// first W / SPLIT) owns S tile stages and is its own TMA producer: it keeps up
// to S of its blocks in flight, following its share of the items (blocks l,
// l+L, ... of each, L = W / SPLIT) and running ahead into the next items
// while it computes.  With SPLIT = 2 a second warp reads the same stages and
// takes the item's upper query rows; a stage is refilled once both warps have
// released it (an "empty" barrier with two arrivals).  At the end of an item
// the W warps combine their online-softmax states through shared memory.
template <typename T, int D, int GMAX, int W, int S, int MB, int SPLIT>
__global__ void __launch_bounds__((W + 1) * 32, 1)
    decode_kernel(const __grid_constant__ CUtensorMap tmap_k,
                  const __grid_constant__ CUtensorMap tmap_v, const DecodeParams prm) {
  constexpr int ELEM = sizeof(T);            // cache bytes per element (1 for FP8)
  constexpr int QELEM = q_elem_bytes<T>();   // q bytes per element
  using Lay = DecodeLayout<ELEM, D, GMAX, W, S, MB, QELEM, SPLIT>;
  constexpr int L = Lay::kLead;              // warps owning stages
  constexpr int RPW = Lay::kRowsPerWarp;     // query rows per warp
  static_assert(SPLIT == 1 || (SPLIT == 2 && GMAX == 16 && W % 2 == 0), "row split: 2 x 8 rows");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const int g = prm.group;
  // query rows of the largest item
  const int rows_max = (prm.max_query_len < prm.group_tokens ? prm.max_query_len
                                                              : prm.group_tokens) * g;
  uint8_t* stages = smem + Lay::kStagesOff;
  uint8_t* ring = smem + Lay::kRingOff;
  int32_t* tables = reinterpret_cast<int32_t*>(smem + Lay::kTablesOff);  // [kRing][kMaxItemBlocks]
  float* merge = reinterpret_cast<float*>(smem + Lay::kMergeOff);
  ItemMeta* meta = reinterpret_cast<ItemMeta*>(smem + Lay::meta_off(rows_max));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Lay::bars_off(rows_max));
  uint64_t* full = bars;                       // [L][S]
  uint64_t* empty = full + L * S;              // [L][S] (SPLIT > 1 only)
  uint64_t* item_full = empty + L * S;         // [kRing]
  uint64_t* item_empty = item_full + kRing;    // [kRing]
  uint64_t* merge_bar = item_empty + kRing;    // [2]
  uint32_t* stage_ok = reinterpret_cast<uint32_t*>(smem + Lay::flags_off(rows_max));  // [L][S]
  volatile uint32_t* abort_flag = stage_ok + L * S;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int i = 0; i < L * S; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], SPLIT);
    }
    for (int i = 0; i < kRing; ++i) {
      mbar_init(&item_full[i], 1);
      mbar_init(&item_empty[i], W);
    }
    mbar_init(&merge_bar[0], W);
    mbar_init(&merge_bar[1], W);
    *abort_flag = 0u;
    fence_mbar_init();
  }
  __syncthreads();
  pdl_wait();  // the plan and the cache writes before this launch are complete

  const int32_t hkv = prm.num_kv_heads;
  if (warp == W) {
    // ================================ scheduler ================================
    const uint32_t per_item = static_cast<uint32_t>(hkv) * prm.row_groups;
    const uint32_t total = prm.counters[1] * per_item;
    uint32_t next = 0;
    if (lane == 0) next = atomicAdd(&prm.counters[0], 1u);
    uint32_t item_seq = 0;
    bool ok = true;
    for (;; ++item_seq) {
      const int r = item_seq % kRing;
      if (item_seq >= kRing) {
        if (lane == 0) ok = mbar_wait(&item_empty[r], ((item_seq / kRing) - 1) & 1);
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok || *abort_flag) break;
      }
      const uint32_t widx = __shfl_sync(0xffffffffu, next, 0);
      if (widx >= total) {
        pdl_trigger();  // this CTA's work is all handed out: let the next kernel launch
        if (lane == 0) {
          meta[r].seq = -1;
          mbar_arrive(&item_full[r]);
          // Every CTA has made its last fetch once it gets here; the last one
          // to finish rearms the counters for the next run of the same plan.
          __threadfence();
          if (atomicAdd(&prm.counters[2], 1u) == gridDim.x - 1) {
            prm.counters[0] = 0u;
            prm.counters[2] = 0u;
          }
        }
        ++item_seq;
        break;
      }
      // fetch the following item now; its value is only needed next time round
      if (lane == 0) next = atomicAdd(&prm.counters[0], 1u);
      // work index -> (planned item, kv head, row group); a (sequence, partition,
      // kv head)'s row groups are adjacent, so they read the same tiles close in time
      const PlanItem pi = prm.items[widx / per_item];
      const uint32_t rem = widx % per_item;
      const int32_t kvh = static_cast<int32_t>(rem / prm.row_groups);
      const int32_t grp = static_cast<int32_t>(rem % prm.row_groups);
      const int32_t blk_begin = pi.blk0;
      // the chunk of query tokens: one per sequence unless query_start_loc is
      // given; a shared-prefix item serves one token of each of q_len sequences
      int32_t q_start = pi.seq, q_len = 1;
      const bool shared = pi.q_start >= 0;
      if (shared) {
        q_start = pi.q_start;
        q_len = pi.q_len;
        if (q_len < 0 || q_len > prm.group_tokens || q_start + q_len > prm.num_q_tokens) {
          if (lane == 0 && kvh == 0) raise_error(PKV_DEVERR_GROUP);
          q_start = 0;
          q_len = 0;
        }
      } else if (prm.query_start_loc) {
        q_start = prm.query_start_loc[pi.seq];
        q_len = prm.query_start_loc[pi.seq + 1] - q_start;
        const int32_t cap = pi.len < prm.max_query_len ? pi.len : prm.max_query_len;
        const bool first = lane == 0 && kvh == 0 && pi.part == 0 && grp == 0;
        if (q_len < 0 || q_len > cap) {
          if (first) raise_error(PKV_DEVERR_LEN);
          q_len = q_len < 0 ? 0 : cap;
        }
        if (q_start < 0 || q_start + q_len > prm.num_q_tokens) {  // rows outside q / out
          if (first) raise_error(PKV_DEVERR_LEN);
          q_start = 0;
          q_len = 0;
        }
      }
      // this row group: chunk tokens t0 .. t0 + tlen - 1; none of its rows sees a
      // key past position len_eff - 1, so only those blocks are read
      const int32_t t0 = grp * prm.group_tokens;
      int32_t tlen = q_len - t0;
      tlen = tlen < 0 ? 0 : (tlen > prm.group_tokens ? prm.group_tokens : tlen);
      const int32_t len_eff = tlen > 0 ? pi.len - (q_len - t0 - tlen) : pi.len;
      int32_t nblk = (len_eff + kBlock - 1) / kBlock - blk_begin;
      nblk = nblk < prm.part_blocks ? nblk : prm.part_blocks;
      nblk = nblk < 0 || tlen == 0 ? 0 : nblk;  // a group without rows reads nothing
      q_start += t0;
      q_len = tlen;
      const int32_t* src = prm.block_tables +
                           static_cast<size_t>(pi.seq) * prm.max_blocks_per_seq + blk_begin;
      int32_t* dst = tables + r * kMaxItemBlocks;
      for (int32_t j = lane; j < nblk; j += 32) dst[j] = src[j];
      __syncwarp();
      if (lane == 0) {
        ItemMeta& mt = meta[r];
        mt.seq = pi.seq;
        mt.kv_head = kvh;
        mt.part = pi.part;
        mt.len = len_eff;
        mt.nparts = pi.nparts;
        mt.blk_begin = blk_begin;
        mt.nblk = nblk;
        mt.q_start = q_start;
        mt.q_len = q_len;
        mt.q_causal = shared ? 1 : q_len;
        const uint32_t row_bytes = static_cast<uint32_t>(g * D * QELEM);  // one token's group
        if (q_len > 0) {
          mbar_arrive_expect_tx(&item_full[r], row_bytes * q_len);
          for (int32_t i = 0; i < q_len; ++i) {
            const uint8_t* qsrc = reinterpret_cast<const uint8_t*>(prm.q) +
                                  (static_cast<size_t>(q_start + i) * prm.num_q_heads + kvh * g) *
                                      D * QELEM;
            bulk_load(ring + r * Lay::kQBytes + i * row_bytes, qsrc, row_bytes, &item_full[r]);
          }
        } else {
          mbar_arrive(&item_full[r]);
        }
      }
    }
    if (!ok) {
      // A wait gave up: tell the decode warps, then wait (bounded) for the q
      // copies still in flight into the ring, so none lands after exit.
      *abort_flag = 1u;
      if (lane == 0) {
        for (uint32_t j = item_seq > kRing ? item_seq - kRing : 0; j < item_seq; ++j) {
          mbar_wait(&item_full[j % kRing], (j / kRing) & 1, kDrainLimitCycles);
        }
      }
    }
    return;
  }

  // ================================ decode warps ================================
  using Bst = Bf16State<D, RPW>;
  using Fst = F32State<D, GMAX>;
  constexpr bool kE5m2 = std::is_same<T, Fp8E5m2Kv>::value;
  constexpr bool kFp8 = std::is_same<T, Fp8Kv>::value || kE5m2;
  constexpr bool kBf16 = sizeof(T) == 2;
  static_assert(SPLIT == 1 || kFp8 || kBf16, "row split needs the tensor-core states");
  typename std::conditional<kFp8, Fp8State<RPW>,
                            typename std::conditional<kBf16, Bst, Fst>::type>::type st;
  const float sc = prm.qk_scale_log2;
  const int per_warp = Lay::merge_floats_per_warp(Lay::slot_rows(rows_max));
  const int lead = warp % L;         // the stage set this warp reads
  const int half = warp / L;         // which RPW query rows of an item it holds
  uint64_t* my_full = full + lead * S;
  uint64_t* my_empty = empty + lead * S;
  uint32_t* my_ok = stage_ok + lead * S;
  uint8_t* my_stages = stages + lead * S * Lay::kStageBytes;

  // Producer cursor over this stage set's blocks: item p_item, block p_blk of it.
  uint32_t cctr = 0, pctr = 0;       // blocks consumed by this warp / issued by its lead
  uint32_t c_item = 0;               // item being consumed
  uint32_t p_item = 0;
  int32_t p_blk = lead;
  bool p_known = false, p_end = false;
  ItemMeta pm{};
  bool ok = true;

  // Issue the stage set's next blocks until S are in flight (lead warps only).
  // With `blocking` the waits for an item's metadata and for a stage's
  // release may block (only when the block is needed now).
  auto produce = [&](bool blocking) {
    while (pctr < cctr + S && !p_end) {
      if (!p_known) {
        if (p_item >= c_item + kRing) return;          // that slot still holds an older item
        const int r = p_item % kRing;
        const uint32_t par = (p_item / kRing) & 1;
        if (blocking) {
          if (!mbar_wait(&item_full[r], par)) {
            ok = false;
            return;
          }
        } else if (!mbar_try_wait(&item_full[r], par)) {
          return;
        }
        pm = meta[r];
        if (pm.seq < 0) {
          p_end = true;
          return;
        }
        p_known = true;
      }
      if (p_blk >= pm.nblk) {
        ++p_item;
        p_blk = warp;
        p_known = false;
        continue;
      }
      const int s_idx = pctr % S;
      if constexpr (SPLIT > 1) {
        // the stage's previous use must have been released by every warp reading it
        if (pctr >= static_cast<uint32_t>(S)) {
          const uint32_t par = ((pctr / S) - 1) & 1;
          if (blocking) {
            if (!mbar_wait(&my_empty[s_idx], par)) {
              ok = false;
              return;
            }
          } else if (!mbar_try_wait(&my_empty[s_idx], par)) {
            return;
          }
        }
      }
      const int32_t entry = tables[(p_item % kRing) * kMaxItemBlocks + p_blk];
      if (lane == 0) {
        const bool valid = entry >= 0 && entry < prm.num_blocks;
        my_ok[s_idx] = valid ? 1u : 0u;
        uint8_t* kdst = my_stages + s_idx * Lay::kStageBytes;
        uint8_t* vdst = kdst + Lay::kTileBytes;
        if (valid) {
          mbar_arrive_expect_tx(&my_full[s_idx], 2 * Lay::kTileBytes);
          const int32_t y = (entry * hkv + pm.kv_head) * kBlock;
#pragma unroll
          for (int c = 0; c < Lay::kChunks; ++c) {
            tma_load_2d(kdst + c * (kBlock * 128), &tmap_k, c * (128 / ELEM), y, &my_full[s_idx]);
            tma_load_2d(vdst + c * (kBlock * 128), &tmap_v, c * (128 / ELEM), y, &my_full[s_idx]);
          }
        } else {
          raise_error(PKV_DEVERR_BLOCK);
          mbar_arrive(&my_full[s_idx]);
        }
      }
      p_blk += L;
      ++pctr;
    }
  };

  for (;; ++c_item) {
    const int r = c_item % kRing;
    if (!mbar_wait(&item_full[r], (c_item / kRing) & 1)) {
      ok = false;
      break;
    }
    const ItemMeta it = meta[r];
    if (it.seq < 0) break;
    const uint8_t* qs = ring + r * Lay::kQBytes;
    const int rows = it.q_len * g;  // query rows of this item
    // this warp's rows: row0 .. row0 + my_rows - 1
    const int row0 = half * RPW;
    const int my_rows = SPLIT == 1 ? rows
                                   : (rows - row0 < 0 ? 0 : (rows - row0 < RPW ? rows - row0 : RPW));
    const uint8_t* my_qs = qs + row0 * D * QELEM;
    if constexpr (kFp8) {
      fp8_begin_item<RPW>(st, my_qs, my_rows, g, it.len, it.q_causal, lane, row0);
    } else if constexpr (kBf16) {
      bf16_begin_item<D, RPW>(st, my_qs, my_rows, g, it.len, it.q_causal, lane, row0);
    } else {
      f32_begin_item<D, GMAX>(st, rows, g, it.len, it.q_causal);
    }
    // bf16 consumes the blocks two at a time (b and b + L), fp32 one at a time.
    constexpr int kStep = (kBf16 || kFp8) ? 2 : 1;
    for (int32_t b = lead; b < it.nblk; b += kStep * L) {
      const int n = (kStep == 2 && b + L < it.nblk) ? 2 : 1;
      if (half == 0 && pctr < cctr + n) {
        produce(true);
        if (!ok || pctr < cctr + n) {
          ok = false;
          break;
        }
      }
      int valid[2] = {0, 0};
      const uint8_t* kt[2];
#pragma unroll
      for (int x = 0; x < kStep; ++x) {
        const uint32_t k = cctr + (x < n ? x : 0);
        const int s_idx = k % S;
        if (x < n && !mbar_wait(&my_full[s_idx], (k / S) & 1)) ok = false;
        kt[x] = my_stages + s_idx * Lay::kStageBytes;
        if (x < n && my_ok[s_idx]) {
          const int v = it.len - (it.blk_begin + b + x * L) * kBlock;
          valid[x] = v > kBlock ? kBlock : v;
        }
      }
      if (!ok) break;
      const int pos0 = (it.blk_begin + b) * kBlock;  // position of the first tile's token 0
      if constexpr (kFp8) {
        if (my_rows > 0)
          fp8_step<RPW, kE5m2>(st, kt[0], kt[0] + Lay::kTileBytes, valid[0], pos0, kt[1],
                               kt[1] + Lay::kTileBytes, valid[1], pos0 + L * kBlock, sc, lane);
      } else if constexpr (kBf16) {
        if (my_rows > 0)
          bf16_step<D, RPW>(st, kt[0], kt[0] + Lay::kTileBytes, valid[0], pos0, kt[1],
                            kt[1] + Lay::kTileBytes, valid[1], pos0 + L * kBlock, sc, lane);
      } else {
        f32_block<D, GMAX>(st, reinterpret_cast<const float*>(qs), kt[0], kt[0] + Lay::kTileBytes,
                           valid[0], pos0, sc, rows, lane);
      }
      __syncwarp();
      if constexpr (SPLIT > 1) {
        // release the stages to the lead (it refills them once every reader has)
        if (lane == 0) {
          for (int x = 0; x < n; ++x) mbar_arrive(&my_empty[(cctr + x) % S]);
        }
      }
      cctr += n;
      if (half == 0) produce(false);
    }
    if (!ok) break;
    // The q tile, metadata and table slice of this item are no longer needed.
    __syncwarp();
    if (lane == 0) mbar_arrive(&item_empty[r]);
    if (half == 0) produce(false);
    // ---- merge the W warps' states ----
    // two buffers: item c uses buffer c & 1 and merge_bar[c & 1];
    // one buffer: merge_bar[0] = states published, merge_bar[1] = combined.
    const int mb = MB == 2 ? (c_item & 1) : 0;
    const uint32_t pub_parity = MB == 2 ? ((c_item >> 1) & 1) : (c_item & 1);
    if (MB == 1 && c_item > 0 && !mbar_wait(&merge_bar[1], (c_item - 1) & 1)) {
      ok = false;
      break;
    }
    float* mslot = merge + (mb * W + warp) * per_warp;
    if constexpr (kFp8) {
      fp8_publish<RPW>(st, mslot, my_rows, lane);
    } else if constexpr (kBf16) {
      bf16_publish<D, RPW>(st, mslot, my_rows, lane);
    } else {
      f32_publish<D, GMAX>(st, mslot, rows, lane);
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&merge_bar[mb]);
    if (!mbar_wait(&merge_bar[mb], pub_parity)) {
      ok = false;
      break;
    }
    combine_and_store<T, D, W, SPLIT, RPW>(prm, it, merge + mb * W * per_warp, per_warp, rows,
                                           warp, lane);
    if constexpr (MB == 1) {
      __syncwarp();
      if (lane == 0) mbar_arrive(&merge_bar[1]);
    }
  }
  if (!ok) {
    // A wait gave up: raise the abort flag and wait (bounded) for the copies
    // this warp still has in flight.
    *abort_flag = 1u;
    for (uint32_t k = cctr; k < pctr; ++k) {
      mbar_wait(&my_full[k % S], (k / S) & 1, kDrainLimitCycles);
    }
  }
}

// ------------------------------------------------------------- merge kernel
// Combines the partial results (m, l, o) of a (query token, query head) row
// whose sequence was split (or read a shared prefix separately) by
// log-sum-exp and stores the final output.  WPR warps serve one row (CTAs of
// kMergeWarps warps, so kMergeWarps / WPR rows per CTA): every warp finds the
// common maximum M and takes every WPR-th partition, so a long row's partials
// stream in on several warps at once; with WPR > 1 warp 0 adds the warps'
// sums in a fixed order.  WPR = 1 suits rows with a few partials (one warp
// per row, no shared-memory step).  Partitions a causal row cannot see carry
// l = 0 and no weight.
constexpr int kMergeWarps = 4;

template <typename T, int D, int WPR>
__global__ void __launch_bounds__(kMergeWarps * 32)
    merge_kernel(void* __restrict__ out, const float* __restrict__ part_o,
                 const float* __restrict__ part_ml, const int32_t* __restrict__ context_lens,
                 const int32_t* __restrict__ query_start_loc,
                 const int32_t* __restrict__ seq_prefix, int32_t num_seqs,
                 int32_t num_q_tokens, int32_t num_q_heads, int32_t max_parts, int32_t max_len,
                 int32_t part_tokens) {
  static_assert(WPR == 1 || WPR == kMergeWarps, "one warp per row, or the whole CTA");
  constexpr int VEC = D / 32;  // floats per lane
  constexpr int RPC = kMergeWarps / WPR;  // rows per CTA
  __shared__ __align__(16) float red[kMergeWarps][D];
  __shared__ float red_w[kMergeWarps];
  pdl_wait();
  pdl_trigger();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int sub = warp % WPR;  // which of the row's partitions this warp takes
  const int64_t row = static_cast<int64_t>(blockIdx.x) * RPC + warp / WPR;
  // (returns below are uniform over the warps that share a row)
  if (row >= static_cast<int64_t>(num_q_tokens) * num_q_heads) return;
  const int32_t t = static_cast<int32_t>(row / num_q_heads);  // query token
  int32_t s = t;                                                // its sequence
  if (query_start_loc) {  // the last sequence whose chunk starts at or before t
    if (t >= query_start_loc[num_seqs]) return;  // rows past the last chunk
    int32_t lo = 0, hi = num_seqs - 1;
    while (lo < hi) {
      const int32_t mid = (lo + hi + 1) / 2;
      if (query_start_loc[mid] <= t) lo = mid; else hi = mid - 1;
    }
    s = lo;
  }
  int32_t L = context_lens[s];
  L = L < 0 ? 0 : (L > max_len ? max_len : L);
  // partials: those of a shared prefix of P blocks (if any), then the sequence's own
  const int32_t P = seq_prefix ? seq_prefix[s] : 0;
  const int32_t n = (P > 0 ? num_parts(P * kBlock, part_tokens) : 0) +
                    num_parts(L - P * kBlock, part_tokens);
  if (n <= 1) return;  // the decode kernel wrote this row directly
  const float* ml = part_ml + row * max_parts * 2;
  float M = -INFINITY;
  for (int p = lane; p < n; p += 32) M = fmaxf(M, ml[2 * p]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
  float acc[VEC];
#pragma unroll
  for (int i = 0; i < VEC; ++i) acc[i] = 0.f;
  float wsum = 0.f;
  const float* po = part_o + row * max_parts * D + lane * VEC;
  if (M != -INFINITY) {
#pragma unroll 4
    for (int p = sub; p < n; p += WPR) {
      const float lp = ml[2 * p + 1];
      const float w = lp > 0.f ? lp * exp2f((ml[2 * p] - M) * kLog2e) : 0.f;
      wsum += w;
      if constexpr (VEC == 4) {
        const float4 v = *reinterpret_cast<const float4*>(po + static_cast<size_t>(p) * D);
        acc[0] = fmaf(w, v.x, acc[0]);
        acc[1] = fmaf(w, v.y, acc[1]);
        acc[2] = fmaf(w, v.z, acc[2]);
        acc[3] = fmaf(w, v.w, acc[3]);
      } else {
        const float2 v = *reinterpret_cast<const float2*>(po + static_cast<size_t>(p) * D);
        acc[0] = fmaf(w, v.x, acc[0]);
        acc[1] = fmaf(w, v.y, acc[1]);
      }
    }
  }
  float tot = wsum;
  if constexpr (WPR > 1) {
#pragma unroll
    for (int i = 0; i < VEC; ++i) red[warp][lane * VEC + i] = acc[i];
    if (lane == 0) red_w[warp] = wsum;
    __syncthreads();
    if (warp != 0) return;
    tot = 0.f;
#pragma unroll
    for (int w = 0; w < kMergeWarps; ++w) tot += red_w[w];
#pragma unroll
    for (int i = 0; i < VEC; ++i) {
      float a = 0.f;
#pragma unroll
      for (int w = 0; w < kMergeWarps; ++w) a += red[w][lane * VEC + i];
      acc[i] = a;
    }
  }
  const float inv = tot > 0.f ? 1.f / tot : 0.f;
  if constexpr (sizeof(T) == 2) {
    __nv_bfloat16* o = reinterpret_cast<__nv_bfloat16*>(out) + row * D + lane * VEC;
    if constexpr (VEC == 4) {
      *reinterpret_cast<uint2*>(o) =
          make_uint2(pack_bf16x2(acc[0] * inv, acc[1] * inv), pack_bf16x2(acc[2] * inv, acc[3] * inv));
    } else {
      *reinterpret_cast<uint32_t*>(o) = pack_bf16x2(acc[0] * inv, acc[1] * inv);
    }
  } else {
    float* o = reinterpret_cast<float*>(out) + row * D + lane * VEC;
#pragma unroll
    for (int i = 0; i < VEC; ++i) o[i] = acc[i] * inv;
  }
}

}  // namespace pkv
