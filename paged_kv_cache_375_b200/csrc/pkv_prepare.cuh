// The prologue of a decode step in one launch: every sequence's new token
// (the one at position L - 1, L = context_lens[s]) is written into its slot of
// the paged pools -- the slot found through the block table as slot indexing
// does, the K/V rows copied (or quantised into FP8 codes) as reshape_and_cache
// does -- while CTA 0 builds the decode plan from the same lengths.  The
// per-block lookup and the 16-token blocks follow the ipipp.com vLLM article,
// section "二、PagedAttention分页原理深度剖析"; the slot of a position is the
// wiki entry's "Flattened 布局与 slot_mapping".
#pragma once

#include "pkv_cache_ops.cuh"
#include "pkv_decode.cuh"

namespace pkv {

// Grid: 1 + ceil(num_seqs / seqs_per_cta) CTAs of kPlanThreads threads.  CTA 0
// plans; CTA c > 0 writes sequences (c - 1) * seqs_per_cta ... with `per`
// threads each (per = min(units, kPlanThreads), units = 16-byte source units
// of one token's K row block).  A sequence with L = 0 has no new token.
template <bool kFp8, bool kE5m2>
__global__ void __launch_bounds__(kPlanThreads)
    decode_prepare_kernel(const uint4* __restrict__ k, const uint4* __restrict__ v,
                          uint8_t* __restrict__ k_cache, uint8_t* __restrict__ v_cache,
                          const int32_t* __restrict__ block_tables,
                          const int32_t* __restrict__ context_lens, int64_t* __restrict__ slots_out,
                          int32_t num_seqs, int32_t num_kv_heads, int32_t units_per_head,
                          int32_t max_blocks_per_seq, int32_t num_blocks, int32_t seqs_per_cta,
                          int32_t per, float k_scale, float v_scale, int32_t max_len,
                          int32_t part_blocks, PlanItem* __restrict__ items,
                          uint32_t* __restrict__ counters) {
  __shared__ uint32_t hist[kPlanBuckets];
  __shared__ uint32_t warp_sums[kPlanThreads / 32];
  pdl_wait();
  pdl_trigger();
  if (blockIdx.x == 0) {
    plan_body(context_lens, num_seqs, max_len, part_blocks, items, counters, hist, warp_sums);
    return;
  }
  const int s_local = threadIdx.x / per;
  if (s_local >= seqs_per_cta) return;
  const int32_t s = (blockIdx.x - 1) * seqs_per_cta + s_local;
  if (s >= num_seqs) return;
  const int first = threadIdx.x % per;
  const int32_t L = context_lens[s];
  if (L == 0) {
    if (slots_out && first == 0) slots_out[s] = -1;
    return;
  }
  // the slot of position L - 1, checked as slot indexing checks it
  int64_t slot = -1;
  const int32_t pos = L - 1;
  if (pos < 0 || pos / kBlock >= max_blocks_per_seq) {
    if (first == 0) raise_error(PKV_DEVERR_POS);
  } else {
    const int32_t phys = block_tables[static_cast<int64_t>(s) * max_blocks_per_seq + pos / kBlock];
    if (phys < 0 || phys >= num_blocks) {
      if (first == 0) raise_error(PKV_DEVERR_BLOCK);
    } else {
      slot = static_cast<int64_t>(phys) * kBlock + pos % kBlock;
    }
  }
  if (slots_out && first == 0) slots_out[s] = slot;
  if (slot < 0) return;
  const int64_t block = slot / kBlock;
  const int32_t offset = static_cast<int32_t>(slot % kBlock);
  const int32_t units = num_kv_heads * units_per_head;
  const uint4* ksrc = k + static_cast<int64_t>(s) * units;
  const uint4* vsrc = v + static_cast<int64_t>(s) * units;
  for (int32_t u = first; u < units; u += per) {
    const int32_t h = u / units_per_head;
    const int32_t within = u % units_per_head;
    const int64_t row = (block * num_kv_heads + h) * kBlock + offset;  // destination row
    if constexpr (kFp8) {
      // 8 bf16 values -> 8 FP8 codes
      const int64_t dst = row * (units_per_head * 8) + within * 8;
      *reinterpret_cast<uint2*>(k_cache + dst) = bf16x8_to_fp8x8<kE5m2>(ksrc[u], k_scale);
      *reinterpret_cast<uint2*>(v_cache + dst) = bf16x8_to_fp8x8<kE5m2>(vsrc[u], v_scale);
    } else {
      const int64_t dst = row * (units_per_head * 16) + within * 16;
      *reinterpret_cast<uint4*>(k_cache + dst) = ksrc[u];
      *reinterpret_cast<uint4*>(v_cache + dst) = vsrc[u];
    }
  }
}

}  // namespace pkv

namespace pkv {

// ------------------------------------------------------- token-list prologue
// The same for any list of new tokens (the tails of parallel samples, the
// chunks of several query tokens): token t of sequence token_seq[t] at
// position token_pos[t] goes to its slot through the block table, checked as
// slot indexing checks it; CTA 0 meanwhile builds the decode plan (kShared:
// the shared-prefix plan) from the context lengths.
struct TokenPrepare {
  const uint4* k;                 // [T][Hkv][D] new K rows (bf16 for FP8 pools)
  const uint4* v;
  uint8_t* k_cache;
  uint8_t* v_cache;
  const int32_t* block_tables;    // [B][MB]
  const int32_t* token_seq;       // [T]
  const int32_t* token_pos;       // [T]
  int64_t* slots_out;             // [T] or NULL
  int32_t num_tokens, num_seqs, num_kv_heads, units_per_head, max_blocks_per_seq, num_blocks;
  int32_t toks_per_cta, per;      // tokens per CTA, threads per token
  float k_scale, v_scale;         // FP8 pools
  // the plan
  const int32_t* context_lens;
  int32_t max_len, part_blocks;
  PlanItem* items;
  uint32_t* counters;
  // the shared-prefix plan
  const int32_t* group_start;
  const int32_t* shared_blocks;
  int32_t num_groups, members_per_item;
  int32_t* seq_prefix;
  int32_t* group_pref;
};

// Grid: 1 + ceil(num_tokens / toks_per_cta) CTAs of kPlanThreads threads.
template <bool kFp8, bool kE5m2, bool kShared>
__global__ void __launch_bounds__(kPlanThreads) token_prepare_kernel(const TokenPrepare a) {
  __shared__ uint32_t hist[kPlanBuckets];
  __shared__ uint32_t warp_sums[kPlanThreads / 32];
  __shared__ int32_t gs_cache[kShared ? kPlanGroupCache : 1];
  pdl_wait();  // the copy-on-write copies before this launch are complete
  pdl_trigger();
  if (blockIdx.x == 0) {
    if constexpr (kShared) {
      plan_shared_body(a.context_lens, a.group_start, a.shared_blocks, a.num_groups, a.num_seqs,
                       a.max_len, a.part_blocks, a.members_per_item, a.items, a.counters,
                       a.seq_prefix, a.group_pref, hist, warp_sums, gs_cache);
    } else {
      plan_body(a.context_lens, a.num_seqs, a.max_len, a.part_blocks, a.items, a.counters, hist,
                warp_sums);
    }
    return;
  }
  const int t_local = threadIdx.x / a.per;
  if (t_local >= a.toks_per_cta) return;
  const int32_t t = (blockIdx.x - 1) * a.toks_per_cta + t_local;
  if (t >= a.num_tokens) return;
  const int first = threadIdx.x % a.per;
  const int32_t units = a.num_kv_heads * a.units_per_head;
  const uint4* ksrc = a.k + static_cast<int64_t>(t) * units;
  const uint4* vsrc = a.v + static_cast<int64_t>(t) * units;
  // the token's rows do not depend on its slot: their first units are loaded
  // while the slot is looked up
  uint4 k0 = make_uint4(0u, 0u, 0u, 0u), v0 = k0;
  if (first < units) {
    k0 = ksrc[first];
    v0 = vsrc[first];
  }
  // the slot of (token_seq[t], token_pos[t]), checked as slot indexing checks it
  int64_t slot = -1;
  const int32_t seq = a.token_seq[t];
  if (seq < 0 || seq >= a.num_seqs) {
    if (first == 0) raise_error(PKV_DEVERR_POS);
  } else {
    const int32_t pos = a.token_pos[t];
    if (pos < 0 || pos / kBlock >= a.max_blocks_per_seq) {
      if (first == 0) raise_error(PKV_DEVERR_POS);
    } else {
      const int32_t phys =
          a.block_tables[static_cast<int64_t>(seq) * a.max_blocks_per_seq + pos / kBlock];
      if (phys < 0 || phys >= a.num_blocks) {
        if (first == 0) raise_error(PKV_DEVERR_BLOCK);
      } else {
        slot = static_cast<int64_t>(phys) * kBlock + pos % kBlock;
      }
    }
  }
  if (a.slots_out && first == 0) a.slots_out[t] = slot;
  if (slot < 0) return;
  const int64_t block = slot / kBlock;
  const int32_t offset = static_cast<int32_t>(slot % kBlock);
  for (int32_t u = first; u < units; u += a.per) {
    const int32_t h = u / a.units_per_head;
    const int32_t within = u % a.units_per_head;
    const int64_t row = (block * a.num_kv_heads + h) * kBlock + offset;  // destination row
    const uint4 kx = u == first ? k0 : ksrc[u];
    const uint4 vx = u == first ? v0 : vsrc[u];
    if constexpr (kFp8) {
      const int64_t dst = row * (a.units_per_head * 8) + within * 8;
      *reinterpret_cast<uint2*>(a.k_cache + dst) = bf16x8_to_fp8x8<kE5m2>(kx, a.k_scale);
      *reinterpret_cast<uint2*>(a.v_cache + dst) = bf16x8_to_fp8x8<kE5m2>(vx, a.v_scale);
    } else {
      const int64_t dst = row * (a.units_per_head * 16) + within * 16;
      *reinterpret_cast<uint4*>(a.k_cache + dst) = kx;
      *reinterpret_cast<uint4*>(a.v_cache + dst) = vx;
    }
  }
}

}  // namespace pkv
