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
