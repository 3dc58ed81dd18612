// pkv_cache_ops.cuh -- the kernels that maintain the paged KV cache on sm_100a:
// slot indexing, reshape_and_cache (scatter of new tokens into their slots)
// and copy_blocks (copy-on-write of shared blocks).
//
//  * Slots: a token at position j of a sequence lives in logical block j/16
//    at offset j%16; the block table names the physical block ("vLLM" wiki
//    entry, wiki.bytelighting.cn, "Flattened 布局与 slot_mapping"; ipipp.com
//    vLLM article, "二、PagedAttention分页原理深度剖析").
//  * copy_blocks serves copy-on-write of blocks shared by several sequences
//    ("vLLM 深读：用 PagedAttention 撑起高并发 LLM 推理", "先看浪费在哪里").
//
// These are byte movers: the element type only fixes the row size.
#pragma once

#include "pkv_device.cuh"

namespace pkv {

// ---------------------------------------------------------------- slot mapping
__global__ void __launch_bounds__(256)
    slot_mapping_kernel(int64_t* __restrict__ slots, const int32_t* __restrict__ block_tables,
                        const int32_t* __restrict__ context_lens,
                        const int32_t* __restrict__ token_seq,
                        const int32_t* __restrict__ token_pos, int32_t num_tokens,
                        int32_t num_seqs, int32_t max_blocks_per_seq, int32_t num_blocks) {
  pdl_wait();
  pdl_trigger();
  const int32_t t = blockIdx.x * blockDim.x + threadIdx.x;
  if (t >= num_tokens) return;
  const int32_t seq = token_seq ? token_seq[t] : t;
  int64_t slot = -1;
  if (seq < 0 || seq >= num_seqs) {
    raise_error(PKV_DEVERR_POS);
  } else {
    const int32_t pos = token_pos ? token_pos[t] : context_lens[seq] - 1;
    if (pos < 0 || pos / kBlock >= max_blocks_per_seq) {
      raise_error(PKV_DEVERR_POS);
    } else {
      const int32_t phys =
          block_tables[static_cast<int64_t>(seq) * max_blocks_per_seq + pos / kBlock];
      if (phys < 0 || phys >= num_blocks) {
        raise_error(PKV_DEVERR_BLOCK);
      } else {
        slot = static_cast<int64_t>(phys) * kBlock + pos % kBlock;
      }
    }
  }
  slots[t] = slot;
}

// ----------------------------------------------------------- reshape_and_cache
// One CTA per token.  Each thread moves 16-byte units of the token's K row
// block ([Hkv][D]) and V row block to their (block, head, offset) rows.
__global__ void __launch_bounds__(256)
    reshape_and_cache_kernel(const uint4* __restrict__ k, const uint4* __restrict__ v,
                             uint8_t* __restrict__ k_cache, uint8_t* __restrict__ v_cache,
                             const int64_t* __restrict__ slot_mapping, int32_t num_kv_heads,
                             int32_t row_bytes, int64_t num_slots) {
  pdl_wait();
  pdl_trigger();
  const int32_t t = blockIdx.x;
  const int64_t slot = slot_mapping[t];
  if (slot < 0) return;  // padding token
  if (slot >= num_slots) {
    if (threadIdx.x == 0) raise_error(PKV_DEVERR_SLOT);
    return;
  }
  const int64_t block = slot / kBlock;
  const int32_t offset = static_cast<int32_t>(slot % kBlock);
  const int32_t units_per_row = row_bytes / 16;
  const int32_t units = num_kv_heads * units_per_row;
  const uint4* ksrc = k + static_cast<int64_t>(t) * units;
  const uint4* vsrc = v + static_cast<int64_t>(t) * units;
  for (int32_t u = threadIdx.x; u < units; u += blockDim.x) {
    const int32_t h = u / units_per_row;
    const int32_t within = u % units_per_row;
    const int64_t dst =
        ((block * num_kv_heads + h) * kBlock + offset) * row_bytes + within * 16;
    const uint4 kv = ksrc[u];
    const uint4 vv = vsrc[u];
    *reinterpret_cast<uint4*>(k_cache + dst) = kv;
    *reinterpret_cast<uint4*>(v_cache + dst) = vv;
  }
}

// Eight bf16 values (16 bytes) to eight FP8 codes (8 bytes, same order):
// code = e4m3(value / scale), the division in float (round to nearest even),
// then round to nearest even onto e4m3, saturating to +-448.
// With kE5m2 the codes are e5m2 (saturating to +-57344).
template <bool kE5m2 = false>
__device__ __forceinline__ uint2 bf16x8_to_fp8x8(uint4 x, float scale) {
  const uint32_t w[4] = {x.x, x.y, x.z, x.w};
  uint32_t codes[2];
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const float a = __fdiv_rn(bf16lo_to_f32(w[2 * i]), scale);
    const float b = __fdiv_rn(bf16hi_to_f32(w[2 * i]), scale);
    const float c = __fdiv_rn(bf16lo_to_f32(w[2 * i + 1]), scale);
    const float d = __fdiv_rn(bf16hi_to_f32(w[2 * i + 1]), scale);
    const uint32_t p0 = kE5m2 ? f32x2_to_e5m2x2(a, b) : f32x2_to_e4m3x2(a, b);
    const uint32_t p1 = kE5m2 ? f32x2_to_e5m2x2(c, d) : f32x2_to_e4m3x2(c, d);
    codes[i] = p0 | (p1 << 16);
  }
  return make_uint2(codes[0], codes[1]);
}

// ------------------------------------------------ reshape_and_cache into FP8
// One CTA per token: each thread turns 8 bf16 values of the token's K (and V)
// into 8 FP8 codes, code = e4m3(value / scale) (or e5m2 with kE5m2) with the
// division in float, rounded to nearest even and saturated to the largest
// finite code, and stores them at the slot.
template <bool kE5m2>
__global__ void __launch_bounds__(256)
    reshape_and_cache_fp8_kernel(const uint4* __restrict__ k, const uint4* __restrict__ v,
                                 uint8_t* __restrict__ k_cache, uint8_t* __restrict__ v_cache,
                                 const int64_t* __restrict__ slot_mapping, int32_t num_kv_heads,
                                 int32_t head_dim, int64_t num_slots, float k_scale,
                                 float v_scale) {
  pdl_wait();
  pdl_trigger();
  const int32_t t = blockIdx.x;
  const int64_t slot = slot_mapping[t];
  if (slot < 0) return;
  if (slot >= num_slots) {
    if (threadIdx.x == 0) raise_error(PKV_DEVERR_SLOT);
    return;
  }
  const int64_t block = slot / kBlock;
  const int32_t offset = static_cast<int32_t>(slot % kBlock);
  const int32_t units_per_row = head_dim / 8;
  const int32_t units = num_kv_heads * units_per_row;
  for (int32_t u = threadIdx.x; u < units; u += blockDim.x) {
    const int32_t h = u / units_per_row;
    const int32_t within = u % units_per_row;
    const int64_t dst = ((block * num_kv_heads + h) * kBlock + offset) * head_dim + within * 8;
#pragma unroll
    for (int c = 0; c < 2; ++c) {
      const uint4 x = (c ? v : k)[static_cast<int64_t>(t) * units + u];
      *reinterpret_cast<uint2*>((c ? v_cache : k_cache) + dst) =
          bf16x8_to_fp8x8<kE5m2>(x, c ? v_scale : k_scale);
    }
  }
}

// ------------------------------------------------------------------ copy_blocks
// Grid: (pair, chunk, cache).  One thread moves one chunk of a block with the
// bulk-copy (TMA) engine: global -> shared, then shared -> global.
constexpr int kCopyChunk = 16384;

__global__ void __launch_bounds__(32)
    copy_blocks_kernel(uint8_t* __restrict__ k_cache, uint8_t* __restrict__ v_cache,
                       const int64_t* __restrict__ pairs, int64_t block_bytes,
                       int32_t num_blocks) {
  __shared__ __align__(128) uint8_t buf[kCopyChunk];
  __shared__ __align__(8) uint64_t bar;
  pdl_wait();
  pdl_trigger();
  if (threadIdx.x != 0) return;
  const int64_t src = pairs[2 * blockIdx.x];
  const int64_t dst = pairs[2 * blockIdx.x + 1];
  if (src < 0 || src >= num_blocks || dst < 0 || dst >= num_blocks) {
    if (blockIdx.y == 0 && blockIdx.z == 0) raise_error(PKV_DEVERR_PAIR);
    return;
  }
  const int64_t off = static_cast<int64_t>(blockIdx.y) * kCopyChunk;
  if (off >= block_bytes) return;
  const uint32_t bytes = static_cast<uint32_t>(
      block_bytes - off < kCopyChunk ? block_bytes - off : kCopyChunk);
  uint8_t* cache = blockIdx.z == 0 ? k_cache : v_cache;
  mbar_init(&bar, 1);
  fence_mbar_init();
  mbar_arrive_expect_tx(&bar, bytes);
  bulk_load(buf, cache + src * block_bytes + off, bytes, &bar);
  if (!mbar_wait(&bar, 0)) {
    // Timeout (flagged).  Give the load a last, shorter bound to land before
    // this CTA's shared memory is released; nothing was issued after it.
    mbar_wait(&bar, 0, kDrainLimitCycles);
    return;
  }
  fence_proxy_async_smem();
  bulk_store(cache + dst * block_bytes + off, buf, bytes);
  bulk_commit();
  bulk_wait_read_all();  // keep the shared buffer alive until the store has read it
}

// ------------------------------------------------------------ wait self-test
// One warp waits, with the same bounded wait the decode kernel uses, on an
// mbarrier phase that nothing completes.  The wait expires, raises
// PKV_DEVERR_TIMEOUT and the kernel returns normally.
__global__ void __launch_bounds__(32) wait_timeout_selftest_kernel() {
  __shared__ __align__(8) uint64_t bar;
  pdl_wait();
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
  }
  __syncwarp();
  mbar_wait(&bar, 0);
}

}  // namespace pkv
