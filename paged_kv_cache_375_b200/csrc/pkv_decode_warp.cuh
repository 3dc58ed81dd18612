// pkv_decode_warp.cuh -- paged decode of short work items, one warp per item.
//
// The same computation as decode_kernel (a sequence's partition of the
// context, one kv head, the GQA group's query rows; ipipp.com vLLM article,
// section "二、PagedAttention分页原理深度剖析": every block found through the
// table), scheduled differently.  decode_kernel spreads each item over all
// eight decode warps of a CTA and merges their states through shared memory
// at the end of the item, which suits long items.  When the plan's items are
// short -- 512-token split-K partitions, or a sequence's own blocks after a
// shared prefix -- that per-item merge and its barrier dominate.  Here every
// warp is a worker of its own:
//  * it takes work units (planned item x kv head) from the plan's counter,
//    one ahead, copies the item's table slice into its own shared memory and
//    loads the item's q rows with one bulk copy per query token;
//  * it owns S tile stages and is its own TMA producer, running ahead across
//    item boundaries;
//  * the tile math is decode_kernel's bf16 path (S^T = K Q^T and O^T += V^T P^T
//    on mma.sync, lazily rescaled online softmax);
//  * at the end of the item it writes the normalised output (single pass) or
//    the partial (o / l, m, l) straight from its registers: no merge between
//    warps, no barrier across the CTA.
// bf16 pools, head_dim 128, one query token per sequence (decode, chunks of
// one token, the shared-prefix plan), items of at most kWarpItemMaxBlocks
// blocks.
#pragma once

#include <type_traits>

#include "pkv_decode.cuh"

namespace pkv {

constexpr int kWarpItemMaxBlocks = 128;  // longest item (blocks) the warp kernel takes

template <int GMAX, int W, int S>
struct WarpDecodeLayout {
  static constexpr int D = 128;
  static constexpr int kTileBytes = kBlock * D * 2;        // one bf16 K (or V) tile: 4 KB
  static constexpr int kStageBytes = 2 * kTileBytes;       // K and V
  static constexpr int kQBytes = GMAX * D * 2;             // the item's query rows
  static constexpr int kTableBytes = 2 * kWarpItemMaxBlocks * 4;  // current and next item
  // per warp: [S stages][q rows][2 table slices]; a multiple of 1024 bytes, so
  // every warp's stages stay 1024-byte aligned (128-byte swizzled TMA boxes)
  static constexpr int kWarpBytes = S * kStageBytes + kQBytes + kTableBytes;
  static_assert(kWarpBytes % 1024 == 0, "per-warp area must keep 1024-byte alignment");
  static constexpr int kBarsOff = W * kWarpBytes;             // full[W][S], qbar[W]
  static constexpr int kTotal = kBarsOff + (W * S + W) * 8 + 1024;  // + alignment slack
};

// One work unit of a decode or shared-prefix plan, as the scheduler of
// decode_kernel derives it (one query token per sequence; a shared-prefix
// item serves one token of each of q_len consecutive sequences).
struct WarpItem {
  int32_t seq, kv_head, part, len, nparts, blk_begin, nblk, q_start, q_len;
};

__device__ __forceinline__ WarpItem warp_item(const DecodeParams& prm, uint32_t widx) {
  const int32_t hkv = prm.num_kv_heads;
  const PlanItem pi = prm.items[widx / hkv];
  WarpItem it;
  it.seq = pi.seq;
  it.kv_head = static_cast<int32_t>(widx % hkv);
  it.part = pi.part;
  it.len = pi.len;
  it.nparts = pi.nparts;
  it.blk_begin = pi.blk0;
  it.q_start = pi.seq;
  it.q_len = 1;
  if (pi.q_start >= 0) {
    it.q_start = pi.q_start;
    it.q_len = pi.q_len;
    if (it.q_len < 0 || it.q_len > prm.group_tokens || it.q_start + it.q_len > prm.num_q_tokens) {
      if (it.kv_head == 0) raise_error(PKV_DEVERR_GROUP);
      it.q_start = 0;
      it.q_len = 0;
    }
  } else if (prm.query_start_loc) {
    // chunks of at most one token (max_query_len 1): the same checks as the
    // scheduler of decode_kernel
    it.q_start = prm.query_start_loc[pi.seq];
    it.q_len = prm.query_start_loc[pi.seq + 1] - it.q_start;
    const int32_t cap = pi.len < prm.max_query_len ? pi.len : prm.max_query_len;
    const bool first = it.kv_head == 0 && pi.part == 0;
    if (it.q_len < 0 || it.q_len > cap) {
      if (first) raise_error(PKV_DEVERR_LEN);
      it.q_len = it.q_len < 0 ? 0 : cap;
    }
    if (it.q_start < 0 || it.q_start + it.q_len > prm.num_q_tokens) {
      if (first) raise_error(PKV_DEVERR_LEN);
      it.q_start = 0;
      it.q_len = 0;
    }
  }
  int32_t nblk = (it.len + kBlock - 1) / kBlock - it.blk_begin;
  nblk = nblk < prm.part_blocks ? nblk : prm.part_blocks;
  it.nblk = (nblk < 0 || it.q_len == 0) ? 0 : nblk;
  return it;
}

template <int GMAX, int W, int S>
__global__ void __launch_bounds__(W * 32, 1)
    decode_warp_kernel(const __grid_constant__ CUtensorMap tmap_k,
                       const __grid_constant__ CUtensorMap tmap_v, const DecodeParams prm) {
  using Lay = WarpDecodeLayout<GMAX, W, S>;
  constexpr int D = 128;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  uint8_t* stages = smem + warp * Lay::kWarpBytes;
  uint8_t* qbuf = stages + S * Lay::kStageBytes;
  int32_t* tabs = reinterpret_cast<int32_t*>(qbuf + Lay::kQBytes);  // [2][kWarpItemMaxBlocks]
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + Lay::kBarsOff) + warp * S;
  uint64_t* qbar = reinterpret_cast<uint64_t*>(smem + Lay::kBarsOff) + W * S + warp;
  if (lane == 0) {
    for (int i = 0; i < S; ++i) mbar_init(&full[i], 1);
    mbar_init(qbar, 1);
    fence_mbar_init();
  }
  __syncwarp();
  pdl_wait();  // the plan and the cache writes before this launch are complete

  const int g = prm.group;
  const int32_t hkv = prm.num_kv_heads;
  const uint32_t total = prm.counters[1] * static_cast<uint32_t>(hkv);
  const float sc = prm.qk_scale_log2;
  const int r = lane >> 2, qd = (lane & 3) * 2;

  // ---- work units: fetched one ahead ----
  auto fetch = [&](WarpItem& it, int slot) -> bool {
    uint32_t widx = 0;
    if (lane == 0) widx = atomicAdd(&prm.counters[0], 1u);
    widx = __shfl_sync(0xffffffffu, widx, 0);
    if (widx >= total) {
      // this warp's last fetch: the last warp of the grid to get here rearms
      // the counters for the next run of the same plan
      if (lane == 0) {
        __threadfence();
        if (atomicAdd(&prm.counters[2], 1u) == gridDim.x * W - 1) {
          prm.counters[0] = 0u;
          prm.counters[2] = 0u;
        }
      }
      pdl_trigger();
      return false;
    }
    it = warp_item(prm, widx);
    const int32_t* src = prm.block_tables + static_cast<size_t>(it.seq) * prm.max_blocks_per_seq +
                         it.blk_begin;
    int32_t* dst = tabs + slot * kWarpItemMaxBlocks;
    for (int32_t j = lane; j < it.nblk; j += 32) dst[j] = src[j];
    __syncwarp();
    return true;
  };
  uint32_t qi = 0;               // q loads issued
  auto load_q = [&](const WarpItem& it) {
    ++qi;
    if (lane == 0) {
      const uint32_t row_bytes = static_cast<uint32_t>(g * D * 2);
      if (it.q_len > 0) {
        mbar_arrive_expect_tx(qbar, row_bytes * it.q_len);
        for (int32_t i = 0; i < it.q_len; ++i) {
          const uint8_t* src = reinterpret_cast<const uint8_t*>(prm.q) +
                               (static_cast<size_t>(it.q_start + i) * prm.num_q_heads +
                                it.kv_head * g) * D * 2;
          bulk_load(qbuf + i * row_bytes, src, row_bytes, qbar);
        }
      } else {
        mbar_arrive(qbar);
      }
    }
  };

  WarpItem cur{}, nxt{};
  int cur_slot = 0;
  bool has_cur = fetch(cur, 0);
  bool has_nxt = has_cur && fetch(nxt, 1);
  if (has_cur) load_q(cur);

  // ---- producer over the block stream: cur's blocks, then nxt's ----
  uint32_t pctr = 0, cctr = 0;   // blocks issued / consumed
  int p_which = 0;               // 0: issuing cur's blocks, 1: nxt's
  int32_t p_blk = 0;
  uint32_t stage_ok = 0;         // bit s: stage s holds a valid tile
  auto produce = [&]() {
    while (pctr < cctr + S) {
      const bool on_cur = p_which == 0;
      if (on_cur ? !has_cur : !has_nxt) return;
      const WarpItem& it = on_cur ? cur : nxt;
      if (p_blk >= it.nblk) {
        if (!on_cur) return;     // never more than one item ahead
        p_which = 1;
        p_blk = 0;
        continue;
      }
      const int s_idx = pctr % S;
      const int slot = on_cur ? cur_slot : cur_slot ^ 1;
      const int32_t entry = tabs[slot * kWarpItemMaxBlocks + p_blk];
      const bool valid = entry >= 0 && entry < prm.num_blocks;
      stage_ok = valid ? (stage_ok | (1u << s_idx)) : (stage_ok & ~(1u << s_idx));
      if (lane == 0) {
        uint8_t* kdst = stages + s_idx * Lay::kStageBytes;
        uint8_t* vdst = kdst + Lay::kTileBytes;
        if (valid) {
          mbar_arrive_expect_tx(&full[s_idx], 2 * Lay::kTileBytes);
          const int32_t y = (entry * hkv + it.kv_head) * kBlock;
#pragma unroll
          for (int c = 0; c < 2; ++c) {
            tma_load_2d(kdst + c * (kBlock * 128), &tmap_k, c * 64, y, &full[s_idx]);
            tma_load_2d(vdst + c * (kBlock * 128), &tmap_v, c * 64, y, &full[s_idx]);
          }
        } else {
          raise_error(PKV_DEVERR_BLOCK);
          mbar_arrive(&full[s_idx]);
        }
      }
      ++p_blk;
      ++pctr;
    }
  };

  bool ok = true;
  uint32_t qc = 0;               // q loads consumed
  // One item with a state of G rows (G = 8 for items of at most 8 query rows,
  // so a 16-row kernel does not spend half its MMAs and exponentials on empty
  // rows; else GMAX).
  auto run_item = [&](auto rows_tag) {
    constexpr int G = decltype(rows_tag)::value;
    using Sg = Bf16State<D, G>;
    Sg st;
    const int rows = cur.q_len * g;
    bf16_begin_item<D, G>(st, qbuf, rows, g, cur.len, 1, lane);
    __syncwarp();                // every lane has its q fragments: the buffer is free
    if (has_nxt) load_q(nxt);
    for (int32_t b = 0; b < cur.nblk; b += 2) {
      const int n = b + 1 < cur.nblk ? 2 : 1;
      if (pctr < cctr + n) produce();
      int valid[2] = {0, 0};
      const uint8_t* kt[2];
#pragma unroll
      for (int x = 0; x < 2; ++x) {
        const uint32_t k = cctr + (x < n ? x : 0);
        const int s_idx = k % S;
        if (x < n && !mbar_wait(&full[s_idx], (k / S) & 1)) ok = false;
        kt[x] = stages + s_idx * Lay::kStageBytes;
        if (x < n && ((stage_ok >> s_idx) & 1u)) {
          const int v = cur.len - (cur.blk_begin + b + x) * kBlock;
          valid[x] = v > kBlock ? kBlock : v;
        }
      }
      if (!ok) return;
      const int pos0 = (cur.blk_begin + b) * kBlock;
      if (rows > 0)
        bf16_step<D, G>(st, kt[0], kt[0] + Lay::kTileBytes, valid[0], pos0, kt[1],
                        kt[1] + Lay::kTileBytes, valid[1], pos0 + kBlock, sc, lane);
      __syncwarp();
      cctr += n;
      produce();
    }
    // ---- the item's result, straight from the fragments: row n = nh*8 + qd + hc,
    // column d = 16 mt + r (and + 8) ----
#pragma unroll
    for (int nh = 0; nh < Sg::NH; ++nh)
#pragma unroll
      for (int hc = 0; hc < 2; ++hc) {
        const int n = nh * 8 + qd + hc;
        if (n < rows) {
          const float l = st.lsum[nh][hc];
          const float inv = l > 0.f ? prm.out_scale / l : 0.f;
          const size_t row = static_cast<size_t>(cur.q_start + n / g) * prm.num_q_heads +
                             cur.kv_head * g + n % g;
          if (cur.nparts == 1) {
            uint16_t* o16 = reinterpret_cast<uint16_t*>(prm.out) + row * D;
#pragma unroll
            for (int mt = 0; mt < Sg::MT; ++mt) {
              o16[mt * 16 + r] = static_cast<uint16_t>(pack_bf16x2(st.o[nh][mt][hc] * inv, 0.f));
              o16[mt * 16 + r + 8] =
                  static_cast<uint16_t>(pack_bf16x2(st.o[nh][mt][hc + 2] * inv, 0.f));
            }
          } else {
            const size_t prow = row * prm.max_parts + cur.part;
            float* po = prm.part_o + prow * D;
#pragma unroll
            for (int mt = 0; mt < Sg::MT; ++mt) {
              po[mt * 16 + r] = st.o[nh][mt][hc] * inv;
              po[mt * 16 + r + 8] = st.o[nh][mt][hc + 2] * inv;
            }
            if (r == 0) {
              const float m = st.m[nh][hc];
              prm.part_ml[prow * 2 + 0] = m == -INFINITY ? -INFINITY : m * kLn2;
              prm.part_ml[prow * 2 + 1] = l;
            }
          }
        }
      }
  };
  while (has_cur) {
    produce();
    if (!mbar_wait(qbar, qc & 1)) { ok = false; break; }
    ++qc;
    if (GMAX > 8 && cur.q_len * g <= 8) {
      run_item(std::integral_constant<int, 8>{});
    } else {
      run_item(std::integral_constant<int, GMAX>{});
    }
    if (!ok) break;
    // ---- next item ----
    if (!has_nxt) break;
    cur = nxt;
    cur_slot ^= 1;
    // the producer either is on nxt already (keep its block) or has issued all
    // of the old item's blocks and not moved on (start the new one at 0)
    if (p_which == 0) p_blk = 0;
    p_which = 0;
    has_nxt = fetch(nxt, cur_slot ^ 1);
  }
  if (!ok) {
    // A wait gave up: wait (bounded) for the copies this warp still has in flight.
    for (uint32_t k = cctr; k < pctr; ++k) {
      mbar_wait(&full[k % S], (k / S) & 1, kDrainLimitCycles);
    }
    for (uint32_t k = qc; k < qi; ++k) mbar_wait(qbar, k & 1, kDrainLimitCycles);
  }
}

}  // namespace pkv
