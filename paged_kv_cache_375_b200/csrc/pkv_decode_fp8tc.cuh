// pkv_decode_fp8tc.cuh -- paged decode over FP8 (e4m3) pools on the tcgen05
// tensor cores.
//
// The same computation as decode_kernel over e4m3 pools (a sequence's context
// or one split-K partition of it, one kv head, the GQA group's query rows; the
// context found block by block through the table: ipipp.com vLLM article,
// section "二、PagedAttention分页原理深度剖析"), with the per-key arithmetic
// moved onto the tensor cores.  decode_kernel widens every code to f16 and runs
// the score and output products on mma.sync: about 270 instructions per
// 16-key tile, which bounds it well below the HBM roofline for one-byte codes.
// Here the codes stay codes: both products are tcgen05.mma kind::f8f6f4 with
// e4m3 operands straight from the TMA stages, over tiles of 128 keys (8 blocks):
//   S^T = K Bq^T   M 128 keys, N 32, K 128 (head_dim)   A = K tile (K-major)
//   O^T = V^T P    M 128 (head_dim), N 32, K 128 keys    A = V tile read MN-major
// The other operands are e4m3 too, each split into two terms so that about 8
// significant bits survive: Bq's 32 rows are 16 "high" rows hi_r = e4m3(c q_r)
// and 16 "low" rows e4m3(16 (c q_r - hi_r)) (c a power of two per query row
// that keeps |c q| <= 256; rows past the group are zero), and P's 32 columns
// are likewise 16 high and 16 low columns of the weights.  S and O therefore
// come out of tensor memory as 32 columns, and s = s_hi + s_lo / 16 (so for O).
//
// Units of up to 16 query rows (one token per sequence with up to 16 heads
// per kv head, or chunks of a few tokens, such as the draft tokens of a
// speculative step: row r = token r / g, head r % g, each token seeing the
// keys up to its own position).  Roles in a CTA of 8 warps
// (persistent over work units, the plan's items x kv heads; two CTAs per SM
// with three K and three V stages each):
//  * warp 0 (one lane) and warp 2 (one lane): TMA producers of the K and the V
//    tiles (one box per 16-token block, 128 one-byte codes wide), the next
//    tile's table entries read ahead.  The K producer also claims the units:
//    one grid-wide counter over the plan's longest-first list, so the CTAs
//    stay evenly loaded to the end; it passes each unit to the other roles
//    through a ring of unit indices in shared memory (full / empty mbarriers);
//  * warp 3: builds each unit's Bq (double-buffered) from the bf16 q rows;
//  * warp 1: tensor-memory allocation, the MMAs and their commits; it zeroes
//    the value rows past the context of a unit's last tile before P V (a zero
//    weight times a NaN code is NaN on a tensor core too);
//  * warps 4-7: thread t owns key t of every tile (TMEM lane t of S) and column
//    t of the output (TMEM lane t of O^T).  Per tile it forms the scaled
//    scores of the unit's rows against the lazily moved running maximum of
//    decode_kernel.  In a tile that every row sees whole, where no score
//    passes its row's maximum by more than the slack (2^8), the four warps
//    only exchange one flag; otherwise (a unit's first tile, a masked tile, a
//    maximum that moves) each row's maximum over the 128 keys is formed (a
//    reduce-scatter over the warp, then the four warps' maxima meet in shared
//    memory at a bounded mbarrier) and O^T is rescaled in tensor memory where
//    it moved.  The thread accumulates its own share of each row's weight
//    sum, writes its key's 32 P bytes and arrives.  At the end of a unit the sums
//    are reduced over the 128 threads and each thread writes its output
//    column (or the partial o / l, m, l of a split sequence).
// S is double-buffered in tensor memory, so the next tile's scores run on the
// tensor core while the softmax works on this tile's.
#pragma once

#include "pkv_decode.cuh"
#include "pkv_prefill.cuh"

namespace pkv {

constexpr int kTcKeys = 128;                     // keys per tile
constexpr int kTcBlocks = kTcKeys / kBlock;      // blocks per tile
constexpr int kTcRing = 8;                       // claimed units in flight
constexpr int kTcRows = 16;                      // query rows per unit, at most
constexpr int kTcN = 2 * kTcRows;                // MMA N: high and low terms
constexpr int kTcThreads = 256;
constexpr uint32_t kTcTmemCols = 128;            // S at columns 0 and 32, O^T at 64
constexpr uint32_t kTcTmemO = 64;
constexpr float kNoMax = 1e30f;                  // a running maximum not yet set

// ST = K stages = V stages.
template <int ST>
struct TcLayout {
  static constexpr int kTileBytes = kTcKeys * 128;             // 16 KB of codes
  static constexpr int kKOff = 0;
  static constexpr int kVOff = kKOff + ST * kTileBytes;
  static constexpr int kBqOff = kVOff + ST * kTileBytes;       // 2 x [32 rows][128 B]
  static constexpr int kBqBytes = kTcN * 128;
  static constexpr int kPOff = kBqOff + 2 * kBqBytes;            // [128 keys][32 B], 32-byte swizzle
  static constexpr int kPBytes = kTcKeys * kTcN;
  static constexpr int kXOff = kPOff + kPBytes;                  // exchange floats
  // xmax [2][4 warps][16], xsum [2][4][16], row scales [2][16]
  static constexpr int kXFloats = 2 * 4 * kTcRows + 2 * 4 * kTcRows + 2 * kTcRows;
  static constexpr int kRingOff = kXOff + kXFloats * 4;         // unit indices [kTcRing]
  static constexpr int kBarsOff = kRingOff + kTcRing * 4;
  // k_full[ST], k_empty[ST], v_full[ST], v_empty[ST], bq_full[2], bq_empty[2],
  // s_full[2], s_free[2], p_full, o_done, xbar, fin, ring_full[R], ring_empty[R]
  static constexpr int kNumBars = 4 * ST + 8 + 4 + 2 * kTcRing;
  static constexpr int kMiscOff = kBarsOff + kNumBars * 8;
  static constexpr int kTotal = kMiscOff + 16 + 1024;
};

// Shared-memory matrix descriptor, any layout (sm_100 format; see
// umma_desc_sw128): layout 2 = 128-byte swizzle, 6 = 32-byte swizzle.
__device__ __forceinline__ uint64_t umma_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo,
                                              uint64_t layout) {
  return static_cast<uint64_t>((saddr >> 4) & 0x3fffu) |
         (static_cast<uint64_t>((lbo >> 4) & 0x3fffu) << 16) |
         (static_cast<uint64_t>((sbo >> 4) & 0x3fffu) << 32) | (1ull << 46) | (layout << 61);
}

// D[tmem] (+)= A * B, kind::f8f6f4 (both operands e4m3 here), fp32 accumulate.
__device__ __forceinline__ void umma_f8(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                        uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Instruction descriptor of kind::f8f6f4 -> fp32 (bits 4-5 = 1): A's format
// in bits 7-9 (0 e4m3, 1 e5m2; the instruction takes A's and B's formats
// separately), B e4m3 (bits 10-12 = 0), A / B major (bits 15 / 16: 1 =
// MN-major), N >> 3 in bits 17-22, M >> 4 in bits 24-28.
__host__ __device__ constexpr uint32_t umma_idesc_f8(int M, int N, int a_fmt, bool a_mn,
                                                     bool b_mn) {
  return (1u << 4) | (static_cast<uint32_t>(a_fmt) << 7) | (a_mn ? (1u << 15) : 0u) |
         (b_mn ? (1u << 16) : 0u) | (static_cast<uint32_t>(N >> 3) << 17) |
         (static_cast<uint32_t>(M >> 4) << 24);
}

// The weights p0, p1 of two rows as two-term e4m3 codes, formed in f16x2: the
// high pair hi = e4m3(p) and the low pair e4m3(16 (p - hi)), p0 in the low
// byte of each.  p - hi is exact in f16 (hi is p rounded to 4 significant
// bits), so the pair keeps about 8 bits of each weight, as through f32.
__device__ __forceinline__ void p_codes2(float p0, float p1, uint32_t& hc, uint32_t& lc) {
  asm("{\n\t.reg .b32 ph, hv, dl, k16;\n\t.reg .b16 h, l;\n\t"
      "cvt.rn.f16x2.f32 ph, %3, %2;\n\t"
      "cvt.rn.satfinite.e4m3x2.f16x2 h, ph;\n\t"
      "cvt.rn.f16x2.e4m3x2 hv, h;\n\t"
      "mov.b32 k16, 0x4C004C00;\n\t"
      "sub.rn.f16x2 dl, ph, hv;\n\t"
      "mul.rn.f16x2 dl, dl, k16;\n\t"
      "cvt.rn.satfinite.e4m3x2.f16x2 l, dl;\n\t"
      "cvt.u32.u16 %0, h;\n\t"
      "cvt.u32.u16 %1, l;\n\t}"
      : "=r"(hc), "=r"(lc)
      : "f"(p0), "f"(p1));
}

// 16 consecutive fp32 columns of this thread's TMEM lane: load (waited for in
// the same statement) and store.
__device__ __forceinline__ void tmem_ld16_wait(uint32_t taddr, float (&v)[16]) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
      "%11, %12, %13, %14, %15}, [%16];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15])
      : "r"(taddr)
      : "memory");
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const float (&v)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
      "%11, %12, %13, %14, %15, %16};" ::"r"(taddr),
      "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])),
      "r"(__float_as_uint(v[3])), "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])),
      "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])), "r"(__float_as_uint(v[8])),
      "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])), "r"(__float_as_uint(v[11])),
      "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])), "r"(__float_as_uint(v[14])),
      "r"(__float_as_uint(v[15]))
      : "memory");
}

// A work unit: planned item x kv head.  Its rows: q_len query tokens (rows
// q_start .. of q and out, the last q_len positions of the context) x the
// group's heads, row r = token r / g, head r % g; at most 16.
struct TcUnit {
  int32_t seq, kv_head, part, len, nparts, blk_begin, nblk, ntiles;
  int32_t end;    // keys at positions < end belong to the unit (its partition's end)
  int32_t q_start, q_len;
};

__device__ __forceinline__ TcUnit tc_unit(const DecodeParams& prm, int32_t u) {
  const PlanItem pi = prm.items[u / prm.num_kv_heads];
  TcUnit w;
  w.seq = pi.seq;
  w.kv_head = u % prm.num_kv_heads;
  w.part = pi.part;
  w.len = pi.len;
  w.nparts = pi.nparts;
  w.blk_begin = pi.blk0;
  w.q_start = pi.seq;
  int32_t q_len = 1;
  if (prm.query_start_loc) {
    // a chunk of several tokens: the scheduler's checks of decode_kernel
    const int32_t q0 = prm.query_start_loc[pi.seq];
    q_len = prm.query_start_loc[pi.seq + 1] - q0;
    const int32_t cap = pi.len < prm.max_query_len ? pi.len : prm.max_query_len;
    const bool first = w.kv_head == 0 && pi.part == 0;
    if (q_len < 0 || q_len > cap) {
      if (first) raise_error(PKV_DEVERR_LEN);
      q_len = q_len < 0 ? 0 : cap;
    }
    if (q0 < 0 || q0 + q_len > prm.num_q_tokens) {
      if (first) raise_error(PKV_DEVERR_LEN);
      q_len = 0;
    }
    w.q_start = q0;
  }
  w.q_len = q_len;
  int32_t nblk = (pi.len + kBlock - 1) / kBlock - pi.blk0;
  nblk = nblk < prm.part_blocks ? nblk : prm.part_blocks;
  w.nblk = (nblk < 0 || q_len == 0) ? 0 : nblk;
  w.ntiles = (w.nblk + kTcBlocks - 1) / kTcBlocks;
  const int32_t part_end = (w.blk_begin + w.nblk) * kBlock;
  w.end = w.len < part_end ? w.len : part_end;
  return w;
}

// One halving step of a reduce-scatter of per-row values over the warp
// (maxima, or sums if SUM): lanes with bit `off` set keep the upper HALF rows,
// the others the lower, each combining them with its partner's copy.
template <int HALF, bool SUM>
__device__ __forceinline__ void scatter_step(float* v, int lane, int off, int& row) {
  const bool upper = lane & off;
#pragma unroll
  for (int i = 0; i < HALF; ++i) {
    const float send = upper ? v[i] : v[HALF + i];
    const float keep = upper ? v[HALF + i] : v[i];
    const float other = __shfl_xor_sync(0xffffffffu, send, off);
    v[i] = SUM ? keep + other : fmaxf(keep, other);
  }
  if (upper) row += HALF;
}

// The maxima (or sums if SUM) of RM rows over the warp's 32 lanes, in RM - 1
// + log2(32 / RM) shuffles: afterwards every lane holds the result for row
// `row`, and the lanes whose low bits (below 32 / RM) are zero are the first
// of each row.
template <int RM, bool SUM = false>
__device__ __forceinline__ float scatter_reduce(const float (&z)[RM], int lane, int& row) {
  float v[RM];
#pragma unroll
  for (int i = 0; i < RM; ++i) v[i] = z[i];
  row = 0;
  int off = 16;
  if constexpr (RM >= 16) { scatter_step<8, SUM>(v, lane, off, row); off >>= 1; }
  if constexpr (RM >= 8) { scatter_step<4, SUM>(v, lane, off, row); off >>= 1; }
  if constexpr (RM >= 4) { scatter_step<2, SUM>(v, lane, off, row); off >>= 1; }
  if constexpr (RM >= 2) { scatter_step<1, SUM>(v, lane, off, row); off >>= 1; }
  float r = v[0];
  for (; off > 0; off >>= 1) {
    const float other = __shfl_xor_sync(0xffffffffu, r, off);
    r = SUM ? r + other : fmaxf(r, other);
  }
  return r;
}

// RM: query rows the softmax handles (4, 8 or 16, at least the unit's rows); the
// operand layouts hold 16 high and 16 low rows.  ST: K and V stages per CTA,
// three, with two CTAs per SM.
template <int RM>
constexpr int tc_stages() { return 3; }

// AF: the pools' code format, A of both products (0 e4m3, 1 e5m2).
template <int RM, int AF, int ST = tc_stages<RM>()>
__global__ void __launch_bounds__(kTcThreads, 2)
    decode_fp8tc_kernel(const __grid_constant__ CUtensorMap tmap_k,
                        const __grid_constant__ CUtensorMap tmap_v, const DecodeParams prm) {
  static_assert(RM == 4 || RM == 8 || RM == 16, "4, 8 or 16 query rows per unit");
  static_assert(AF == 0 || AF == 1, "e4m3 or e5m2 pools");
  using Lay = TcLayout<ST>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                           ~static_cast<uintptr_t>(1023));
  uint8_t* sK = sm + Lay::kKOff;
  uint8_t* sV = sm + Lay::kVOff;
  uint8_t* sBq = sm + Lay::kBqOff;
  uint8_t* sP = sm + Lay::kPOff;
  float* xmax = reinterpret_cast<float*>(sm + Lay::kXOff);  // [2][4][16]
  float* xsum = xmax + 2 * 4 * kTcRows;                      // [2][4][16]
  // [Bq buffer][row]: the score scale of the row in log2 units over its c, 0
  // for rows past the unit's
  float* row_sc = xsum + 2 * 4 * kTcRows;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + Lay::kBarsOff);
  uint64_t* k_full = bars;
  uint64_t* k_empty = k_full + ST;
  uint64_t* v_full = k_empty + ST;
  uint64_t* v_empty = v_full + ST;
  uint64_t* bq_full = v_empty + ST;
  uint64_t* bq_empty = bq_full + 2;
  uint64_t* s_full = bq_empty + 2;
  uint64_t* s_free = s_full + 2;
  uint64_t* p_full = s_free + 2;
  uint64_t* o_done = p_full + 1;
  uint64_t* xbar = o_done + 1;
  uint64_t* fin = xbar + 1;
  uint64_t* ring_full = fin + 1;
  uint64_t* ring_empty = ring_full + kTcRing;
  int32_t* ring = reinterpret_cast<int32_t*>(sm + Lay::kRingOff);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + Lay::kMiscOff);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int i = 0; i < ST; ++i) {
      mbar_init(&k_full[i], 1);
      mbar_init(&k_empty[i], 1);
      mbar_init(&v_full[i], 1);
      mbar_init(&v_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bq_full[i], 1);
      mbar_init(&bq_empty[i], 5);  // the unit's last scores (a commit) + the 4 softmax warps
      mbar_init(&s_full[i], 1);
      mbar_init(&s_free[i], 4);
    }
    mbar_init(p_full, 4);
    mbar_init(o_done, 1);
    mbar_init(xbar, 4);
    mbar_init(fin, 1);
    for (int i = 0; i < kTcRing; ++i) {
      mbar_init(&ring_full[i], 1);
      mbar_init(&ring_empty[i], 7);  // V producer, Bq builder, MMA warp, 4 softmax warps
    }
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kTcTmemCols);
    tmem_relinquish();
  }
  pdl_wait();  // the plan and the cache writes before this launch are complete
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int32_t hkv = prm.num_kv_heads;
  const int32_t total = static_cast<int32_t>(prm.counters[1]) * hkv;
  const int g = prm.group;
  // the n-th claimed unit, from the ring (all lanes of a warp; lane 0
  // releases the slot); u < 0 after the last
  auto take_unit = [&](uint32_t n, int32_t& u) -> bool {
    const int slot = n % kTcRing;
    if (!warp_wait(&ring_full[slot], (n / kTcRing) & 1)) return false;
    u = ring[slot];
    __syncwarp();
    if (lane == 0) mbar_arrive(&ring_empty[slot]);
    return true;
  };

  if (warp == 0 || warp == 2) {
    // ===================================================== TMA producers
    if (lane == 0) {
      const bool is_k = warp == 0;
      const CUtensorMap* map = is_k ? &tmap_k : &tmap_v;
      uint8_t* stage_base = is_k ? sK : sV;
      uint64_t* full_bar = is_k ? k_full : v_full;
      uint64_t* empty_bar = is_k ? k_empty : v_empty;
      prefetch_tensormap(map);
      auto read_rows = [&](const TcUnit& w, int32_t j, int32_t (&rows)[kTcBlocks],
                           int32_t& nb) {
        const int32_t* table = prm.block_tables +
                               static_cast<int64_t>(w.seq) * prm.max_blocks_per_seq + w.blk_begin;
        nb = min(kTcBlocks, w.nblk - j * kTcBlocks);
#pragma unroll
        for (int b = 0; b < kTcBlocks; ++b) rows[b] = b < nb ? table[j * kTcBlocks + b] : 0;
      };
      // Units are claimed from the grid-wide counter, largest first (the plan
      // sorts its items by size), by the K producer, which passes each one
      // on through the ring; every other role takes them from the ring in
      // the same order, so that no CTA is left with a long tail of work.
      uint32_t rn = 0;
      auto next_unit = [&](TcUnit& w) -> bool {  // the next unit with tiles
        for (;;) {
          const int slot = rn % kTcRing;
          int32_t u;
          if (is_k) {
            const uint32_t ui = atomicAdd(&prm.counters[0], 1u);
            u = ui < static_cast<uint32_t>(total) ? static_cast<int32_t>(ui) : -1;
            if (u < 0) {
              // this CTA's last claim: the last CTA of the grid to get here
              // rearms the counters for the next run of the same plan
              __threadfence();
              if (atomicAdd(&prm.counters[2], 1u) == gridDim.x - 1) {
                prm.counters[0] = 0u;
                prm.counters[2] = 0u;
              }
            }
            if (rn >= kTcRing && !mbar_wait(&ring_empty[slot], ((rn / kTcRing) + 1) & 1))
              return false;
            ring[slot] = u;
            mbar_arrive(&ring_full[slot]);
          } else {
            if (!mbar_wait(&ring_full[slot], (rn / kTcRing) & 1)) return false;
            u = ring[slot];
            mbar_arrive(&ring_empty[slot]);
          }
          ++rn;
          if (u < 0) return false;
          w = tc_unit(prm, u);
          if (w.ntiles > 0) return true;
        }
      };
      // the stream of (unit, tile), the next tile's table entries read ahead
      TcUnit w{};
      int32_t j = 0;
      bool more = next_unit(w);
      int32_t rows[kTcBlocks], nb = 0;
      if (more) read_rows(w, 0, rows, nb);
      uint32_t c = 0;
      while (more) {
        int32_t jn = j + 1;
        TcUnit wn = w;
        bool more_n = true;
        if (jn >= w.ntiles) {
          jn = 0;
          more_n = next_unit(wn);
        }
        int32_t rows_n[kTcBlocks], nb_n = 0;
        if (more_n) read_rows(wn, jn, rows_n, nb_n);
        const int st = c % ST;
        if (c >= ST && !mbar_wait(&empty_bar[st], ((c / ST) + 1) & 1)) break;
        mbar_arrive_expect_tx(&full_bar[st], static_cast<uint32_t>(nb) * (kBlock * 128));
        for (int b = 0; b < nb; ++b) {
          int32_t pb = rows[b];
          if (pb < 0 || pb >= prm.num_blocks) {
            if (is_k) raise_error(PKV_DEVERR_BLOCK);
            pb = 0;
          }
          tma_load_2d(stage_base + st * Lay::kTileBytes + b * (kBlock * 128), map, 0,
                      (pb * hkv + w.kv_head) * kBlock, &full_bar[st]);
        }
        ++c;
        more = more_n;
        j = jn;
        w = wn;
        nb = nb_n;
#pragma unroll
        for (int b = 0; b < kTcBlocks; ++b) rows[b] = rows_n[b];
      }
    }
  } else if (warp == 3) {
    // ===================================================== Bq builder
    uint32_t n = 0;
    bool ok = true;
    for (; ok; ++n) {
      int32_t u;
      if (!take_unit(n, u)) { ok = false; break; }
      if (u < 0) break;
      const TcUnit w = tc_unit(prm, u);
      const int b = n & 1;
      if (n >= 2 && !warp_wait(&bq_empty[b], ((n >> 1) + 1) & 1)) { ok = false; break; }
      uint8_t* bq = sBq + b * Lay::kBqBytes;
      {
        // the unit's row `row` (token row / g, head row % g), its codes 0-63
        // from lane row and 64-127 from lane 16 + row: high terms in row
        // `row` of Bq, low in 16 + row
        const int row = lane & (kTcRows - 1), part = lane >> 4;
        float c = 1.f;
        const bool live = row < w.q_len * g;
        const size_t qrow = live ? static_cast<size_t>(w.q_start + row / g) * prm.num_q_heads +
                                       w.kv_head * g + row % g
                                 : 0;
        const uint4* src = reinterpret_cast<const uint4*>(
                               static_cast<const __nv_bfloat16*>(prm.q) + qrow * 128) +
                           part * 8;
        float mx = 0.f;
        if (live) {
#pragma unroll 4
          for (int i = 0; i < 8; ++i) {
            const uint4 v = src[i];
            const uint32_t vv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int k = 0; k < 4; ++k)
              mx = fmaxf(mx, fmaxf(fabsf(bf16lo_to_f32(vv[k])), fabsf(bf16hi_to_f32(vv[k]))));
          }
        }
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));  // the row's other half
        // c = 2^(7 - e) with mx = f 2^e, f in [0.5, 1): |c q| < 128
        if (live && mx > 0.f && isfinite(mx)) {
          int e;
          frexpf(mx, &e);
          c = ldexpf(1.f, 7 - e);
        }
        // 16 codes (one 16-byte chunk of each of the two rows) per step, two
        // per conversion; rows of 128 codes with the 128-byte swizzle
#pragma unroll 2
        for (int cq = 0; cq < 4; ++cq) {
          const int ch = part * 4 + cq;
          uint32_t hi[4] = {0u, 0u, 0u, 0u}, lo[4] = {0u, 0u, 0u, 0u};
          if (live) {
#pragma unroll
            for (int half = 0; half < 2; ++half) {
              const uint4 v = src[2 * cq + half];
              const uint32_t vv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
              for (int k = 0; k < 4; ++k) {
                const float x0 = bf16lo_to_f32(vv[k]) * c, x1 = bf16hi_to_f32(vv[k]) * c;
                const uint32_t hc = f32x2_to_e4m3x2(x0, x1);
                const uint32_t hv = e4m3x2_to_f16x2(hc);
                const uint32_t lc = f32x2_to_e4m3x2((x0 - f16lo_to_f32(hv)) * 16.f,
                                                    (x1 - f16hi_to_f32(hv)) * 16.f);
                const int byte = half * 8 + 2 * k;  // even: the pair fills half a word
                hi[byte >> 2] |= hc << (8 * (byte & 3));
                lo[byte >> 2] |= lc << (8 * (byte & 3));
              }
            }
          }
          *reinterpret_cast<uint4*>(bq + swz128(row, ch * 16)) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
          *reinterpret_cast<uint4*>(bq + swz128(kTcRows + row, ch * 16)) =
              make_uint4(lo[0], lo[1], lo[2], lo[3]);
        }
        if (part == 0) row_sc[b * kTcRows + row] = live ? prm.qk_scale_log2 / c : 0.f;
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bq_full[b]);
    }
  } else if (warp == 1) {
    // ===================================================== MMA issue
    constexpr uint32_t idesc_s = umma_idesc_f8(kTcKeys, kTcN, AF, false, false);
    constexpr uint32_t idesc_o = umma_idesc_f8(128, kTcN, AF, true, true);
    const uint32_t k_base = smem_addr(sK), v_base = smem_addr(sV);
    const uint32_t bq_base = smem_addr(sBq), p_base = smem_addr(sP);
    uint32_t n = 0, c = 0, sc = 0, pc = 0;
    bool ok = true;
    for (; ok; ++n) {
      int32_t u;
      if (!take_unit(n, u)) { ok = false; break; }
      if (u < 0) break;
      const TcUnit w = tc_unit(prm, u);
      const int b = n & 1;
      if (!warp_wait(&bq_full[b], (n >> 1) & 1)) { ok = false; break; }
      const uint32_t c0 = c;
      if (w.ntiles == 0) {
        if (lane == 0) umma_commit(&bq_empty[b]);
        __syncwarp();
      }
      // Two streams of MMAs, issued as their inputs arrive: the scores of
      // tile ns (up to two tiles ahead: S has two buffers) once its K stage
      // is full and its S buffer free, and P V of tile np once P and the V
      // stage are ready.  Neither waits behind the other, so a late K tile
      // does not hold back the P V that the softmax needs before its next P.
      // The warp polls (every lane tests, so each one has observed a phase
      // before it touches the data behind it); a poll that sees no progress
      // for kWaitLimitCycles flags a timeout.
      int32_t ns = 0, np = 0;
      long long idle_since = -1;
      while (np < w.ntiles) {
        bool progress = false;
        if (np < ns) {
          const uint32_t cc = c0 + np;
          const int st = cc % ST;
          if (__all_sync(0xffffffffu, mbar_test(p_full, pc & 1) &&
                                          mbar_test(&v_full[st], (cc / ST) & 1))) {
            ++pc;
            // keys of this tile inside the context; P V runs over whole 32-key
            // steps, the value rows past the context within them are zeroed first
            const int32_t valid = min(kTcKeys, w.end - (w.blk_begin + np * kTcBlocks) * kBlock);
            const int ksteps = (valid + 31) / 32;
            const int zero_end = ksteps * 32;
            uint8_t* vt = sV + st * Lay::kTileBytes;
            if (valid < zero_end) {
              for (int i = lane; i < (zero_end - valid) * 8; i += 32) {
                const int row = valid + i / 8, ch = i % 8;
                *reinterpret_cast<uint4*>(vt + row * 128 + ch * 16) = make_uint4(0u, 0u, 0u, 0u);
              }
              fence_proxy_async_smem();
              __syncwarp();
            }
            tc_fence_after();
            if (lane == 0) {
              for (int kk = 0; kk < ksteps; ++kk)
                umma_f8(tmem + kTcTmemO,
                        umma_desc(v_base + st * Lay::kTileBytes + kk * 4096, 16384, 1024, 2),
                        umma_desc(p_base + kk * 1024, 16, 256, 6), idesc_o,
                        (np > 0 || kk > 0) ? 1u : 0u);
              umma_commit(&v_empty[st]);
              umma_commit(o_done);
            }
            __syncwarp();
            ++np;
            progress = true;
          }
        }
        if (ns < w.ntiles && ns <= np + 2) {
          const uint32_t cc = c0 + ns;
          const int st = cc % ST;
          const int sb = sc & 1;
          if (__all_sync(0xffffffffu, mbar_test(&k_full[st], (cc / ST) & 1) &&
                                          (sc < 2 || mbar_test(&s_free[sb], ((sc >> 1) + 1) & 1)))) {
            tc_fence_after();
            if (lane == 0) {
#pragma unroll
              for (int ks = 0; ks < 4; ++ks)
                umma_f8(tmem + sb * kTcN,
                        umma_desc(k_base + st * Lay::kTileBytes + ks * 32, 16, 1024, 2),
                        umma_desc(bq_base + b * Lay::kBqBytes + ks * 32, 16, 1024, 2), idesc_s,
                        ks > 0 ? 1u : 0u);
              umma_commit(&s_full[sb]);
              umma_commit(&k_empty[st]);
              if (ns + 1 == w.ntiles) umma_commit(&bq_empty[b]);  // the unit's last scores read Bq
            }
            __syncwarp();
            ++sc;
            ++ns;
            progress = true;
          }
        }
        if (progress) {
          idle_since = -1;
        } else if (idle_since < 0) {
          idle_since = clock64();
        } else if (clock64() - idle_since > kWaitLimitCycles) {
          if (lane == 0) raise_error(PKV_DEVERR_TIMEOUT);
          ok = false;
          break;
        }
      }
      if (!ok) break;
      c = c0 + w.ntiles;
    }
    if (lane == 0) {
      umma_commit(fin);
      mbar_wait(fin, 0, kDrainLimitCycles);
    }
    __syncwarp();
  } else if (warp >= 4) {
    // ===================================================== softmax
    const int t = threadIdx.x - 128;  // key of a tile, and output column
    const int wi = warp - 4;
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(wi * 32) << 16);
    uint32_t n = 0, sc = 0, od = 0, xc = 0;
    bool ok = true;
    for (; ok; ++n) {
      int32_t u;
      if (!take_unit(n, u)) { ok = false; break; }
      if (u < 0) break;
      const TcUnit w = tc_unit(prm, u);
      const int rows = w.q_len * g;  // the unit's query rows
      const int b = n & 1;
      // nm: minus the running maximum (lazily moved, log2 units); kNoMax
      // marks a row without a visible key yet, and rows past the unit's
      // (zero rows of Bq, scale 0) are pinned so that they never move nor weigh
      float nm[RM], l[RM];
#pragma unroll
      for (int r = 0; r < RM; ++r) {
        nm[r] = r < rows ? kNoMax : -kNoMax;
        l[r] = 0.f;
      }
      // the unit's row scales, read from shared memory at every tile; the Bq
      // buffer is released at the end of the unit (and once the MMAs that
      // read it are done)
      if (!warp_wait(&bq_full[b], (n >> 1) & 1)) { ok = false; break; }
      const float* ic = row_sc + b * kTcRows;
      for (int32_t j = 0; j < w.ntiles; ++j) {
        const int sb = sc & 1;
        if (!warp_wait(&s_full[sb], (sc >> 1) & 1)) { ok = false; break; }
        ++sc;
        tc_fence_after();
        float s[kTcN];
        tmem_ld32_wait(lane_base + sb * kTcN, s);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&s_free[sb]);
        const int32_t pos0 = (w.blk_begin + j * kTcBlocks) * kBlock;  // the tile's first key
        // every key of the tile in the context and before the chunk: every
        // row sees all of them
        const bool full = pos0 + kTcKeys <= w.end && pos0 + kTcKeys - 1 <= w.len - w.q_len;
        float tt[RM];  // the scores, high and low terms joined
#pragma unroll
        for (int r = 0; r < RM; ++r) tt[r] = fmaf(s[kTcRows + r], 0.0625f, s[r]);
        // Common case: an unmasked tile in which no row's maximum moves by
        // more than the slack; the warps then only agree on that (one flag
        // each).  Otherwise (a unit's first tile, a masked tile, a moved
        // maximum) the rows' maxima over the tile are formed and exchanged.
        bool slow = j == 0 || !full;
        if (!slow) {
          bool up = false;
#pragma unroll
          for (int r = 0; r < RM; ++r) up |= fmaf(tt[r], ic[r], nm[r]) > kRescaleSlack;
          const bool wup = __any_sync(0xffffffffu, up);
          float* xf = xmax + (xc & 1) * 4 * kTcRows;
          if (lane == 0) xf[wi * kTcRows] = wup ? 1.f : 0.f;
          __syncwarp();
          if (lane == 0) mbar_arrive(xbar);
          if (!warp_wait(xbar, xc & 1)) { ok = false; break; }
          ++xc;
          slow = (xf[0] + xf[kTcRows]) + (xf[2 * kTcRows] + xf[3 * kTcRows]) != 0.f;
        }
        float dd[RM];  // scaled score minus the running maximum (log2 units)
        bool waited = false;
        if (!slow) {
#pragma unroll
          for (int r = 0; r < RM; ++r) dd[r] = fmaf(tt[r], ic[r], nm[r]);
        } else {
          // key pos is seen by the rows of tokens i >= pos - (len - q_len),
          // i.e. rows r >= thr (all rows for keys before the chunk)
          const int32_t pos = pos0 + t;
          const bool in_ctx = pos < w.end;
          const int32_t thr = (pos - (w.len - w.q_len)) * g;
          float z[RM];
#pragma unroll
          for (int r = 0; r < RM; ++r)
            z[r] = (in_ctx && r < rows && r >= thr) ? tt[r] * ic[r] : -INFINITY;
          // each row's maximum over the warp's 32 keys: reduce-scatter; then
          // the four warps' maxima meet in shared memory
          int row;
          const float v1 = scatter_reduce<RM>(z, lane, row);
          float* xm = xmax + (xc & 1) * 4 * kTcRows;
          if ((lane & (32 / RM - 1)) == 0) xm[wi * kTcRows + row] = v1;
          __syncwarp();
          if (lane == 0) mbar_arrive(xbar);
          if (!warp_wait(xbar, xc & 1)) { ok = false; break; }
          ++xc;
          float alpha[RM];
          bool any_grow = false;
#pragma unroll
          for (int r = 0; r < RM; ++r) {
            const float mt = fmaxf(fmaxf(xm[r], xm[kTcRows + r]),
                                   fmaxf(xm[2 * kTcRows + r], xm[3 * kTcRows + r]));
            const bool grow = mt > kRescaleSlack - nm[r];
            alpha[r] = grow ? fast_exp2(-(nm[r] + mt)) : 1.f;  // 0 without an earlier key
            if (grow) nm[r] = -mt;
            any_grow |= grow;
            l[r] *= alpha[r];
            dd[r] = z[r] + nm[r];  // -inf for masked keys
          }
          if (j > 0 && any_grow) {  // the same decision in every thread
            // O^T rescaled once the P V of the tile before has completed
            if (!warp_wait(o_done, od & 1)) { ok = false; break; }
            ++od;
            waited = true;
            tc_fence_after();
            // the high columns (0 .. 15), then the low ones
#pragma unroll 1
            for (int hl = 0; hl < 2; ++hl) {
              float o[16];
              tmem_ld16_wait(lane_base + kTcTmemO + hl * kTcRows, o);
#pragma unroll
              for (int r = 0; r < RM; ++r) o[r] *= alpha[r];
              tmem_st16(lane_base + kTcTmemO + hl * kTcRows, o);
            }
            tmem_wait_st();
          }
        }
        // this key's weights (at most 2^slack), high and low e4m3 terms, and
        // the running sums, two rows per conversion
        uint32_t ph[4] = {0u, 0u, 0u, 0u}, pl[4] = {0u, 0u, 0u, 0u};
#pragma unroll
        for (int r = 0; r < RM; r += 2) {
          const float p0 = fast_exp2(dd[r]), p1 = fast_exp2(dd[r + 1]);
          l[r] += p0;
          l[r + 1] += p1;
          uint32_t hc, lc;
          p_codes2(p0, p1, hc, lc);
          ph[r >> 2] |= hc << (8 * (r & 3));
          pl[r >> 2] |= lc << (8 * (r & 3));
        }
        if (j > 0 && !waited) {
          // P is single-buffered: the P V of the tile before must be done
          if (!warp_wait(o_done, od & 1)) { ok = false; break; }
          ++od;
          tc_fence_after();
        }
        // key t's row of P: [16 high | 16 low] bytes, 32-byte swizzle
        const uint32_t swz = (static_cast<uint32_t>(t) >> 2) & 1u;
        *reinterpret_cast<uint4*>(sP + t * kTcN + ((0u ^ swz) << 4)) =
            make_uint4(ph[0], ph[1], ph[2], ph[3]);
        *reinterpret_cast<uint4*>(sP + t * kTcN + ((1u ^ swz) << 4)) =
            make_uint4(pl[0], pl[1], pl[2], pl[3]);
        fence_proxy_async_smem();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(p_full);
      }
      if (!ok) break;
      __syncwarp();
      if (lane == 0) mbar_arrive(&bq_empty[b]);
      // ---- the unit's result ----
      // row sums over the 128 threads (each holds its keys' share): a
      // reduce-scatter over the warp, then the four warps' sums meet in
      // shared memory
      int srow;
      const float lw = scatter_reduce<RM, true>(l, lane, srow);
      float* xs = xsum + b * 4 * kTcRows;
      if ((lane & (32 / RM - 1)) == 0) xs[wi * kTcRows + srow] = lw;
      __syncwarp();
      if (lane == 0) mbar_arrive(xbar);
      if (!warp_wait(xbar, xc & 1)) { ok = false; break; }
      ++xc;
      // lane r < RM works out row r's sum, output factor and output row once;
      // the loop below takes them from that lane
      float l_my = 0.f, inv_my = 0.f;
      int64_t qrow_my = 0;
      if (lane < RM) {
        l_my = (xs[lane] + xs[kTcRows + lane]) + (xs[2 * kTcRows + lane] + xs[3 * kTcRows + lane]);
        inv_my = l_my > 0.f ? prm.out_scale / l_my : 0.f;
        qrow_my = static_cast<int64_t>(w.q_start + lane / g) * prm.num_q_heads +
                  w.kv_head * g + lane % g;
      }
      float o[32];
#pragma unroll
      for (int i = 0; i < 32; ++i) o[i] = 0.f;
      if (w.ntiles > 0) {
        if (!warp_wait(o_done, od & 1)) { ok = false; break; }
        ++od;
        tc_fence_after();
        tmem_ld32_wait(lane_base + kTcTmemO, o);
      }
#pragma unroll
      for (int r = 0; r < RM; ++r) {
        if (r < rows) {  // the same in every thread
          const size_t qrow = static_cast<size_t>(__shfl_sync(0xffffffffu, qrow_my, r));
          const float inv = __shfl_sync(0xffffffffu, inv_my, r);
          const float acc = fmaf(o[kTcRows + r], 0.0625f, o[r]);
          if (w.nparts == 1) {
            reinterpret_cast<uint16_t*>(prm.out)[qrow * 128 + t] =
                static_cast<uint16_t>(pack_bf16x2(acc * inv, 0.f));
          } else {
            const size_t prow = qrow * prm.max_parts + w.part;
            const float lr = __shfl_sync(0xffffffffu, l_my, r);
            prm.part_o[prow * 128 + t] = acc * inv;
            if (t == 0) {
              prm.part_ml[prow * 2 + 0] = nm[r] >= kNoMax ? -INFINITY : -nm[r] * kLn2;
              prm.part_ml[prow * 2 + 1] = lr;
            }
          }
        }
      }
      tc_fence_before();
    }
  }
  pdl_trigger();
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTcTmemCols);
  }
}

}  // namespace pkv
