// pkv_prefill.cuh -- causal chunks of many query tokens over the paged cache,
// on the 5th-generation tensor cores (tcgen05.mma, accumulators in TMEM).
//
// What is computed is the multi-token attention of the decode library: the n
// new tokens of a sequence are the last n positions of its context L (written
// into their slots first, "vLLM" wiki entry, section "Flattened 布局与
// slot_mapping"), and chunk token i attends to keys 0 .. L - n + i through the
// block table, visited block by block (ipipp.com vLLM article, section
// "二、PagedAttention分页原理深度剖析").  Long chunks are what chunked prefill
// produces (vampireachao.github.io "vllm", section "第二层：请求不该排队等整批").
//
// Why a second kernel: the decode kernel serves at most 16 query rows per kv
// head per work item, so a chunk of n tokens re-reads its keys and values
// ceil(n*g/16) times on mma.sync.  Here a work unit is a tile of 128 query rows
// of one kv head (row r = token i * g + head h of the GQA group, i.e.
// floor(128/g) consecutive chunk tokens with all g heads): every KV tile is
// read once per 128 rows, and the products run on tcgen05 at M = 128:
//   S  = Q K^T   (M 128 rows, N 128 keys, K = head_dim)   into TMEM
//   O += P V     (M 128 rows, N = head_dim, K = 128 keys) into TMEM
//
// Roles in a CTA of 13 warps (one CTA per SM, persistent over work units):
//  * warps 0, 3 (K) and 2, 12 (V), one lane each: TMA producers.  Warp 0
//    loads the unit's Q tile (a 3-D tensor map over q [T][Hq][D], box {64 d,
//    g heads, tokens}); per KV tile of 128 keys, warps 0 and 3 load blocks 0-3
//    and 4-7 of K through the block table (the 2-D pool map, one box per
//    block and 64-column half), warps 2 and 12 the same of V.  Stages are
//    128-byte swizzled, laid out [half][128 keys][128 B]; a K stage is
//    released when its scores are computed, a V stage when its P V is.
//  * warp 1: TMEM allocation; one lane issues the MMAs and commits them to
//    mbarriers, polling two streams (the scores of the next tiles, P V of the
//    tile whose P is ready) so that neither waits behind the other; the warp
//    zeroes the value rows past the context in the last block of the context
//    (NaN padding times a zero weight is still NaN on a tensor core).
//  * warps 4-11 (two warpgroups; warp w reads TMEM lanes 32(w%4) ...): softmax.
//    Query row r belongs to one thread of each warpgroup, which take keys 0-63
//    and 64-127 of every tile.  Each reads its 64 scores from TMEM, masks keys
//    past the row's causal limit, swaps its maximum with its partner through
//    shared memory, keeps a running maximum in log2 units that moves only when
//    it grows by more than 8 (the output row in TMEM is then rescaled, each
//    thread its half of the columns), writes its half of P in bf16 pairs into
//    tensor memory (the A operand of P V) and sums its weights.  At the end the
//    two sums are added, and each thread reads its half of the output row from
//    TMEM, divides by the sum and stores bf16.
// TMEM: S double-buffered at columns 0 and 128 (the MMA of the next tile's
// scores runs while the softmax works on this tile's), O at 256, P
// double-buffered at 384 and 448 (the softmax writes the next tile's P while
// the tensor core still reads this one's).
#pragma once

#include "pkv_device.cuh"

namespace pkv {

constexpr int kPfRows = 128;       // query rows per tile: the MMA's M
constexpr int kPfKeys = 128;       // keys per KV tile: N of S = Q K^T, K of O += P V
constexpr int kPfBlocksPerTile = kPfKeys / kBlock;
constexpr int kPfKStages = 3;      // K tile stages (a K stage frees as soon as its scores are done)
constexpr int kPfVStages = 2;      // V tile stages
constexpr int kPfThreads = 416;    // warps 0, 3 (K) and 2, 12 (V) producers, warp 1 MMA,
                                   // warps 4-11 softmax
constexpr int kPfKProducers = 2;
constexpr int kPfVProducers = 2;
constexpr int kPfSoftmaxWarps = 8;  // two warpgroups: keys 0-63 and 64-127 of every row
constexpr int kPfMaxSeqs = 2048;   // sequences per call (per-CTA tile prefix in shared memory)
constexpr uint32_t kPfTmemCols = 512;  // S buffers at columns 0 and 128, O at 256, P at 384 and 448
constexpr uint32_t kPfTmemO = 2 * kPfKeys;        // O: head_dim columns of fp32
constexpr uint32_t kPfTmemP = 3 * kPfKeys;        // P: two buffers of bf16 pairs, kPfKeys / 2 columns each
constexpr float kPfRescaleSlack = 8.f; // the running max moves when it grows by more (log2)

struct PrefillParams {
  void* out;                       // bf16 [num_q_tokens][Hq][D]
  const int32_t* block_tables;     // [B][max_blocks_per_seq]
  const int32_t* context_lens;     // [B]
  const int32_t* query_start_loc;  // [B + 1]
  int32_t num_seqs, num_q_tokens, num_q_heads, num_kv_heads, group;
  int32_t tokens_per_tile;         // floor(128 / group)
  int32_t max_blocks_per_seq, num_blocks, max_len;
  float qk_scale_log2;             // scale * log2(e)
};

// Shared-memory layout (offsets from a 1024-byte aligned base).
template <int D>
struct PfLayout {
  static constexpr int kHalves = D / 64;                       // 128-byte column halves
  static constexpr int kQBytes = kHalves * kPfRows * 128;      // [half][128 rows][128 B]
  static constexpr int kKvBytes = kHalves * kPfKeys * 128;     // one K (or V) stage
  static constexpr int kQOff = 0;
  static constexpr int kKOff = kQOff + kQBytes;
  static constexpr int kVOff = kKOff + kPfKStages * kKvBytes;
  static constexpr int kPrefixOff = kVOff + kPfVStages * kKvBytes;
  static constexpr int kBarsOff = kPrefixOff + (kPfMaxSeqs + 8) * 4;
  // q_full, q_empty, k_full[SK], k_empty[SK], v_full[SV], v_empty[SV], s_full[2],
  // s_free[2], p_full[2], pv_done[2], final, xchg[4] (the two softmax warps of each row
  // quarter)
  static constexpr int kNumBars = 2 + 2 * kPfKStages + 2 * kPfVStages + 4 + 5 + 4;
  static constexpr int kMiscOff = kBarsOff + kNumBars * 8;     // tmem base, abort flag
  // row maxima exchanged between the two softmax warpgroups: [parity][half][row],
  // then the row sums [half][row]
  static constexpr int kXchgOff = kMiscOff + 16;
  static constexpr int kTotal = kXchgOff + (4 + 2) * kPfRows * 4 + 1024;  // + alignment slack
};

// ------------------------------------------------------------ tcgen05 helpers
__device__ __forceinline__ void tmem_alloc(uint32_t* dst_smem, uint32_t cols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                   smem_addr(dst_smem)),
               "r"(cols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t cols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(cols)
               : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// D[tmem] (+)= A[smem] * B[smem]^T per the instruction descriptor; bf16 in,
// fp32 accumulate.  Issued by one thread.
__device__ __forceinline__ void umma_f16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                         uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// The same with A in tensor memory (M rows on the lanes, two 16-bit
// elements per 32-bit column along K).
__device__ __forceinline__ void umma_f16_tmem_a(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc,
                                                uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// The barrier's arrival fires once every MMA this thread issued before has
// completed.
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::
                   "r"(smem_addr(bar))
               : "memory");
}

// 32 consecutive fp32 columns of this thread's TMEM lane (warp w of a
// warpgroup reads lanes 32(w%4) .. 32(w%4)+31), loaded and waited for in one
// statement.
__device__ __forceinline__ void tmem_ld32_wait(uint32_t taddr, float (&v)[32]) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr)
      : "memory");
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

// 64 consecutive fp32 columns of this thread's TMEM lane, loaded and waited
// for in one statement.
__device__ __forceinline__ void tmem_ld64_wait(uint32_t taddr, float (&v)[64]) {
  uint32_t r[64];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x64.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32, %33, %34, %35, %36, %37, %38, %39, %40, %41, %42, %43, %44, %45, %46, %47, %48, %49, %50, %51, %52, %53, %54, %55, %56, %57, %58, %59, %60, %61, %62, %63}, [%64];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31]), "=r"(r[32]), "=r"(r[33]), "=r"(r[34]), "=r"(r[35]), "=r"(r[36]), "=r"(r[37]), "=r"(r[38]), "=r"(r[39]), "=r"(r[40]), "=r"(r[41]), "=r"(r[42]), "=r"(r[43]), "=r"(r[44]), "=r"(r[45]), "=r"(r[46]), "=r"(r[47]), "=r"(r[48]), "=r"(r[49]), "=r"(r[50]), "=r"(r[51]), "=r"(r[52]), "=r"(r[53]), "=r"(r[54]), "=r"(r[55]), "=r"(r[56]), "=r"(r[57]), "=r"(r[58]), "=r"(r[59]), "=r"(r[60]), "=r"(r[61]), "=r"(r[62]), "=r"(r[63])
      : "r"(taddr)
      : "memory");
#pragma unroll
  for (int i = 0; i < 64; ++i) v[i] = __uint_as_float(r[i]);
}

// 128 consecutive fp32 columns of this thread's TMEM lane, loaded and waited
// for in one statement, so no use of the registers can precede the wait.
__device__ __forceinline__ void tmem_ld128_wait(uint32_t taddr, float (&v)[128]) {
  uint32_t r[128];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x128.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32, %33, %34, %35, %36, %37, %38, %39, %40, %41, %42, %43, %44, %45, %46, %47, %48, %49, %50, %51, %52, %53, %54, %55, %56, %57, %58, %59, %60, %61, %62, %63, %64, %65, %66, %67, %68, %69, %70, %71, %72, %73, %74, %75, %76, %77, %78, %79, %80, %81, %82, %83, %84, %85, %86, %87, %88, %89, %90, %91, %92, %93, %94, %95, %96, %97, %98, %99, %100, %101, %102, %103, %104, %105, %106, %107, %108, %109, %110, %111, %112, %113, %114, %115, %116, %117, %118, %119, %120, %121, %122, %123, %124, %125, %126, %127}, [%128];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31]), "=r"(r[32]), "=r"(r[33]), "=r"(r[34]), "=r"(r[35]), "=r"(r[36]), "=r"(r[37]), "=r"(r[38]), "=r"(r[39]), "=r"(r[40]), "=r"(r[41]), "=r"(r[42]), "=r"(r[43]), "=r"(r[44]), "=r"(r[45]), "=r"(r[46]), "=r"(r[47]), "=r"(r[48]), "=r"(r[49]), "=r"(r[50]), "=r"(r[51]), "=r"(r[52]), "=r"(r[53]), "=r"(r[54]), "=r"(r[55]), "=r"(r[56]), "=r"(r[57]), "=r"(r[58]), "=r"(r[59]), "=r"(r[60]), "=r"(r[61]), "=r"(r[62]), "=r"(r[63]), "=r"(r[64]), "=r"(r[65]), "=r"(r[66]), "=r"(r[67]), "=r"(r[68]), "=r"(r[69]), "=r"(r[70]), "=r"(r[71]), "=r"(r[72]), "=r"(r[73]), "=r"(r[74]), "=r"(r[75]), "=r"(r[76]), "=r"(r[77]), "=r"(r[78]), "=r"(r[79]), "=r"(r[80]), "=r"(r[81]), "=r"(r[82]), "=r"(r[83]), "=r"(r[84]), "=r"(r[85]), "=r"(r[86]), "=r"(r[87]), "=r"(r[88]), "=r"(r[89]), "=r"(r[90]), "=r"(r[91]), "=r"(r[92]), "=r"(r[93]), "=r"(r[94]), "=r"(r[95]), "=r"(r[96]), "=r"(r[97]), "=r"(r[98]), "=r"(r[99]), "=r"(r[100]), "=r"(r[101]), "=r"(r[102]), "=r"(r[103]), "=r"(r[104]), "=r"(r[105]), "=r"(r[106]), "=r"(r[107]), "=r"(r[108]), "=r"(r[109]), "=r"(r[110]), "=r"(r[111]), "=r"(r[112]), "=r"(r[113]), "=r"(r[114]), "=r"(r[115]), "=r"(r[116]), "=r"(r[117]), "=r"(r[118]), "=r"(r[119]), "=r"(r[120]), "=r"(r[121]), "=r"(r[122]), "=r"(r[123]), "=r"(r[124]), "=r"(r[125]), "=r"(r[126]), "=r"(r[127])
      : "r"(taddr)
      : "memory");
#pragma unroll
  for (int i = 0; i < 128; ++i) v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const float (&v)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
      "%11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, "
      "%28, %29, %30, %31, %32};" ::"r"(taddr),
      "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])),
      "r"(__float_as_uint(v[3])), "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])),
      "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])), "r"(__float_as_uint(v[8])),
      "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])), "r"(__float_as_uint(v[11])),
      "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])), "r"(__float_as_uint(v[14])),
      "r"(__float_as_uint(v[15])), "r"(__float_as_uint(v[16])), "r"(__float_as_uint(v[17])),
      "r"(__float_as_uint(v[18])), "r"(__float_as_uint(v[19])), "r"(__float_as_uint(v[20])),
      "r"(__float_as_uint(v[21])), "r"(__float_as_uint(v[22])), "r"(__float_as_uint(v[23])),
      "r"(__float_as_uint(v[24])), "r"(__float_as_uint(v[25])), "r"(__float_as_uint(v[26])),
      "r"(__float_as_uint(v[27])), "r"(__float_as_uint(v[28])), "r"(__float_as_uint(v[29])),
      "r"(__float_as_uint(v[30])), "r"(__float_as_uint(v[31]))
      : "memory");
}

__device__ __forceinline__ void tmem_st32u(uint32_t taddr, const uint32_t (&v)[32]) {
  float f[32];
#pragma unroll
  for (int i = 0; i < 32; ++i) f[i] = __uint_as_float(v[i]);
  tmem_st32(taddr, f);
}

__device__ __forceinline__ void tmem_wait_st() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// Shared-memory matrix descriptor of a 128-byte swizzled operand (sm_100
// format: start >> 4 in bits 0-13, leading byte offset >> 4 in 16-29, stride
// byte offset >> 4 in 32-45, version 1 in 46-47, layout 2 = 128-byte swizzle
// in 61-63).  K-major tiles: rows of 128 B, 8-row groups `sbo` apart (the
// leading offset is unused and set to 16 B).  MN-major tiles: 64-element
// column groups `lbo` apart, 8-row groups of the K dimension `sbo` apart.
__device__ __forceinline__ uint64_t umma_desc_sw128(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  return static_cast<uint64_t>((saddr >> 4) & 0x3fffu) |
         (static_cast<uint64_t>((lbo >> 4) & 0x3fffu) << 16) |
         (static_cast<uint64_t>((sbo >> 4) & 0x3fffu) << 32) | (1ull << 46) | (2ull << 61);
}

// Instruction descriptor of kind::f16: fp32 accumulator (bits 4-5 = 1), A and
// B bf16 (bits 7-9 = 1, 10-12 = 1), A K-major (bit 15 = 0), B K-major or
// MN-major (bit 16), N >> 3 in bits 17-22, M >> 4 in bits 24-28.
__host__ __device__ constexpr uint32_t umma_idesc_bf16(int M, int N, bool b_mn_major) {
  return (1u << 4) | (1u << 7) | (1u << 10) | (b_mn_major ? (1u << 16) : 0u) |
         (static_cast<uint32_t>(N >> 3) << 17) | (static_cast<uint32_t>(M >> 4) << 24);
}

// 3-D tiled tensor load global -> shared, completing on `bar`; x innermost
// (16-byte aligned).
__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* map, int32_t x,
                                            int32_t y, int32_t z, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(smem_addr(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(smem_addr(bar))
      : "memory");
}

// A bounded wait whose outcome is the same for the whole warp (the TMEM loads
// and stores that follow are warp-collective).
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity) {
  return __all_sync(0xffffffffu, mbar_wait(bar, parity));
}

// ------------------------------------------------------------ work units
// A unit is (sequence s, query tile t, kv head).  Tiles of a sequence are
// counted from its last (the tile with the most keys) to its first.
struct PfUnit {
  int32_t seq, kv_head;
  int32_t L;          // context length (validated)
  int32_t q_len;      // chunk tokens of the sequence
  int32_t q_row0;     // flattened index of the tile's first query token
  int32_t tok0;       // chunk index of the tile's first token
  int32_t ntok;       // tokens of the tile
  int32_t nkv;        // keys the tile's rows can see: 0 .. nkv-1
  int32_t ntiles;     // KV tiles
};

__device__ __forceinline__ int32_t pf_tiles_of(int32_t q_len, int32_t tpt) {
  return (q_len + tpt - 1) / tpt;
}

// Length and chunk of sequence s after validation (invalid ones give an empty chunk
// and raise PKV_DEVERR_LEN).
__device__ __forceinline__ void pf_seq(const PrefillParams& p, int32_t s, int32_t& L,
                                       int32_t& q0, int32_t& q_len, bool flag) {
  L = p.context_lens[s];
  if (L < 0 || L > p.max_len) {
    if (flag) raise_error(PKV_DEVERR_LEN);
    L = L < 0 ? 0 : p.max_len;
  }
  q0 = p.query_start_loc[s];
  const int32_t q1 = p.query_start_loc[s + 1];
  q_len = q1 - q0;
  if (q0 < 0 || q1 > p.num_q_tokens || q_len < 0 || q_len > L) {
    if (flag) raise_error(PKV_DEVERR_LEN);
    q_len = 0;
  }
}

__device__ __forceinline__ PfUnit pf_unit(const PrefillParams& p, const int32_t* prefix,
                                          int32_t u) {
  PfUnit w;
  const int32_t idx = u / p.num_kv_heads;
  w.kv_head = u - idx * p.num_kv_heads;
  // last s with prefix[s] <= idx
  int32_t lo = 0, hi = p.num_seqs - 1;
  while (lo < hi) {
    const int32_t mid = (lo + hi + 1) >> 1;
    if (prefix[mid] <= idx) lo = mid; else hi = mid - 1;
  }
  w.seq = lo;
  int32_t q0;
  pf_seq(p, lo, w.L, q0, w.q_len, false);
  const int32_t tpt = p.tokens_per_tile;
  const int32_t nt = pf_tiles_of(w.q_len, tpt);
  const int32_t tile = nt - 1 - (idx - prefix[lo]);
  w.tok0 = tile * tpt;
  w.ntok = min(tpt, w.q_len - w.tok0);
  w.q_row0 = q0 + w.tok0;
  w.nkv = w.L - w.q_len + w.tok0 + w.ntok;   // last visible key + 1
  w.ntiles = (w.nkv + kPfKeys - 1) / kPfKeys;
  return w;
}

// ------------------------------------------------------------ the kernel
template <int D>
__global__ void __launch_bounds__(kPfThreads, 1)
    prefill_kernel(const __grid_constant__ CUtensorMap map_q,
                   const __grid_constant__ CUtensorMap map_k,
                   const __grid_constant__ CUtensorMap map_v, const PrefillParams p) {
  using Lay = PfLayout<D>;
  constexpr int H = Lay::kHalves;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                           ~static_cast<uintptr_t>(1023));
  uint8_t* sQ = sm + Lay::kQOff;
  uint8_t* sK = sm + Lay::kKOff;
  uint8_t* sV = sm + Lay::kVOff;
  int32_t* prefix = reinterpret_cast<int32_t*>(sm + Lay::kPrefixOff);
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + Lay::kBarsOff);
  uint64_t* q_full = bars;
  uint64_t* q_empty = bars + 1;
  uint64_t* k_full = bars + 2;
  uint64_t* k_empty = k_full + kPfKStages;
  uint64_t* v_full = k_empty + kPfKStages;
  uint64_t* v_empty = v_full + kPfVStages;
  uint64_t* s_full = v_empty + kPfVStages;
  uint64_t* s_free = s_full + 2;
  uint64_t* p_full = s_free + 2;
  // [tile & 1]: the softmax warps have written that tile's P.  One barrier per
  // P buffer: the warps of different row quarters may be a tile apart.
  uint64_t* pv_done = p_full + 2;  // [tile & 1]: that tile's P V has completed
  uint64_t* fin = pv_done + 2;
  uint64_t* xchg = fin + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + Lay::kMiscOff);
  volatile uint32_t* abort_flag = tmem_slot + 1;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    for (int i = 0; i < kPfKStages; ++i) {
      mbar_init(&k_full[i], kPfKProducers);  // every producer warp of the stream
      mbar_init(&k_empty[i], 1);
    }
    for (int i = 0; i < kPfVStages; ++i) {
      mbar_init(&v_full[i], kPfVProducers);
      mbar_init(&v_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&s_free[i], kPfSoftmaxWarps);
    }
    mbar_init(&p_full[0], kPfSoftmaxWarps);
    mbar_init(&p_full[1], kPfSoftmaxWarps);
    mbar_init(&pv_done[0], 1);
    mbar_init(&pv_done[1], 1);
    mbar_init(fin, 1);
    for (int i = 0; i < 4; ++i) mbar_init(&xchg[i], 2);
    *abort_flag = 0u;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kPfTmemCols);
    tmem_relinquish();
  }
  pdl_wait();
  // tile prefix over the sequences (every CTA builds its own copy)
  {
    const int B = p.num_seqs;
    const int per = (B + kPfThreads - 1) / kPfThreads;
    const int s0 = threadIdx.x * per;
    int32_t local = 0;
    for (int s = s0; s < s0 + per && s < B; ++s) {
      int32_t L, q0, ql;
      pf_seq(p, s, L, q0, ql, blockIdx.x == 0);
      local += pf_tiles_of(ql, p.tokens_per_tile);
    }
    // exclusive scan of the 256 thread sums
    int32_t incl = local;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int32_t n = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += n;
    }
    __shared__ int32_t warp_tot[kPfThreads / 32];
    if (lane == 31) warp_tot[warp] = incl;
    __syncthreads();
    int32_t base = 0;
    for (int w = 0; w < warp; ++w) base += warp_tot[w];
    int32_t run = base + incl - local;
    for (int s = s0; s < s0 + per && s < B; ++s) {
      prefix[s] = run;
      int32_t L, q0, ql;
      pf_seq(p, s, L, q0, ql, false);
      run += pf_tiles_of(ql, p.tokens_per_tile);
    }
    if (threadIdx.x == kPfThreads - 1) prefix[B] = run;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int32_t total_units = prefix[p.num_seqs] * p.num_kv_heads;
  const int g = p.group;
  const uint32_t qrow_bytes = 128u * static_cast<uint32_t>(g * p.tokens_per_tile);

  if (warp == 0 || warp == 2 || warp == 3 || warp == 12) {
    // ===================================================== TMA producers
    // Warps 0 and 3 (one lane each) load the K tiles, blocks 0-3 and 4-7 of
    // each, warp 0 also the Q tile; warps 2 and 12 load the V tiles the same
    // way.  A K stage is free once the tile's scores are computed, a V stage
    // only once its P V is, so the next K tiles are not held up behind the
    // current P V.  Two warps per stream: one warp issues tensor copies at
    // about 14 bytes a cycle, below what the tile pipeline consumes (four K
    // and three V warps measured slower again).  (Two lanes of one warp would
    // not do: while one waits on its barrier the other's path does not run.)
    if (lane == 0) {
      const bool is_k = warp == 0 || warp == 3;
      const int nprod = is_k ? kPfKProducers : kPfVProducers;
      const int part = (warp == 3 || warp == 12) ? 1 : 0;
      const CUtensorMap* map = is_k ? &map_k : &map_v;
      uint8_t* stage_base = is_k ? sK : sV;
      uint64_t* full_bar = is_k ? k_full : v_full;
      uint64_t* empty_bar = is_k ? k_empty : v_empty;
      const uint32_t nst = is_k ? kPfKStages : kPfVStages;
      if (is_k) prefetch_tensormap(&map_q);
      prefetch_tensormap(map);
      // The stream of (unit, KV tile) this CTA loads.  The block-table entries
      // of the next tile are read before waiting for a free stage, so their
      // latency is off the critical path.
      int32_t u = blockIdx.x, j = 0;
      PfUnit w{};
      if (u < total_units) w = pf_unit(p, prefix, u);
      auto read_rows = [&](const PfUnit& wu, int32_t jj, int32_t (&rows)[kPfBlocksPerTile],
                           int32_t& nblk) {
        const int32_t* table = p.block_tables + static_cast<int64_t>(wu.seq) * p.max_blocks_per_seq;
        const int32_t blk0 = jj * kPfBlocksPerTile;
        nblk = min(kPfBlocksPerTile, (wu.nkv - jj * kPfKeys + kBlock - 1) / kBlock);
#pragma unroll
        for (int b = 0; b < kPfBlocksPerTile; ++b) rows[b] = b < nblk ? table[blk0 + b] : 0;
      };
      int32_t rows[kPfBlocksPerTile], nblk = 0;
      if (u < total_units) read_rows(w, 0, rows, nblk);
      uint32_t qc = 0, kvc = 0;
      bool ok = true;
      while (u < total_units) {
        // the tile after this one (possibly the first of the next unit)
        int32_t un = u, jn = j + 1;
        PfUnit wn = w;
        if (jn >= w.ntiles) {
          un = u + gridDim.x;
          jn = 0;
          if (un < total_units) wn = pf_unit(p, prefix, un);
        }
        int32_t rows_n[kPfBlocksPerTile], nblk_n = 0;
        if (un < total_units) read_rows(wn, jn, rows_n, nblk_n);
        // this tile
        const int st = kvc % nst;
        if (kvc >= nst && !mbar_wait(&empty_bar[st], ((kvc / nst) + 1) & 1)) {
          ok = false;
          break;
        }
        // this warp's blocks of the tile: [8 part / nprod, 8 (part + 1) / nprod)
        const int b0 = part * kPfBlocksPerTile / nprod;
        const int b1 = min(nblk, (part + 1) * kPfBlocksPerTile / nprod);
        mbar_arrive_expect_tx(&full_bar[st],
                              static_cast<uint32_t>(max(b1 - b0, 0)) * H * (kBlock * 128));
        for (int b = b0; b < b1; ++b) {
          int32_t pb = rows[b];
          if (pb < 0 || pb >= p.num_blocks) {
            if (is_k) raise_error(PKV_DEVERR_BLOCK);
            pb = 0;
          }
          const int32_t y = (pb * p.num_kv_heads + w.kv_head) * kBlock;
#pragma unroll
          for (int h = 0; h < H; ++h)
            tma_load_2d(stage_base + st * Lay::kKvBytes + h * (kPfKeys * 128) +
                            b * (kBlock * 128),
                        map, h * 64, y, &full_bar[st]);
        }
        ++kvc;
        if (is_k && part == 0 && j == 0) {
          // the unit's Q tile, once the previous unit's last scores are done
          // (its first K tile is already on its way)
          if (qc > 0 && !mbar_wait(q_empty, (qc - 1) & 1)) { ok = false; break; }
          mbar_arrive_expect_tx(q_full, qrow_bytes * H);
#pragma unroll
          for (int h = 0; h < H; ++h)
            tma_load_3d(sQ + h * (kPfRows * 128), &map_q, h * 64, w.kv_head * g, w.q_row0,
                        q_full);
          ++qc;
        }
        u = un;
        j = jn;
        w = wn;
        nblk = nblk_n;
#pragma unroll
        for (int b = 0; b < kPfBlocksPerTile; ++b) rows[b] = rows_n[b];
      }
      if (!ok) *abort_flag = 1u;
    }
  } else if (warp == 1) {
    // ===================================================== MMA issue
    constexpr uint32_t idesc_s = umma_idesc_bf16(kPfRows, kPfKeys, false);
    constexpr uint32_t idesc_o = umma_idesc_bf16(kPfRows, D, true);
    const uint32_t q_base = smem_addr(sQ);
    const uint32_t k_base = smem_addr(sK), v_base = smem_addr(sV);
    uint32_t qc = 0, kvc = 0, sc = 0;
    bool ok = true;
    for (int32_t u = blockIdx.x; u < total_units && ok; u += gridDim.x) {
      const PfUnit w = pf_unit(p, prefix, u);
      if (!warp_wait(q_full, qc & 1)) { ok = false; break; }
      ++qc;
      const uint32_t kv0 = kvc;
      // Two streams of MMAs, issued as their inputs arrive: S_ns = Q K_ns^T
      // into S buffer sc % 2 (up to two tiles ahead of P V: S has two
      // buffers) and O += P_np V_np.  Neither waits behind the other, so a
      // finished P goes to the tensor core at once.  Every lane tests the
      // barriers, so each one has observed a phase before it touches the data
      // behind it; no progress for kWaitLimitCycles flags a timeout.
      int32_t ns = 0, np = 0;
      long long idle_since = -1;
      while (np < w.ntiles) {
        bool progress = false;
        if (np < ns) {
          const uint32_t c = kv0 + np;
          const int st = c % kPfVStages;
          if (__all_sync(0xffffffffu, mbar_test(&p_full[c & 1], (c >> 1) & 1) &&
                                          mbar_test(&v_full[st], (c / kPfVStages) & 1))) {
            const int32_t j = np;
            const int32_t nblk =
                min(kPfBlocksPerTile, (w.nkv - j * kPfKeys + kBlock - 1) / kBlock);
            // value rows past the context in the context's last block: zero them
            // (their weights are zero, but NaN or Inf there would still poison O)
            const int32_t last_blk = (w.L - 1) / kBlock;
            const int32_t tail = w.L % kBlock;
            if (tail != 0 && last_blk >= j * kPfBlocksPerTile &&
                last_blk < j * kPfBlocksPerTile + nblk) {
              const int b = last_blk - j * kPfBlocksPerTile;
              const int nrows = kBlock - tail;
              for (int i = lane; i < nrows * 8 * H; i += 32) {
                const int h = i / (nrows * 8);
                const int rr = (i / 8) % nrows + tail;
                const int chunk = i % 8;
                *reinterpret_cast<uint4*>(sV + st * Lay::kKvBytes + h * (kPfKeys * 128) +
                                          (b * kBlock + rr) * 128 + chunk * 16) =
                    make_uint4(0u, 0u, 0u, 0u);
              }
              fence_proxy_async_smem();
              __syncwarp();
            }
            tc_fence_after();
            if (lane == 0) {
              for (int b = 0; b < nblk; ++b) {
                // A = P from tensor memory: the 16 keys of block b are columns 8b .. 8b+7
                const uint32_t voff = b * (kBlock * 128);
                umma_f16_tmem_a(tmem + kPfTmemO,
                                tmem + kPfTmemP + (c & 1) * (kPfKeys / 2) + b * (kBlock / 2),
                                umma_desc_sw128(v_base + st * Lay::kKvBytes + voff,
                                                kPfKeys * 128, 1024),
                                idesc_o, (j > 0 || b > 0) ? 1u : 0u);
              }
              umma_commit(&v_empty[st]);
              umma_commit(&pv_done[c & 1]);
            }
            __syncwarp();
            ++np;
            progress = true;
          }
        }
        if (ns < w.ntiles && ns <= np + 2) {
          const uint32_t c = kv0 + ns;
          const int st = c % kPfKStages;
          const int sb = sc & 1;
          if (__all_sync(0xffffffffu, mbar_test(&k_full[st], (c / kPfKStages) & 1) &&
                                          (sc < 2 || mbar_test(&s_free[sb], ((sc >> 1) + 1) & 1)))) {
            tc_fence_after();
            if (lane == 0) {
#pragma unroll
              for (int ks = 0; ks < D / 16; ++ks) {
                const uint32_t off = (ks >> 2) * (kPfRows * 128) + (ks & 3) * 32;
                const uint32_t koff = (ks >> 2) * (kPfKeys * 128) + (ks & 3) * 32;
                umma_f16(tmem + sb * kPfKeys, umma_desc_sw128(q_base + off, 16, 1024),
                         umma_desc_sw128(k_base + st * Lay::kKvBytes + koff, 16, 1024), idesc_s,
                         ks > 0 ? 1u : 0u);
              }
              umma_commit(&s_full[sb]);
              umma_commit(&k_empty[st]);  // the K tile is free once the scores are
              if (ns + 1 == w.ntiles) umma_commit(q_empty);  // the unit's last S reads Q
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
      kvc = kv0 + w.ntiles;
    }
    if (!ok) *abort_flag = 1u;
    // every MMA issued has completed before TMEM is released
    if (lane == 0) {
      umma_commit(fin);
      mbar_wait(fin, 0, kDrainLimitCycles);
    }
    __syncwarp();
  } else if (warp >= 4) {
    // ===================================================== softmax
    // Warp w reads TMEM lanes 32 (w % 4) ..: thread r owns query row r; the
    // warpgroup `half` takes keys 64 half .. 64 half + 63 of every tile and
    // columns D/2 half .. of the output.  The partner warps (w and w + 4) swap
    // their row maxima each tile through shared memory, meeting at an mbarrier
    // (two arrivals, a bounded wait like every other).
    const int r = (warp & 3) * 32 + lane;  // query row of the tile = TMEM lane
    const int half = (warp - 4) >> 2;
    constexpr int KH = kPfKeys / 2;          // keys per half
    constexpr int DH = D / 2;                // output columns per half
    const uint32_t lane_base = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);
    float* xmax = reinterpret_cast<float*>(sm + Lay::kXchgOff);  // [2][2][128]
    float* xsum = xmax + 4 * kPfRows;                            // [2][128]
    uint64_t* my_xchg = &xchg[warp & 3];
    uint32_t xc = 0;  // uses of my_xchg
    const float sc_log2 = p.qk_scale_log2;
    const int32_t rows_used = g * p.tokens_per_tile;
    const int i_tok = r / g, h_in = r - (r / g) * g;
    uint32_t sc = 0;
    bool ok = true;
    for (int32_t u = blockIdx.x; u < total_units && ok; u += gridDim.x) {
      const PfUnit w = pf_unit(p, prefix, u);
      const bool row_ok = r < rows_used && i_tok < w.ntok;
      const int32_t lim = row_ok ? w.L - w.q_len + w.tok0 + i_tok : -1;  // last visible key
      // smallest limit over the warp's rows: tiles wholly below it need no mask
      int32_t lim_min = lim;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) lim_min = min(lim_min, __shfl_xor_sync(0xffffffffu, lim_min, o));
      float m = -INFINITY, l = 0.f;
      for (int32_t j = 0; j < w.ntiles; ++j) {
        const int sb = sc & 1;
        const uint32_t t = sc;  // this tile's place in the CTA's sequence of tiles
        if (!warp_wait(&s_full[sb], (sc >> 1) & 1)) { ok = false; break; }
        ++sc;
        tc_fence_after();
        float s[KH];
        tmem_ld64_wait(lane_base + sb * kPfKeys + half * KH, s);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&s_free[sb]);
        // scores in log2 units; keys past the row's causal limit (and past the
        // context, and past the blocks loaded for a short last tile) get -inf
        const int32_t pos0 = j * kPfKeys + half * KH;
        float mxp[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) mxp[e] = -INFINITY;
        float ks = 1.f;  // the part of the scale still to apply, inside the exponent
        if (pos0 + KH - 1 <= lim_min && sc_log2 >= 0.f) {
          // unmasked, scale >= 0: the maximum of the raw scores, scaled once;
          // each score's scaling joins its exponent's subtraction
#pragma unroll
          for (int c = 0; c < KH; ++c) mxp[c & 7] = fmaxf(mxp[c & 7], s[c]);  // eight chains
          ks = sc_log2;
        } else if (pos0 + KH - 1 <= lim_min) {
#pragma unroll
          for (int c = 0; c < KH; ++c) {
            s[c] *= sc_log2;
            mxp[c & 7] = fmaxf(mxp[c & 7], s[c]);
          }
        } else {
#pragma unroll
          for (int c = 0; c < KH; ++c) {
            s[c] = pos0 + c <= lim ? s[c] * sc_log2 : -INFINITY;
            mxp[c & 7] = fmaxf(mxp[c & 7], s[c]);
          }
        }
        float mx = fmaxf(fmaxf(fmaxf(mxp[0], mxp[1]), fmaxf(mxp[2], mxp[3])),
                         fmaxf(fmaxf(mxp[4], mxp[5]), fmaxf(mxp[6], mxp[7]))) * ks;
        // the row's maximum over both halves
        xmax[((j & 1) * 2 + half) * kPfRows + r] = mx;
        __syncwarp();
        if (lane == 0) mbar_arrive(my_xchg);
        if (!warp_wait(my_xchg, xc & 1)) { ok = false; break; }
        ++xc;
        mx = fmaxf(mx, xmax[((j & 1) * 2 + (half ^ 1)) * kPfRows + r]);
        const bool grow = mx > m + kPfRescaleSlack;
        const float alpha = grow ? fast_exp2(m - mx) : 1.f;  // 0 when m = -inf
        if (grow) m = mx;
        // P = 2^(s - m) in bf16 (packed pairs, in registers) and the sum of the
        // weights, before waiting for the previous tile's P V: the exponentials
        // overlap that MMA
        const float mu = m == -INFINITY ? 0.f : m;
        uint32_t pk[KH / 2];
        float lsp[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) lsp[e] = 0.f;
#pragma unroll
        for (int c = 0; c < KH / 2; ++c) {
          const float p0 = fast_exp2(fmaf(s[2 * c], ks, -mu));
          const float p1 = fast_exp2(fmaf(s[2 * c + 1], ks, -mu));
          pk[c] = pack_bf16x2(p0, p1);
          lsp[c & 7] += p0 + p1;
        }
        const float lsum = ((lsp[0] + lsp[1]) + (lsp[2] + lsp[3])) +
                           ((lsp[4] + lsp[5]) + (lsp[6] + lsp[7]));
        l = l * alpha + lsum;
        // P buffer t & 1 is free once P V of tile t - 2 has completed (tile k's
        // P V completes phase k / 2 of pv_done[k & 1]); O may be rescaled only
        // once P V of tile t - 1 has
        if (t >= 2) {
          if (!warp_wait(&pv_done[t & 1], ((t - 2) >> 1) & 1)) { ok = false; break; }
          tc_fence_after();
        }
        if (j > 0) {
          // rows whose maximum moved rescale their output columns (warp-uniform:
          // the other rows of the warp multiply by 1)
          if (__any_sync(0xffffffffu, grow)) {
            if (!warp_wait(&pv_done[(t - 1) & 1], ((t - 1) >> 1) & 1)) { ok = false; break; }
            tc_fence_after();
#pragma unroll 1
            for (int c = 0; c < DH / 32; ++c) {
              float o[32];
              tmem_ld32_wait(lane_base + kPfTmemO + half * DH + c * 32, o);
#pragma unroll
              for (int i = 0; i < 32; ++i) o[i] *= alpha;
              tmem_st32(lane_base + kPfTmemO + half * DH + c * 32, o);
            }
            tmem_wait_st();
          }
        }
        // this half's 64 keys of row r into tensor memory, two bf16 a column
        // (keys 2c and 2c+1 in column c, the lower key in the low half): the
        // A operand of P V
        tmem_st32u(lane_base + kPfTmemP + (t & 1) * (kPfKeys / 2) + half * (KH / 2), pk);
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&p_full[t & 1]);
      }
      if (!ok) break;
      if (w.ntiles > 0) {
        // the row's weight sum over both halves
        xsum[half * kPfRows + r] = l;
        __syncwarp();
        if (lane == 0) mbar_arrive(my_xchg);
        if (!warp_wait(my_xchg, xc & 1)) { ok = false; break; }
        ++xc;
        l += xsum[(half ^ 1) * kPfRows + r];
        // the unit's last P V (tile sc - 1)
        if (!warp_wait(&pv_done[(sc - 1) & 1], ((sc - 1) >> 1) & 1)) { ok = false; break; }
        tc_fence_after();
        const float inv = l > 0.f ? 1.f / l : 0.f;
        __nv_bfloat16* orow = static_cast<__nv_bfloat16*>(p.out) +
                              (static_cast<int64_t>(w.q_row0 + i_tok) * p.num_q_heads +
                               w.kv_head * g + h_in) * D + half * DH;
#pragma unroll 1
        for (int c = 0; c < DH / 32; ++c) {
          float o[32];
          tmem_ld32_wait(lane_base + kPfTmemO + half * DH + c * 32, o);
          if (row_ok) {
#pragma unroll
            for (int v4 = 0; v4 < 4; ++v4) {
              uint4 pkd;
              pkd.x = pack_bf16x2(o[8 * v4 + 0] * inv, o[8 * v4 + 1] * inv);
              pkd.y = pack_bf16x2(o[8 * v4 + 2] * inv, o[8 * v4 + 3] * inv);
              pkd.z = pack_bf16x2(o[8 * v4 + 4] * inv, o[8 * v4 + 5] * inv);
              pkd.w = pack_bf16x2(o[8 * v4 + 6] * inv, o[8 * v4 + 7] * inv);
              *reinterpret_cast<uint4*>(orow + c * 32 + v4 * 8) = pkd;
            }
          }
        }
        tc_fence_before();
      }
    }
    if (!ok) *abort_flag = 1u;
  }
  pdl_trigger();
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kPfTmemCols);
  }
}

}  // namespace pkv
