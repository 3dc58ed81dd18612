// pkv_api.cu -- host side of the C ABI declared in include/pkv.h: argument
// validation, work planning, TMA tensor-map encoding and kernel launches.
// Everything is one translation unit so the kernels share the device error
// word without relocatable device code.
#include <cudaTypedefs.h>

#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>
#include <vector>

#include "pkv.h"
#include "pkv_cache_ops.cuh"
#include "pkv_decode.cuh"
#include "pkv_decode_fp8tc.cuh"
#include "pkv_decode_warp.cuh"
#include "pkv_device.cuh"
#include "pkv_prefill.cuh"
#include "pkv_prepare.cuh"

namespace {

thread_local std::string g_last_error;

pkv_status fail(pkv_status st, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof buf, fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return st;
}

pkv_status cuda_fail(cudaError_t e, const char* what) {
  return fail(PKV_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

// Launch with programmatic stream serialisation, so the kernel can begin while
// the previous kernel in the stream drains (every kernel here waits for its
// prerequisites with griddepcontrol.wait before touching global memory).
template <typename... KArgs, typename... Args>
cudaError_t launch(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
                   cudaStream_t stream, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Make the device that owns `p` current for this library's runtime.  The
// library carries its own CUDA runtime, whose current device is independent
// of the caller's (e.g. PyTorch's), so every call that launches work binds
// the device of its output buffer first.  Also rejects host pointers.
pkv_status bind_device(const void* p, const char* what) {
  cudaPointerAttributes a;
  cudaError_t e = cudaPointerGetAttributes(&a, p);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return cuda_fail(e, "cudaPointerGetAttributes");
  }
  if (a.type != cudaMemoryTypeDevice && a.type != cudaMemoryTypeManaged)
    return fail(PKV_ERR_SHAPE, "%s is not device memory", what);
  int cur = -1;
  e = cudaGetDevice(&cur);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (cur != a.device) {
    e = cudaSetDevice(a.device);
    if (e != cudaSuccess) return cuda_fail(e, "cudaSetDevice");
  }
  return PKV_OK;
}

bool is_fp8(int t) { return t == PKV_FP8_E4M3 || t == PKV_FP8_E5M2; }
int elem_bytes(pkv_dtype t) { return t == PKV_BF16 ? 2 : (is_fp8(t) ? 1 : 4); }

// Checks shared by every call.  `need_seq` also checks the per-sequence fields.
pkv_status check_dims(const pkv_dims* d, bool need_seq) {
  if (!d) return fail(PKV_ERR_NULL, "dims is NULL");
  if (d->dtype != PKV_F32 && d->dtype != PKV_BF16 && !is_fp8(d->dtype))
    return fail(PKV_ERR_UNSUPPORTED, "dtype %d not supported (fp32, bf16, fp8 e4m3)",
                (int)d->dtype);
  if (is_fp8(d->dtype) && d->head_dim != 128)
    return fail(PKV_ERR_UNSUPPORTED, "FP8 caches need head_dim 128");
  if (d->block_size != pkv::kBlock)
    return fail(PKV_ERR_UNSUPPORTED, "block_size %d not supported (16)", d->block_size);
  if (d->head_dim != 64 && d->head_dim != 128)
    return fail(PKV_ERR_UNSUPPORTED, "head_dim %d not supported (64 or 128)", d->head_dim);
  if (d->num_kv_heads <= 0 || d->num_blocks <= 0)
    return fail(PKV_ERR_SHAPE, "num_kv_heads and num_blocks must be positive");
  // rows of the pool seen by the TMA tensor map must fit a signed 32-bit coordinate
  if (static_cast<int64_t>(d->num_blocks) * d->num_kv_heads * pkv::kBlock >= (1ll << 31))
    return fail(PKV_ERR_SHAPE, "num_blocks * num_kv_heads * 16 must be < 2^31");
  if (need_seq) {
    if (d->num_seqs < 0 || d->num_q_heads <= 0 || d->max_blocks_per_seq <= 0)
      return fail(PKV_ERR_SHAPE, "num_seqs >= 0, num_q_heads > 0, max_blocks_per_seq > 0 required");
    if (d->num_q_heads % d->num_kv_heads != 0)
      return fail(PKV_ERR_SHAPE, "num_q_heads %d is not a multiple of num_kv_heads %d",
                  d->num_q_heads, d->num_kv_heads);
    if (d->num_q_heads / d->num_kv_heads > 16)
      return fail(PKV_ERR_UNSUPPORTED, "query heads per kv head %d > 16",
                  d->num_q_heads / d->num_kv_heads);
  }
  return PKV_OK;
}

int device_sm_count() {
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 148;
  return sms > 0 ? sms : 148;
}

struct DecodePlan {
  int32_t part_tokens = 0;
  int32_t part_blocks = 0;
  int32_t max_parts = 0;
  int32_t max_len = 0;       // lengths above this are clamped (and flagged)
  int32_t num_q_tokens = 0;  // query rows of q and out (num_seqs for decode)
  // shared-prefix plans: sequences one shared-prefix item serves (x group <= 16 rows)
  bool shared = false;
  int32_t members_per_item = 0;
  size_t items_off = 0, part_o_off = 0, part_ml_off = 0, total = 0;
  size_t seq_prefix_off = 0, group_pref_off = 0;
};

size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Partition choice.  Aim at about 16 items of work per SM at the longest
// length: P = the power of two >= B*Hkv*max_len / (16*SMs), within
// [512, 8192] tokens.  When that covers the longest sequence the decode is
// single-pass (the planner then orders whole sequences longest first).
//
// Shared-prefix plans of bf16 head_dim-128 caches run on decode_warp_kernel,
// whose work is handed out per warp: there the aim is about 16 items per
// warp (eight per SM), so a long prefix is cut into several items that
// different warps read at once.
int32_t choose_partition(const pkv_dims* d, int32_t max_len, int32_t requested,
                         bool per_warp = false) {
  if (requested > 0) return requested;
  const int64_t units = static_cast<int64_t>(d->num_seqs) * d->num_kv_heads;
  const int64_t target = units * max_len / (16ll * device_sm_count() * (per_warp ? 8 : 1));
  int64_t p = 512;
  while (p < target && p < pkv::kMaxItemBlocks * pkv::kBlock) p *= 2;
  if (p >= max_len)
    return max_len < pkv::kBlock ? pkv::kBlock
                                 : static_cast<int32_t>(round_up(max_len, pkv::kBlock));
  return static_cast<int32_t>(p);
}

// num_q_tokens < 0: one query token per sequence (decode).  shared: the
// shared-prefix plan (decode only), whose sequences may have one partial more
// (the prefix is split from the rest at a block boundary) and whose work list
// holds up to two items per partial row.
pkv_status make_plan(const pkv_dims* d, int32_t max_context_len, int32_t partition_tokens,
                     DecodePlan* plan, int32_t num_q_tokens = -1, bool shared = false) {
  pkv_status st = check_dims(d, true);
  if (st != PKV_OK) return st;
  if (max_context_len < 0) return fail(PKV_ERR_SHAPE, "max_context_len must be >= 0");
  if (partition_tokens < 0 || partition_tokens % pkv::kBlock != 0)
    return fail(PKV_ERR_SHAPE, "partition_tokens must be 0 or a positive multiple of 16");
  if (partition_tokens > pkv::kMaxItemBlocks * pkv::kBlock)
    return fail(PKV_ERR_UNSUPPORTED, "partition_tokens must be <= %d",
                pkv::kMaxItemBlocks * pkv::kBlock);
  const int64_t table_len = static_cast<int64_t>(d->max_blocks_per_seq) * pkv::kBlock;
  const int32_t max_len =
      static_cast<int32_t>(max_context_len < table_len ? max_context_len : table_len);
  DecodePlan p;
  p.max_len = max_len;
  p.num_q_tokens = num_q_tokens < 0 ? d->num_seqs : num_q_tokens;
  p.part_tokens = choose_partition(d, max_len, partition_tokens,
                                   shared && d->dtype == PKV_BF16 && d->head_dim == 128);
  p.part_blocks = p.part_tokens / pkv::kBlock;
  p.max_parts = max_len <= 0 ? 1 : (max_len + p.part_tokens - 1) / p.part_tokens;
  const size_t B = static_cast<size_t>(d->num_seqs);
  size_t max_items = B * p.max_parts;
  if (shared) {
    const int group = d->num_q_heads / d->num_kv_heads;
    p.shared = true;
    p.members_per_item = group <= 8 ? 16 / group : 1;
    p.max_parts += 1;
    max_items = 2 * B * p.max_parts;
  }
  const size_t rows = static_cast<size_t>(p.num_q_tokens) * d->num_q_heads * p.max_parts;
  p.items_off = 256;
  size_t off = round_up(p.items_off + max_items * sizeof(pkv::PlanItem), 256);
  if (shared) {
    p.seq_prefix_off = off;
    off = round_up(off + B * sizeof(int32_t), 256);
    p.group_pref_off = off;
    off = round_up(off + B * sizeof(int32_t), 256);
  }
  if (p.max_parts > 1) {
    p.part_o_off = off;
    off = round_up(off + rows * d->head_dim * sizeof(float), 256);
    p.part_ml_off = off;
    off = round_up(off + rows * 2 * sizeof(float), 256);
  }
  p.total = off;
  *plan = p;
  return PKV_OK;
}

// cuTensorMapEncodeTiled, resolved from the driver once.
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault,
                                         &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess) {
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    }
  });
  return fn;
}

// A 2-D view of one cache pool: rows = (block, kv head, slot), columns = the
// head dimension.  The box is 16 rows x 128 bytes with 128-byte swizzling, so
// one (block, kv head) tile arrives as D*elem/128 swizzled [16][128 B] chunks.
pkv_status encode_pool_map(CUtensorMap* map, const void* pool, const pkv_dims* d) {
  auto enc = tensor_map_encoder();
  if (!enc) return fail(PKV_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
  const int e = elem_bytes(d->dtype);
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(d->head_dim),
                        static_cast<cuuint64_t>(d->num_blocks) * d->num_kv_heads * pkv::kBlock};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(d->head_dim) * e};
  cuuint32_t box[2] = {static_cast<cuuint32_t>(128 / e), static_cast<cuuint32_t>(pkv::kBlock)};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(map,
                   d->dtype == PKV_BF16       ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                   : is_fp8(d->dtype)         ? CU_TENSOR_MAP_DATA_TYPE_UINT8
                                              : CU_TENSOR_MAP_DATA_TYPE_FLOAT32,
                   2, const_cast<void*>(pool), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(PKV_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
  return PKV_OK;
}

// Kernel configuration: W decode warps per CTA (one CTA per SM), S tile
// stages per stage set, MB merge buffers, SPLIT warps reading each stage set
// (W / SPLIT sets).  Eight decode warps with two stages each hide the latency
// of the per-tile math best (measured on B200).  With 16 query rows per kv
// head at head_dim 128 one warp's state does not fit its registers and a
// second merge buffer does not fit shared memory: fourteen warps in pairs,
// each pair sharing the stages of one set and taking 8 rows apiece, one merge
// buffer (15 warps with the scheduler keep 128 registers per thread: at most
// four warps per SM sub-partition).  fp32 tiles are twice as large: four warps.
template <typename T, int D, int GMAX>
struct DecodeCfg {
  static constexpr bool kPairs = D == 128 && GMAX == 16;
  static constexpr int W = kPairs ? 14 : 8, S = 2, MB = kPairs ? 1 : 2, SPLIT = kPairs ? 2 : 1;
};
template <int D, int GMAX>
struct DecodeCfg<float, D, GMAX> {
  static constexpr int W = 4, S = 2, MB = (D == 128 && GMAX == 16) ? 1 : 2, SPLIT = 1;
};
// FP8 tiles carry half the bytes of bf16 ones for the same math (plus the
// code conversions), so the kernel is bound by per-tile latency rather than
// by HBM: more decode warps hide more of it.  Up to 8 query rows the state
// fits 128 registers and 15 decode warps run (one merge buffer to fit shared
// memory); measured on B200 on the Llama-3-8B-shaped batch: 15 warps 4.49
// TB/s, 11 warps 4.25, 8 warps with 4 stages 3.78.  With 16 rows one warp
// holds all of them (11 warps, 168 registers): paired warps would each widen
// the same codes to f16, and the conversions dominate (spec verification:
// 11 single warps 2.93 TB/s, 7 pairs 2.49).  Two stages per warp keep
// 88-120 KB per SM in flight.
template <int D, int GMAX>
struct DecodeCfg<pkv::Fp8Kv, D, GMAX> {
  static constexpr int W = GMAX == 16 ? 11 : 15, S = 2, MB = 1, SPLIT = 1;
};
template <int D, int GMAX>
struct DecodeCfg<pkv::Fp8E5m2Kv, D, GMAX> : DecodeCfg<pkv::Fp8Kv, D, GMAX> {};

// Largest dynamic shared memory already enabled per kernel, per device.
struct SmemAttr {
  const void* fn;
  int device;
  int bytes;
};
std::mutex g_attr_mu;
std::vector<SmemAttr> g_attr;

cudaError_t ensure_smem(const void* fn, int bytes) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(g_attr_mu);
  for (auto& a : g_attr) {
    if (a.fn == fn && a.device == dev) {
      if (a.bytes >= bytes) return cudaSuccess;
      e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
      if (e == cudaSuccess) a.bytes = bytes;
      return e;
    }
  }
  e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess) g_attr.push_back({fn, dev, bytes});
  return e;
}

template <typename T, int D, int GMAX>
pkv_status launch_decode(const CUtensorMap& mk, const CUtensorMap& mv,
                         const pkv::DecodeParams& prm, int64_t work_units, int rows_max,
                         cudaStream_t stream) {
  constexpr int W = DecodeCfg<T, D, GMAX>::W, S = DecodeCfg<T, D, GMAX>::S;
  constexpr int MB = DecodeCfg<T, D, GMAX>::MB, SPLIT = DecodeCfg<T, D, GMAX>::SPLIT;
  using Lay = pkv::DecodeLayout<sizeof(T), D, GMAX, W, S, MB, pkv::q_elem_bytes<T>(), SPLIT>;
  const int smem = Lay::total_bytes(rows_max);
  int dev = 0, max_optin = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&max_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
  if (smem > max_optin)
    return fail(PKV_ERR_UNSUPPORTED, "decode needs %d bytes of shared memory (> %d)", smem,
                max_optin);
  auto kern = pkv::decode_kernel<T, D, GMAX, W, S, MB, SPLIT>;
  cudaError_t e = ensure_smem(reinterpret_cast<const void*>(kern), smem);
  if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(decode)");
  int per_sm = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, (W + 1) * 32, smem);
  if (e != cudaSuccess) return cuda_fail(e, "occupancy query (decode)");
  if (per_sm < 1) per_sm = 1;
  int64_t grid = static_cast<int64_t>(device_sm_count()) * per_sm;
  if (grid > work_units) grid = work_units;
  if (grid < 1) grid = 1;
  e = launch(kern, dim3(static_cast<unsigned>(grid)), dim3((W + 1) * 32), smem, stream, mk, mv,
             prm);
  if (e != cudaSuccess) return cuda_fail(e, "decode launch");
  return PKV_OK;
}

// Short items (split-K partitions of at most kWarpItemMaxBlocks blocks, the
// shared-prefix plan) of bf16 head_dim-128 decode: one warp per item; for up
// to 8 query rows eight warps per CTA with 3 tile stages each, for 16 rows
// (the 16-row state needs 239 registers) six warps with 4 stages (measured on
// the parallel-sampling batch: 8 x 2 stages 0.116 ms, 7 x 3 0.110, 6 x 4
// 0.106; on the long-context batch at 512-token partitions 8 x 3 beat 6 x 4).
template <int GMAX>
pkv_status launch_decode_warp(const CUtensorMap& mk, const CUtensorMap& mv,
                              const pkv::DecodeParams& prm, int64_t work_units,
                              cudaStream_t stream) {
  constexpr int W = GMAX <= 8 ? 8 : 6, S = GMAX <= 8 ? 3 : 4;
  using Lay = pkv::WarpDecodeLayout<GMAX, W, S>;
  auto kern = pkv::decode_warp_kernel<GMAX, W, S>;
  cudaError_t e = ensure_smem(reinterpret_cast<const void*>(kern), Lay::kTotal);
  if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(decode_warp)");
  int64_t grid = device_sm_count();
  const int64_t need = (work_units + W - 1) / W;
  if (grid > need) grid = need;
  if (grid < 1) grid = 1;
  e = launch(kern, dim3(static_cast<unsigned>(grid)), dim3(W * 32), Lay::kTotal, stream, mk, mv,
             prm);
  if (e != cudaSuccess) return cuda_fail(e, "decode_warp launch");
  return PKV_OK;
}

// Decode over FP8 pools on the tcgen05 tensor cores (units of up to RM query
// rows, plain or split-K plans); AF: 0 e4m3 pools, 1 e5m2.
template <int RM, int AF>
pkv_status launch_decode_fp8tc(const CUtensorMap& mk, const CUtensorMap& mv,
                               const pkv::DecodeParams& prm, int64_t work_units,
                               cudaStream_t stream) {
  constexpr int ST = pkv::tc_stages<RM>();
  auto kern = pkv::decode_fp8tc_kernel<RM, AF, ST>;
  constexpr int smem = pkv::TcLayout<ST>::kTotal;
  cudaError_t e = ensure_smem(reinterpret_cast<const void*>(kern), smem);
  if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(decode_fp8tc)");
  // persistent: two CTAs per SM
  int64_t grid = static_cast<int64_t>(device_sm_count()) * 2;
  if (grid > work_units) grid = work_units;
  if (grid < 1) grid = 1;
  e = launch(kern, dim3(static_cast<unsigned>(grid)), dim3(pkv::kTcThreads), smem, stream, mk,
             mv, prm);
  if (e != cudaSuccess) return cuda_fail(e, "decode_fp8tc launch");
  return PKV_OK;
}

// The query rows of an item (chunk length x group) go on the MMA's N side:
// up to 8 or up to 16 rows.
template <typename T, int D>
pkv_status launch_decode_d(const CUtensorMap& mk, const CUtensorMap& mv,
                           const pkv::DecodeParams& prm, int64_t work_units, int rows_max,
                           cudaStream_t stream) {
  if (rows_max <= 8) return launch_decode<T, D, 8>(mk, mv, prm, work_units, rows_max, stream);
  if (rows_max <= 16) return launch_decode<T, D, 16>(mk, mv, prm, work_units, rows_max, stream);
  return fail(PKV_ERR_UNSUPPORTED, "query rows per kv head (chunk length x group = %d) > 16",
              rows_max);
}

pkv_status check_workspace(const DecodePlan& plan, const void* workspace, size_t bytes) {
  if (!workspace) return fail(PKV_ERR_WORKSPACE, "workspace is NULL");
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    return fail(PKV_ERR_WORKSPACE, "workspace must be 256-byte aligned");
  if (bytes < plan.total)
    return fail(PKV_ERR_WORKSPACE, "workspace has %zu bytes, %zu needed", bytes, plan.total);
  return PKV_OK;
}

// The merge: one warp per row when a row has at most 8 partials (the common
// case: a few partitions, or a shared prefix and the sequence's own blocks),
// else the CTA's kMergeWarps warps per row.
template <typename T>
pkv_status launch_merge(void* out, const DecodePlan& plan, uint8_t* ws,
                        const int32_t* context_lens, const int32_t* query_start_loc,
                        const pkv_dims* d, cudaStream_t stream) {
  const int64_t rows = static_cast<int64_t>(plan.num_q_tokens) * d->num_q_heads;
  if (rows > 0x7fffffff) return fail(PKV_ERR_UNSUPPORTED, "too many query rows for the merge");
  const bool warp_rows = plan.max_parts <= 8;
  const int64_t per_cta = warp_rows ? pkv::kMergeWarps : 1;
  const unsigned grid = static_cast<unsigned>((rows + per_cta - 1) / per_cta);
  const float* po = reinterpret_cast<const float*>(ws + plan.part_o_off);
  const float* pml = reinterpret_cast<const float*>(ws + plan.part_ml_off);
  const bool d128 = d->head_dim == 128;
  auto kern = warp_rows ? (d128 ? pkv::merge_kernel<T, 128, 1> : pkv::merge_kernel<T, 64, 1>)
                        : (d128 ? pkv::merge_kernel<T, 128, pkv::kMergeWarps>
                                : pkv::merge_kernel<T, 64, pkv::kMergeWarps>);
  cudaError_t e = launch(kern, dim3(grid), dim3(pkv::kMergeWarps * 32), 0, stream, out, po, pml,
                         context_lens, query_start_loc,
                         plan.shared ? reinterpret_cast<const int32_t*>(ws + plan.seq_prefix_off)
                                     : nullptr,
                         d->num_seqs, plan.num_q_tokens, d->num_q_heads,
                         plan.max_parts, plan.max_len, plan.part_tokens);
  if (e != cudaSuccess) return cuda_fail(e, "merge launch");
  return PKV_OK;
}

// Scratch for pkv_paged_attention_decode_static: callers that cannot
// allocate device memory use this fixed array instead of a workspace of their
// own.  Every device that loads the library holds it until the process exits.
static __device__ __align__(256) uint8_t g_static_workspace[PKV_STATIC_WORKSPACE_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_static_ws_mu;
void* g_static_ws_ptr[kMaxDevices] = {};

// Device address of g_static_workspace on the current device, looked up once
// per device (host code cannot use the array's name as a device pointer).  The
// caller binds the device first.  The lookup may load the module, which a
// stream capture does not allow, so the first call on a device refuses a
// capturing stream.  The cached address belongs to the device's primary
// context: it does not survive a cudaDeviceReset.
pkv_status static_workspace(cudaStream_t stream, void** ptr) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return fail(PKV_ERR_UNSUPPORTED, "device %d out of range", dev);
  std::lock_guard<std::mutex> lock(g_static_ws_mu);
  if (!g_static_ws_ptr[dev]) {
    cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
    e = cudaStreamIsCapturing(stream, &cap);
    if (e != cudaSuccess) return cuda_fail(e, "cudaStreamIsCapturing");
    if (cap != cudaStreamCaptureStatusNone)
      return fail(PKV_ERR_UNSUPPORTED,
                  "the first pkv_paged_attention_decode_static call on device %d looks up the "
                  "built-in scratch and must not be made while its stream is being captured",
                  dev);
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_static_workspace);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(static workspace)");
    g_static_ws_ptr[dev] = p;
  }
  *ptr = g_static_ws_ptr[dev];
  return PKV_OK;
}

// Every operand of a call must live on the device that owns `out` (the device
// bind_device made current): the kernels run there and read all of them.
pkv_status check_same_device(const void* const* ptrs, const char* const* names, int n) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  for (int i = 0; i < n; ++i) {
    cudaPointerAttributes a;
    e = cudaPointerGetAttributes(&a, ptrs[i]);
    if (e != cudaSuccess) {
      cudaGetLastError();
      return cuda_fail(e, "cudaPointerGetAttributes");
    }
    if (a.type != cudaMemoryTypeDevice && a.type != cudaMemoryTypeManaged)
      return fail(PKV_ERR_SHAPE, "%s is not device memory", names[i]);
    if (a.device != dev)
      return fail(PKV_ERR_SHAPE, "%s is on device %d but out is on device %d", names[i],
                  a.device, dev);
  }
  return PKV_OK;
}

// Decode (and merge) over a plan already in the workspace.  query_start_loc
// NULL: one query token per sequence; otherwise chunks of up to max_query_len
// causal query tokens.
pkv_status run_decode(void* out, const void* q, const void* k_cache, const void* v_cache,
                      const int32_t* block_tables, const int32_t* context_lens,
                      const int32_t* query_start_loc, int32_t max_query_len, float scale,
                      const pkv_dims* d, const DecodePlan& plan, void* workspace,
                      size_t workspace_bytes, void* cuda_stream, float k_scale = 1.f,
                      float v_scale = 1.f) {
  pkv_status st;
  if (d->num_seqs == 0 || plan.num_q_tokens == 0) return PKV_OK;
  if (!out || !q || !k_cache || !v_cache || !block_tables || !context_lens)
    return fail(PKV_ERR_NULL, "a tensor pointer is NULL");
  if (!aligned16(out) || !aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache))
    return fail(PKV_ERR_ALIGN, "out, q and the caches must be 16-byte aligned");
  if ((st = check_workspace(plan, workspace, workspace_bytes)) != PKV_OK) return st;
  if (!std::isfinite(scale)) return fail(PKV_ERR_SHAPE, "scale must be finite");
  if (!(k_scale > 0.f) || !(v_scale > 0.f) || !std::isfinite(k_scale) || !std::isfinite(v_scale))
    return fail(PKV_ERR_SHAPE, "k_scale and v_scale must be finite and positive");
  if (max_query_len < 1) return fail(PKV_ERR_SHAPE, "max_query_len must be >= 1");
  const int group = d->num_q_heads / d->num_kv_heads;
  if (group > 16)
    return fail(PKV_ERR_UNSUPPORTED, "%d query heads per kv head (at most 16)", group);
  // Up to 16 query rows per item (an item's rows share one MMA tile); a longer
  // chunk is split into row groups of whole tokens, each read against the
  // keys its rows can see.
  // A shared-prefix plan serves one token of up to members_per_item sequences per item.
  if (plan.shared) max_query_len = plan.members_per_item;
  const int group_tokens = max_query_len * group <= 16 ? max_query_len : 16 / group;
  const int row_groups = (max_query_len + group_tokens - 1) / group_tokens;
  const int rows_max = group_tokens * group;
  if ((st = bind_device(out, "out")) != PKV_OK) return st;
  CUtensorMap mk, mv;
  if ((st = encode_pool_map(&mk, k_cache, d)) != PKV_OK) return st;
  if ((st = encode_pool_map(&mv, v_cache, d)) != PKV_OK) return st;
  cudaStream_t stream = static_cast<cudaStream_t>(cuda_stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);

  pkv::DecodeParams prm;
  prm.out = out;
  prm.q = q;
  prm.block_tables = block_tables;
  prm.items = reinterpret_cast<pkv::PlanItem*>(ws + plan.items_off);
  prm.counters = reinterpret_cast<uint32_t*>(ws);
  prm.part_o = plan.max_parts > 1 ? reinterpret_cast<float*>(ws + plan.part_o_off) : nullptr;
  prm.part_ml = plan.max_parts > 1 ? reinterpret_cast<float*>(ws + plan.part_ml_off) : nullptr;
  prm.query_start_loc = query_start_loc;
  prm.max_query_len = max_query_len;
  prm.group_tokens = group_tokens;
  prm.row_groups = row_groups;
  prm.num_q_tokens = plan.num_q_tokens;
  prm.num_q_heads = d->num_q_heads;
  prm.num_kv_heads = d->num_kv_heads;
  prm.group = group;
  prm.max_blocks_per_seq = d->max_blocks_per_seq;
  prm.num_blocks = d->num_blocks;
  prm.max_parts = plan.max_parts;
  prm.part_blocks = plan.part_blocks;
  prm.qk_scale_log2 = scale * pkv::kLog2e * k_scale;
  prm.out_scale = v_scale;
  const int64_t units = static_cast<int64_t>(d->num_seqs) * plan.max_parts * d->num_kv_heads *
                        (plan.shared ? 2 : row_groups);
  if (is_fp8(d->dtype) && !plan.shared && row_groups == 1) {
    // FP8 codes, every sequence's query rows (chunk tokens x group, at most
    // 16) in one unit: the tensor-core path
    if (d->dtype == PKV_FP8_E4M3)
      st = rows_max <= 4   ? launch_decode_fp8tc<4, 0>(mk, mv, prm, units, stream)
           : rows_max <= 8 ? launch_decode_fp8tc<8, 0>(mk, mv, prm, units, stream)
                           : launch_decode_fp8tc<16, 0>(mk, mv, prm, units, stream);
    else
      st = rows_max <= 4   ? launch_decode_fp8tc<4, 1>(mk, mv, prm, units, stream)
           : rows_max <= 8 ? launch_decode_fp8tc<8, 1>(mk, mv, prm, units, stream)
                           : launch_decode_fp8tc<16, 1>(mk, mv, prm, units, stream);
  } else if (d->dtype == PKV_FP8_E4M3) {
    st = launch_decode_d<pkv::Fp8Kv, 128>(mk, mv, prm, units, rows_max, stream);
  } else if (d->dtype == PKV_FP8_E5M2) {
    st = launch_decode_d<pkv::Fp8E5m2Kv, 128>(mk, mv, prm, units, rows_max, stream);
  } else if (d->dtype == PKV_BF16 && d->head_dim == 128 &&
             (!query_start_loc || max_query_len == 1) &&
             rows_max <= 16 && plan.part_blocks <= pkv::kWarpItemMaxBlocks &&
             (plan.max_parts > 1 || plan.shared)) {
    // short items: a warp per item, no merge across warps
    st = rows_max <= 8 ? launch_decode_warp<8>(mk, mv, prm, units, stream)
                       : launch_decode_warp<16>(mk, mv, prm, units, stream);
  } else if (d->dtype == PKV_BF16) {
    st = d->head_dim == 128
             ? launch_decode_d<__nv_bfloat16, 128>(mk, mv, prm, units, rows_max, stream)
             : launch_decode_d<__nv_bfloat16, 64>(mk, mv, prm, units, rows_max, stream);
  } else {
    st = d->head_dim == 128 ? launch_decode_d<float, 128>(mk, mv, prm, units, rows_max, stream)
                            : launch_decode_d<float, 64>(mk, mv, prm, units, rows_max, stream);
  }
  if (st != PKV_OK) return st;
  if (plan.max_parts > 1) {
    st = d->dtype != PKV_F32
             ? launch_merge<__nv_bfloat16>(out, plan, ws, context_lens, query_start_loc, d, stream)
             : launch_merge<float>(out, plan, ws, context_lens, query_start_loc, d, stream);
  }
  return st;
}

}  // namespace

namespace {

// Slot indexing + the new tokens' writes + the plan in one launch (see
// pkv_decode_prepare).
pkv_status decode_prepare(const void* k, const void* v, void* k_cache, void* v_cache,
                          const int32_t* block_tables, const int32_t* context_lens,
                          int64_t* slot_mapping_out, bool fp8, float k_scale, float v_scale,
                          const pkv_dims* dims, int32_t max_context_len,
                          int32_t partition_tokens, void* workspace, size_t workspace_bytes,
                          void* cuda_stream) {
  DecodePlan plan;
  pkv_status st = make_plan(dims, max_context_len, partition_tokens, &plan);
  if (st != PKV_OK) return st;
  if (fp8) {
    if (!is_fp8(dims->dtype)) return fail(PKV_ERR_UNSUPPORTED, "dims->dtype must be FP8");
    if (!(k_scale > 0.f) || !(v_scale > 0.f) || !std::isfinite(k_scale) ||
        !std::isfinite(v_scale))
      return fail(PKV_ERR_SHAPE, "k_scale and v_scale must be finite and positive");
  } else if (is_fp8(dims->dtype)) {
    return fail(PKV_ERR_UNSUPPORTED, "FP8 pools need their scales: use pkv_decode_prepare_fp8");
  }
  if (dims->num_seqs == 0) return PKV_OK;
  if (!k || !v || !k_cache || !v_cache || !block_tables || !context_lens)
    return fail(PKV_ERR_NULL, "a tensor pointer is NULL");
  if (!aligned16(k) || !aligned16(v) || !aligned16(k_cache) || !aligned16(v_cache))
    return fail(PKV_ERR_ALIGN, "k, v and the caches must be 16-byte aligned");
  if ((st = check_workspace(plan, workspace, workspace_bytes)) != PKV_OK) return st;
  if ((st = bind_device(k_cache, "k_cache")) != PKV_OK) return st;
  // 16-byte units of one head's source row: bf16 / fp32 rows as stored, FP8
  // rows as their bf16 inputs
  const int src_row_bytes = dims->head_dim * (fp8 ? 2 : elem_bytes(dims->dtype));
  const int units_per_head = src_row_bytes / 16;
  const int units = dims->num_kv_heads * units_per_head;
  const int per = units < pkv::kPlanThreads ? units : pkv::kPlanThreads;
  const int seqs_per_cta = pkv::kPlanThreads / per;
  const unsigned grid = 1u + static_cast<unsigned>((dims->num_seqs + seqs_per_cta - 1) / seqs_per_cta);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  auto kern = !fp8 ? pkv::decode_prepare_kernel<false, false>
              : dims->dtype == PKV_FP8_E5M2 ? pkv::decode_prepare_kernel<true, true>
                                            : pkv::decode_prepare_kernel<true, false>;
  cudaError_t e = launch(kern, dim3(grid), dim3(pkv::kPlanThreads), 0,
                         static_cast<cudaStream_t>(cuda_stream), static_cast<const uint4*>(k),
                         static_cast<const uint4*>(v), static_cast<uint8_t*>(k_cache),
                         static_cast<uint8_t*>(v_cache), block_tables, context_lens,
                         slot_mapping_out, dims->num_seqs, dims->num_kv_heads, units_per_head,
                         dims->max_blocks_per_seq, dims->num_blocks, seqs_per_cta, per, k_scale,
                         v_scale, plan.max_len, plan.part_blocks,
                         reinterpret_cast<pkv::PlanItem*>(ws + plan.items_off),
                         reinterpret_cast<uint32_t*>(ws));
  if (e != cudaSuccess) return cuda_fail(e, "decode prepare launch");
  return PKV_OK;
}

}  // namespace

namespace {

// The run and one-shot calls for several query tokens; `fp8` selects the FP8
// entry points (FP8 pools and their scales) or the plain ones (bf16 / fp32).
pkv_status check_multi_pools(const pkv_dims* dims, bool fp8, float k_scale, float v_scale) {
  if (fp8) {
    if (!is_fp8(dims->dtype)) return fail(PKV_ERR_UNSUPPORTED, "dims->dtype must be FP8");
    if (!(k_scale > 0.f) || !(v_scale > 0.f) || !std::isfinite(k_scale) ||
        !std::isfinite(v_scale))
      return fail(PKV_ERR_SHAPE, "k_scale and v_scale must be finite and positive");
  } else if (is_fp8(dims->dtype)) {
    return fail(PKV_ERR_UNSUPPORTED,
                "FP8 pools need their scales: use the _fp8 calls for several query tokens");
  }
  return PKV_OK;
}

pkv_status multi_run(void* out, const void* q, const void* k_cache, const void* v_cache,
                     const int32_t* block_tables, const int32_t* context_lens,
                     const int32_t* query_start_loc, int32_t num_q_tokens, int32_t max_query_len,
                     float scale, bool fp8, float k_scale, float v_scale, const pkv_dims* dims,
                     int32_t max_context_len, int32_t partition_tokens, void* workspace,
                     size_t workspace_bytes, void* cuda_stream) {
  if (num_q_tokens < 0) return fail(PKV_ERR_SHAPE, "num_q_tokens must be >= 0");
  DecodePlan plan;
  pkv_status st = make_plan(dims, max_context_len, partition_tokens, &plan, num_q_tokens);
  if (st != PKV_OK) return st;
  if ((st = check_multi_pools(dims, fp8, k_scale, v_scale)) != PKV_OK) return st;
  if (dims->num_seqs == 0 || num_q_tokens == 0) return PKV_OK;
  if (!query_start_loc) return fail(PKV_ERR_NULL, "query_start_loc is NULL");
  return run_decode(out, q, k_cache, v_cache, block_tables, context_lens, query_start_loc,
                    max_query_len, scale, dims, plan, workspace, workspace_bytes, cuda_stream,
                    k_scale, v_scale);
}

pkv_status multi_one_shot(void* out, const void* q, const void* k_cache, const void* v_cache,
                          const int32_t* block_tables, const int32_t* context_lens,
                          const int32_t* query_start_loc, int32_t num_q_tokens,
                          int32_t max_query_len, float scale, bool fp8, float k_scale,
                          float v_scale, const pkv_dims* dims, int32_t max_context_len,
                          int32_t partition_tokens, void* workspace, size_t workspace_bytes,
                          void* cuda_stream) {
  if (num_q_tokens < 0) return fail(PKV_ERR_SHAPE, "num_q_tokens must be >= 0");
  DecodePlan plan;
  pkv_status st = make_plan(dims, max_context_len, partition_tokens, &plan, num_q_tokens);
  if (st != PKV_OK) return st;
  if ((st = check_multi_pools(dims, fp8, k_scale, v_scale)) != PKV_OK) return st;
  if (dims->num_seqs == 0 || num_q_tokens == 0) return PKV_OK;
  if (!query_start_loc) return fail(PKV_ERR_NULL, "query_start_loc is NULL");
  if (max_query_len < 1) return fail(PKV_ERR_SHAPE, "max_query_len must be >= 1");
  if ((st = check_workspace(plan, workspace, workspace_bytes)) != PKV_OK) return st;
  st = pkv_decode_plan(context_lens, dims, max_context_len, partition_tokens, workspace,
                       workspace_bytes, cuda_stream);
  if (st != PKV_OK) return st;
  return run_decode(out, q, k_cache, v_cache, block_tables, context_lens, query_start_loc,
                    max_query_len, scale, dims, plan, workspace, workspace_bytes, cuda_stream,
                    k_scale, v_scale);
}

}  // namespace

namespace {

// The token-list prologue (see pkv_decode_prepare_tokens).
pkv_status prepare_tokens(const void* k, const void* v, void* k_cache, void* v_cache,
                          const int32_t* block_tables, const int32_t* context_lens,
                          const int32_t* token_seq, const int32_t* token_pos, int32_t num_tokens,
                          int64_t* slot_mapping_out, float k_scale, float v_scale,
                          const int32_t* group_start, const int32_t* shared_blocks,
                          int32_t num_groups, const pkv_dims* dims, int32_t max_context_len,
                          int32_t partition_tokens, void* workspace, size_t workspace_bytes,
                          void* cuda_stream) {
  const bool shared = group_start != nullptr;
  DecodePlan plan;
  pkv_status st = make_plan(dims, max_context_len, partition_tokens, &plan, -1, shared);
  if (st != PKV_OK) return st;
  const bool fp8 = is_fp8(dims->dtype);
  if (fp8 && (!(k_scale > 0.f) || !(v_scale > 0.f) || !std::isfinite(k_scale) ||
              !std::isfinite(v_scale)))
    return fail(PKV_ERR_SHAPE, "k_scale and v_scale must be finite and positive for FP8 pools");
  if (num_tokens < 0) return fail(PKV_ERR_SHAPE, "num_tokens must be >= 0");
  if (shared && (num_groups < 0 || num_groups > dims->num_seqs))
    return fail(PKV_ERR_SHAPE, "num_groups must be in [0, num_seqs]");
  if (dims->num_seqs == 0) return PKV_OK;
  if (!k_cache || !v_cache || !block_tables || !context_lens)
    return fail(PKV_ERR_NULL, "a tensor pointer is NULL");
  if (num_tokens > 0 && (!k || !v || !token_seq || !token_pos))
    return fail(PKV_ERR_NULL, "k, v, token_seq or token_pos is NULL");
  if (shared && num_groups > 0 && !shared_blocks) return fail(PKV_ERR_NULL, "shared_blocks is NULL");
  if (!aligned16(k) || !aligned16(v) || !aligned16(k_cache) || !aligned16(v_cache))
    return fail(PKV_ERR_ALIGN, "k, v and the caches must be 16-byte aligned");
  if ((st = check_workspace(plan, workspace, workspace_bytes)) != PKV_OK) return st;
  if ((st = bind_device(k_cache, "k_cache")) != PKV_OK) return st;
  // 16-byte units of one head's source row: bf16 / fp32 rows as stored, FP8
  // rows as their bf16 inputs
  const int units_per_head = dims->head_dim * (fp8 ? 2 : elem_bytes(dims->dtype)) / 16;
  const int units = dims->num_kv_heads * units_per_head;
  const int per = units < pkv::kPlanThreads ? units : pkv::kPlanThreads;
  const int toks_per_cta = pkv::kPlanThreads / per;
  const unsigned grid =
      1u + static_cast<unsigned>((static_cast<int64_t>(num_tokens) + toks_per_cta - 1) / toks_per_cta);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  pkv::TokenPrepare a{};
  a.k = static_cast<const uint4*>(k);
  a.v = static_cast<const uint4*>(v);
  a.k_cache = static_cast<uint8_t*>(k_cache);
  a.v_cache = static_cast<uint8_t*>(v_cache);
  a.block_tables = block_tables;
  a.token_seq = token_seq;
  a.token_pos = token_pos;
  a.slots_out = slot_mapping_out;
  a.num_tokens = num_tokens;
  a.num_seqs = dims->num_seqs;
  a.num_kv_heads = dims->num_kv_heads;
  a.units_per_head = units_per_head;
  a.max_blocks_per_seq = dims->max_blocks_per_seq;
  a.num_blocks = dims->num_blocks;
  a.toks_per_cta = toks_per_cta;
  a.per = per;
  a.k_scale = k_scale;
  a.v_scale = v_scale;
  a.context_lens = context_lens;
  a.max_len = plan.max_len;
  a.part_blocks = plan.part_blocks;
  a.items = reinterpret_cast<pkv::PlanItem*>(ws + plan.items_off);
  a.counters = reinterpret_cast<uint32_t*>(ws);
  if (shared) {
    a.group_start = group_start;
    a.shared_blocks = shared_blocks;
    a.num_groups = num_groups;
    a.members_per_item = plan.members_per_item;
    a.seq_prefix = reinterpret_cast<int32_t*>(ws + plan.seq_prefix_off);
    a.group_pref = reinterpret_cast<int32_t*>(ws + plan.group_pref_off);
  }
  const bool e5m2 = dims->dtype == PKV_FP8_E5M2;
  auto kern = shared ? (!fp8 ? pkv::token_prepare_kernel<false, false, true>
                             : e5m2 ? pkv::token_prepare_kernel<true, true, true>
                                    : pkv::token_prepare_kernel<true, false, true>)
                     : (!fp8 ? pkv::token_prepare_kernel<false, false, false>
                             : e5m2 ? pkv::token_prepare_kernel<true, true, false>
                                    : pkv::token_prepare_kernel<true, false, false>);
  cudaError_t e = launch(kern, dim3(grid), dim3(pkv::kPlanThreads), 0,
                         static_cast<cudaStream_t>(cuda_stream), a);
  if (e != cudaSuccess) return cuda_fail(e, "token prologue launch");
  return PKV_OK;
}

}  // namespace

namespace {

// The shared-prefix decode: its plan, and the run over it (bf16 / fp32 pools,
// or FP8 pools with their scales when `fp8`).
pkv_status plan_shared(const int32_t* context_lens, const int32_t* group_start,
                       const int32_t* shared_blocks, int32_t num_groups, const pkv_dims* dims,
                       int32_t max_context_len, int32_t partition_tokens, void* workspace,
                       size_t workspace_bytes, void* cuda_stream) {
  DecodePlan plan;
  pkv_status st = make_plan(dims, max_context_len, partition_tokens, &plan, -1, true);
  if (st != PKV_OK) return st;
  if (num_groups < 0 || num_groups > dims->num_seqs)
    return fail(PKV_ERR_SHAPE, "num_groups must be in [0, num_seqs]");
  if (dims->num_seqs == 0) return PKV_OK;
  if (!context_lens || !group_start || (num_groups > 0 && !shared_blocks))
    return fail(PKV_ERR_NULL, "context_lens, group_start or shared_blocks is NULL");
  if ((st = check_workspace(plan, workspace, workspace_bytes)) != PKV_OK) return st;
  if ((st = bind_device(workspace, "workspace")) != PKV_OK) return st;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  cudaError_t e = launch(pkv::plan_shared_kernel, dim3(1), dim3(pkv::kPlanThreads), 0,
                         static_cast<cudaStream_t>(cuda_stream), context_lens, group_start,
                         shared_blocks, num_groups, dims->num_seqs, plan.max_len,
                         plan.part_blocks, plan.members_per_item,
                         reinterpret_cast<pkv::PlanItem*>(ws + plan.items_off),
                         reinterpret_cast<uint32_t*>(ws),
                         reinterpret_cast<int32_t*>(ws + plan.seq_prefix_off),
                         reinterpret_cast<int32_t*>(ws + plan.group_pref_off));
  if (e != cudaSuccess) return cuda_fail(e, "shared-prefix plan launch");
  return PKV_OK;
}

pkv_status check_pool_kind(const pkv_dims* dims, bool fp8, float k_scale, float v_scale) {
  if (fp8) {
    if (!is_fp8(dims->dtype)) return fail(PKV_ERR_UNSUPPORTED, "dims->dtype must be FP8");
    if (!(k_scale > 0.f) || !(v_scale > 0.f) || !std::isfinite(k_scale) ||
        !std::isfinite(v_scale))
      return fail(PKV_ERR_SHAPE, "k_scale and v_scale must be finite and positive");
  } else if (is_fp8(dims->dtype)) {
    return fail(PKV_ERR_UNSUPPORTED, "FP8 pools need their scales: use the _fp8 calls");
  }
  return PKV_OK;
}

pkv_status run_shared(void* out, const void* q, const void* k_cache, const void* v_cache,
                      const int32_t* block_tables, const int32_t* context_lens, float scale,
                      bool fp8, float k_scale, float v_scale, const pkv_dims* dims,
                      int32_t max_context_len, int32_t partition_tokens, void* workspace,
                      size_t workspace_bytes, void* cuda_stream) {
  DecodePlan plan;
  pkv_status st = make_plan(dims, max_context_len, partition_tokens, &plan, -1, true);
  if (st != PKV_OK) return st;
  if ((st = check_pool_kind(dims, fp8, k_scale, v_scale)) != PKV_OK) return st;
  return run_decode(out, q, k_cache, v_cache, block_tables, context_lens, nullptr, 1, scale,
                    dims, plan, workspace, workspace_bytes, cuda_stream, k_scale, v_scale);
}

pkv_status shared_one_shot(void* out, const void* q, const void* k_cache, const void* v_cache,
                           const int32_t* block_tables, const int32_t* context_lens,
                           const int32_t* group_start, const int32_t* shared_blocks,
                           int32_t num_groups, float scale, bool fp8, float k_scale,
                           float v_scale, const pkv_dims* dims, int32_t max_context_len,
                           int32_t partition_tokens, void* workspace, size_t workspace_bytes,
                           void* cuda_stream) {
  DecodePlan plan;
  pkv_status st = make_plan(dims, max_context_len, partition_tokens, &plan, -1, true);
  if (st != PKV_OK) return st;
  if ((st = check_pool_kind(dims, fp8, k_scale, v_scale)) != PKV_OK) return st;
  if (dims->num_seqs == 0) return PKV_OK;
  // Check everything the run needs before launching the plan.
  if (!out || !q || !k_cache || !v_cache || !block_tables || !context_lens)
    return fail(PKV_ERR_NULL, "a tensor pointer is NULL");
  if (!aligned16(out) || !aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache))
    return fail(PKV_ERR_ALIGN, "out, q and the caches must be 16-byte aligned");
  if (!std::isfinite(scale)) return fail(PKV_ERR_SHAPE, "scale must be finite");
  st = plan_shared(context_lens, group_start, shared_blocks, num_groups, dims, max_context_len,
                   partition_tokens, workspace, workspace_bytes, cuda_stream);
  if (st != PKV_OK) return st;
  return run_decode(out, q, k_cache, v_cache, block_tables, context_lens, nullptr, 1, scale,
                    dims, plan, workspace, workspace_bytes, cuda_stream, k_scale, v_scale);
}

}  // namespace

namespace {

// A 3-D view of q [num_q_tokens][Hq][D] (bf16) for the prefill kernel: the box
// is {64 columns, the g heads of one kv head, tokens_per_tile tokens}, so one
// load brings the tile's 128 query rows (token-major, head-minor) of one
// 128-byte column half, 128-byte swizzled.
pkv_status encode_q_map(CUtensorMap* map, const void* q, int32_t num_q_tokens, const pkv_dims* d,
                        int group, int tokens_per_tile) {
  auto enc = tensor_map_encoder();
  if (!enc) return fail(PKV_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(d->head_dim),
                        static_cast<cuuint64_t>(d->num_q_heads),
                        static_cast<cuuint64_t>(num_q_tokens)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(d->head_dim) * 2,
                           static_cast<cuuint64_t>(d->num_q_heads) * d->head_dim * 2};
  cuuint32_t box[3] = {64u, static_cast<cuuint32_t>(group),
                       static_cast<cuuint32_t>(tokens_per_tile)};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(q), dims, strides,
                   box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(PKV_ERR_CUDA, "cuTensorMapEncodeTiled (q) failed (%d)", (int)r);
  return PKV_OK;
}

template <int D>
pkv_status launch_prefill(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                          const pkv::PrefillParams& prm, int64_t units_bound,
                          cudaStream_t stream) {
  auto kern = pkv::prefill_kernel<D>;
  constexpr int smem = pkv::PfLayout<D>::kTotal;
  cudaError_t e = ensure_smem(reinterpret_cast<const void*>(kern), smem);
  if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(prefill)");
  const int64_t sms = device_sm_count();
  const int grid = static_cast<int>(units_bound < sms ? units_bound : sms);
  e = launch(kern, dim3(grid), dim3(pkv::kPfThreads), smem, stream, mq, mk, mv, prm);
  if (e != cudaSuccess) return cuda_fail(e, "prefill launch");
  return PKV_OK;
}

}  // namespace

extern "C" {

int32_t pkv_decode_partition_tokens(const pkv_dims* dims, int32_t max_context_len,
                                    int32_t partition_tokens) {
  DecodePlan plan;
  if (make_plan(dims, max_context_len, partition_tokens, &plan) != PKV_OK) return 0;
  return plan.part_tokens;
}

int32_t pkv_decode_shared_partition_tokens(const pkv_dims* dims, int32_t max_context_len,
                                           int32_t partition_tokens) {
  DecodePlan plan;
  if (make_plan(dims, max_context_len, partition_tokens, &plan, -1, true) != PKV_OK) return 0;
  return plan.part_tokens;
}

size_t pkv_decode_workspace_bytes(const pkv_dims* dims, int32_t max_context_len,
                                  int32_t partition_tokens) {
  DecodePlan plan;
  if (make_plan(dims, max_context_len, partition_tokens, &plan) != PKV_OK) return 0;
  return plan.total;
}

pkv_status pkv_decode_workspace_layout(const pkv_dims* dims, int32_t max_context_len,
                                       int32_t partition_tokens, int32_t* max_parts,
                                       size_t* part_o_offset, size_t* part_ml_offset) {
  DecodePlan plan;
  pkv_status st = make_plan(dims, max_context_len, partition_tokens, &plan);
  if (st != PKV_OK) return st;
  if (max_parts) *max_parts = plan.max_parts;
  if (plan.max_parts <= 1) return fail(PKV_ERR_SHAPE, "single-pass decode has no partials");
  if (part_o_offset) *part_o_offset = plan.part_o_off;
  if (part_ml_offset) *part_ml_offset = plan.part_ml_off;
  return PKV_OK;
}

pkv_status pkv_decode_plan(const int32_t* context_lens, const pkv_dims* dims,
                           int32_t max_context_len, int32_t partition_tokens, void* workspace,
                           size_t workspace_bytes, void* cuda_stream) {
  DecodePlan plan;
  pkv_status st = make_plan(dims, max_context_len, partition_tokens, &plan);
  if (st != PKV_OK) return st;
  if (dims->num_seqs == 0) return PKV_OK;
  if (!context_lens) return fail(PKV_ERR_NULL, "context_lens is NULL");
  if ((st = check_workspace(plan, workspace, workspace_bytes)) != PKV_OK) return st;
  if ((st = bind_device(workspace, "workspace")) != PKV_OK) return st;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  cudaError_t e = launch(pkv::plan_kernel, dim3(1), dim3(pkv::kPlanThreads), 0,
                         static_cast<cudaStream_t>(cuda_stream), context_lens, dims->num_seqs,
                         plan.max_len, plan.part_blocks,
                         reinterpret_cast<pkv::PlanItem*>(ws + plan.items_off),
                         reinterpret_cast<uint32_t*>(ws));
  if (e != cudaSuccess) return cuda_fail(e, "plan launch");
  return PKV_OK;
}

pkv_status pkv_decode_prepare(const void* k, const void* v, void* k_cache, void* v_cache,
                              const int32_t* block_tables, const int32_t* context_lens,
                              int64_t* slot_mapping_out, const pkv_dims* dims,
                              int32_t max_context_len, int32_t partition_tokens, void* workspace,
                              size_t workspace_bytes, void* cuda_stream) {
  return decode_prepare(k, v, k_cache, v_cache, block_tables, context_lens, slot_mapping_out,
                        false, 1.f, 1.f, dims, max_context_len, partition_tokens, workspace,
                        workspace_bytes, cuda_stream);
}

pkv_status pkv_decode_prepare_fp8(const void* k, const void* v, void* k_cache, void* v_cache,
                                  const int32_t* block_tables, const int32_t* context_lens,
                                  int64_t* slot_mapping_out, float k_scale, float v_scale,
                                  const pkv_dims* dims, int32_t max_context_len,
                                  int32_t partition_tokens, void* workspace,
                                  size_t workspace_bytes, void* cuda_stream) {
  return decode_prepare(k, v, k_cache, v_cache, block_tables, context_lens, slot_mapping_out,
                        true, k_scale, v_scale, dims, max_context_len, partition_tokens,
                        workspace, workspace_bytes, cuda_stream);
}

pkv_status pkv_decode_run(void* out, const void* q, const void* k_cache, const void* v_cache,
                          const int32_t* block_tables, const int32_t* context_lens, float scale,
                          const pkv_dims* dims, int32_t max_context_len,
                          int32_t partition_tokens, void* workspace, size_t workspace_bytes,
                          void* cuda_stream) {
  DecodePlan plan;
  pkv_status st = make_plan(dims, max_context_len, partition_tokens, &plan);
  if (st != PKV_OK) return st;
  if (is_fp8(dims->dtype))
    return fail(PKV_ERR_UNSUPPORTED, "FP8 caches need their scales: use pkv_decode_run_fp8");
  return run_decode(out, q, k_cache, v_cache, block_tables, context_lens, nullptr, 1, scale,
                    dims, plan, workspace, workspace_bytes, cuda_stream);
}

pkv_status pkv_paged_attention_decode(void* out, const void* q, const void* k_cache,
                                      const void* v_cache, const int32_t* block_tables,
                                      const int32_t* context_lens, float scale,
                                      const pkv_dims* dims, int32_t max_context_len,
                                      int32_t partition_tokens, void* workspace,
                                      size_t workspace_bytes, void* cuda_stream) {
  DecodePlan plan;
  pkv_status st = make_plan(dims, max_context_len, partition_tokens, &plan);
  if (st != PKV_OK) return st;
  if (is_fp8(dims->dtype))
    return fail(PKV_ERR_UNSUPPORTED,
                "FP8 caches need their scales: use pkv_paged_attention_decode_fp8");
  if (dims->num_seqs == 0) return PKV_OK;
  // Check everything the run needs before launching the plan.
  if (!out || !q || !k_cache || !v_cache || !block_tables || !context_lens)
    return fail(PKV_ERR_NULL, "a tensor pointer is NULL");
  if (!aligned16(out) || !aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache))
    return fail(PKV_ERR_ALIGN, "out, q and the caches must be 16-byte aligned");
  if ((st = check_workspace(plan, workspace, workspace_bytes)) != PKV_OK) return st;
  if (!std::isfinite(scale)) return fail(PKV_ERR_SHAPE, "scale must be finite");
  st = pkv_decode_plan(context_lens, dims, max_context_len, partition_tokens, workspace,
                       workspace_bytes, cuda_stream);
  if (st != PKV_OK) return st;
  return pkv_decode_run(out, q, k_cache, v_cache, block_tables, context_lens, scale, dims,
                        max_context_len, partition_tokens, workspace, workspace_bytes,
                        cuda_stream);
}

size_t pkv_multi_workspace_bytes(const pkv_dims* dims, int32_t num_q_tokens,
                                 int32_t max_context_len, int32_t partition_tokens) {
  DecodePlan plan;
  if (num_q_tokens < 0) return 0;
  if (make_plan(dims, max_context_len, partition_tokens, &plan, num_q_tokens) != PKV_OK) return 0;
  return plan.total;
}


pkv_status pkv_multi_run(void* out, const void* q, const void* k_cache, const void* v_cache,
                         const int32_t* block_tables, const int32_t* context_lens,
                         const int32_t* query_start_loc, int32_t num_q_tokens,
                         int32_t max_query_len, float scale, const pkv_dims* dims,
                         int32_t max_context_len, int32_t partition_tokens, void* workspace,
                         size_t workspace_bytes, void* cuda_stream) {
  return multi_run(out, q, k_cache, v_cache, block_tables, context_lens, query_start_loc,
                   num_q_tokens, max_query_len, scale, false, 1.f, 1.f, dims, max_context_len,
                   partition_tokens, workspace, workspace_bytes, cuda_stream);
}

pkv_status pkv_paged_attention_multi(void* out, const void* q, const void* k_cache,
                                     const void* v_cache, const int32_t* block_tables,
                                     const int32_t* context_lens, const int32_t* query_start_loc,
                                     int32_t num_q_tokens, int32_t max_query_len, float scale,
                                     const pkv_dims* dims, int32_t max_context_len,
                                     int32_t partition_tokens, void* workspace,
                                     size_t workspace_bytes, void* cuda_stream) {
  return multi_one_shot(out, q, k_cache, v_cache, block_tables, context_lens, query_start_loc,
                        num_q_tokens, max_query_len, scale, false, 1.f, 1.f, dims,
                        max_context_len, partition_tokens, workspace, workspace_bytes,
                        cuda_stream);
}

pkv_status pkv_multi_run_fp8(void* out, const void* q, const void* k_cache, const void* v_cache,
                             const int32_t* block_tables, const int32_t* context_lens,
                             const int32_t* query_start_loc, int32_t num_q_tokens,
                             int32_t max_query_len, float scale, float k_scale, float v_scale,
                             const pkv_dims* dims, int32_t max_context_len,
                             int32_t partition_tokens, void* workspace, size_t workspace_bytes,
                             void* cuda_stream) {
  return multi_run(out, q, k_cache, v_cache, block_tables, context_lens, query_start_loc,
                   num_q_tokens, max_query_len, scale, true, k_scale, v_scale, dims,
                   max_context_len, partition_tokens, workspace, workspace_bytes, cuda_stream);
}

pkv_status pkv_paged_attention_multi_fp8(void* out, const void* q, const void* k_cache,
                                         const void* v_cache, const int32_t* block_tables,
                                         const int32_t* context_lens,
                                         const int32_t* query_start_loc, int32_t num_q_tokens,
                                         int32_t max_query_len, float scale, float k_scale,
                                         float v_scale, const pkv_dims* dims,
                                         int32_t max_context_len, int32_t partition_tokens,
                                         void* workspace, size_t workspace_bytes,
                                         void* cuda_stream) {
  return multi_one_shot(out, q, k_cache, v_cache, block_tables, context_lens, query_start_loc,
                        num_q_tokens, max_query_len, scale, true, k_scale, v_scale, dims,
                        max_context_len, partition_tokens, workspace, workspace_bytes,
                        cuda_stream);
}

pkv_status pkv_decode_run_fp8(void* out, const void* q, const void* k_cache,
                              const void* v_cache, const int32_t* block_tables,
                              const int32_t* context_lens, float scale, float k_scale,
                              float v_scale, const pkv_dims* dims, int32_t max_context_len,
                              int32_t partition_tokens, void* workspace, size_t workspace_bytes,
                              void* cuda_stream) {
  DecodePlan plan;
  pkv_status st = make_plan(dims, max_context_len, partition_tokens, &plan);
  if (st != PKV_OK) return st;
  if (!is_fp8(dims->dtype)) return fail(PKV_ERR_UNSUPPORTED, "dims->dtype must be FP8");
  return run_decode(out, q, k_cache, v_cache, block_tables, context_lens, nullptr, 1, scale,
                    dims, plan, workspace, workspace_bytes, cuda_stream, k_scale, v_scale);
}

pkv_status pkv_paged_attention_decode_fp8(void* out, const void* q, const void* k_cache,
                                          const void* v_cache, const int32_t* block_tables,
                                          const int32_t* context_lens, float scale,
                                          float k_scale, float v_scale, const pkv_dims* dims,
                                          int32_t max_context_len, int32_t partition_tokens,
                                          void* workspace, size_t workspace_bytes,
                                          void* cuda_stream) {
  DecodePlan plan;
  pkv_status st = make_plan(dims, max_context_len, partition_tokens, &plan);
  if (st != PKV_OK) return st;
  if (!is_fp8(dims->dtype)) return fail(PKV_ERR_UNSUPPORTED, "dims->dtype must be FP8");
  if (!(k_scale > 0.f) || !(v_scale > 0.f) || !std::isfinite(k_scale) || !std::isfinite(v_scale))
    return fail(PKV_ERR_SHAPE, "k_scale and v_scale must be finite and positive");
  if (dims->num_seqs == 0) return PKV_OK;
  if ((st = check_workspace(plan, workspace, workspace_bytes)) != PKV_OK) return st;
  st = pkv_decode_plan(context_lens, dims, max_context_len, partition_tokens, workspace,
                       workspace_bytes, cuda_stream);
  if (st != PKV_OK) return st;
  return run_decode(out, q, k_cache, v_cache, block_tables, context_lens, nullptr, 1, scale,
                    dims, plan, workspace, workspace_bytes, cuda_stream, k_scale, v_scale);
}

size_t pkv_decode_shared_workspace_bytes(const pkv_dims* dims, int32_t max_context_len,
                                         int32_t partition_tokens) {
  DecodePlan plan;
  if (make_plan(dims, max_context_len, partition_tokens, &plan, -1, true) != PKV_OK) return 0;
  return plan.total;
}

pkv_status pkv_decode_shared_workspace_layout(const pkv_dims* dims, int32_t max_context_len,
                                              int32_t partition_tokens, int32_t* max_parts,
                                              size_t* part_o_offset, size_t* part_ml_offset,
                                              size_t* seq_prefix_offset) {
  DecodePlan plan;
  pkv_status st = make_plan(dims, max_context_len, partition_tokens, &plan, -1, true);
  if (st != PKV_OK) return st;
  if (max_parts) *max_parts = plan.max_parts;
  if (part_o_offset) *part_o_offset = plan.part_o_off;
  if (part_ml_offset) *part_ml_offset = plan.part_ml_off;
  if (seq_prefix_offset) *seq_prefix_offset = plan.seq_prefix_off;
  return PKV_OK;
}

pkv_status pkv_decode_plan_shared(const int32_t* context_lens, const int32_t* group_start,
                                  const int32_t* shared_blocks, int32_t num_groups,
                                  const pkv_dims* dims, int32_t max_context_len,
                                  int32_t partition_tokens, void* workspace,
                                  size_t workspace_bytes, void* cuda_stream) {
  return plan_shared(context_lens, group_start, shared_blocks, num_groups, dims,
                     max_context_len, partition_tokens, workspace, workspace_bytes, cuda_stream);
}

pkv_status pkv_decode_run_shared(void* out, const void* q, const void* k_cache,
                                 const void* v_cache, const int32_t* block_tables,
                                 const int32_t* context_lens, float scale, const pkv_dims* dims,
                                 int32_t max_context_len, int32_t partition_tokens,
                                 void* workspace, size_t workspace_bytes, void* cuda_stream) {
  return run_shared(out, q, k_cache, v_cache, block_tables, context_lens, scale, false, 1.f,
                    1.f, dims, max_context_len, partition_tokens, workspace, workspace_bytes,
                    cuda_stream);
}

pkv_status pkv_decode_run_shared_fp8(void* out, const void* q, const void* k_cache,
                                     const void* v_cache, const int32_t* block_tables,
                                     const int32_t* context_lens, float scale, float k_scale,
                                     float v_scale, const pkv_dims* dims,
                                     int32_t max_context_len, int32_t partition_tokens,
                                     void* workspace, size_t workspace_bytes,
                                     void* cuda_stream) {
  return run_shared(out, q, k_cache, v_cache, block_tables, context_lens, scale, true, k_scale,
                    v_scale, dims, max_context_len, partition_tokens, workspace,
                    workspace_bytes, cuda_stream);
}

pkv_status pkv_paged_attention_decode_shared(
    void* out, const void* q, const void* k_cache, const void* v_cache,
    const int32_t* block_tables, const int32_t* context_lens, const int32_t* group_start,
    const int32_t* shared_blocks, int32_t num_groups, float scale, const pkv_dims* dims,
    int32_t max_context_len, int32_t partition_tokens, void* workspace, size_t workspace_bytes,
    void* cuda_stream) {
  return shared_one_shot(out, q, k_cache, v_cache, block_tables, context_lens, group_start,
                         shared_blocks, num_groups, scale, false, 1.f, 1.f, dims,
                         max_context_len, partition_tokens, workspace, workspace_bytes,
                         cuda_stream);
}

pkv_status pkv_paged_attention_decode_shared_fp8(
    void* out, const void* q, const void* k_cache, const void* v_cache,
    const int32_t* block_tables, const int32_t* context_lens, const int32_t* group_start,
    const int32_t* shared_blocks, int32_t num_groups, float scale, float k_scale, float v_scale,
    const pkv_dims* dims, int32_t max_context_len, int32_t partition_tokens, void* workspace,
    size_t workspace_bytes, void* cuda_stream) {
  return shared_one_shot(out, q, k_cache, v_cache, block_tables, context_lens, group_start,
                         shared_blocks, num_groups, scale, true, k_scale, v_scale, dims,
                         max_context_len, partition_tokens, workspace, workspace_bytes,
                         cuda_stream);
}

pkv_status pkv_decode_prepare_tokens(const void* k, const void* v, void* k_cache, void* v_cache,
                                     const int32_t* block_tables, const int32_t* context_lens,
                                     const int32_t* token_seq, const int32_t* token_pos,
                                     int32_t num_tokens, int64_t* slot_mapping_out,
                                     float k_scale, float v_scale, const int32_t* group_start,
                                     const int32_t* shared_blocks, int32_t num_groups,
                                     const pkv_dims* dims, int32_t max_context_len,
                                     int32_t partition_tokens, void* workspace,
                                     size_t workspace_bytes, void* cuda_stream) {
  return prepare_tokens(k, v, k_cache, v_cache, block_tables, context_lens, token_seq, token_pos,
                        num_tokens, slot_mapping_out, k_scale, v_scale, group_start,
                        shared_blocks, num_groups, dims, max_context_len, partition_tokens,
                        workspace, workspace_bytes, cuda_stream);
}

pkv_status pkv_reshape_and_cache_fp8(const void* k, const void* v, void* k_cache, void* v_cache,
                                     const int64_t* slot_mapping, int32_t num_tokens,
                                     float k_scale, float v_scale, const pkv_dims* dims,
                                     void* cuda_stream) {
  pkv_status st = check_dims(dims, false);
  if (st != PKV_OK) return st;
  if (!is_fp8(dims->dtype)) return fail(PKV_ERR_UNSUPPORTED, "dims->dtype must be FP8");
  if (!(k_scale > 0.f) || !(v_scale > 0.f) || !std::isfinite(k_scale) || !std::isfinite(v_scale))
    return fail(PKV_ERR_SHAPE, "k_scale and v_scale must be finite and positive");
  if (num_tokens < 0) return fail(PKV_ERR_SHAPE, "num_tokens must be >= 0");
  if (num_tokens == 0) return PKV_OK;
  if (!k || !v || !k_cache || !v_cache || !slot_mapping)
    return fail(PKV_ERR_NULL, "a tensor pointer is NULL");
  if (!aligned16(k) || !aligned16(v) || !aligned16(k_cache) || !aligned16(v_cache))
    return fail(PKV_ERR_ALIGN, "k, v and the caches must be 16-byte aligned");
  if ((st = bind_device(k_cache, "k_cache")) != PKV_OK) return st;
  const int units = dims->num_kv_heads * dims->head_dim / 8;
  const int threads = units < 256 ? (units + 31) / 32 * 32 : 256;
  auto kern = dims->dtype == PKV_FP8_E5M2 ? pkv::reshape_and_cache_fp8_kernel<true>
                                          : pkv::reshape_and_cache_fp8_kernel<false>;
  cudaError_t e = launch(kern, dim3(num_tokens), dim3(threads), 0,
                         static_cast<cudaStream_t>(cuda_stream), static_cast<const uint4*>(k),
                         static_cast<const uint4*>(v), static_cast<uint8_t*>(k_cache),
                         static_cast<uint8_t*>(v_cache), slot_mapping, dims->num_kv_heads,
                         dims->head_dim, static_cast<int64_t>(dims->num_blocks) * pkv::kBlock,
                         k_scale, v_scale);
  if (e != cudaSuccess) return cuda_fail(e, "reshape_and_cache_fp8 launch");
  return PKV_OK;
}

pkv_status pkv_paged_prefill(void* out, const void* q, const void* k_cache, const void* v_cache,
                             const int32_t* block_tables, const int32_t* context_lens,
                             const int32_t* query_start_loc, int32_t num_q_tokens, float scale,
                             const pkv_dims* dims, int32_t max_context_len, void* cuda_stream) {
  pkv_status st = check_dims(dims, true);
  if (st != PKV_OK) return st;
  if (dims->dtype != PKV_BF16)
    return fail(PKV_ERR_UNSUPPORTED, "pkv_paged_prefill runs on bf16 pools only");
  if (dims->num_seqs > pkv::kPfMaxSeqs)
    return fail(PKV_ERR_UNSUPPORTED, "pkv_paged_prefill takes at most %d sequences a call",
                pkv::kPfMaxSeqs);
  if (num_q_tokens < 0 || max_context_len < 0)
    return fail(PKV_ERR_SHAPE, "num_q_tokens and max_context_len must be >= 0");
  if (dims->num_seqs == 0 || num_q_tokens == 0) return PKV_OK;
  if (!out || !q || !k_cache || !v_cache || !block_tables || !context_lens || !query_start_loc)
    return fail(PKV_ERR_NULL, "a tensor pointer is NULL");
  if (!aligned16(out) || !aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache))
    return fail(PKV_ERR_ALIGN, "out, q and the caches must be 16-byte aligned");
  if (!std::isfinite(scale)) return fail(PKV_ERR_SHAPE, "scale must be finite");
  if ((st = bind_device(out, "out")) != PKV_OK) return st;
  const int group = dims->num_q_heads / dims->num_kv_heads;
  const int tpt = pkv::kPfRows / group;
  CUtensorMap mq, mk, mv;
  if ((st = encode_q_map(&mq, q, num_q_tokens, dims, group, tpt)) != PKV_OK) return st;
  if ((st = encode_pool_map(&mk, k_cache, dims)) != PKV_OK) return st;
  if ((st = encode_pool_map(&mv, v_cache, dims)) != PKV_OK) return st;
  const int64_t table_len = static_cast<int64_t>(dims->max_blocks_per_seq) * pkv::kBlock;
  pkv::PrefillParams prm;
  prm.out = out;
  prm.block_tables = block_tables;
  prm.context_lens = context_lens;
  prm.query_start_loc = query_start_loc;
  prm.num_seqs = dims->num_seqs;
  prm.num_q_tokens = num_q_tokens;
  prm.num_q_heads = dims->num_q_heads;
  prm.num_kv_heads = dims->num_kv_heads;
  prm.group = group;
  prm.tokens_per_tile = tpt;
  prm.max_blocks_per_seq = dims->max_blocks_per_seq;
  prm.num_blocks = dims->num_blocks;
  prm.max_len = static_cast<int32_t>(max_context_len < table_len ? max_context_len : table_len);
  prm.qk_scale_log2 = scale * pkv::kLog2e;
  // tiles of all chunks together: at most ceil(T / tpt) + B
  const int64_t units_bound =
      (static_cast<int64_t>(num_q_tokens + tpt - 1) / tpt + dims->num_seqs) * dims->num_kv_heads;
  cudaStream_t stream = static_cast<cudaStream_t>(cuda_stream);
  return dims->head_dim == 128 ? launch_prefill<128>(mq, mk, mv, prm, units_bound, stream)
                               : launch_prefill<64>(mq, mk, mv, prm, units_bound, stream);
}

pkv_status pkv_paged_attention_decode_static(void* out, const void* q, const void* k_cache,
                                             const void* v_cache, const int32_t* block_tables,
                                             const int32_t* context_lens, float scale,
                                             const pkv_dims* dims, int32_t max_context_len,
                                             int32_t partition_tokens, void* cuda_stream) {
  DecodePlan plan;
  pkv_status st = make_plan(dims, max_context_len, partition_tokens, &plan);
  if (st != PKV_OK) return st;
  if (plan.total > PKV_STATIC_WORKSPACE_BYTES)
    return fail(PKV_ERR_WORKSPACE,
                "this decode needs %zu bytes of scratch but the built-in scratch holds %u; "
                "call pkv_paged_attention_decode with a workspace of your own",
                plan.total, (unsigned)PKV_STATIC_WORKSPACE_BYTES);
  if (dims->num_seqs == 0) return PKV_OK;
  if (!out || !q || !k_cache || !v_cache || !block_tables || !context_lens)
    return fail(PKV_ERR_NULL, "a tensor pointer is NULL");
  // The scratch address is per device: bind the device that owns `out` (the
  // device the kernels run on) before looking it up.
  if ((st = bind_device(out, "out")) != PKV_OK) return st;
  const void* const ptrs[] = {q, k_cache, v_cache, block_tables, context_lens};
  const char* const names[] = {"q", "k_cache", "v_cache", "block_tables", "context_lens"};
  if ((st = check_same_device(ptrs, names, 5)) != PKV_OK) return st;
  void* ws = nullptr;
  if ((st = static_workspace(static_cast<cudaStream_t>(cuda_stream), &ws)) != PKV_OK) return st;
  return pkv_paged_attention_decode(out, q, k_cache, v_cache, block_tables, context_lens, scale,
                                    dims, max_context_len, partition_tokens, ws,
                                    PKV_STATIC_WORKSPACE_BYTES, cuda_stream);
}

pkv_status pkv_reshape_and_cache(const void* k, const void* v, void* k_cache, void* v_cache,
                                 const int64_t* slot_mapping, int32_t num_tokens,
                                 const pkv_dims* dims, void* cuda_stream) {
  pkv_status st = check_dims(dims, false);
  if (st != PKV_OK) return st;
  if (is_fp8(dims->dtype))
    return fail(PKV_ERR_UNSUPPORTED, "FP8 caches quantise on write: use pkv_reshape_and_cache_fp8");
  if (num_tokens < 0) return fail(PKV_ERR_SHAPE, "num_tokens must be >= 0");
  if (num_tokens == 0) return PKV_OK;
  if (!k || !v || !k_cache || !v_cache || !slot_mapping)
    return fail(PKV_ERR_NULL, "a tensor pointer is NULL");
  if (!aligned16(k) || !aligned16(v) || !aligned16(k_cache) || !aligned16(v_cache))
    return fail(PKV_ERR_ALIGN, "k, v and the caches must be 16-byte aligned");
  if ((st = bind_device(k_cache, "k_cache")) != PKV_OK) return st;
  const int row_bytes = dims->head_dim * elem_bytes(dims->dtype);
  const int units = dims->num_kv_heads * row_bytes / 16;
  int threads = units < 256 ? (units + 31) / 32 * 32 : 256;
  cudaError_t e = launch(pkv::reshape_and_cache_kernel, dim3(num_tokens), dim3(threads), 0,
                         static_cast<cudaStream_t>(cuda_stream), static_cast<const uint4*>(k),
                         static_cast<const uint4*>(v), static_cast<uint8_t*>(k_cache),
                         static_cast<uint8_t*>(v_cache), slot_mapping, dims->num_kv_heads,
                         row_bytes, static_cast<int64_t>(dims->num_blocks) * pkv::kBlock);
  if (e != cudaSuccess) return cuda_fail(e, "reshape_and_cache launch");
  return PKV_OK;
}

pkv_status pkv_copy_blocks(void* k_cache, void* v_cache, const int64_t* pairs,
                           int32_t num_pairs, const pkv_dims* dims, void* cuda_stream) {
  pkv_status st = check_dims(dims, false);
  if (st != PKV_OK) return st;
  if (num_pairs < 0) return fail(PKV_ERR_SHAPE, "num_pairs must be >= 0");
  if (num_pairs == 0) return PKV_OK;
  if (!k_cache || !v_cache || !pairs) return fail(PKV_ERR_NULL, "a pointer is NULL");
  if (!aligned16(k_cache) || !aligned16(v_cache))
    return fail(PKV_ERR_ALIGN, "the caches must be 16-byte aligned");
  if ((st = bind_device(k_cache, "k_cache")) != PKV_OK) return st;
  const int64_t block_bytes = static_cast<int64_t>(dims->num_kv_heads) * pkv::kBlock *
                              dims->head_dim * elem_bytes(dims->dtype);
  const unsigned chunks =
      static_cast<unsigned>((block_bytes + pkv::kCopyChunk - 1) / pkv::kCopyChunk);
  if (chunks > 65535) return fail(PKV_ERR_UNSUPPORTED, "block too large for copy_blocks");
  dim3 grid(static_cast<unsigned>(num_pairs), chunks, 2);
  cudaError_t e = launch(pkv::copy_blocks_kernel, grid, dim3(32), 0,
                         static_cast<cudaStream_t>(cuda_stream), static_cast<uint8_t*>(k_cache),
                         static_cast<uint8_t*>(v_cache), pairs, block_bytes, dims->num_blocks);
  if (e != cudaSuccess) return cuda_fail(e, "copy_blocks launch");
  return PKV_OK;
}

pkv_status pkv_validate_copy_pairs(const int64_t* pairs_host, int32_t num_pairs,
                                   int32_t num_blocks) {
  if (num_pairs < 0 || num_blocks <= 0) return fail(PKV_ERR_SHAPE, "bad counts");
  if (num_pairs == 0) return PKV_OK;
  if (!pairs_host) return fail(PKV_ERR_NULL, "pairs_host is NULL");
  std::vector<uint8_t> role(static_cast<size_t>(num_blocks), 0);  // bit0 src, bit1 dst
  for (int32_t i = 0; i < num_pairs; ++i) {
    const int64_t s = pairs_host[2 * i], t = pairs_host[2 * i + 1];
    if (s < 0 || s >= num_blocks || t < 0 || t >= num_blocks)
      return fail(PKV_ERR_PAIRS, "pair %d (%lld, %lld) outside [0, %d)", i, (long long)s,
                  (long long)t, num_blocks);
    if (role[t] & 2u) return fail(PKV_ERR_PAIRS, "destination %lld repeats", (long long)t);
    role[s] |= 1u;
    role[t] |= 2u;
  }
  for (int32_t i = 0; i < num_blocks; ++i) {
    if (role[i] == 3u) return fail(PKV_ERR_PAIRS, "block %d is both a source and a destination", i);
  }
  return PKV_OK;
}

pkv_status pkv_slot_mapping(int64_t* slot_mapping, const int32_t* block_tables,
                            const int32_t* context_lens, const int32_t* token_seq,
                            const int32_t* token_pos, int32_t num_tokens, const pkv_dims* dims,
                            void* cuda_stream) {
  pkv_status st = check_dims(dims, true);
  if (st != PKV_OK) return st;
  if (num_tokens < 0) return fail(PKV_ERR_SHAPE, "num_tokens must be >= 0");
  if (num_tokens == 0) return PKV_OK;
  if (!slot_mapping || !block_tables) return fail(PKV_ERR_NULL, "a pointer is NULL");
  if (!token_pos && !context_lens)
    return fail(PKV_ERR_NULL, "context_lens is needed when token_pos is NULL");
  if (!token_seq && num_tokens > dims->num_seqs)
    return fail(PKV_ERR_SHAPE, "without token_seq there is one token per sequence");
  if ((st = bind_device(slot_mapping, "slot_mapping")) != PKV_OK) return st;
  const unsigned grid = static_cast<unsigned>((num_tokens + 255) / 256);
  cudaError_t e = launch(pkv::slot_mapping_kernel, dim3(grid), dim3(256), 0,
                         static_cast<cudaStream_t>(cuda_stream), slot_mapping, block_tables,
                         context_lens, token_seq, token_pos, num_tokens, dims->num_seqs,
                         dims->max_blocks_per_seq, dims->num_blocks);
  if (e != cudaSuccess) return cuda_fail(e, "slot_mapping launch");
  return PKV_OK;
}

pkv_status pkv_selftest_wait_timeout(void* cuda_stream) {
  cudaError_t e = launch(pkv::wait_timeout_selftest_kernel, dim3(1), dim3(32), 0,
                         static_cast<cudaStream_t>(cuda_stream));
  if (e != cudaSuccess) return cuda_fail(e, "self-test launch");
  return PKV_OK;
}

pkv_status pkv_check_device_error(void* cuda_stream, uint32_t* bits_out) {
  cudaError_t e;
  if (cuda_stream) {
    // read the error word of the device that owns the stream
    int dev = -1, cur = -1;
    e = cudaStreamGetDevice(static_cast<cudaStream_t>(cuda_stream), &dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaStreamGetDevice");
    if (cudaGetDevice(&cur) == cudaSuccess && cur != dev) {
      e = cudaSetDevice(dev);
      if (e != cudaSuccess) return cuda_fail(e, "cudaSetDevice");
    }
  }
  e = cudaStreamSynchronize(static_cast<cudaStream_t>(cuda_stream));
  if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
  unsigned int bits = 0;
  e = cudaMemcpyFromSymbol(&bits, pkv::g_device_error, sizeof bits);
  if (e != cudaSuccess) return cuda_fail(e, "reading the device error word");
  const unsigned int zero = 0;
  e = cudaMemcpyToSymbol(pkv::g_device_error, &zero, sizeof zero);
  if (e != cudaSuccess) return cuda_fail(e, "clearing the device error word");
  if (bits_out) *bits_out = bits;
  if (bits & PKV_DEVERR_TIMEOUT) return fail(PKV_ERR_DEVICE_TIMEOUT, "device wait timed out (bits 0x%x)", bits);
  if (bits) return fail(PKV_ERR_DEVICE_INDEX, "device index error (bits 0x%x)", bits);
  return PKV_OK;
}

const char* pkv_status_string(pkv_status status) {
  switch (status) {
    case PKV_OK: return "ok";
    case PKV_ERR_NULL: return "null pointer";
    case PKV_ERR_SHAPE: return "inconsistent shape";
    case PKV_ERR_UNSUPPORTED: return "unsupported configuration";
    case PKV_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
    case PKV_ERR_PAIRS: return "invalid copy pairs";
    case PKV_ERR_CUDA: return "CUDA error";
    case PKV_ERR_DEVICE_INDEX: return "invalid index met on the device";
    case PKV_ERR_ALIGN: return "pointer not 16-byte aligned";
    case PKV_ERR_DEVICE_TIMEOUT: return "device wait timed out";
    case PKV_ERR_NO_BLOCKS: return "no KV block left in the pool";
    case PKV_ERR_NOT_FOUND: return "unknown or duplicate sequence id";
  }
  return "unknown status";
}

const char* pkv_last_error_message(void) { return g_last_error.c_str(); }

}  // extern "C"
