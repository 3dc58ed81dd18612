/*
 * pkv.h -- C ABI of the B200 (sm_100a) paged KV-cache decode library.
 *
 * The operations are those of PagedAttention decode as the pages state the
 * problem:
 *  - the KV cache is cut into fixed-size blocks of 16 tokens; a per-sequence
 *    block table maps each logical block to a physical block of one shared
 *    pool, and attention visits the sequence block by block, looking up each
 *    block and loading it (ipipp.com vLLM article, section
 *    "二、PagedAttention分页原理深度剖析");
 *  - new tokens reach their physical slot through slot_mapping ("vLLM" wiki
 *    entry, wiki.bytelighting.cn, section "Flattened 布局与 slot_mapping");
 *  - blocks shared by several sequences are reference counted and copied on
 *    write ("vLLM 深读：用 PagedAttention 撑起高并发 LLM 推理", section
 *    "先看浪费在哪里").
 * Beyond one query token per sequence the same decode kernel serves chunks of
 * several causal query tokens (pkv_paged_attention_multi), batches whose
 * consecutive sequences share their leading blocks, each such block read once
 * for the group (pkv_paged_attention_decode_shared), and pools of FP8 (e4m3
 * or e5m2) codes with per-pool scales (the *_fp8 calls).  The host block
 * manager that produces tables, slots, copy pairs and shared-prefix groups is
 * declared in pkv_block_manager.h.
 *
 * Conventions for every call:
 *  - Pointers are DEVICE pointers unless the argument says "host".  The caller
 *    owns every buffer; the library never allocates device memory.  Scratch
 *    memory (the decode workspace) is passed in by the caller.
 *  - Every call is asynchronous on `cuda_stream` (a cudaStream_t; NULL is the
 *    legacy default stream).  A returned PKV_OK means the work was validated
 *    and enqueued, not that it has finished.
 *  - The return value reports what the host can see: bad arguments, an
 *    unsupported shape, a workspace that is too small, a failed launch.
 *  - Indices the host cannot see (block-table entries, slots, copy pairs,
 *    context lengths, all in device memory) are checked by the kernels.  An
 *    invalid one is skipped -- never dereferenced -- and a bit is set in a
 *    per-device error word; pkv_check_device_error() reads and clears it.  No
 *    kernel traps, asserts or waits without a bound: every internal wait gives
 *    up after about one second and reports PKV_DEVERR_TIMEOUT.
 *  - All device pointers must be 16-byte aligned.  Calls that launch work make
 *    the device owning their output buffer current (the library carries its
 *    own CUDA runtime, so the caller's current device is not seen); a host
 *    pointer where device memory is expected is rejected with PKV_ERR_SHAPE.
 *    The stream must belong to that device.
 *
 * Layouts (row-major, innermost last):
 *  - q, out         [num_seqs][num_q_heads][head_dim], dtype of the cache
 *                   (bf16 for FP8 pools)
 *  - k, v (new)     [num_tokens][num_kv_heads][head_dim]
 *  - k_cache,v_cache[num_blocks][num_kv_heads][16][head_dim]  ("HND": one
 *                   (block, kv head) tile of 16 tokens is contiguous)
 *  - block_tables   int32 [num_seqs][max_blocks_per_seq]; entries at or past
 *                   ceil(context_len/16) are never read
 *  - context_lens   int32 [num_seqs]; the length includes the token being
 *                   decoded; 0 is allowed and gives a zero output
 *  - slot_mapping   int64 [num_tokens]; slot = block*16 + offset; negative
 *                   slots mark padding tokens and are skipped
 *  - pairs          int64 [num_pairs][2] = (src block, dst block)
 *  - query head h reads kv head h / (num_q_heads / num_kv_heads).
 */
#ifndef PKV_H
#define PKV_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum pkv_status {
    PKV_OK = 0,
    PKV_ERR_NULL = 1,          /* a required pointer is NULL */
    PKV_ERR_SHAPE = 2,         /* inconsistent sizes (e.g. Hq % Hkv != 0, negative counts) */
    PKV_ERR_UNSUPPORTED = 3,   /* block_size != 16, head_dim not 64/128, group > 16, dtype */
    PKV_ERR_WORKSPACE = 4,     /* workspace NULL, misaligned or smaller than required */
    PKV_ERR_PAIRS = 5,         /* copy pairs: out of range, repeated dst, or dst also a src */
    PKV_ERR_CUDA = 6,          /* a CUDA runtime call or a launch failed */
    PKV_ERR_DEVICE_INDEX = 7,  /* a kernel met an invalid index (see the error bits) */
    PKV_ERR_ALIGN = 8,         /* a pointer is not 16-byte aligned */
    PKV_ERR_DEVICE_TIMEOUT = 9,/* a kernel's bounded wait expired */
    PKV_ERR_NO_BLOCKS = 10,    /* block manager: the pool has no block left */
    PKV_ERR_NOT_FOUND = 11     /* block manager: unknown (or already used) sequence id */
} pkv_status;

typedef enum pkv_dtype {
    PKV_F32 = 0,       /* IEEE binary32 */
    PKV_BF16 = 1,      /* bfloat16; arithmetic in fp32, output rounded to nearest even */
    PKV_FP8_E4M3 = 2,  /* caches hold FP8 e4m3 codes (one byte; value = code x the pool's
                          scale); q, out and the new K/V are bf16; head_dim 128 only */
    PKV_FP8_E5M2 = 3   /* the same with e5m2 codes (1-5-2, bias 15: the upper byte of an
                          IEEE binary16; widening to f16 is a byte move) */
} pkv_dtype;

/* Bits of the per-device error word. */
#define PKV_DEVERR_BLOCK   0x1u   /* block-table entry outside [0, num_blocks) */
#define PKV_DEVERR_SLOT    0x2u   /* slot beyond num_blocks*16 */
#define PKV_DEVERR_LEN     0x4u   /* context length < 0 or > max_blocks_per_seq*16 or > max_context_len */
#define PKV_DEVERR_PAIR    0x8u   /* copy pair outside [0, num_blocks) */
#define PKV_DEVERR_POS     0x10u  /* slot-mapping position outside the block table */
#define PKV_DEVERR_TIMEOUT 0x20u  /* a bounded wait gave up */
#define PKV_DEVERR_GROUP   0x40u  /* shared-prefix groups: bounds not nondecreasing in
                                     [0, num_seqs], or a shared block count < 0 or past
                                     a member's full blocks */

typedef struct pkv_dims {
    int32_t num_seqs;            /* B */
    int32_t num_q_heads;         /* Hq */
    int32_t num_kv_heads;        /* Hkv; Hq % Hkv == 0, Hq/Hkv <= 16 */
    int32_t head_dim;            /* D: 64 or 128 */
    int32_t block_size;          /* must be 16 */
    int32_t num_blocks;          /* NB, physical blocks in each of the K and V pools */
    int32_t max_blocks_per_seq;  /* MB, width of block_tables */
    pkv_dtype dtype;             /* of q, out, k, v and both caches */
} pkv_dims;

/*
 * Partition size the decode will use for `partition_tokens` (0 = automatic):
 * a multiple of 16.  A sequence longer than the partition is split into
 * partitions computed independently and merged by log-sum-exp.  When the
 * result is >= max_context_len the decode runs single-pass.
 * Returns 0 for invalid dims.
 */
int32_t pkv_decode_partition_tokens(const pkv_dims *dims, int32_t max_context_len,
                                    int32_t partition_tokens);

/*
 * Bytes of device workspace pkv_paged_attention_decode needs for these
 * arguments (work list, scheduling counters and, when sequences are split,
 * the per-partition partial results).  Returns 0 for invalid dims.
 */
size_t pkv_decode_workspace_bytes(const pkv_dims *dims, int32_t max_context_len,
                                  int32_t partition_tokens);

/*
 * Offsets inside the workspace of the split-K partial results, for tests that
 * inspect them: part_o is float [B][Hq][max_parts][D] (each partition's
 * normalised output), part_ml is float [B][Hq][max_parts][2] = (m, l) with
 * l = sum exp(scale*q.k - m) over the partition.  m is the partition's max of
 * scale*q.k for fp32; for bf16 it is a reference value at most 8 ln 2 below
 * that max (the kernel only moves its running max when it grows by more than
 * that), which the merge treats the same way.  Only partitions of sequences
 * with more than one partition are written.
 * Returns PKV_ERR_SHAPE when the decode would run single-pass.
 */
pkv_status pkv_decode_workspace_layout(const pkv_dims *dims, int32_t max_context_len,
                                       int32_t partition_tokens, int32_t *max_parts,
                                       size_t *part_o_offset, size_t *part_ml_offset);

/*
 * Paged decode attention: for each sequence s and query head h,
 *   out[s][h] = softmax_j(scale * q[s][h] . K_j) V_j   over j < context_lens[s],
 * with K_j, V_j read from physical block block_tables[s][j/16], slot j%16,
 * kv head h/(Hq/Hkv).  One query token per sequence.
 *
 * max_context_len (host) must be >= every context length; it sizes the
 * partitions and the workspace (a larger value is always safe; a length above
 * it is clamped and flagged PKV_DEVERR_LEN).  partition_tokens: 0 = automatic,
 * else a multiple of 16 no larger than 8192 (e.g. 512); a sequence longer
 * than 8192 tokens is therefore always split.  workspace: device scratch of at least
 * pkv_decode_workspace_bytes() bytes, 256-byte aligned, not shared with a
 * decode that may run concurrently.  Launches a planning kernel, the decode
 * kernel and, when some sequence is split, the merge kernel, in that order
 * (pkv_decode_plan followed by pkv_decode_run).
 */
pkv_status pkv_paged_attention_decode(void *out, const void *q, const void *k_cache,
                                      const void *v_cache, const int32_t *block_tables,
                                      const int32_t *context_lens, float scale,
                                      const pkv_dims *dims, int32_t max_context_len,
                                      int32_t partition_tokens, void *workspace,
                                      size_t workspace_bytes, void *cuda_stream);

/*
 * Several query tokens per sequence: chunks of new tokens (tokens proposed by
 * speculative decoding and being verified, or a slice of a prompt).  The
 * chunk of sequence s is rows query_start_loc[s] .. query_start_loc[s+1]-1
 * of q and out (int32 [num_seqs+1], device, non-decreasing, the cu_seqlens of
 * the flattened layout); its i-th token sits at position L - n + i, where
 * L = context_lens[s] already counts the chunk (its K/V written by
 * reshape_and_cache first) and n is the chunk length, and attends causally
 * to keys 0 .. L - n + i:
 *   out[row][h] = softmax_{j <= L-n+i}(scale * q[row][h] . K_j) V_j.
 * q, out: [num_q_tokens][Hq][D].  max_query_len (host) bounds every chunk;
 * Hq/Hkv must be at most 16.  Chunks of any length are accepted: the rows of
 * one kv head are taken 16 (whole tokens) at a time, each group of rows
 * reading only the keys it can see, so a long chunk (a prompt prefilled in
 * one call) re-reads the KV once per group.  A chunk longer than max_query_len or than its context
 * is clamped, and a chunk reaching outside rows [0, num_q_tokens) is skipped;
 * both are flagged PKV_DEVERR_LEN.  With n = 1 everywhere this is
 * pkv_paged_attention_decode.  Workspace: pkv_multi_workspace_bytes().
 * bf16 and fp32 pools; FP8 pools go through pkv_paged_attention_multi_fp8
 * and pkv_multi_run_fp8 (below), which take the pools' scales (the plain
 * calls return PKV_ERR_UNSUPPORTED for them).
 */
size_t pkv_multi_workspace_bytes(const pkv_dims *dims, int32_t num_q_tokens,
                                 int32_t max_context_len, int32_t partition_tokens);

pkv_status pkv_paged_attention_multi(void *out, const void *q, const void *k_cache,
                                     const void *v_cache, const int32_t *block_tables,
                                     const int32_t *context_lens, const int32_t *query_start_loc,
                                     int32_t num_q_tokens, int32_t max_query_len, float scale,
                                     const pkv_dims *dims, int32_t max_context_len,
                                     int32_t partition_tokens, void *workspace,
                                     size_t workspace_bytes, void *cuda_stream);

/*
 * The same operation as pkv_paged_attention_multi, for long chunks (chunked
 * prefill: vampireachao.github.io "vllm", section "第二层：请求不该排队等整批";
 * the flattened layout of the "vLLM" wiki entry, section "Flattened 布局与
 * slot_mapping"): chunk token i of sequence s, at position L - n + i of its
 * context, attends to keys 0 .. L - n + i found block by block through the
 * table.  Runs on the tcgen05 tensor cores with the accumulators in tensor
 * memory: a work unit is 128 query rows (floor(128/g) chunk tokens times the
 * g query heads of one kv head), and every 128-key tile of K and V is read
 * once per unit.  For chunks of a few tokens the decode kernel behind
 * pkv_paged_attention_multi is the better fit.
 *  - bf16 pools only (PKV_ERR_UNSUPPORTED otherwise); head_dim 64 or 128;
 *    Hq/Hkv at most 16; at most 2048 sequences a call.
 *  - q, out: bf16 [num_q_tokens][Hq][D]; query_start_loc int32 [B+1] (device).
 *  - No workspace, no split-K: the call allocates nothing and needs none.
 *  - Device-side errors as for the multi call: a chunk longer than its
 *    context or outside [0, num_q_tokens) is skipped and flags
 *    PKV_DEVERR_LEN; a length past the table or max_context_len is clamped
 *    and flagged PKV_DEVERR_LEN; a table entry outside [0, num_blocks) is
 *    read as block 0 and flags PKV_DEVERR_BLOCK.
 */
pkv_status pkv_paged_prefill(void *out, const void *q, const void *k_cache, const void *v_cache,
                             const int32_t *block_tables, const int32_t *context_lens,
                             const int32_t *query_start_loc, int32_t num_q_tokens, float scale,
                             const pkv_dims *dims, int32_t max_context_len, void *cuda_stream);

/*
 * The run half of pkv_paged_attention_multi, over a plan made by
 * pkv_decode_plan (the plan depends only on the context lengths); the same
 * rules as pkv_decode_run apply, with the workspace sized by
 * pkv_multi_workspace_bytes.
 */
pkv_status pkv_multi_run(void *out, const void *q, const void *k_cache, const void *v_cache,
                         const int32_t *block_tables, const int32_t *context_lens,
                         const int32_t *query_start_loc, int32_t num_q_tokens,
                         int32_t max_query_len, float scale, const pkv_dims *dims,
                         int32_t max_context_len, int32_t partition_tokens, void *workspace,
                         size_t workspace_bytes, void *cuda_stream);

/*
 * The two halves of pkv_paged_attention_decode, for callers that decode
 * several layers (several cache pools) with the same context lengths: plan
 * once per step, run once per layer.
 *
 * pkv_decode_plan launches the planning kernel: it reads context_lens and
 * writes the work list into the workspace.  pkv_decode_run launches the
 * decode kernel (and the merge kernel when some sequence is split) using the
 * plan found in the workspace; every argument it shares with the plan call
 * (dims, max_context_len, partition_tokens, the workspace and context_lens'
 * contents) must be the same as at planning time, and runs using one plan
 * must not overlap on the GPU.  After a device error, plan again.
 */
pkv_status pkv_decode_plan(const int32_t *context_lens, const pkv_dims *dims,
                           int32_t max_context_len, int32_t partition_tokens, void *workspace,
                           size_t workspace_bytes, void *cuda_stream);

pkv_status pkv_decode_run(void *out, const void *q, const void *k_cache, const void *v_cache,
                          const int32_t *block_tables, const int32_t *context_lens, float scale,
                          const pkv_dims *dims, int32_t max_context_len,
                          int32_t partition_tokens, void *workspace, size_t workspace_bytes,
                          void *cuda_stream);

/*
 * Decode with built-in scratch, for callers that cannot allocate device
 * memory.  There is no counterpart in the paper: it is a convenience of this
 * library.  Some callers cannot call cudaMalloc themselves -- for instance an
 * engine that hands almost all HBM to its KV-cache pool at start-up and lets
 * nothing else allocate, or a host runtime that reaches this library only
 * through the C ABI and owns no device allocator.  This entry point takes the
 * same arguments as pkv_paged_attention_decode minus the workspace: the
 * scratch is a fixed array of PKV_STATIC_WORKSPACE_BYTES inside the library,
 * reserved on every GPU that loads the library until the process exits.
 *  - The call allocates nothing.  It runs on the device that owns `out`;
 *    q, the caches, block_tables and context_lens must be on that device too
 *    (else PKV_ERR_SHAPE).  The first call on a device makes that device
 *    current for the library, looks up the array's device address there
 *    (cudaGetSymbolAddress) and caches it for the rest of the process; make
 *    that first call before any stream capture (a first call on a capturing
 *    stream returns PKV_ERR_UNSUPPORTED).  The cached address does not
 *    survive a cudaDeviceReset of that device.
 *  - A decode whose pkv_decode_workspace_bytes() exceeds
 *    PKV_STATIC_WORKSPACE_BYTES is rejected with PKV_ERR_WORKSPACE (the
 *    message gives both sizes); use pkv_paged_attention_decode with a
 *    caller-provided workspace instead.
 *  - All calls in the process share the one array per device, and each call
 *    leaves its contents behind.  Nothing in it needs to start at zero (the
 *    planning kernel resets the counters it uses), but calls that overlap on
 *    the GPU -- on different streams, or from different host threads -- race
 *    on it and must be serialised by the caller.
 */
#define PKV_STATIC_WORKSPACE_BYTES (32u << 20)

pkv_status pkv_paged_attention_decode_static(void *out, const void *q, const void *k_cache,
                                             const void *v_cache, const int32_t *block_tables,
                                             const int32_t *context_lens, float scale,
                                             const pkv_dims *dims, int32_t max_context_len,
                                             int32_t partition_tokens, void *cuda_stream);

/*
 * The prologue of a decode step in one launch (no counterpart of its own in
 * the pages: it fuses three of their steps).  For every sequence s with
 * L = context_lens[s] >= 1 the new token at position L - 1 is written:
 * slot = block_tables[s][(L-1)/16] * 16 + (L-1) % 16 (slot indexing, the
 * wiki entry's "Flattened 布局与 slot_mapping"), then k[s], v[s] ([num_seqs]
 * [Hkv][D], same dtype as the pools) are copied into that slot as
 * pkv_reshape_and_cache does; and the decode plan is built into `workspace`
 * exactly as pkv_decode_plan builds it (same arguments, same workspace
 * size).  The plan is built by one CTA while the others write the tokens.
 * slot_mapping_out (int64 [num_seqs], may be NULL) receives each sequence's
 * slot, -1 for L = 0 (no new token, nothing written) or a flagged entry.
 * Equivalent to pkv_slot_mapping (context-length mode) + pkv_reshape_and_cache
 * + pkv_decode_plan, except that L = 0 is not an error here.  Device-side
 * errors: PKV_DEVERR_POS (L - 1 past the table), PKV_DEVERR_BLOCK (entry out
 * of range), PKV_DEVERR_LEN (lengths, as the plan).  Follow it with
 * pkv_decode_run (or pkv_decode_run_fp8) on the same workspace.
 * pkv_decode_prepare_fp8: FP8 pools; k, v are bf16 and quantised as
 * pkv_reshape_and_cache_fp8 does.
 */
pkv_status pkv_decode_prepare(const void *k, const void *v, void *k_cache, void *v_cache,
                              const int32_t *block_tables, const int32_t *context_lens,
                              int64_t *slot_mapping_out, const pkv_dims *dims,
                              int32_t max_context_len, int32_t partition_tokens, void *workspace,
                              size_t workspace_bytes, void *cuda_stream);

pkv_status pkv_decode_prepare_fp8(const void *k, const void *v, void *k_cache, void *v_cache,
                                  const int32_t *block_tables, const int32_t *context_lens,
                                  int64_t *slot_mapping_out, float k_scale, float v_scale,
                                  const pkv_dims *dims, int32_t max_context_len,
                                  int32_t partition_tokens, void *workspace,
                                  size_t workspace_bytes, void *cuda_stream);

/*
 * The prologue for any list of new tokens in one launch: the tails of parallel
 * samples, a chunk of several query tokens per sequence.  Token t (k[t], v[t],
 * [num_tokens][Hkv][D]) of sequence token_seq[t] at position token_pos[t]
 * (int32 [num_tokens] each, device) is written into its slot
 * block_tables[seq][pos/16] * 16 + pos % 16 exactly as pkv_slot_mapping (token
 * mode) followed by pkv_reshape_and_cache (or pkv_reshape_and_cache_fp8 for
 * FP8 pools, with k_scale and v_scale; they are ignored otherwise) does, with
 * the same device-side checks (PKV_DEVERR_POS, PKV_DEVERR_BLOCK; a flagged
 * token is skipped); slot_mapping_out (int64 [num_tokens], may be NULL)
 * receives the slots, -1 for flagged tokens.  In the same launch one CTA
 * builds the decode plan from context_lens: with group_start == NULL the plan
 * of pkv_decode_plan (follow with pkv_decode_run, pkv_multi_run or their
 * _fp8 forms; workspace sized for that run), else the shared-prefix plan of
 * pkv_decode_plan_shared over (group_start, shared_blocks, num_groups)
 * (follow with pkv_decode_run_shared or its _fp8 form; workspace
 * pkv_decode_shared_workspace_bytes).  Copy-on-write copies (pkv_copy_blocks)
 * issued before it on the stream complete before any token is written.
 * Two tokens with the same slot leave it unspecified.
 */
pkv_status pkv_decode_prepare_tokens(const void *k, const void *v, void *k_cache, void *v_cache,
                                     const int32_t *block_tables, const int32_t *context_lens,
                                     const int32_t *token_seq, const int32_t *token_pos,
                                     int32_t num_tokens, int64_t *slot_mapping_out,
                                     float k_scale, float v_scale, const int32_t *group_start,
                                     const int32_t *shared_blocks, int32_t num_groups,
                                     const pkv_dims *dims, int32_t max_context_len,
                                     int32_t partition_tokens, void *workspace,
                                     size_t workspace_bytes, void *cuda_stream);

/*
 * FP8 KV cache.  The pages list FP8 among the quantisation formats and note
 * that memory saved holds more KV blocks ("vLLM 深读", section "引擎的分层结构";
 * "vllm" by vampireachao, "第三层：图、核、量化"); here the cache itself is FP8:
 * each pool has one scale, a cached element is code x scale.
 *  - pkv_reshape_and_cache_fp8: k, v are bf16 [T][Hkv][D]; each value x is
 *    stored as code = e4m3(x / scale) (division in float, round to nearest
 *    even, saturate to +-448); slots as in pkv_reshape_and_cache.
 *  - pkv_paged_attention_decode_fp8 / pkv_decode_run_fp8: as the bf16 calls,
 *    over e4m3 pools with their k_scale and v_scale; q and out are bf16.
 *    Arithmetic when every sequence's query rows (its chunk's tokens x heads
 *    per kv head, for the longest chunk) number at most 16 and there is no
 *    shared prefix: the codes (e4m3
 *    or e5m2) enter the tensor cores as they are, q (times a power of two per
 *    row) and the softmax weights as two e4m3 terms each (the rounded value
 *    and 16 x its rounding remainder, about 8 significant bits), products
 *    accumulate in fp32.  Otherwise: codes are widened exactly to f16, q is
 *    rounded to f16 (|q| above 65504 saturates), products accumulate in fp32.
 * dims->dtype must be PKV_FP8_E4M3 or PKV_FP8_E5M2 (the plain calls reject
 * both; for e5m2 read e5m2 for e4m3 above, saturating to +-57344); copy_blocks,
 * slot mapping and the planner work on FP8 pools unchanged.
 */
pkv_status pkv_reshape_and_cache_fp8(const void *k, const void *v, void *k_cache, void *v_cache,
                                     const int64_t *slot_mapping, int32_t num_tokens,
                                     float k_scale, float v_scale, const pkv_dims *dims,
                                     void *cuda_stream);

pkv_status pkv_paged_attention_decode_fp8(void *out, const void *q, const void *k_cache,
                                          const void *v_cache, const int32_t *block_tables,
                                          const int32_t *context_lens, float scale,
                                          float k_scale, float v_scale, const pkv_dims *dims,
                                          int32_t max_context_len, int32_t partition_tokens,
                                          void *workspace, size_t workspace_bytes,
                                          void *cuda_stream);

/* Several causal query tokens per sequence (pkv_paged_attention_multi,
 * pkv_multi_run) over FP8 pools: q and out bf16, arithmetic as for
 * pkv_paged_attention_decode_fp8. */
pkv_status pkv_paged_attention_multi_fp8(void *out, const void *q, const void *k_cache,
                                         const void *v_cache, const int32_t *block_tables,
                                         const int32_t *context_lens,
                                         const int32_t *query_start_loc, int32_t num_q_tokens,
                                         int32_t max_query_len, float scale, float k_scale,
                                         float v_scale, const pkv_dims *dims,
                                         int32_t max_context_len, int32_t partition_tokens,
                                         void *workspace, size_t workspace_bytes,
                                         void *cuda_stream);

pkv_status pkv_multi_run_fp8(void *out, const void *q, const void *k_cache, const void *v_cache,
                             const int32_t *block_tables, const int32_t *context_lens,
                             const int32_t *query_start_loc, int32_t num_q_tokens,
                             int32_t max_query_len, float scale, float k_scale, float v_scale,
                             const pkv_dims *dims, int32_t max_context_len,
                             int32_t partition_tokens, void *workspace, size_t workspace_bytes,
                             void *cuda_stream);

pkv_status pkv_decode_run_fp8(void *out, const void *q, const void *k_cache,
                              const void *v_cache, const int32_t *block_tables,
                              const int32_t *context_lens, float scale, float k_scale,
                              float v_scale, const pkv_dims *dims, int32_t max_context_len,
                              int32_t partition_tokens, void *workspace, size_t workspace_bytes,
                              void *cuda_stream);

/*
 * Decode for batches whose consecutive sequences share their leading blocks:
 * parallel samples of one prompt, or requests behind one system prompt (the
 * pages' prefix sharing with reference counts and copy-on-write: "vLLM 深读：
 * 用 PagedAttention 撑起高并发 LLM 推理", section "先看浪费在哪里").  The result
 * is pkv_paged_attention_decode's, but a shared block is read from HBM once
 * per kv head for its whole group instead of once per sequence.
 *
 * Group i covers sequences group_start[i] .. group_start[i+1] - 1
 * (group_start: int32 [num_groups + 1], device, nondecreasing within
 * [0, num_seqs]; num_groups <= num_seqs; a sequence in no group has no shared
 * prefix).  shared_blocks: int32 [num_groups], device.  Definition: every
 * member s of group i reads its first P = shared_blocks[i] blocks through the
 * FIRST member's table row and blocks P .. through its own row, i.e.
 *   out[s][h] = softmax_j(scale * q[s][h] . K_j) V_j   over j < context_lens[s]
 * with K_j, V_j from block_tables[j < 16P ? first : s][j/16], slot j%16.  When
 * the members' tables really hold the same first P entries (what a block
 * manager's fork gives) this is exactly pkv_paged_attention_decode; the
 * tables are not compared.  Groups of fewer than two members read no shared
 * prefix (their count is not looked at).  Otherwise P larger than a member's
 * full blocks (context_len/16, rounded down) is lowered to them and a negative
 * P raised to 0; both, and group bounds that are not nondecreasing in
 * [0, num_seqs] (then no group is used), are flagged PKV_DEVERR_GROUP.
 *
 * How it runs: the plan makes, per group, items over the shared blocks that
 * take one query token of each of up to 16/(Hq/Hkv) members at once (all
 * Hq/Hkv heads of each, at most 16 query rows; one member per item when
 * Hq/Hkv > 8), and ordinary items over each sequence's own blocks; every
 * member's prefix and own partial results are merged by log-sum-exp (so the
 * merge kernel always runs).  Workspace: pkv_decode_shared_workspace_bytes()
 * (different from the plain decode's).  Plan/run split as pkv_decode_plan /
 * pkv_decode_run, with the same rules; the plan also depends on group_start
 * and shared_blocks.  The _fp8 calls take FP8 pools and their scales.
 * pkv_decode_shared_workspace_layout: offsets of the partial results (as
 * pkv_decode_workspace_layout) and of seq_prefix, int32 [num_seqs] = P used
 * for each sequence after the plan (for tests).
 */
/*
 * Partition size (tokens) the shared-prefix plan uses for these arguments
 * (0 = automatic; otherwise the request).  Its automatic choice differs from
 * pkv_decode_partition_tokens for bf16 head_dim-128 caches: those plans run
 * one warp per work item, so the prefix and the sequences' own blocks are cut
 * finer (about 16 items per warp, at least 512 tokens each).  Returns 0 for
 * invalid dims.
 */
int32_t pkv_decode_shared_partition_tokens(const pkv_dims *dims, int32_t max_context_len,
                                           int32_t partition_tokens);

size_t pkv_decode_shared_workspace_bytes(const pkv_dims *dims, int32_t max_context_len,
                                         int32_t partition_tokens);

pkv_status pkv_decode_shared_workspace_layout(const pkv_dims *dims, int32_t max_context_len,
                                              int32_t partition_tokens, int32_t *max_parts,
                                              size_t *part_o_offset, size_t *part_ml_offset,
                                              size_t *seq_prefix_offset);

pkv_status pkv_paged_attention_decode_shared(
    void *out, const void *q, const void *k_cache, const void *v_cache,
    const int32_t *block_tables, const int32_t *context_lens, const int32_t *group_start,
    const int32_t *shared_blocks, int32_t num_groups, float scale, const pkv_dims *dims,
    int32_t max_context_len, int32_t partition_tokens, void *workspace, size_t workspace_bytes,
    void *cuda_stream);

pkv_status pkv_paged_attention_decode_shared_fp8(
    void *out, const void *q, const void *k_cache, const void *v_cache,
    const int32_t *block_tables, const int32_t *context_lens, const int32_t *group_start,
    const int32_t *shared_blocks, int32_t num_groups, float scale, float k_scale, float v_scale,
    const pkv_dims *dims, int32_t max_context_len, int32_t partition_tokens, void *workspace,
    size_t workspace_bytes, void *cuda_stream);

pkv_status pkv_decode_plan_shared(const int32_t *context_lens, const int32_t *group_start,
                                  const int32_t *shared_blocks, int32_t num_groups,
                                  const pkv_dims *dims, int32_t max_context_len,
                                  int32_t partition_tokens, void *workspace,
                                  size_t workspace_bytes, void *cuda_stream);

pkv_status pkv_decode_run_shared(void *out, const void *q, const void *k_cache,
                                 const void *v_cache, const int32_t *block_tables,
                                 const int32_t *context_lens, float scale, const pkv_dims *dims,
                                 int32_t max_context_len, int32_t partition_tokens,
                                 void *workspace, size_t workspace_bytes, void *cuda_stream);

pkv_status pkv_decode_run_shared_fp8(void *out, const void *q, const void *k_cache,
                                     const void *v_cache, const int32_t *block_tables,
                                     const int32_t *context_lens, float scale, float k_scale,
                                     float v_scale, const pkv_dims *dims,
                                     int32_t max_context_len, int32_t partition_tokens,
                                     void *workspace, size_t workspace_bytes,
                                     void *cuda_stream);

/*
 * reshape_and_cache: for every token t with slot_mapping[t] >= 0, copy the
 * bytes of k[t][h][:] and v[t][h][:] to k_cache / v_cache at block
 * slot/16, kv head h, offset slot%16, for every kv head h.  The copy is
 * bit-exact (no conversion).  Negative slots are skipped; a slot >=
 * num_blocks*16 is skipped and flagged PKV_DEVERR_SLOT.  Two tokens with the
 * same non-negative slot in one call leave that slot unspecified.
 * dims->num_seqs and dims->max_blocks_per_seq are not used.
 */
pkv_status pkv_reshape_and_cache(const void *k, const void *v, void *k_cache, void *v_cache,
                                 const int64_t *slot_mapping, int32_t num_tokens,
                                 const pkv_dims *dims, void *cuda_stream);

/*
 * copy_blocks (copy-on-write): for each pair (src, dst) copy every byte of K
 * block src to K block dst and of V block src to V block dst (all kv heads,
 * all 16 slots).  Pairs are applied as if every source were read before any
 * destination is written; that is only guaranteed when no destination repeats
 * and no destination is also a source, which pkv_validate_copy_pairs() checks
 * on a host copy.  A pair outside [0, num_blocks) is skipped and flagged
 * PKV_DEVERR_PAIR.  dims->num_seqs and dims->max_blocks_per_seq are not used.
 */
pkv_status pkv_copy_blocks(void *k_cache, void *v_cache, const int64_t *pairs,
                           int32_t num_pairs, const pkv_dims *dims, void *cuda_stream);

/*
 * Host-side check of copy pairs (pairs_host is a HOST pointer): every index in
 * [0, num_blocks), no repeated destination, no destination that is also a
 * source.  Returns PKV_OK or PKV_ERR_PAIRS.
 */
pkv_status pkv_validate_copy_pairs(const int64_t *pairs_host, int32_t num_pairs,
                                   int32_t num_blocks);

/*
 * Slot indexing: slot_mapping[t] = block_tables[seq][pos/16]*16 + pos%16 with
 * seq = token_seq[t] (or t when token_seq is NULL) and pos = token_pos[t] (or
 * context_lens[seq]-1 when token_pos is NULL: the decode token).  A position
 * outside the table or a table entry outside [0, num_blocks) gives slot -1
 * and sets PKV_DEVERR_POS / PKV_DEVERR_BLOCK.  context_lens may be NULL when
 * token_pos is given.
 */
pkv_status pkv_slot_mapping(int64_t *slot_mapping, const int32_t *block_tables,
                            const int32_t *context_lens, const int32_t *token_seq,
                            const int32_t *token_pos, int32_t num_tokens,
                            const pkv_dims *dims, void *cuda_stream);

/*
 * Synchronises cuda_stream, then reads and clears the error word of the
 * device that owns the stream (the library's current device for a NULL
 * stream).  *bits_out (may be NULL) receives the PKV_DEVERR_* bits.
 * Returns PKV_OK, PKV_ERR_DEVICE_TIMEOUT (timeout bit set),
 * PKV_ERR_DEVICE_INDEX (other bits) or PKV_ERR_CUDA.
 */
pkv_status pkv_check_device_error(void *cuda_stream, uint32_t *bits_out);

/*
 * Diagnostic: launches one warp that waits, with the kernels' own bounded
 * wait, on a barrier nothing completes.  After about a second the wait gives
 * up and sets PKV_DEVERR_TIMEOUT; the kernel then returns and the context
 * stays usable.  Shows that a stalled wait turns into an error status
 * rather than a hang.  Asynchronous on cuda_stream.
 */
pkv_status pkv_selftest_wait_timeout(void *cuda_stream);

/* Static text for a status code. */
const char *pkv_status_string(pkv_status status);

/* Details of the last non-OK status returned on the calling host thread. */
const char *pkv_last_error_message(void);

#ifdef __cplusplus
}
#endif

#endif /* PKV_H */
