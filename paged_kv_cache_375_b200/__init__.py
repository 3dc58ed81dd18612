"""Paged KV-cache decode attention for NVIDIA B200 (sm_100a).

A thin ctypes binding over the C ABI of ``libpkv.so`` (declared in
``include/pkv.h``).  It only marshals arguments -- shapes, pointers, the
current CUDA stream and a cached workspace -- every step runs in the library's
CUDA kernels.  There is no CPU fallback: if the library is missing, importing
the operations raises.

Operations (the pages' statement of the problem: 16-token blocks, a
per-sequence block table, slot_mapping, copy-on-write of shared blocks):

  paged_attention_decode(out, q, k_cache, v_cache, block_tables, context_lens,
                         scale, num_kv_heads, ...)
  reshape_and_cache(k, v, k_cache, v_cache, slot_mapping)
  copy_blocks(k_cache, v_cache, pairs)
  slot_mapping(block_tables, context_lens=None, token_seq=None, token_pos=None)
  DecodePlan(...)            plan once per step (optionally writing the new tokens
                             in the same launch), run once per layer
  paged_attention_multi(...) several causal query tokens per sequence
  paged_attention_decode_shared(...), SharedDecodePlan
                             decode reading a prefix shared by consecutive
                             sequences once per group
  *_fp8 variants             FP8 (e4m3 or e5m2) pools with per-pool scales
  BlockManager               host-side block bookkeeping with prefix caching; its
                             prefix_order / shared_prefix_groups feed the
                             shared-prefix decode
  check_device_error()
"""
from __future__ import annotations

import ctypes
import os
import threading

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libpkv.so")

PKV_F32, PKV_BF16, PKV_FP8_E4M3, PKV_FP8_E5M2 = 0, 1, 2, 3
FP8_DTYPES = (torch.float8_e4m3fn, torch.float8_e5m2)   # pool dtypes of the *_fp8 calls
DEVERR_BLOCK, DEVERR_SLOT, DEVERR_LEN, DEVERR_PAIR, DEVERR_POS, DEVERR_TIMEOUT = (
    0x1, 0x2, 0x4, 0x8, 0x10, 0x20)
DEVERR_GROUP = 0x40

STATUS_NAMES = {0: "PKV_OK", 1: "PKV_ERR_NULL", 2: "PKV_ERR_SHAPE", 3: "PKV_ERR_UNSUPPORTED",
                4: "PKV_ERR_WORKSPACE", 5: "PKV_ERR_PAIRS", 6: "PKV_ERR_CUDA",
                7: "PKV_ERR_DEVICE_INDEX", 8: "PKV_ERR_ALIGN", 9: "PKV_ERR_DEVICE_TIMEOUT",
                10: "PKV_ERR_NO_BLOCKS", 11: "PKV_ERR_NOT_FOUND"}


class PkvError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{STATUS_NAMES.get(status, status)}: {message}")
        self.status = status


class PkvDims(ctypes.Structure):
    _fields_ = [("num_seqs", ctypes.c_int32), ("num_q_heads", ctypes.c_int32),
                ("num_kv_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
                ("block_size", ctypes.c_int32), ("num_blocks", ctypes.c_int32),
                ("max_blocks_per_seq", ctypes.c_int32), ("dtype", ctypes.c_int32)]


_lib = None
_lib_lock = threading.Lock()


def load_library() -> ctypes.CDLL:
    """Load libpkv.so (built in-tree by ``paged_kv_cache_375_b200.build``)."""
    global _lib
    with _lib_lock:
        if _lib is not None:
            return _lib
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m paged_kv_cache_375_b200.build` (no CPU fallback exists)")
        lib = ctypes.CDLL(LIB_PATH)
        P, i32, sz, f32 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_size_t, ctypes.c_float
        D = ctypes.POINTER(PkvDims)
        sig = {
            "pkv_decode_partition_tokens": (i32, [D, i32, i32]),
            "pkv_decode_shared_partition_tokens": (i32, [D, i32, i32]),
            "pkv_decode_workspace_bytes": (sz, [D, i32, i32]),
            "pkv_decode_workspace_layout": (ctypes.c_int, [D, i32, i32, P, P, P]),
            "pkv_paged_attention_decode": (ctypes.c_int, [P, P, P, P, P, P, f32, D, i32, i32, P,
                                                          sz, P]),
            "pkv_decode_plan": (ctypes.c_int, [P, D, i32, i32, P, sz, P]),
            "pkv_decode_prepare": (ctypes.c_int, [P, P, P, P, P, P, P, D, i32, i32, P, sz, P]),
            "pkv_decode_prepare_fp8": (ctypes.c_int, [P, P, P, P, P, P, P, f32, f32, D, i32, i32,
                                                      P, sz, P]),
            "pkv_multi_workspace_bytes": (sz, [D, i32, i32, i32]),
            "pkv_multi_run": (ctypes.c_int, [P, P, P, P, P, P, P, i32, i32, f32, D, i32, i32, P,
                                             sz, P]),
            "pkv_paged_attention_multi": (ctypes.c_int, [P, P, P, P, P, P, P, i32, i32, f32, D,
                                                         i32, i32, P, sz, P]),
            "pkv_decode_run": (ctypes.c_int, [P, P, P, P, P, P, f32, D, i32, i32, P, sz, P]),
            "pkv_paged_prefill": (ctypes.c_int, [P, P, P, P, P, P, P, i32, f32, D, i32, P]),
            "pkv_reshape_and_cache": (ctypes.c_int, [P, P, P, P, P, i32, D, P]),
            "pkv_reshape_and_cache_fp8": (ctypes.c_int, [P, P, P, P, P, i32, f32, f32, D, P]),
            "pkv_paged_attention_decode_fp8": (ctypes.c_int, [P, P, P, P, P, P, f32, f32, f32, D,
                                                              i32, i32, P, sz, P]),
            "pkv_decode_run_fp8": (ctypes.c_int, [P, P, P, P, P, P, f32, f32, f32, D, i32, i32,
                                                  P, sz, P]),
            "pkv_paged_attention_multi_fp8": (ctypes.c_int, [P, P, P, P, P, P, P, i32, i32, f32,
                                                             f32, f32, D, i32, i32, P, sz, P]),
            "pkv_multi_run_fp8": (ctypes.c_int, [P, P, P, P, P, P, P, i32, i32, f32, f32, f32, D,
                                                 i32, i32, P, sz, P]),
            "pkv_decode_prepare_tokens": (ctypes.c_int, [P, P, P, P, P, P, P, P, i32, P, f32, f32,
                                                         P, P, i32, D, i32, i32, P, sz, P]),
            "pkv_decode_shared_workspace_bytes": (sz, [D, i32, i32]),
            "pkv_decode_shared_workspace_layout": (ctypes.c_int, [D, i32, i32, P, P, P, P]),
            "pkv_paged_attention_decode_shared": (ctypes.c_int, [P, P, P, P, P, P, P, P, i32,
                                                                 f32, D, i32, i32, P, sz, P]),
            "pkv_paged_attention_decode_shared_fp8": (ctypes.c_int, [P, P, P, P, P, P, P, P,
                                                                     i32, f32, f32, f32, D, i32,
                                                                     i32, P, sz, P]),
            "pkv_decode_plan_shared": (ctypes.c_int, [P, P, P, i32, D, i32, i32, P, sz, P]),
            "pkv_decode_run_shared": (ctypes.c_int, [P, P, P, P, P, P, f32, D, i32, i32, P, sz,
                                                     P]),
            "pkv_decode_run_shared_fp8": (ctypes.c_int, [P, P, P, P, P, P, f32, f32, f32, D, i32,
                                                         i32, P, sz, P]),
            "pkv_copy_blocks": (ctypes.c_int, [P, P, P, i32, D, P]),
            "pkv_validate_copy_pairs": (ctypes.c_int, [P, i32, i32]),
            "pkv_slot_mapping": (ctypes.c_int, [P, P, P, P, P, i32, D, P]),
            "pkv_check_device_error": (ctypes.c_int, [P, P]),
            "pkv_selftest_wait_timeout": (ctypes.c_int, [P]),
            "pkv_status_string": (ctypes.c_char_p, [ctypes.c_int]),
            "pkv_bm_create": (P, [i32, i32, ctypes.c_uint64, i32]),
            "pkv_bm_destroy": (None, [P]),
            "pkv_bm_add_sequence": (ctypes.c_int, [P, ctypes.c_int64, P, i32, P]),
            "pkv_bm_fork": (ctypes.c_int, [P, ctypes.c_int64, ctypes.c_int64]),
            "pkv_bm_append_tokens": (ctypes.c_int, [P, P, P, i32, P]),
            "pkv_bm_slots": (ctypes.c_int, [P, ctypes.c_int64, i32, i32, P]),
            "pkv_bm_free_sequence": (ctypes.c_int, [P, ctypes.c_int64]),
            "pkv_bm_take_copies": (i32, [P, P, i32]),
            "pkv_bm_block_tables": (ctypes.c_int, [P, P, i32, i32, P, P]),
            "pkv_bm_stats": (ctypes.c_int, [P, P, P, P, P]),
            "pkv_bm_refcount": (i32, [P, i32]),
            "pkv_bm_shared_prefix_groups": (ctypes.c_int, [P, P, i32, i32, P, P, P]),
            "pkv_bm_prefix_order": (ctypes.c_int, [P, P, i32, P]),
            "pkv_last_error_message": (ctypes.c_char_p, []),
        }
        for name, (res, args) in sig.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
        return lib


def _check(status: int):
    if status != 0:
        lib = load_library()
        raise PkvError(status, lib.pkv_last_error_message().decode())


def _dtype_code(t: torch.dtype) -> int:
    if t == torch.bfloat16:
        return PKV_BF16
    if t == torch.float32:
        return PKV_F32
    if t == torch.float8_e4m3fn:
        return PKV_FP8_E4M3
    if t == torch.float8_e5m2:
        return PKV_FP8_E5M2
    raise TypeError(f"dtype {t} not supported (bfloat16, float32, float8_e4m3fn or float8_e5m2 "
                    "caches)")


def _stream_ptr(device: torch.device):
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _p(t: torch.Tensor | None):
    return ctypes.c_void_p(t.data_ptr() if t is not None else 0)


def _need_fp8_pools(k_cache: torch.Tensor, v_cache: torch.Tensor, device):
    _need(k_cache, "k_cache", device=device)
    if k_cache.dtype not in FP8_DTYPES:
        raise TypeError(f"k_cache must be float8_e4m3fn or float8_e5m2, got {k_cache.dtype}")
    _need(v_cache, "v_cache", k_cache.dtype, device)


def _need(t: torch.Tensor, name: str, dtype=None, device=None):
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if device is not None and t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device}")


def make_dims(num_seqs: int, num_q_heads: int, k_cache: torch.Tensor,
              max_blocks_per_seq: int) -> PkvDims:
    nb, hkv, bs, d = k_cache.shape
    return PkvDims(num_seqs, num_q_heads, hkv, d, bs, nb, max_blocks_per_seq,
                   _dtype_code(k_cache.dtype))


def decode_partition_tokens(dims: PkvDims, max_context_len: int, partition_tokens: int = 0) -> int:
    return load_library().pkv_decode_partition_tokens(ctypes.byref(dims), max_context_len,
                                                      partition_tokens)


def decode_shared_partition_tokens(dims: PkvDims, max_context_len: int,
                                   partition_tokens: int = 0) -> int:
    """Partition size of the shared-prefix plan (see pkv_decode_shared_partition_tokens)."""
    return load_library().pkv_decode_shared_partition_tokens(ctypes.byref(dims), max_context_len,
                                                             partition_tokens)


def decode_workspace_bytes(dims: PkvDims, max_context_len: int, partition_tokens: int = 0) -> int:
    return load_library().pkv_decode_workspace_bytes(ctypes.byref(dims), max_context_len,
                                                     partition_tokens)


def decode_workspace_layout(dims: PkvDims, max_context_len: int, partition_tokens: int = 0):
    """(max_parts, part_o_offset, part_ml_offset) of the split-K partials in the workspace."""
    mp = ctypes.c_int32()
    po = ctypes.c_size_t()
    pm = ctypes.c_size_t()
    _check(load_library().pkv_decode_workspace_layout(
        ctypes.byref(dims), max_context_len, partition_tokens, ctypes.byref(mp),
        ctypes.byref(po), ctypes.byref(pm)))
    return mp.value, po.value, pm.value


_ws_cache: dict = {}


def workspace(device: torch.device, nbytes: int) -> torch.Tensor:
    """A cached uint8 workspace of at least nbytes for (device, current stream).

    Decodes issued on one stream run in order, so they can share it; another
    stream gets its own.
    """
    key = (device, torch.cuda.current_stream(device).cuda_stream)
    buf = _ws_cache.get(key)
    if buf is None or buf.numel() < nbytes:
        buf = torch.empty(max(nbytes, 256), dtype=torch.uint8, device=device)
        _ws_cache[key] = buf
    return buf


def paged_attention_decode(out: torch.Tensor, q: torch.Tensor, k_cache: torch.Tensor,
                           v_cache: torch.Tensor, block_tables: torch.Tensor,
                           context_lens: torch.Tensor, scale: float, num_kv_heads: int, *,
                           max_context_len: int | None = None, partition_tokens: int = 0,
                           workspace_tensor: torch.Tensor | None = None) -> torch.Tensor:
    """out[s][h] = softmax(scale * q[s][h] . K^T) V over the paged context of sequence s.

    q, out: [B][Hq][D]; k_cache, v_cache: [NB][Hkv][16][D]; block_tables: int32 [B][MB];
    context_lens: int32 [B].  max_context_len defaults to MB*16 (always safe; a tighter
    value gives a smaller workspace and better partitioning).
    """
    dev = q.device
    _need(q, "q", device=dev)
    _need(out, "out", q.dtype, dev)
    _need(k_cache, "k_cache", q.dtype, dev)
    _need(v_cache, "v_cache", q.dtype, dev)
    _need(block_tables, "block_tables", torch.int32, dev)
    _need(context_lens, "context_lens", torch.int32, dev)
    if k_cache.dim() != 4 or v_cache.shape != k_cache.shape:
        raise ValueError("k_cache and v_cache must both be [num_blocks][num_kv_heads][16][head_dim]")
    if k_cache.shape[1] != num_kv_heads:
        raise ValueError(f"k_cache has {k_cache.shape[1]} kv heads, num_kv_heads={num_kv_heads}")
    B, hq, d = q.shape
    if out.shape != q.shape or block_tables.dim() != 2 or block_tables.shape[0] != B \
            or context_lens.shape != (B,) or k_cache.shape[3] != d:
        raise ValueError("inconsistent shapes")
    dims = make_dims(B, hq, k_cache, block_tables.shape[1])
    mcl = block_tables.shape[1] * k_cache.shape[2] if max_context_len is None else int(max_context_len)
    need = decode_workspace_bytes(dims, mcl, partition_tokens)
    if need == 0:
        raise PkvError(2, load_library().pkv_last_error_message().decode())
    ws = workspace_tensor if workspace_tensor is not None else workspace(dev, need)
    _check(load_library().pkv_paged_attention_decode(
        _p(out), _p(q), _p(k_cache), _p(v_cache), _p(block_tables), _p(context_lens),
        float(scale), ctypes.byref(dims), mcl, partition_tokens, _p(ws), ws.numel(),
        _stream_ptr(dev)))
    return out


def paged_attention_multi(out: torch.Tensor, q: torch.Tensor, k_cache: torch.Tensor,
                          v_cache: torch.Tensor, block_tables: torch.Tensor,
                          context_lens: torch.Tensor, query_start_loc: torch.Tensor,
                          scale: float, num_kv_heads: int, max_query_len: int, *,
                          max_context_len: int | None = None, partition_tokens: int = 0,
                          workspace_tensor: torch.Tensor | None = None) -> torch.Tensor:
    """Causal attention of several query tokens per sequence over the paged context.

    q, out: [T][Hq][D]; query_start_loc: int32 [B+1] (sequence s owns rows
    query_start_loc[s] .. query_start_loc[s+1]-1, at positions L-n .. L-1 of its context,
    L = context_lens[s] including the chunk).  Any chunk length; Hq/Hkv <= 16.
    """
    dev = q.device
    _need(q, "q", device=dev)
    _need(out, "out", q.dtype, dev)
    _need(k_cache, "k_cache", q.dtype, dev)
    _need(v_cache, "v_cache", q.dtype, dev)
    _need(block_tables, "block_tables", torch.int32, dev)
    _need(context_lens, "context_lens", torch.int32, dev)
    _need(query_start_loc, "query_start_loc", torch.int32, dev)
    if k_cache.dim() != 4 or v_cache.shape != k_cache.shape or k_cache.shape[1] != num_kv_heads:
        raise ValueError("k_cache and v_cache must be [num_blocks][num_kv_heads][16][head_dim]")
    T, hq, d = q.shape
    B = context_lens.shape[0]
    if out.shape != q.shape or query_start_loc.shape != (B + 1,) or block_tables.shape[0] != B:
        raise ValueError("inconsistent shapes")
    dims = make_dims(B, hq, k_cache, block_tables.shape[1])
    mcl = block_tables.shape[1] * k_cache.shape[2] if max_context_len is None else int(max_context_len)
    lib = load_library()
    need = lib.pkv_multi_workspace_bytes(ctypes.byref(dims), T, mcl, partition_tokens)
    if need == 0:
        raise PkvError(2, lib.pkv_last_error_message().decode())
    ws = workspace_tensor if workspace_tensor is not None else workspace(dev, need)
    _check(lib.pkv_paged_attention_multi(
        _p(out), _p(q), _p(k_cache), _p(v_cache), _p(block_tables), _p(context_lens),
        _p(query_start_loc), T, int(max_query_len), float(scale), ctypes.byref(dims), mcl,
        partition_tokens, _p(ws), ws.numel(), _stream_ptr(dev)))
    return out


def paged_prefill(out: torch.Tensor, q: torch.Tensor, k_cache: torch.Tensor,
                  v_cache: torch.Tensor, block_tables: torch.Tensor, context_lens: torch.Tensor,
                  query_start_loc: torch.Tensor, scale: float, num_kv_heads: int, *,
                  max_context_len: int | None = None) -> torch.Tensor:
    """The same causal attention as paged_attention_multi, on the tcgen05 tensor cores
    with 128-row query tiles: for long chunks (chunked prefill, whole prompts).

    bf16 only; q, out: [T][Hq][D]; query_start_loc: int32 [B+1].  Needs no workspace.
    """
    dev = q.device
    _need(q, "q", torch.bfloat16, dev)
    _need(out, "out", torch.bfloat16, dev)
    _need(k_cache, "k_cache", torch.bfloat16, dev)
    _need(v_cache, "v_cache", torch.bfloat16, dev)
    _need(block_tables, "block_tables", torch.int32, dev)
    _need(context_lens, "context_lens", torch.int32, dev)
    _need(query_start_loc, "query_start_loc", torch.int32, dev)
    if k_cache.dim() != 4 or v_cache.shape != k_cache.shape or k_cache.shape[1] != num_kv_heads:
        raise ValueError("k_cache and v_cache must be [num_blocks][num_kv_heads][16][head_dim]")
    T, hq, d = q.shape
    B = context_lens.shape[0]
    if out.shape != q.shape or query_start_loc.shape != (B + 1,) or block_tables.shape[0] != B \
            or k_cache.shape[3] != d:
        raise ValueError("inconsistent shapes")
    dims = make_dims(B, hq, k_cache, block_tables.shape[1])
    mcl = block_tables.shape[1] * k_cache.shape[2] if max_context_len is None else int(max_context_len)
    _check(load_library().pkv_paged_prefill(
        _p(out), _p(q), _p(k_cache), _p(v_cache), _p(block_tables), _p(context_lens),
        _p(query_start_loc), T, float(scale), ctypes.byref(dims), mcl, _stream_ptr(dev)))
    return out


def _check_fp8_decode(out, q, k_cache, v_cache, block_tables, context_lens):
    dev = q.device
    _need(q, "q", torch.bfloat16, dev)
    _need(out, "out", torch.bfloat16, dev)
    _need_fp8_pools(k_cache, v_cache, dev)
    _need(block_tables, "block_tables", torch.int32, dev)
    _need(context_lens, "context_lens", torch.int32, dev)
    if k_cache.dim() != 4 or v_cache.shape != k_cache.shape:
        raise ValueError("k_cache and v_cache must both be [num_blocks][num_kv_heads][16][head_dim]")
    B, hq, d = q.shape
    if out.shape != q.shape or block_tables.dim() != 2 or block_tables.shape[0] != B \
            or context_lens.shape != (B,) or k_cache.shape[3] != d:
        raise ValueError("inconsistent shapes")


def paged_attention_decode_fp8(out: torch.Tensor, q: torch.Tensor, k_cache: torch.Tensor,
                               v_cache: torch.Tensor, block_tables: torch.Tensor,
                               context_lens: torch.Tensor, scale: float, k_scale: float,
                               v_scale: float, *, max_context_len: int | None = None,
                               partition_tokens: int = 0,
                               workspace_tensor: torch.Tensor | None = None) -> torch.Tensor:
    """paged_attention_decode over FP8 (float8_e4m3fn or float8_e5m2) caches whose elements stand for
    code * k_scale and code * v_scale; q and out are bfloat16, head_dim 128."""
    _check_fp8_decode(out, q, k_cache, v_cache, block_tables, context_lens)
    dev = q.device
    dims = make_dims(q.shape[0], q.shape[1], k_cache, block_tables.shape[1])
    mcl = block_tables.shape[1] * k_cache.shape[2] if max_context_len is None else int(max_context_len)
    need = decode_workspace_bytes(dims, mcl, partition_tokens)
    if need == 0:
        raise PkvError(2, load_library().pkv_last_error_message().decode())
    ws = workspace_tensor if workspace_tensor is not None else workspace(dev, need)
    _check(load_library().pkv_paged_attention_decode_fp8(
        _p(out), _p(q), _p(k_cache), _p(v_cache), _p(block_tables), _p(context_lens),
        float(scale), float(k_scale), float(v_scale), ctypes.byref(dims), mcl, partition_tokens,
        _p(ws), ws.numel(), _stream_ptr(dev)))
    return out


def paged_attention_multi_fp8(out: torch.Tensor, q: torch.Tensor, k_cache: torch.Tensor,
                              v_cache: torch.Tensor, block_tables: torch.Tensor,
                              context_lens: torch.Tensor, query_start_loc: torch.Tensor,
                              scale: float, k_scale: float, v_scale: float, max_query_len: int,
                              *, max_context_len: int | None = None, partition_tokens: int = 0,
                              workspace_tensor: torch.Tensor | None = None) -> torch.Tensor:
    """paged_attention_multi over FP8 (float8_e4m3fn or float8_e5m2) pools with their scales; q and out
    are bfloat16, head_dim 128."""
    dev = q.device
    _need(q, "q", torch.bfloat16, dev)
    _need(out, "out", torch.bfloat16, dev)
    _need_fp8_pools(k_cache, v_cache, dev)
    _need(block_tables, "block_tables", torch.int32, dev)
    _need(context_lens, "context_lens", torch.int32, dev)
    _need(query_start_loc, "query_start_loc", torch.int32, dev)
    if k_cache.dim() != 4 or v_cache.shape != k_cache.shape:
        raise ValueError("k_cache and v_cache must be [num_blocks][num_kv_heads][16][head_dim]")
    T, hq, d = q.shape
    B = context_lens.shape[0]
    if out.shape != q.shape or query_start_loc.shape != (B + 1,) or block_tables.shape[0] != B \
            or k_cache.shape[3] != d:
        raise ValueError("inconsistent shapes")
    dims = make_dims(B, hq, k_cache, block_tables.shape[1])
    mcl = block_tables.shape[1] * k_cache.shape[2] if max_context_len is None else int(max_context_len)
    lib = load_library()
    need = lib.pkv_multi_workspace_bytes(ctypes.byref(dims), T, mcl, partition_tokens)
    if need == 0:
        raise PkvError(2, lib.pkv_last_error_message().decode())
    ws = workspace_tensor if workspace_tensor is not None else workspace(dev, need)
    _check(lib.pkv_paged_attention_multi_fp8(
        _p(out), _p(q), _p(k_cache), _p(v_cache), _p(block_tables), _p(context_lens),
        _p(query_start_loc), T, int(max_query_len), float(scale), float(k_scale),
        float(v_scale), ctypes.byref(dims), mcl, partition_tokens, _p(ws), ws.numel(),
        _stream_ptr(dev)))
    return out


def _prepare_tokens(lib, dims, k_cache, v_cache, block_tables, context_lens, new_k, new_v,
                    token_seq, token_pos, k_scale, v_scale, slot_mapping_out, group_start,
                    shared_blocks, num_groups, max_context_len, partition_tokens, ws, dev):
    """The token-list prologue (pkv_decode_prepare_tokens): writes and plan in one launch."""
    fp8 = k_cache.dtype in FP8_DTYPES
    src = torch.bfloat16 if fp8 else k_cache.dtype
    _need(new_k, "new_k", src, dev)
    _need(new_v, "new_v", src, dev)
    _need(token_seq, "token_seq", torch.int32, dev)
    _need(token_pos, "token_pos", torch.int32, dev)
    _need(k_cache, "k_cache", device=dev)
    if v_cache is None:
        raise ValueError("v_cache is needed to write the new tokens")
    _need(v_cache, "v_cache", k_cache.dtype, dev)
    T = token_seq.shape[0]
    if new_k.shape != (T, k_cache.shape[1], k_cache.shape[3]) or new_v.shape != new_k.shape \
            or token_pos.shape != (T,) or v_cache.shape != k_cache.shape:
        raise ValueError("new_k, new_v must be [num_tokens][num_kv_heads][head_dim], "
                         "token_seq and token_pos int32 [num_tokens]")
    if slot_mapping_out is not None:
        _need(slot_mapping_out, "slot_mapping_out", torch.int64, dev)
        if slot_mapping_out.shape != (T,):
            raise ValueError("slot_mapping_out must be int64 [num_tokens]")
    if fp8 and (k_scale is None or v_scale is None):
        raise ValueError("FP8 pools need k_scale and v_scale")
    _check(lib.pkv_decode_prepare_tokens(
        _p(new_k), _p(new_v), _p(k_cache), _p(v_cache), _p(block_tables), _p(context_lens),
        _p(token_seq), _p(token_pos), T, _p(slot_mapping_out),
        float(k_scale) if fp8 else 1.0, float(v_scale) if fp8 else 1.0, _p(group_start),
        _p(shared_blocks), num_groups, ctypes.byref(dims), max_context_len, partition_tokens,
        _p(ws), ws.numel(), _stream_ptr(dev)))


class DecodePlan:
    """A decode plan for one step: the work list built from context_lens, kept in a
    workspace.  ``run`` decodes one layer's cache pools with it; plan once per step, run
    once per layer (the context lengths are the same for every layer).

    With ``new_k``/``new_v`` ([B][Hkv][D]; bf16 for FP8 pools) and ``v_cache``, the same
    launch also writes every sequence's new token (position L - 1) into its slot of
    ``k_cache``/``v_cache`` (quantised with ``k_scale``/``v_scale`` for FP8 pools) and,
    if given, each slot into ``slot_mapping_out`` (int64 [B]): slot indexing,
    reshape_and_cache and the plan in one launch.  With ``token_seq``/``token_pos`` (int32
    [T]) the new tokens are any list instead ([T][Hkv][D]; ``slot_mapping_out`` int64 [T]),
    e.g. the chunks of several query tokens per sequence."""

    def __init__(self, block_tables: torch.Tensor, context_lens: torch.Tensor, num_q_heads: int,
                 k_cache: torch.Tensor, *, max_context_len: int | None = None,
                 partition_tokens: int = 0, workspace_tensor: torch.Tensor | None = None,
                 new_k: torch.Tensor | None = None, new_v: torch.Tensor | None = None,
                 v_cache: torch.Tensor | None = None, k_scale: float | None = None,
                 v_scale: float | None = None, slot_mapping_out: torch.Tensor | None = None,
                 token_seq: torch.Tensor | None = None, token_pos: torch.Tensor | None = None):
        dev = context_lens.device
        _need(block_tables, "block_tables", torch.int32, dev)
        _need(context_lens, "context_lens", torch.int32, dev)
        self.block_tables, self.context_lens = block_tables, context_lens
        self.dims = make_dims(context_lens.shape[0], num_q_heads, k_cache, block_tables.shape[1])
        self.max_context_len = (block_tables.shape[1] * k_cache.shape[2] if max_context_len is None
                                else int(max_context_len))
        self.partition_tokens = partition_tokens
        need = decode_workspace_bytes(self.dims, self.max_context_len, partition_tokens)
        if need == 0:
            raise PkvError(2, load_library().pkv_last_error_message().decode())
        if workspace_tensor is None:
            workspace_tensor = torch.empty(need, dtype=torch.uint8, device=dev)
        if workspace_tensor.numel() < need:
            raise ValueError(f"workspace_tensor has {workspace_tensor.numel()} bytes, {need} needed")
        self.workspace = workspace_tensor
        lib = load_library()
        if new_k is None:
            _check(lib.pkv_decode_plan(_p(context_lens), ctypes.byref(self.dims),
                                       self.max_context_len, partition_tokens,
                                       _p(self.workspace), self.workspace.numel(),
                                       _stream_ptr(dev)))
            return
        if token_seq is not None:
            _prepare_tokens(lib, self.dims, k_cache, v_cache, block_tables, context_lens, new_k,
                            new_v, token_seq, token_pos, k_scale, v_scale, slot_mapping_out, None,
                            None, 0, self.max_context_len, partition_tokens, self.workspace, dev)
            return
        fp8 = k_cache.dtype in FP8_DTYPES
        src = torch.bfloat16 if fp8 else k_cache.dtype
        _need(new_k, "new_k", src, dev)
        _need(new_v, "new_v", src, dev)
        _need(k_cache, "k_cache", device=dev)
        if v_cache is None:
            raise ValueError("v_cache is needed to write the new tokens")
        _need(v_cache, "v_cache", k_cache.dtype, dev)
        B = context_lens.shape[0]
        if new_k.shape != (B, k_cache.shape[1], k_cache.shape[3]) or new_v.shape != new_k.shape \
                or v_cache.shape != k_cache.shape:
            raise ValueError("new_k, new_v must be [num_seqs][num_kv_heads][head_dim]")
        if slot_mapping_out is not None:
            _need(slot_mapping_out, "slot_mapping_out", torch.int64, dev)
            if slot_mapping_out.shape != (B,):
                raise ValueError("slot_mapping_out must be int64 [num_seqs]")
        args = [_p(new_k), _p(new_v), _p(k_cache), _p(v_cache), _p(block_tables),
                _p(context_lens), _p(slot_mapping_out)]
        tail = [ctypes.byref(self.dims), self.max_context_len, partition_tokens,
                _p(self.workspace), self.workspace.numel(), _stream_ptr(dev)]
        if fp8:
            if k_scale is None or v_scale is None:
                raise ValueError("FP8 pools need k_scale and v_scale")
            _check(lib.pkv_decode_prepare_fp8(*args, float(k_scale), float(v_scale), *tail))
        else:
            _check(lib.pkv_decode_prepare(*args, *tail))

    def run_multi(self, out: torch.Tensor, q: torch.Tensor, k_cache: torch.Tensor,
                  v_cache: torch.Tensor, query_start_loc: torch.Tensor, max_query_len: int,
                  scale: float) -> torch.Tensor:
        """Several causal query tokens per sequence (see paged_attention_multi) over this
        plan; the plan's workspace must hold pkv_multi_workspace_bytes for q's rows."""
        dev = q.device
        _need(q, "q", device=dev)
        _need(out, "out", q.dtype, dev)
        _need(query_start_loc, "query_start_loc", torch.int32, dev)
        need = load_library().pkv_multi_workspace_bytes(ctypes.byref(self.dims), q.shape[0],
                                                        self.max_context_len,
                                                        self.partition_tokens)
        if need == 0 or self.workspace.numel() < need:
            raise PkvError(4, f"workspace too small for {q.shape[0]} query rows ({need} bytes)")
        _check(load_library().pkv_multi_run(
            _p(out), _p(q), _p(k_cache), _p(v_cache), _p(self.block_tables),
            _p(self.context_lens), _p(query_start_loc), q.shape[0], int(max_query_len),
            float(scale), ctypes.byref(self.dims), self.max_context_len, self.partition_tokens,
            _p(self.workspace), self.workspace.numel(), _stream_ptr(dev)))
        return out

    def run_multi_fp8(self, out: torch.Tensor, q: torch.Tensor, k_cache: torch.Tensor,
                      v_cache: torch.Tensor, query_start_loc: torch.Tensor, max_query_len: int,
                      scale: float, k_scale: float, v_scale: float) -> torch.Tensor:
        """run_multi over FP8 pools (see paged_attention_multi_fp8)."""
        dev = q.device
        _need(q, "q", torch.bfloat16, dev)
        _need(out, "out", torch.bfloat16, dev)
        _need_fp8_pools(k_cache, v_cache, dev)
        _need(query_start_loc, "query_start_loc", torch.int32, dev)
        lib = load_library()
        need = lib.pkv_multi_workspace_bytes(ctypes.byref(self.dims), q.shape[0],
                                             self.max_context_len, self.partition_tokens)
        if need == 0 or self.workspace.numel() < need:
            raise PkvError(4, f"workspace too small for {q.shape[0]} query rows ({need} bytes)")
        _check(lib.pkv_multi_run_fp8(
            _p(out), _p(q), _p(k_cache), _p(v_cache), _p(self.block_tables),
            _p(self.context_lens), _p(query_start_loc), q.shape[0], int(max_query_len),
            float(scale), float(k_scale), float(v_scale), ctypes.byref(self.dims),
            self.max_context_len, self.partition_tokens, _p(self.workspace),
            self.workspace.numel(), _stream_ptr(dev)))
        return out

    def run(self, out: torch.Tensor, q: torch.Tensor, k_cache: torch.Tensor,
            v_cache: torch.Tensor, scale: float) -> torch.Tensor:
        dev = q.device
        _need(q, "q", device=dev)
        _need(out, "out", q.dtype, dev)
        _need(k_cache, "k_cache", q.dtype, dev)
        _need(v_cache, "v_cache", q.dtype, dev)
        if out.shape != q.shape or q.shape[0] != self.dims.num_seqs \
                or tuple(k_cache.shape) != (self.dims.num_blocks, self.dims.num_kv_heads, 16,
                                            self.dims.head_dim) or v_cache.shape != k_cache.shape:
            raise ValueError("inconsistent shapes")
        _check(load_library().pkv_decode_run(
            _p(out), _p(q), _p(k_cache), _p(v_cache), _p(self.block_tables),
            _p(self.context_lens), float(scale), ctypes.byref(self.dims), self.max_context_len,
            self.partition_tokens, _p(self.workspace), self.workspace.numel(), _stream_ptr(dev)))
        return out

    def run_fp8(self, out: torch.Tensor, q: torch.Tensor, k_cache: torch.Tensor,
                v_cache: torch.Tensor, scale: float, k_scale: float,
                v_scale: float) -> torch.Tensor:
        """``run`` over FP8 caches (see paged_attention_decode_fp8)."""
        _check_fp8_decode(out, q, k_cache, v_cache, self.block_tables, self.context_lens)
        if q.shape[0] != self.dims.num_seqs or tuple(k_cache.shape) != (
                self.dims.num_blocks, self.dims.num_kv_heads, 16, self.dims.head_dim):
            raise ValueError("inconsistent shapes")
        # the pools' own FP8 format (the plan itself does not depend on it)
        dims = PkvDims(*[getattr(self.dims, f) for f, _ in PkvDims._fields_[:-1]],
                       _dtype_code(k_cache.dtype))
        _check(load_library().pkv_decode_run_fp8(
            _p(out), _p(q), _p(k_cache), _p(v_cache), _p(self.block_tables),
            _p(self.context_lens), float(scale), float(k_scale), float(v_scale),
            ctypes.byref(dims), self.max_context_len, self.partition_tokens, _p(self.workspace),
            self.workspace.numel(), _stream_ptr(q.device)))
        return out


def decode_shared_workspace_bytes(dims: PkvDims, max_context_len: int,
                                  partition_tokens: int = 0) -> int:
    return load_library().pkv_decode_shared_workspace_bytes(ctypes.byref(dims), max_context_len,
                                                            partition_tokens)


def decode_shared_workspace_layout(dims: PkvDims, max_context_len: int,
                                   partition_tokens: int = 0):
    """(max_parts, part_o_offset, part_ml_offset, seq_prefix_offset) in a shared-prefix
    decode's workspace."""
    mp = ctypes.c_int32()
    po, pm, sp = ctypes.c_size_t(), ctypes.c_size_t(), ctypes.c_size_t()
    _check(load_library().pkv_decode_shared_workspace_layout(
        ctypes.byref(dims), max_context_len, partition_tokens, ctypes.byref(mp),
        ctypes.byref(po), ctypes.byref(pm), ctypes.byref(sp)))
    return mp.value, po.value, pm.value, sp.value


def _check_groups(group_start: torch.Tensor, shared_blocks: torch.Tensor, dev, num_seqs: int):
    _need(group_start, "group_start", torch.int32, dev)
    _need(shared_blocks, "shared_blocks", torch.int32, dev)
    G = shared_blocks.shape[0]
    if group_start.dim() != 1 or shared_blocks.dim() != 1 or group_start.shape[0] != G + 1:
        raise ValueError("group_start must be int32 [num_groups + 1], shared_blocks int32 "
                         "[num_groups]")
    if G > num_seqs:
        raise ValueError("num_groups must be <= num_seqs")
    return G


class SharedDecodePlan:
    """A decode plan for batches whose consecutive sequences share leading blocks.

    Group i is sequences ``group_start[i] .. group_start[i+1]-1`` (int32 [G+1], device);
    every member reads its first ``shared_blocks[i]`` blocks (int32 [G], device) through the
    first member's table row, so the shared blocks are read once per kv head for the whole
    group.  With tables that really share those blocks the result is exactly
    paged_attention_decode's.  Plan once per step, ``run`` (``run_fp8``) once per layer.
    With ``new_k``/``new_v`` ([T][Hkv][D]), ``v_cache`` and ``token_seq``/``token_pos``
    (int32 [T]) the same launch also writes those tokens into their slots (quantised with
    ``k_scale``/``v_scale`` for FP8 pools), as slot indexing + reshape_and_cache would."""

    def __init__(self, block_tables: torch.Tensor, context_lens: torch.Tensor,
                 group_start: torch.Tensor, shared_blocks: torch.Tensor, num_q_heads: int,
                 k_cache: torch.Tensor, *, max_context_len: int | None = None,
                 partition_tokens: int = 0, workspace_tensor: torch.Tensor | None = None,
                 new_k: torch.Tensor | None = None, new_v: torch.Tensor | None = None,
                 v_cache: torch.Tensor | None = None, token_seq: torch.Tensor | None = None,
                 token_pos: torch.Tensor | None = None, k_scale: float | None = None,
                 v_scale: float | None = None, slot_mapping_out: torch.Tensor | None = None):
        dev = context_lens.device
        _need(block_tables, "block_tables", torch.int32, dev)
        _need(context_lens, "context_lens", torch.int32, dev)
        B = context_lens.shape[0]
        G = _check_groups(group_start, shared_blocks, dev, B)
        self.block_tables, self.context_lens = block_tables, context_lens
        self.group_start, self.shared_blocks = group_start, shared_blocks
        self.dims = make_dims(B, num_q_heads, k_cache, block_tables.shape[1])
        self.max_context_len = (block_tables.shape[1] * k_cache.shape[2] if max_context_len is None
                                else int(max_context_len))
        self.partition_tokens = partition_tokens
        need = decode_shared_workspace_bytes(self.dims, self.max_context_len, partition_tokens)
        if need == 0:
            raise PkvError(2, load_library().pkv_last_error_message().decode())
        if workspace_tensor is None:
            workspace_tensor = torch.empty(need, dtype=torch.uint8, device=dev)
        if workspace_tensor.numel() < need:
            raise ValueError(f"workspace_tensor has {workspace_tensor.numel()} bytes, {need} needed")
        self.workspace = workspace_tensor
        if new_k is not None:
            _prepare_tokens(load_library(), self.dims, k_cache, v_cache, block_tables,
                            context_lens, new_k, new_v, token_seq, token_pos, k_scale, v_scale,
                            slot_mapping_out, group_start, shared_blocks, G,
                            self.max_context_len, partition_tokens, self.workspace, dev)
            return
        _check(load_library().pkv_decode_plan_shared(
            _p(context_lens), _p(group_start), _p(shared_blocks), G, ctypes.byref(self.dims),
            self.max_context_len, partition_tokens, _p(self.workspace), self.workspace.numel(),
            _stream_ptr(dev)))

    def _shapes(self, q, k_cache):
        if q.shape[0] != self.dims.num_seqs or tuple(k_cache.shape) != (
                self.dims.num_blocks, self.dims.num_kv_heads, 16, self.dims.head_dim):
            raise ValueError("inconsistent shapes")

    def run(self, out: torch.Tensor, q: torch.Tensor, k_cache: torch.Tensor,
            v_cache: torch.Tensor, scale: float) -> torch.Tensor:
        dev = q.device
        _need(q, "q", device=dev)
        _need(out, "out", q.dtype, dev)
        _need(k_cache, "k_cache", q.dtype, dev)
        _need(v_cache, "v_cache", q.dtype, dev)
        if out.shape != q.shape or v_cache.shape != k_cache.shape:
            raise ValueError("inconsistent shapes")
        self._shapes(q, k_cache)
        _check(load_library().pkv_decode_run_shared(
            _p(out), _p(q), _p(k_cache), _p(v_cache), _p(self.block_tables),
            _p(self.context_lens), float(scale), ctypes.byref(self.dims), self.max_context_len,
            self.partition_tokens, _p(self.workspace), self.workspace.numel(), _stream_ptr(dev)))
        return out

    def run_fp8(self, out: torch.Tensor, q: torch.Tensor, k_cache: torch.Tensor,
                v_cache: torch.Tensor, scale: float, k_scale: float,
                v_scale: float) -> torch.Tensor:
        """``run`` over FP8 caches (see paged_attention_decode_fp8)."""
        _check_fp8_decode(out, q, k_cache, v_cache, self.block_tables, self.context_lens)
        self._shapes(q, k_cache)
        dims = PkvDims(*[getattr(self.dims, f) for f, _ in PkvDims._fields_[:-1]],
                       _dtype_code(k_cache.dtype))
        _check(load_library().pkv_decode_run_shared_fp8(
            _p(out), _p(q), _p(k_cache), _p(v_cache), _p(self.block_tables),
            _p(self.context_lens), float(scale), float(k_scale), float(v_scale),
            ctypes.byref(dims), self.max_context_len, self.partition_tokens, _p(self.workspace),
            self.workspace.numel(), _stream_ptr(q.device)))
        return out


def paged_attention_decode_shared(out: torch.Tensor, q: torch.Tensor, k_cache: torch.Tensor,
                                  v_cache: torch.Tensor, block_tables: torch.Tensor,
                                  context_lens: torch.Tensor, group_start: torch.Tensor,
                                  shared_blocks: torch.Tensor, scale: float, *,
                                  k_scale: float | None = None, v_scale: float | None = None,
                                  max_context_len: int | None = None, partition_tokens: int = 0,
                                  workspace_tensor: torch.Tensor | None = None) -> torch.Tensor:
    """Decode with shared prefixes read once per group (see SharedDecodePlan), in one call:
    the plan, the decode and the merge.  FP8 pools take k_scale and v_scale."""
    dev = q.device
    fp8 = k_cache.dtype in FP8_DTYPES
    if fp8:
        _check_fp8_decode(out, q, k_cache, v_cache, block_tables, context_lens)
        if k_scale is None or v_scale is None:
            raise ValueError("FP8 pools need k_scale and v_scale")
    else:
        _need(q, "q", device=dev)
        _need(out, "out", q.dtype, dev)
        _need(k_cache, "k_cache", q.dtype, dev)
        _need(v_cache, "v_cache", q.dtype, dev)
        _need(block_tables, "block_tables", torch.int32, dev)
        _need(context_lens, "context_lens", torch.int32, dev)
    B, hq, d = q.shape
    if out.shape != q.shape or block_tables.dim() != 2 or block_tables.shape[0] != B \
            or context_lens.shape != (B,) or k_cache.dim() != 4 or v_cache.shape != k_cache.shape \
            or k_cache.shape[3] != d:
        raise ValueError("inconsistent shapes")
    G = _check_groups(group_start, shared_blocks, dev, B)
    dims = make_dims(B, hq, k_cache, block_tables.shape[1])
    mcl = block_tables.shape[1] * k_cache.shape[2] if max_context_len is None else int(max_context_len)
    need = decode_shared_workspace_bytes(dims, mcl, partition_tokens)
    if need == 0:
        raise PkvError(2, load_library().pkv_last_error_message().decode())
    ws = workspace_tensor if workspace_tensor is not None else workspace(dev, need)
    lib = load_library()
    head = [_p(out), _p(q), _p(k_cache), _p(v_cache), _p(block_tables), _p(context_lens),
            _p(group_start), _p(shared_blocks), G, float(scale)]
    tail = [ctypes.byref(dims), mcl, partition_tokens, _p(ws), ws.numel(), _stream_ptr(dev)]
    if fp8:
        _check(lib.pkv_paged_attention_decode_shared_fp8(*head, float(k_scale), float(v_scale),
                                                         *tail))
    else:
        _check(lib.pkv_paged_attention_decode_shared(*head, *tail))
    return out


def reshape_and_cache(k: torch.Tensor, v: torch.Tensor, k_cache: torch.Tensor,
                      v_cache: torch.Tensor, slot_mapping: torch.Tensor) -> None:
    """Write k, v ([T][Hkv][D]) into the caches at slot_mapping (int64 [T]); -1 skips."""
    dev = k.device
    _need(k, "k", k_cache.dtype, dev)
    _need(v, "v", k_cache.dtype, dev)
    _need(k_cache, "k_cache", device=dev)
    _need(v_cache, "v_cache", k_cache.dtype, dev)
    _need(slot_mapping, "slot_mapping", torch.int64, dev)
    T = slot_mapping.shape[0]
    if k.shape != v.shape or k.shape[0] != T or k.shape[1:] != (k_cache.shape[1], k_cache.shape[3]):
        raise ValueError("k, v must be [num_tokens][num_kv_heads][head_dim]")
    dims = make_dims(0, k_cache.shape[1], k_cache, 1)
    _check(load_library().pkv_reshape_and_cache(_p(k), _p(v), _p(k_cache), _p(v_cache),
                                                _p(slot_mapping), T, ctypes.byref(dims),
                                                _stream_ptr(dev)))


def reshape_and_cache_fp8(k: torch.Tensor, v: torch.Tensor, k_cache: torch.Tensor,
                          v_cache: torch.Tensor, slot_mapping: torch.Tensor, k_scale: float,
                          v_scale: float) -> None:
    """Quantise bf16 k, v ([T][Hkv][128]) to e4m3 codes (value / scale, nearest even,
    saturated) and write them into the FP8 caches (float8_e4m3fn or float8_e5m2) at
    slot_mapping; -1 skips."""
    dev = k.device
    _need(k, "k", torch.bfloat16, dev)
    _need(v, "v", torch.bfloat16, dev)
    _need_fp8_pools(k_cache, v_cache, dev)
    _need(slot_mapping, "slot_mapping", torch.int64, dev)
    T = slot_mapping.shape[0]
    if k.shape != v.shape or k.shape[0] != T or k.shape[1:] != (k_cache.shape[1], k_cache.shape[3]) \
            or v_cache.shape != k_cache.shape:
        raise ValueError("k, v must be [num_tokens][num_kv_heads][head_dim]")
    dims = make_dims(0, k_cache.shape[1], k_cache, 1)
    _check(load_library().pkv_reshape_and_cache_fp8(_p(k), _p(v), _p(k_cache), _p(v_cache),
                                                    _p(slot_mapping), T, float(k_scale),
                                                    float(v_scale), ctypes.byref(dims),
                                                    _stream_ptr(dev)))


def validate_copy_pairs(pairs_host: torch.Tensor, num_blocks: int) -> None:
    pr = pairs_host.detach().to("cpu", torch.int64).contiguous().reshape(-1, 2)
    _check(load_library().pkv_validate_copy_pairs(ctypes.c_void_p(pr.data_ptr()), pr.shape[0],
                                                  num_blocks))


def copy_blocks(k_cache: torch.Tensor, v_cache: torch.Tensor, pairs: torch.Tensor,
                validate: bool = True) -> None:
    """Copy-on-write: copy K and V block src to dst for each (src, dst) row of pairs.

    pairs may live on the CPU (it is validated there, then copied to the device) or on the
    device (validated only when ``validate`` and after a device-to-host copy).
    """
    dev = k_cache.device
    _need(k_cache, "k_cache", device=dev)
    _need(v_cache, "v_cache", k_cache.dtype, dev)
    pr = pairs.reshape(-1, 2)
    if pr.shape[0] == 0:
        return
    if validate:
        validate_copy_pairs(pr, k_cache.shape[0])
    pr_dev = pr.to(dev, torch.int64).contiguous()
    dims = make_dims(0, k_cache.shape[1], k_cache, 1)
    _check(load_library().pkv_copy_blocks(_p(k_cache), _p(v_cache), _p(pr_dev), pr_dev.shape[0],
                                          ctypes.byref(dims), _stream_ptr(dev)))


def slot_mapping(block_tables: torch.Tensor, num_blocks: int, *,
                 context_lens: torch.Tensor | None = None, token_seq: torch.Tensor | None = None,
                 token_pos: torch.Tensor | None = None, num_tokens: int | None = None,
                 out: torch.Tensor | None = None) -> torch.Tensor:
    """Slots of tokens: block_tables[seq][pos // 16] * 16 + pos % 16, computed on the GPU.

    Without token_pos the position is context_lens[seq] - 1 (the decode token); without
    token_seq token t belongs to sequence t.
    """
    dev = block_tables.device
    _need(block_tables, "block_tables", torch.int32, dev)
    for name, t in (("context_lens", context_lens), ("token_seq", token_seq),
                    ("token_pos", token_pos)):
        if t is not None:
            _need(t, name, torch.int32, dev)
    B = block_tables.shape[0]
    if num_tokens is None:
        num_tokens = token_pos.shape[0] if token_pos is not None else (
            token_seq.shape[0] if token_seq is not None else B)
    if out is None:
        out = torch.empty(num_tokens, dtype=torch.int64, device=dev)
    dims = PkvDims(B, 1, 1, 64, 16, num_blocks, block_tables.shape[1], PKV_BF16)
    _check(load_library().pkv_slot_mapping(_p(out), _p(block_tables), _p(context_lens),
                                           _p(token_seq), _p(token_pos), num_tokens,
                                           ctypes.byref(dims), _stream_ptr(dev)))
    return out


def check_device_error(device: torch.device | None = None) -> int:
    """Synchronise the current stream, read and clear the device error bits.

    Raises PkvError when a kernel met an invalid index or a wait timed out.
    """
    dev = device or torch.device("cuda", torch.cuda.current_device())
    bits = ctypes.c_uint32()
    status = load_library().pkv_check_device_error(_stream_ptr(dev), ctypes.byref(bits))
    if status not in (0, 7, 9):
        _check(status)
    if status != 0:
        raise PkvError(status, f"device error bits 0x{bits.value:x}")
    return bits.value


def device_error_bits(device: torch.device | None = None) -> int:
    """Like check_device_error, but returns the bits instead of raising."""
    dev = device or torch.device("cuda", torch.cuda.current_device())
    bits = ctypes.c_uint32()
    status = load_library().pkv_check_device_error(_stream_ptr(dev), ctypes.byref(bits))
    if status not in (0, 7, 9):
        _check(status)
    return bits.value


def selftest_wait_timeout(device: torch.device | None = None) -> None:
    """Launch the bounded-wait self-test (about one second); read the result with
    device_error_bits()."""
    dev = device or torch.device("cuda", torch.cuda.current_device())
    _check(load_library().pkv_selftest_wait_timeout(_stream_ptr(dev)))


class BlockManager:
    """Host-side KV-block bookkeeping (the library's native block manager).

    Hands out blocks of ``block_size`` tokens from a scattered pool, keeps block tables,
    shares blocks between forked sequences with reference counts and emits copy-on-write
    pairs, and (with ``prefix_caching``) reuses cached full prompt blocks found through a
    chain of block hashes, evicting unreferenced cached blocks least recently used first.
    Take the queued copies (``take_copies``) after each append call, before sequences
    are freed, and apply them with ``copy_blocks`` before the step's writes.
    """

    def __init__(self, num_blocks: int, block_size: int = 16, seed: int = 0,
                 prefix_caching: bool = False):
        import numpy as np
        self._np = np
        self._lib = load_library()
        self._h = self._lib.pkv_bm_create(num_blocks, block_size, seed, int(prefix_caching))
        if not self._h:
            raise PkvError(2, "invalid block manager sizes")
        self.num_blocks, self.block_size = num_blocks, block_size

    def close(self):
        if self._h:
            self._lib.pkv_bm_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def _arr(self, a, dtype):
        a = self._np.ascontiguousarray(a, dtype=dtype)
        return a, a.ctypes.data_as(ctypes.c_void_p)

    def add_sequence(self, seq_id: int, tokens) -> int:
        """Start a sequence with its prompt; returns the number of prompt tokens found cached."""
        t, tp = self._arr(tokens, self._np.int32)
        cached = ctypes.c_int32(0)
        _bm_check(self._lib.pkv_bm_add_sequence(self._h, seq_id, tp, t.shape[0],
                                                ctypes.byref(cached)))
        return cached.value

    def fork(self, parent: int, child: int) -> None:
        _bm_check(self._lib.pkv_bm_fork(self._h, parent, child))

    def append_tokens(self, seq_ids, tokens, out=None):
        """Append one token to each sequence; returns the int64 slots of the new tokens
        (written into ``out`` when given)."""
        s, sp = self._arr(seq_ids, self._np.int64)
        t, tp = self._arr(tokens, self._np.int32)
        assert s.shape == t.shape
        if out is None:
            out = self._np.empty(s.shape[0], dtype=self._np.int64)
        assert out.dtype == self._np.int64 and out.flags["C_CONTIGUOUS"] and out.shape == s.shape
        _bm_check(self._lib.pkv_bm_append_tokens(self._h, sp, tp, s.shape[0],
                                                 out.ctypes.data_as(ctypes.c_void_p)))
        return out

    def slots(self, seq_id: int, pos_begin: int, pos_end: int):
        out = self._np.empty(max(0, pos_end - pos_begin), dtype=self._np.int64)
        _bm_check(self._lib.pkv_bm_slots(self._h, seq_id, pos_begin, pos_end,
                                         out.ctypes.data_as(ctypes.c_void_p)))
        return out

    def free_sequence(self, seq_id: int) -> None:
        _bm_check(self._lib.pkv_bm_free_sequence(self._h, seq_id))

    def take_copies(self):
        """The queued (src, dst) copy-on-write pairs, as int64 [P][2]."""
        n = -self._lib.pkv_bm_take_copies(self._h, None, 0)
        out = self._np.empty((max(n, 0), 2), dtype=self._np.int64)
        got = self._lib.pkv_bm_take_copies(self._h, out.ctypes.data_as(ctypes.c_void_p), n)
        return out[:max(got, 0)]

    def block_tables(self, seq_ids, max_blocks: int, tables=None, lens=None):
        """(tables int32 [n][max_blocks] padded with -1, context lengths int32 [n]); written
        into ``tables`` / ``lens`` when given (e.g. pinned buffers reused every step)."""
        s, sp = self._arr(seq_ids, self._np.int64)
        if tables is None:
            tables = self._np.empty((s.shape[0], max_blocks), dtype=self._np.int32)
        if lens is None:
            lens = self._np.empty(s.shape[0], dtype=self._np.int32)
        assert tables.dtype == self._np.int32 and tables.shape == (s.shape[0], max_blocks)
        assert lens.dtype == self._np.int32 and lens.shape == (s.shape[0],)
        assert tables.flags["C_CONTIGUOUS"] and lens.flags["C_CONTIGUOUS"]
        _bm_check(self._lib.pkv_bm_block_tables(self._h, sp, s.shape[0], max_blocks,
                                                tables.ctypes.data_as(ctypes.c_void_p),
                                                lens.ctypes.data_as(ctypes.c_void_p)))
        return tables, lens

    def prefix_order(self, seq_ids):
        """Positions of seq_ids in an order where sequences beginning with the same physical
        blocks are consecutive (int32 [n]); lay out q, out and the tables in it."""
        s, sp = self._arr(seq_ids, self._np.int64)
        out = self._np.empty(s.shape[0], dtype=self._np.int32)
        _bm_check(self._lib.pkv_bm_prefix_order(self._h, sp, s.shape[0],
                                                out.ctypes.data_as(ctypes.c_void_p)))
        return out

    def shared_prefix_groups(self, seq_ids, min_shared_blocks: int = 1):
        """(group_start int32 [G+1], shared_blocks int32 [G]) for paged_attention_decode_shared
        over these sequences in this order: runs of consecutive sequences whose tables begin
        with the same physical blocks (at least min_shared_blocks full ones)."""
        s, sp = self._arr(seq_ids, self._np.int64)
        n = s.shape[0]
        gs = self._np.empty(n + 1, dtype=self._np.int32)
        sb = self._np.empty(max(n, 1), dtype=self._np.int32)
        g = ctypes.c_int32()
        _bm_check(self._lib.pkv_bm_shared_prefix_groups(
            self._h, sp, n, int(min_shared_blocks), gs.ctypes.data_as(ctypes.c_void_p),
            sb.ctypes.data_as(ctypes.c_void_p), ctypes.byref(g)))
        return gs[:g.value + 1].copy(), sb[:g.value].copy()

    def stats(self) -> dict:
        v = [ctypes.c_int32() for _ in range(4)]
        _bm_check(self._lib.pkv_bm_stats(self._h, *[ctypes.byref(x) for x in v]))
        return dict(zip(("free", "evictable", "used", "sequences"), (x.value for x in v)))

    def refcount(self, block: int) -> int:
        return self._lib.pkv_bm_refcount(self._h, block)


def _bm_check(status: int):
    if status != 0:
        name = STATUS_NAMES.get(status, status)
        raise PkvError(status, load_library().pkv_status_string(status).decode() + f" ({name})")
