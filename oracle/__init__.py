"""The float64 CPU oracle for paged KV-cache decode attention.

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the CPU
baseline leg of ``bench.py`` are the only callers.  The product path (the CUDA
library and its binding) never imports this package.

The arithmetic lives in ``pkv_oracle.c`` (plain C, double precision); this
module compiles it on demand with gcc and marshals numpy arrays through
ctypes.  See the header of ``pkv_oracle.c`` for the passages each function
follows and for the readings taken where the pages are silent.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "pkv_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
# Tests that plant mistakes in a copy of the oracle point this at the copy.
_LIB_OVERRIDE = os.environ.get("PKV_ORACLE_LIB_OVERRIDE")
_lock = threading.Lock()
_lib = None

F32 = 0
BF16 = 1
E4M3 = 2

_STATUS = {
    0: "ok",
    1: "bad argument",
    2: "block-table entry out of range",
    3: "context length out of range",
    4: "slot out of range",
    5: "copy pair out of range",
    6: "out of memory",
}


class OracleError(RuntimeError):
    def __init__(self, status: int):
        super().__init__(f"oracle status {status}: {_STATUS.get(status, 'unknown')}")
        self.status = status


def build(force: bool = False) -> str:
    """Compile pkv_oracle.c into liboracle.so (gcc, -O2, C11, pthreads)."""
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    tmp = _LIB_PATH + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-pthread",
           "-Wall", "-Wextra", "-o", tmp, _SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is None:
            if _LIB_OVERRIDE:
                lib = ctypes.CDLL(_LIB_OVERRIDE)
            else:
                build()
                lib = ctypes.CDLL(_LIB_PATH)
            P = ctypes.c_void_p
            i32, i64, f32 = ctypes.c_int32, ctypes.c_int64, ctypes.c_float
            lib.oracle_slot_mapping.argtypes = [P, i32, i32, P, P, i32, P]
            lib.oracle_reshape_and_cache.argtypes = [P, P, P, P, P, i32, i32, i32, i32, i32, i64]
            lib.oracle_copy_blocks.argtypes = [P, P, P, i32, i64, i64]
            lib.oracle_paged_decode.argtypes = [P, P, P, P, i32, P, P, i32, i32, i32, i32,
                                                i32, i64, i32, f32, P, i64, i32]
            lib.oracle_partition_stats.argtypes = [P, P, P, i32, P, P, i32, i32, i32, i32,
                                                   i32, i64, i32, f32, i32, i32, i32, i32,
                                                   P, P, P]
            lib.oracle_lse_merge.argtypes = [P, P, P, i32, i32, P]
            lib.oracle_paged_multi.argtypes = [P, P, P, P, i32, P, P, P, i32, i32, i32, i32,
                                               i32, i64, i32, f32, i32]
            lib.oracle_paged_decode_fp8.argtypes = [P, P, P, P, f32, f32, P, P, i32, i32, i32,
                                                    i32, i32, i64, i32, f32, P, i64, i32]
            lib.oracle_reshape_and_cache_fp8.argtypes = [P, P, P, P, P, i32, i32, i32, i32, i64,
                                                         f32, f32]
            lib.oracle_paged_multi_fp8.argtypes = [P, P, P, P, f32, f32, P, P, P, i32, i32, i32,
                                                   i32, i32, i64, i32, f32, i32]
            lib.oracle_e4m3_quantize.argtypes = [P, i64, f32, P]
            lib.oracle_e5m2_quantize.argtypes = [P, i64, f32, P]
            lib.oracle_e5m2_values.argtypes = [P, i64, P]
            lib.oracle_reshape_and_cache_e5m2.argtypes = [P, P, P, P, P, i32, i32, i32, i32, i64,
                                                          f32, f32]
            lib.oracle_paged_decode_e5m2.argtypes = [P, P, P, P, f32, f32, P, P, i32, i32, i32,
                                                     i32, i32, i64, i32, f32, P, i64, i32]
            lib.oracle_paged_multi_e5m2.argtypes = [P, P, P, P, f32, f32, P, P, P, i32, i32, i32,
                                                    i32, i32, i64, i32, f32, i32]
            lib.oracle_e4m3_values.argtypes = [P, i64, P]
            lib.oracle_lse_merge_f32.argtypes = [P, P, P, i32, i32, P]
            for name in ("oracle_slot_mapping", "oracle_reshape_and_cache",
                         "oracle_copy_blocks", "oracle_paged_decode", "oracle_paged_multi",
                         "oracle_paged_decode_fp8", "oracle_reshape_and_cache_fp8",
                         "oracle_paged_multi_fp8", "oracle_e5m2_quantize",
                         "oracle_e5m2_values", "oracle_reshape_and_cache_e5m2",
                         "oracle_paged_decode_e5m2", "oracle_paged_multi_e5m2",
                         "oracle_e4m3_quantize", "oracle_e4m3_values",
                         "oracle_partition_stats", "oracle_lse_merge",
                         "oracle_lse_merge_f32"):
                getattr(lib, name).restype = ctypes.c_int
            _lib = lib
    return _lib


def _ptr(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"], "oracle arrays must be C-contiguous"
    return a.ctypes.data_as(ctypes.c_void_p)


def _check(status: int):
    if status != 0:
        raise OracleError(status)


def _dtype_code(arr: np.ndarray) -> int:
    """fp32 arrays are float32; bf16 arrays are carried as their uint16 bits."""
    if arr.dtype == np.float32:
        return F32
    if arr.dtype == np.uint16:
        return BF16
    raise TypeError(f"oracle takes float32 or bf16-as-uint16 arrays, got {arr.dtype}")


def slot_mapping(block_tables: np.ndarray, token_seq: np.ndarray, token_pos: np.ndarray,
                 block_size: int = 16) -> np.ndarray:
    bt = np.ascontiguousarray(block_tables, dtype=np.int32)
    ts = np.ascontiguousarray(token_seq, dtype=np.int32)
    tp = np.ascontiguousarray(token_pos, dtype=np.int32)
    out = np.empty(ts.shape[0], dtype=np.int64)
    _check(_load().oracle_slot_mapping(_ptr(bt), bt.shape[1], block_size, _ptr(ts),
                                       _ptr(tp), ts.shape[0], _ptr(out)))
    return out


def reshape_and_cache(k: np.ndarray, v: np.ndarray, k_cache: np.ndarray, v_cache: np.ndarray,
                      slot_mapping_: np.ndarray) -> None:
    """In place on k_cache / v_cache ([NB][Hkv][BS][D]); k, v are [T][Hkv][D]."""
    sm = np.ascontiguousarray(slot_mapping_, dtype=np.int64)
    nb, hkv, bs, d = k_cache.shape
    assert k.shape == v.shape and k.shape[1:] == (hkv, d) and k.dtype == k_cache.dtype
    _check(_load().oracle_reshape_and_cache(_ptr(k), _ptr(v), _ptr(k_cache), _ptr(v_cache),
                                            _ptr(sm), sm.shape[0], hkv, d, k.itemsize, bs, nb))


def copy_blocks(k_cache: np.ndarray, v_cache: np.ndarray, pairs: np.ndarray) -> None:
    """In place; pairs is [P][2] (src, dst)."""
    pr = np.ascontiguousarray(pairs, dtype=np.int64).reshape(-1, 2)
    nb = k_cache.shape[0]
    block_bytes = k_cache.nbytes // nb
    _check(_load().oracle_copy_blocks(_ptr(k_cache), _ptr(v_cache), _ptr(pr), pr.shape[0],
                                      block_bytes, nb))


def paged_decode(q: np.ndarray, k_cache: np.ndarray, v_cache: np.ndarray,
                 block_tables: np.ndarray, context_lens: np.ndarray, scale: float,
                 tasks: np.ndarray | None = None, threads: int | None = None) -> np.ndarray:
    """Float64 attention output.

    q: [B][Hq][D]; caches: [NB][Hkv][BS][D] (float32, or uint16 holding bf16 bits).
    Returns [B][Hq][D] doubles, or [n][D] for tasks = [n][2] (seq, q_head) pairs.
    """
    code = _dtype_code(k_cache)
    assert q.dtype == k_cache.dtype == v_cache.dtype
    B, Hq, D = q.shape
    NB, Hkv, BS, D2 = k_cache.shape
    assert D2 == D and v_cache.shape == k_cache.shape
    bt = np.ascontiguousarray(block_tables, dtype=np.int32)
    cl = np.ascontiguousarray(context_lens, dtype=np.int32)
    threads = threads or len(os.sched_getaffinity(0))
    if tasks is None:
        out = np.empty((B, Hq, D), dtype=np.float64)
        tp, n = None, B * Hq
    else:
        tk = np.ascontiguousarray(tasks, dtype=np.int32).reshape(-1, 2)
        out = np.empty((tk.shape[0], D), dtype=np.float64)
        tp, n = _ptr(tk), tk.shape[0]
    _check(_load().oracle_paged_decode(_ptr(out), _ptr(q), _ptr(k_cache), _ptr(v_cache), code,
                                       _ptr(bt), _ptr(cl), B, Hq, Hkv, D, BS, NB, bt.shape[1],
                                       float(scale), tp, n, threads))
    return out


def paged_multi(q: np.ndarray, k_cache: np.ndarray, v_cache: np.ndarray,
                block_tables: np.ndarray, context_lens: np.ndarray,
                query_start_loc: np.ndarray, scale: float, threads: int | None = None) -> np.ndarray:
    """Float64 output of several causal query tokens per sequence.

    q: [T][Hq][D] (sequence s owns rows query_start_loc[s] .. query_start_loc[s+1]-1);
    returns [T][Hq][D] doubles.
    """
    code = _dtype_code(k_cache)
    assert q.dtype == k_cache.dtype == v_cache.dtype
    T, Hq, D = q.shape
    NB, Hkv, BS, _ = k_cache.shape
    bt = np.ascontiguousarray(block_tables, dtype=np.int32)
    cl = np.ascontiguousarray(context_lens, dtype=np.int32)
    qsl = np.ascontiguousarray(query_start_loc, dtype=np.int32)
    assert qsl.shape[0] == cl.shape[0] + 1 and qsl[-1] <= T
    out = np.zeros((T, Hq, D), dtype=np.float64)
    threads = threads or len(os.sched_getaffinity(0))
    _check(_load().oracle_paged_multi(_ptr(out), _ptr(q), _ptr(k_cache), _ptr(v_cache), code,
                                      _ptr(bt), _ptr(cl), _ptr(qsl), cl.shape[0], Hq, Hkv, D, BS,
                                      NB, bt.shape[1], float(scale), threads))
    return out


def e4m3_quantize(x: np.ndarray, scale: float = 1.0) -> np.ndarray:
    """uint8 e4m3 codes of float32 x / scale (the division in float32)."""
    xf = np.ascontiguousarray(x, dtype=np.float32)
    out = np.empty(xf.shape, dtype=np.uint8)
    _check(_load().oracle_e4m3_quantize(_ptr(xf), xf.size, float(scale), _ptr(out)))
    return out


def e5m2_quantize(x: np.ndarray, scale: float = 1.0) -> np.ndarray:
    """uint8 e5m2 codes of float32 x / scale (the division in float32)."""
    xf = np.ascontiguousarray(x, dtype=np.float32)
    out = np.empty(xf.shape, dtype=np.uint8)
    _check(_load().oracle_e5m2_quantize(_ptr(xf), xf.size, float(scale), _ptr(out)))
    return out


def e5m2_values(codes: np.ndarray) -> np.ndarray:
    """Exact values of e5m2 codes (no scale), as float64."""
    c = np.ascontiguousarray(codes, dtype=np.uint8)
    out = np.empty(c.shape, dtype=np.float64)
    _check(_load().oracle_e5m2_values(_ptr(c), c.size, _ptr(out)))
    return out


def e4m3_values(codes: np.ndarray) -> np.ndarray:
    """Exact values of e4m3 codes (no scale), as float64."""
    c = np.ascontiguousarray(codes, dtype=np.uint8)
    out = np.empty(c.shape, dtype=np.float64)
    _check(_load().oracle_e4m3_values(_ptr(c), c.size, _ptr(out)))
    return out


_FP8 = ("e4m3", "e5m2")


def reshape_and_cache_fp8(k: np.ndarray, v: np.ndarray, k_cache: np.ndarray,
                          v_cache: np.ndarray, slot_mapping_: np.ndarray, k_scale: float,
                          v_scale: float, fmt: str = "e4m3") -> None:
    """In place on uint8 FP8 pools [NB][Hkv][BS][D] (fmt "e4m3" or "e5m2"); k, v are bf16
    bits [T][Hkv][D]."""
    assert fmt in _FP8
    sm = np.ascontiguousarray(slot_mapping_, dtype=np.int64)
    nb, hkv, bs, d = k_cache.shape
    assert k.dtype == np.uint16 and k_cache.dtype == np.uint8 and k.shape[1:] == (hkv, d)
    fn = (_load().oracle_reshape_and_cache_fp8 if fmt == "e4m3" else
          _load().oracle_reshape_and_cache_e5m2)
    _check(fn(_ptr(k), _ptr(v), _ptr(k_cache), _ptr(v_cache), _ptr(sm), sm.shape[0], hkv, d, bs,
              nb, float(k_scale), float(v_scale)))


def paged_decode_fp8(q: np.ndarray, k_cache: np.ndarray, v_cache: np.ndarray, k_scale: float,
                     v_scale: float, block_tables: np.ndarray, context_lens: np.ndarray,
                     scale: float, tasks: np.ndarray | None = None,
                     threads: int | None = None, fmt: str = "e4m3") -> np.ndarray:
    """Float64 decode over FP8 pools (uint8 codes times the pool's scale; fmt "e4m3" or
    "e5m2"); q is bf16 bits."""
    assert fmt in _FP8
    assert q.dtype == np.uint16 and k_cache.dtype == np.uint8 == v_cache.dtype
    B, Hq, D = q.shape
    NB, Hkv, BS, _ = k_cache.shape
    bt = np.ascontiguousarray(block_tables, dtype=np.int32)
    cl = np.ascontiguousarray(context_lens, dtype=np.int32)
    threads = threads or len(os.sched_getaffinity(0))
    if tasks is None:
        out = np.empty((B, Hq, D), dtype=np.float64)
        tp, n = None, B * Hq
    else:
        tk = np.ascontiguousarray(tasks, dtype=np.int32).reshape(-1, 2)
        out = np.empty((tk.shape[0], D), dtype=np.float64)
        tp, n = _ptr(tk), tk.shape[0]
    fn = _load().oracle_paged_decode_fp8 if fmt == "e4m3" else _load().oracle_paged_decode_e5m2
    _check(fn(_ptr(out), _ptr(q), _ptr(k_cache), _ptr(v_cache), float(k_scale), float(v_scale),
              _ptr(bt), _ptr(cl), B, Hq, Hkv, D, BS, NB, bt.shape[1], float(scale), tp, n,
              threads))
    return out


def paged_multi_fp8(q: np.ndarray, k_cache: np.ndarray, v_cache: np.ndarray, k_scale: float,
                    v_scale: float, block_tables: np.ndarray, context_lens: np.ndarray,
                    query_start_loc: np.ndarray, scale: float,
                    threads: int | None = None, fmt: str = "e4m3") -> np.ndarray:
    """paged_multi over FP8 pools (uint8 codes times the pool's scale; fmt "e4m3" or
    "e5m2"); q is bf16 bits."""
    assert fmt in _FP8
    assert q.dtype == np.uint16 and k_cache.dtype == np.uint8 == v_cache.dtype
    T, Hq, D = q.shape
    NB, Hkv, BS, _ = k_cache.shape
    bt = np.ascontiguousarray(block_tables, dtype=np.int32)
    cl = np.ascontiguousarray(context_lens, dtype=np.int32)
    qsl = np.ascontiguousarray(query_start_loc, dtype=np.int32)
    assert qsl.shape[0] == cl.shape[0] + 1 and qsl[-1] <= T
    out = np.zeros((T, Hq, D), dtype=np.float64)
    threads = threads or len(os.sched_getaffinity(0))
    fn = _load().oracle_paged_multi_fp8 if fmt == "e4m3" else _load().oracle_paged_multi_e5m2
    _check(fn(_ptr(out), _ptr(q), _ptr(k_cache), _ptr(v_cache), float(k_scale), float(v_scale),
              _ptr(bt), _ptr(cl), _ptr(qsl), cl.shape[0], Hq, Hkv, D, BS, NB, bt.shape[1],
              float(scale), threads))
    return out


def partition_stats(q, k_cache, v_cache, block_tables, context_lens, scale, seq, q_head,
                    t0, t1):
    """(m, l, o) of one query over tokens [t0, t1): max score, sum of exp, normalised out."""
    code = _dtype_code(k_cache)
    B, Hq, D = q.shape
    NB, Hkv, BS, _ = k_cache.shape
    bt = np.ascontiguousarray(block_tables, dtype=np.int32)
    cl = np.ascontiguousarray(context_lens, dtype=np.int32)
    m = np.zeros(1, dtype=np.float64)
    l = np.zeros(1, dtype=np.float64)
    o = np.zeros(D, dtype=np.float64)
    _check(_load().oracle_partition_stats(_ptr(q), _ptr(k_cache), _ptr(v_cache), code, _ptr(bt),
                                          _ptr(cl), B, Hq, Hkv, D, BS, NB, bt.shape[1],
                                          float(scale), seq, q_head, t0, t1, _ptr(m), _ptr(l),
                                          _ptr(o)))
    return float(m[0]), float(l[0]), o


def lse_merge(m: np.ndarray, l: np.ndarray, o: np.ndarray) -> np.ndarray:
    """Merge partial results: m, l are [P], o is [P][D]; float64 or float32 inputs."""
    lib = _load()
    o = np.ascontiguousarray(o)
    P, D = o.shape
    out = np.empty(D, dtype=np.float64)
    if o.dtype == np.float32:
        m32 = np.ascontiguousarray(m, dtype=np.float32)
        l32 = np.ascontiguousarray(l, dtype=np.float32)
        _check(lib.oracle_lse_merge_f32(_ptr(m32), _ptr(l32), _ptr(o), P, D, _ptr(out)))
    else:
        m64 = np.ascontiguousarray(m, dtype=np.float64)
        l64 = np.ascontiguousarray(l, dtype=np.float64)
        o64 = np.ascontiguousarray(o, dtype=np.float64)
        _check(lib.oracle_lse_merge(_ptr(m64), _ptr(l64), _ptr(o64), P, D, _ptr(out)))
    return out
