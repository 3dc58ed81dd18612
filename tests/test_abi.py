"""The C-ABI library loads, exports every entry point its headers declare, and
its host-side logic (argument checks, workspace sizing, partition choice,
copy-pair validation) behaves as documented.  No GPU is needed: nothing here
launches a kernel."""
import ctypes
import os
import re
import subprocess

import pytest

import paged_kv_cache_375_b200 as pkv
from paged_kv_cache_375_b200 import build as pkv_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "pkv.h")
HEADERS = sorted(os.path.join(ROOT, "include", f) for f in os.listdir(os.path.join(ROOT, "include"))
                 if f.endswith(".h"))


@pytest.fixture(scope="module")
def lib():
    pkv_build.build()
    return pkv.load_library()


def declared_functions(headers=None):
    names = set()
    for h in headers or HEADERS:
        text = re.sub(r"/\*.*?\*/", "", open(h).read(), flags=re.S)
        names.update(re.findall(r"\b(pkv_[a-z0-9_]+)\s*\(", text))
    return sorted(names)


def test_header_declares_the_boundary():
    assert len(HEADERS) >= 2 and HEADER in HEADERS
    names = declared_functions([HEADER])
    for required in ("pkv_paged_attention_decode", "pkv_reshape_and_cache", "pkv_copy_blocks",
                     "pkv_slot_mapping", "pkv_check_device_error", "pkv_decode_workspace_bytes"):
        assert required in names


def test_every_declared_symbol_is_exported(lib):
    out = subprocess.run(["nm", "-D", "--defined-only", pkv.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\sT\s(\w+)$", out, flags=re.M))
    for name in declared_functions():
        assert name in exported, name
        assert getattr(lib, name) is not None


def test_library_is_built_for_sm100a_only(lib):
    # the build flags pin the architecture; the ELF carries the sm_100a cubin
    assert "arch=compute_100a,code=sm_100a" in " ".join(pkv_build.NVCC_FLAGS)


def test_status_strings(lib):
    for code in range(10):
        assert lib.pkv_status_string(code).decode() != "unknown status"
    assert lib.pkv_status_string(99).decode() == "unknown status"


def dims(B=4, hq=8, hkv=2, d=128, bs=16, nb=100, mb=8, dtype=pkv.PKV_BF16):
    return pkv.PkvDims(B, hq, hkv, d, bs, nb, mb, dtype)


def test_workspace_single_pass_has_no_partials():
    d = dims(B=256, hq=32, hkv=8, nb=40000, mb=512)
    assert pkv.decode_partition_tokens(d, 8192) >= 8192
    n = pkv.decode_workspace_bytes(d, 8192)
    assert 0 < n < 64 * 1024
    with pytest.raises(pkv.PkvError):
        pkv.decode_workspace_layout(d, 8192)


def test_workspace_split_k_sizes():
    # long contexts, few sequences: about 16 items per SM -> 4096-token partitions
    d = dims(B=8, hq=64, hkv=8, nb=81920, mb=8192)
    P = pkv.decode_partition_tokens(d, 131072)
    assert P == 4096
    max_parts, po, pm = pkv.decode_workspace_layout(d, 131072)
    assert max_parts == 32
    assert po % 256 == 0 and pm % 256 == 0 and pm >= po + 8 * 64 * 32 * 128 * 4
    assert pkv.decode_workspace_bytes(d, 131072) >= pm + 8 * 64 * 32 * 2 * 4
    max_parts, _, _ = pkv.decode_workspace_layout(d, 131072, 512)
    assert max_parts == 256


def test_partition_rule_is_a_power_of_two_in_range():
    for B, mcl in ((1, 131072), (4, 20000), (64, 2048), (256, 8192), (2, 100)):
        d = dims(B=B, hq=32, hkv=8, nb=81920, mb=8192)
        P = pkv.decode_partition_tokens(d, mcl)
        if P < mcl:
            assert P in (512, 1024, 2048, 4096, 8192)
        else:
            assert P % 16 == 0 and P < mcl + 16


def test_explicit_partition_is_honoured():
    d = dims()
    assert pkv.decode_partition_tokens(d, 100, 32) == 32
    mp, _, _ = pkv.decode_workspace_layout(d, 100, 32)
    assert mp == 4


@pytest.mark.parametrize("bad", [
    dict(bs=8), dict(d=96), dict(hq=6, hkv=4), dict(hq=34, hkv=2), dict(nb=0),
    dict(dtype=7), dict(mb=0), dict(B=-1)])
def test_bad_dims_are_rejected(bad):
    assert pkv.decode_workspace_bytes(dims(**bad), 64) == 0


def test_bad_partition_is_rejected():
    assert pkv.decode_workspace_bytes(dims(), 64, 24) == 0


def test_decode_rejects_null_and_small_workspace(lib):
    d = dims()
    null = ctypes.c_void_p(0)
    st = lib.pkv_paged_attention_decode(null, null, null, null, null, null, 1.0,
                                        ctypes.byref(d), 64, 0, null, 0, null)
    assert pkv.STATUS_NAMES[st] == "PKV_ERR_NULL"
    fake = ctypes.c_void_p(1 << 20)   # never dereferenced: rejected before any launch
    st = lib.pkv_paged_attention_decode(fake, fake, fake, fake, fake, fake, 1.0,
                                        ctypes.byref(d), 64, 0, fake, 16, null)
    assert pkv.STATUS_NAMES[st] == "PKV_ERR_WORKSPACE"
    assert b"needed" in lib.pkv_last_error_message()
    odd = ctypes.c_void_p((1 << 20) + 8)
    st = lib.pkv_paged_attention_decode(odd, fake, fake, fake, fake, fake, 1.0,
                                        ctypes.byref(d), 64, 0, fake, 1 << 20, null)
    assert pkv.STATUS_NAMES[st] == "PKV_ERR_ALIGN"


def test_static_decode_binds_the_output_device_before_the_scratch_lookup(lib):
    """The built-in scratch's address is per device, so the no-allocation decode must make
    the device that owns `out` current before looking it up.  With host buffers and a
    nonzero batch the call therefore fails while binding `out` (at the pointer query on a
    machine without a GPU, with 'not device memory' on one), never at the lookup."""
    import numpy as np
    fn = lib.pkv_paged_attention_decode_static
    P, i32 = ctypes.c_void_p, ctypes.c_int32
    fn.argtypes = [P, P, P, P, P, P, ctypes.c_float, ctypes.POINTER(pkv.PkvDims), i32, i32, P]
    fn.restype = ctypes.c_int
    d = dims()
    bufs = [np.zeros(1 << 14, dtype=np.uint8) for _ in range(6)]
    ptrs = [P(b.ctypes.data) for b in bufs]
    st = fn(*ptrs, 1.0, ctypes.byref(d), 64, 0, P(0))
    msg = lib.pkv_last_error_message()
    assert st != 0
    assert b"cudaGetSymbolAddress" not in msg and b"cudaGetDevice" not in msg, msg
    assert b"cudaPointerGetAttributes" in msg or b"out is not device memory" in msg, msg


def test_empty_batch_is_a_no_op(lib):
    d = dims(B=0)
    null = ctypes.c_void_p(0)
    assert lib.pkv_paged_attention_decode(null, null, null, null, null, null, 1.0,
                                          ctypes.byref(d), 0, 0, null, 0, null) == 0
    assert lib.pkv_reshape_and_cache(null, null, null, null, null, 0, ctypes.byref(d), null) == 0
    assert lib.pkv_copy_blocks(null, null, null, 0, ctypes.byref(d), null) == 0


def _validate(pairs, nb):
    import torch
    t = torch.tensor(pairs, dtype=torch.int64).reshape(-1, 2)
    return pkv.validate_copy_pairs(t, nb)


def test_copy_pair_validation():
    _validate([[0, 1], [2, 3]], 4)
    _validate([], 4)
    for bad in ([[0, 4]], [[-1, 2]], [[0, 1], [2, 1]], [[0, 1], [1, 2]], [[0, 1], [2, 0]]):
        with pytest.raises(pkv.PkvError) as e:
            _validate(bad, 4)
        assert e.value.status == 5


def test_product_path_does_not_touch_the_oracle():
    """The binding and the CUDA sources never import, include or link the oracle."""
    pkg = os.path.join(ROOT, "paged_kv_cache_375_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                text = open(os.path.join(dirpath, f)).read()
                assert "oracle" not in text.lower(), f


def test_shared_prefix_workspace_sizes():
    """The shared-prefix plan keeps partials even when the plain decode is single pass, one
    partial more per row, room for two items per (sequence, partition) and the per-sequence
    and per-group block counts."""
    d = dims(B=256, hq=32, hkv=8, nb=40000, mb=512)
    assert pkv.decode_workspace_bytes(d, 1600) < pkv.decode_shared_workspace_bytes(d, 1600)
    # bf16 head_dim 128: the automatic partition aims at ~16 items per warp (one warp per
    # item), at least 512 tokens: 512 here, so 4 partitions of the context + 1
    assert pkv.decode_shared_partition_tokens(d, 1600) == 512
    assert pkv.decode_partition_tokens(d, 1600) >= 1600       # the plain plan: single pass
    max_parts, po, pm, sp = pkv.decode_shared_workspace_layout(d, 1600)
    assert max_parts == 5
    assert pkv.decode_shared_workspace_layout(d, 1600, 2048)[0] == 2
    assert sp % 256 == 0 and po % 256 == 0 and pm % 256 == 0
    assert sp >= 256 + 2 * 256 * 5 * 32            # counters, then 2*B*max_parts items
    assert po >= sp + 2 * 256 * 4                  # seq_prefix, group block counts
    assert pm >= po + 256 * 32 * 5 * 128 * 4
    assert pkv.decode_shared_workspace_bytes(d, 1600) >= pm + 256 * 32 * 5 * 2 * 4
    # split-K: one partial more than the plain decode's
    d = dims(B=8, hq=64, hkv=8, nb=81920, mb=8192)
    assert pkv.decode_shared_workspace_layout(d, 131072, 512)[0] == \
        pkv.decode_workspace_layout(d, 131072, 512)[0] + 1
    assert pkv.decode_shared_workspace_bytes(dims(bs=8), 64) == 0


def test_shared_prefix_calls_reject_bad_arguments(lib):
    d = dims()
    null = ctypes.c_void_p(0)
    fake = ctypes.c_void_p(1 << 20)   # never dereferenced: rejected before any launch
    big = 1 << 24

    def one_shot(num_groups, dd=d, fp8=False, ws=big):
        args = [fake] * 8 + [num_groups, 1.0]
        if fp8:
            return lib.pkv_paged_attention_decode_shared_fp8(*args, 1.0, 1.0, ctypes.byref(dd),
                                                             64, 0, fake, ws, null)
        return lib.pkv_paged_attention_decode_shared(*args, ctypes.byref(dd), 64, 0, fake, ws,
                                                     null)

    assert pkv.STATUS_NAMES[one_shot(d.num_seqs + 1)] == "PKV_ERR_SHAPE"
    assert pkv.STATUS_NAMES[one_shot(-1)] == "PKV_ERR_SHAPE"
    assert pkv.STATUS_NAMES[one_shot(2, ws=64)] == "PKV_ERR_WORKSPACE"
    assert pkv.STATUS_NAMES[one_shot(2, fp8=True)] == "PKV_ERR_UNSUPPORTED"   # bf16 pools
    fp8 = dims(dtype=pkv.PKV_FP8_E4M3)
    assert pkv.STATUS_NAMES[one_shot(2, dd=fp8)] == "PKV_ERR_UNSUPPORTED"     # scales needed
    st = lib.pkv_paged_attention_decode_shared(null, *[fake] * 7, 2, 1.0, ctypes.byref(d), 64,
                                               0, fake, big, null)
    assert pkv.STATUS_NAMES[st] == "PKV_ERR_NULL"
    st = lib.pkv_decode_plan_shared(fake, null, fake, 2, ctypes.byref(d), 64, 0, fake, big, null)
    assert pkv.STATUS_NAMES[st] == "PKV_ERR_NULL"
    empty = dims(B=0)
    assert lib.pkv_paged_attention_decode_shared(*[null] * 8, 0, 1.0, ctypes.byref(empty), 0, 0,
                                                 null, 0, null) == 0


def test_token_prologue_rejects_bad_arguments(lib):
    d = dims()
    null = ctypes.c_void_p(0)
    fake = ctypes.c_void_p(1 << 20)
    odd = ctypes.c_void_p((1 << 20) + 8)
    big = 1 << 24

    def call(k=fake, T=4, ks=1.0, vs=1.0, gs=null, G=0, dd=d, ws=big):
        return pkv.STATUS_NAMES[lib.pkv_decode_prepare_tokens(
            k, fake, fake, fake, fake, fake, fake, fake, T, null, ks, vs, gs, fake, G,
            ctypes.byref(dd), 64, 0, fake, ws, null)]

    assert call(T=-1) == "PKV_ERR_SHAPE"
    assert call(k=null) == "PKV_ERR_NULL"
    assert call(k=odd) == "PKV_ERR_ALIGN"
    assert call(ws=64) == "PKV_ERR_WORKSPACE"
    assert call(gs=fake, G=d.num_seqs + 1) == "PKV_ERR_SHAPE"
    fp8 = dims(dtype=pkv.PKV_FP8_E5M2)
    assert call(dd=fp8, ks=0.0) == "PKV_ERR_SHAPE"
    assert call(dd=fp8, vs=float("inf")) == "PKV_ERR_SHAPE"
    # the shared plan needs the larger workspace
    need_plain = pkv.decode_workspace_bytes(d, 64)
    assert call(gs=fake, G=2, ws=need_plain) == "PKV_ERR_WORKSPACE"
    assert call(dd=dims(B=0)) == "PKV_OK"
