"""The decode entry point that allocates nothing (pkv_paged_attention_decode_static).

Some callers of this library cannot allocate device memory themselves: an
engine that gives nearly all HBM to its KV-cache pool and lets nothing else
allocate, or a host runtime that only reaches the library through its C ABI.
For them the library keeps a fixed scratch array on each GPU.  This test calls
that entry point through the C ABI twice in a row -- a split-K batch (the
scratch holds partial results) and then a different single-pass batch -- and
checks each output against the ordinary entry point's and against the float64
oracle, within the tolerance of the other parity tests.  It also checks that the
call refuses operands that are not on the output's device.  It lives in its own
file, collected last, so that a run stopping at the first failure has already
run every other test.
"""
import ctypes
import os
import subprocess
import sys

import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_375_b200 as pkv
import workloads

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
pytestmark = pytest.mark.gpu


def _static_fn():
    lib = pkv.load_library()
    fn = lib.pkv_paged_attention_decode_static
    P, i32 = ctypes.c_void_p, ctypes.c_int32
    fn.argtypes = [P, P, P, P, P, P, ctypes.c_float, ctypes.POINTER(pkv.PkvDims), i32, i32, P]
    fn.restype = ctypes.c_int
    return lib, fn


def _decode_both(b, partition_tokens):
    dev = b.q.device
    bt = torch.from_numpy(b.block_tables).to(dev)
    cl = torch.from_numpy(b.context_lens).to(dev)
    dims = pkv.make_dims(b.num_seqs, b.num_q_heads, b.k_cache, b.max_blocks_per_seq)
    mcl = b.max_context_len
    ref = torch.empty_like(b.q)
    pkv.paged_attention_decode(ref, b.q, b.k_cache, b.v_cache, bt, cl, b.scale, b.num_kv_heads,
                               max_context_len=mcl, partition_tokens=partition_tokens)
    lib, fn = _static_fn()
    out = torch.full_like(b.q, float("nan"))
    stream = ctypes.c_void_p(torch.cuda.current_stream(dev).cuda_stream)
    st = fn(ctypes.c_void_p(out.data_ptr()), ctypes.c_void_p(b.q.data_ptr()),
            ctypes.c_void_p(b.k_cache.data_ptr()), ctypes.c_void_p(b.v_cache.data_ptr()),
            ctypes.c_void_p(bt.data_ptr()), ctypes.c_void_p(cl.data_ptr()), b.scale,
            ctypes.byref(dims), mcl, partition_tokens, stream)
    assert st == 0, lib.pkv_last_error_message().decode()
    assert pkv.device_error_bits(dev) == 0
    return ref, out


def _assert_close(ref, out, dtype):
    a = np.asarray(ref, dtype=np.float64) if isinstance(ref, np.ndarray) else \
        ref.double().cpu().numpy()
    b = out.double().cpu().numpy()
    assert np.isfinite(b).all()
    if dtype == "f32":
        assert np.abs(a - b).max() <= 1e-5
    else:
        assert (np.abs(a - b) <= 2e-2 + 1e-2 * np.abs(a)).all()


def _oracle(b):
    h = b.host()
    return oracle.paged_decode(h["q"], h["k_cache"], h["v_cache"], b.block_tables,
                               b.context_lens, b.scale)


def test_static_scratch_decode_matches_workspace_decode_twice(cuda_device):
    # first call: sequences split into 256-token partitions, partials live in the scratch
    b1 = workloads.random_batch(901, [5, 300, 777, 1500, 2049], 32, 8, 128, "bf16",
                                device=cuda_device)
    ref1, out1 = _decode_both(b1, 256)
    _assert_close(ref1, out1, "bf16")
    _assert_close(_oracle(b1), out1, "bf16")
    # second call, right after: another shape and single pass, same scratch
    b2 = workloads.random_batch(902, [1, 17, 64, 200], 8, 8, 64, "f32", device=cuda_device)
    ref2, out2 = _decode_both(b2, 0)
    _assert_close(ref2, out2, "f32")
    _assert_close(_oracle(b2), out2, "f32")


def test_static_scratch_refuses_operands_off_the_output_device(cuda_device):
    """The call runs on the device that owns `out`; an operand elsewhere (here q in host
    memory) is refused before anything is looked up or launched."""
    b = workloads.random_batch(903, [20, 40], 8, 2, 64, "bf16", device=cuda_device)
    lib, fn = _static_fn()
    bt = torch.from_numpy(b.block_tables).to(cuda_device)
    cl = torch.from_numpy(b.context_lens).to(cuda_device)
    q_host = b.q.cpu()
    out = torch.empty_like(b.q)
    dims = pkv.make_dims(b.num_seqs, b.num_q_heads, b.k_cache, b.max_blocks_per_seq)
    st = fn(ctypes.c_void_p(out.data_ptr()), ctypes.c_void_p(q_host.data_ptr()),
            ctypes.c_void_p(b.k_cache.data_ptr()), ctypes.c_void_p(b.v_cache.data_ptr()),
            ctypes.c_void_p(bt.data_ptr()), ctypes.c_void_p(cl.data_ptr()), b.scale,
            ctypes.byref(dims), b.max_context_len, 0,
            ctypes.c_void_p(torch.cuda.current_stream(cuda_device).cuda_stream))
    assert pkv.STATUS_NAMES[st] == "PKV_ERR_SHAPE"
    assert b"q is not device memory" in lib.pkv_last_error_message()


_FIRST_CALL_IN_CAPTURE = r"""
import ctypes, sys, torch
sys.path.insert(0, sys.argv[1])
import paged_kv_cache_375_b200 as pkv, workloads
dev = torch.device("cuda:0")
b = workloads.random_batch(904, [20, 40], 8, 2, 64, "bf16", device=dev)
bt = torch.from_numpy(b.block_tables).to(dev)
cl = torch.from_numpy(b.context_lens).to(dev)
out = torch.empty_like(b.q)
lib = pkv.load_library()
fn = lib.pkv_paged_attention_decode_static
P, i32 = ctypes.c_void_p, ctypes.c_int32
fn.argtypes = [P, P, P, P, P, P, ctypes.c_float, ctypes.POINTER(pkv.PkvDims), i32, i32, P]
dims = pkv.make_dims(b.num_seqs, b.num_q_heads, b.k_cache, b.max_blocks_per_seq)
args = [P(out.data_ptr()), P(b.q.data_ptr()), P(b.k_cache.data_ptr()), P(b.v_cache.data_ptr()),
        P(bt.data_ptr()), P(cl.data_ptr()), b.scale, ctypes.byref(dims), b.max_context_len, 0]
torch.cuda.synchronize()
s = torch.cuda.Stream(device=dev)
g = torch.cuda.CUDAGraph()
with torch.cuda.graph(g, stream=s):
    st = fn(*args, P(s.cuda_stream))
msg = lib.pkv_last_error_message().decode()
del g
print("status", pkv.STATUS_NAMES[st], msg)
"""


def test_static_scratch_first_call_refuses_a_capturing_stream(cuda_device):
    """In a fresh process the first call on a device must look up the scratch's address;
    made on a stream under capture, it returns an error that names the rule instead of
    failing inside the capture."""
    r = subprocess.run([sys.executable, "-c", _FIRST_CALL_IN_CAPTURE, ROOT], capture_output=True,
                       text=True, timeout=300, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    line = [ln for ln in r.stdout.splitlines() if ln.startswith("status")][-1]
    assert "PKV_ERR_UNSUPPORTED" in line and "stream is being captured" in line, line


def test_static_scratch_rejects_decodes_that_do_not_fit(cuda_device):
    lib, fn = _static_fn()
    # 8 sequences x 64 heads x 256 partitions of partials need ~68 MB > the built-in 32 MiB
    dims = pkv.PkvDims(8, 64, 8, 128, 16, 81920, 8192, pkv.PKV_BF16)
    null = ctypes.c_void_p(0)
    st = fn(null, null, null, null, null, null, 1.0, ctypes.byref(dims), 131072, 512, null)
    assert pkv.STATUS_NAMES[st] == "PKV_ERR_WORKSPACE"
    assert b"built-in scratch" in lib.pkv_last_error_message()
