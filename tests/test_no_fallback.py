"""The product path has no CPU fallback: every operation of the binding refuses host
tensors with an error instead of computing anything on the CPU, and the binding refuses
to load without the CUDA library.  Runs without a GPU."""
import os
import subprocess
import sys

import pytest
import torch

import paged_kv_cache_375_b200 as pkv

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _host_batch(B=2, hq=8, hkv=2, d=64, nb=8, mb=2):
    q = torch.zeros((B, hq, d), dtype=torch.bfloat16)
    kc = torch.zeros((nb, hkv, 16, d), dtype=torch.bfloat16)
    bt = torch.zeros((B, mb), dtype=torch.int32)
    cl = torch.ones(B, dtype=torch.int32)
    return q, kc, bt, cl


def test_decode_calls_refuse_host_tensors():
    q, kc, bt, cl = _host_batch()
    out = torch.empty_like(q)
    with pytest.raises(ValueError, match="CUDA tensor"):
        pkv.paged_attention_decode(out, q, kc, kc.clone(), bt, cl, 0.125, 2)
    gs = torch.tensor([0, 2], dtype=torch.int32)
    sb = torch.tensor([1], dtype=torch.int32)
    with pytest.raises(ValueError, match="CUDA tensor"):
        pkv.paged_attention_decode_shared(out, q, kc, kc.clone(), bt, cl, gs, sb, 0.125)
    with pytest.raises(ValueError, match="CUDA tensor"):
        pkv.DecodePlan(bt, cl, 8, kc)
    with pytest.raises(ValueError, match="CUDA tensor"):
        pkv.SharedDecodePlan(bt, cl, gs, sb, 8, kc)
    qsl = torch.tensor([0, 1, 2], dtype=torch.int32)
    with pytest.raises(ValueError, match="CUDA tensor"):
        pkv.paged_attention_multi(out, q, kc, kc.clone(), bt, cl, qsl, 0.125, 2, 1)


def test_cache_ops_refuse_host_tensors():
    q, kc, bt, cl = _host_batch()
    k = torch.zeros((2, 2, 64), dtype=torch.bfloat16)
    slots = torch.zeros(2, dtype=torch.int64)
    with pytest.raises(ValueError, match="CUDA tensor"):
        pkv.reshape_and_cache(k, k.clone(), kc, kc.clone(), slots)
    with pytest.raises(ValueError, match="CUDA tensor"):
        pkv.slot_mapping(bt, 8, context_lens=cl)
    with pytest.raises(ValueError, match="CUDA tensor"):
        pkv.copy_blocks(kc, kc.clone(), torch.tensor([[0, 1]], dtype=torch.int64))
    k8 = torch.zeros((2, 2, 128), dtype=torch.bfloat16)
    kc8 = torch.zeros((8, 2, 16, 128), dtype=torch.uint8).view(torch.float8_e4m3fn)
    with pytest.raises(ValueError, match="CUDA tensor"):
        pkv.reshape_and_cache_fp8(k8, k8.clone(), kc8, kc8.clone(), slots, 1.0, 1.0)


def test_binding_refuses_to_load_without_the_library(tmp_path):
    """A copy of the package without libpkv.so raises when an operation needs the library."""
    import shutil
    dst = tmp_path / "paged_kv_cache_375_b200"
    shutil.copytree(os.path.join(ROOT, "paged_kv_cache_375_b200"), dst,
                    ignore=shutil.ignore_patterns("*.so", "__pycache__", "*.tmp*"))
    code = ("import paged_kv_cache_375_b200 as p\n"
            "try:\n    p.load_library()\nexcept RuntimeError as e:\n"
            "    print('refused:', 'no CPU fallback' in str(e))\n")
    r = subprocess.run([sys.executable, "-c", code], cwd=tmp_path, capture_output=True,
                       text=True, timeout=300)
    assert "refused: True" in r.stdout, r.stdout + r.stderr
