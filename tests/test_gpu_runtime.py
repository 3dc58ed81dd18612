"""Runtime behaviour on the GPU: a plan reused for several runs (several layers'
pools), back-to-back decodes on one stream, and the bounded-wait failure path
(a wait that nothing completes turns into an error status, and the context
stays usable), and decode steps captured in CUDA graphs and replayed, checked
against eager launches and against the oracle."""
import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_375_b200 as pkv
import workloads
from gpu_util import check_close, dev_i32, host_bits, oracle_caches_after_step

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("partition", [0, 256])
def test_one_plan_serves_several_runs(cuda_device, partition):
    lens = [3, 100, 640, 1999, 16, 700]
    b = workloads.random_batch(71, lens, 32, 8, 128, "bf16", device=cuda_device)
    # a second "layer": other pools and queries with the same tables and lengths
    gen = torch.Generator(device=cuda_device).manual_seed(72)
    k2 = torch.randn(b.k_cache.shape, generator=gen, device=cuda_device).to(torch.bfloat16)
    v2 = torch.randn(b.v_cache.shape, generator=gen, device=cuda_device).to(torch.bfloat16)
    q2 = torch.randn(b.q.shape, generator=gen, device=cuda_device).to(torch.bfloat16)
    bt = dev_i32(b.block_tables, cuda_device)
    cl = dev_i32(b.context_lens, cuda_device)
    mcl = b.max_context_len
    plan = pkv.DecodePlan(bt, cl, b.num_q_heads, b.k_cache, max_context_len=mcl,
                          partition_tokens=partition)
    outs = []
    for _ in range(3):
        for q, k, v in ((b.q, b.k_cache, b.v_cache), (q2, k2, v2)):
            outs.append(plan.run(torch.empty_like(q), q, k, v, b.scale))
    ref1 = pkv.paged_attention_decode(torch.empty_like(b.q), b.q, b.k_cache, b.v_cache, bt, cl,
                                      b.scale, 8, max_context_len=mcl, partition_tokens=partition)
    ref2 = pkv.paged_attention_decode(torch.empty_like(q2), q2, k2, v2, bt, cl, b.scale, 8,
                                      max_context_len=mcl, partition_tokens=partition)
    assert pkv.device_error_bits() == 0
    for i, o in enumerate(outs):
        ref = ref1 if i % 2 == 0 else ref2
        assert torch.equal(o.view(torch.int16), ref.view(torch.int16)), f"run {i}"


def test_back_to_back_decodes_are_deterministic(cuda_device):
    b = workloads.random_batch(73, list(range(1, 400, 7)), 16, 2, 128, "bf16", device=cuda_device)
    bt = dev_i32(b.block_tables, cuda_device)
    cl = dev_i32(b.context_lens, cuda_device)
    outs = [pkv.paged_attention_decode(torch.empty_like(b.q), b.q, b.k_cache, b.v_cache, bt, cl,
                                       b.scale, 2, max_context_len=b.max_context_len)
            for _ in range(20)]
    assert pkv.device_error_bits() == 0
    for o in outs[1:]:
        assert torch.equal(o.view(torch.int16), outs[0].view(torch.int16))


def test_expired_wait_reports_timeout_and_context_survives(cuda_device):
    assert pkv.device_error_bits() == 0
    pkv.selftest_wait_timeout(cuda_device)
    bits = pkv.device_error_bits()
    assert bits & pkv.DEVERR_TIMEOUT
    with pytest.raises(pkv.PkvError):
        pkv.selftest_wait_timeout(cuda_device)
        pkv.check_device_error(cuda_device)
    # the context is still usable: a decode afterwards is correct
    b = workloads.c1_tiny_fp32(device=cuda_device)
    host = b.host()
    out = torch.empty_like(b.q)
    pkv.paged_attention_decode(out, b.q, b.k_cache, b.v_cache, dev_i32(b.block_tables, cuda_device),
                               dev_i32(b.context_lens, cuda_device), b.scale, b.num_kv_heads,
                               max_context_len=b.max_context_len)
    ref = oracle.paged_decode(host["q"], host["k_cache"], host["v_cache"], b.block_tables,
                              b.context_lens, b.scale)
    check_close(out, ref, "f32", "after timeout")
    assert pkv.device_error_bits() == 0


def test_decode_step_captured_in_a_cuda_graph_matches_eager(cuda_device):
    """Slot indexing, reshape_and_cache, plan and decode captured once into a CUDA graph
    and replayed give bit-identical results to eager launches, and every replay meets
    the tolerance against the oracle (pools byte for byte)."""
    b = workloads.random_batch(74, [5, 17, 300, 1200, 2100], 32, 8, 128, "bf16",
                               device=cuda_device, new_token=True)
    host = b.host()
    k_ref, v_ref = oracle_caches_after_step(b, host)
    ref = oracle.paged_decode(host["q"], k_ref, v_ref, b.block_tables, b.context_lens, b.scale)
    bt = dev_i32(b.block_tables, cuda_device)
    cl = dev_i32(b.context_lens, cuda_device)
    mcl = b.max_context_len
    ws = torch.empty(pkv.decode_workspace_bytes(
        pkv.make_dims(b.num_seqs, b.num_q_heads, b.k_cache, b.max_blocks_per_seq), mcl, 512),
        dtype=torch.uint8, device=cuda_device)
    slots = torch.empty(b.num_seqs, dtype=torch.int64, device=cuda_device)
    out = torch.empty_like(b.q)

    def step():
        pkv.slot_mapping(bt, b.num_blocks, context_lens=cl, out=slots)
        pkv.reshape_and_cache(b.new_k, b.new_v, b.k_cache, b.v_cache, slots)
        plan = pkv.DecodePlan(bt, cl, b.num_q_heads, b.k_cache, max_context_len=mcl,
                              partition_tokens=512, workspace_tensor=ws)
        plan.run(out, b.q, b.k_cache, b.v_cache, b.scale)

    step()
    torch.cuda.synchronize()
    eager = out.clone()
    out.zero_()
    s = torch.cuda.Stream(device=cuda_device)
    s.wait_stream(torch.cuda.current_stream(cuda_device))
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        step()                                   # warm the per-kernel settings outside capture
        torch.cuda.synchronize()
        out.zero_()
        with torch.cuda.graph(g, stream=s):
            step()
    torch.cuda.synchronize()
    for _ in range(3):
        out.zero_()
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(out.view(torch.int16), eager.view(torch.int16))
        check_close(out, ref, "bf16", "graph replay")
    assert pkv.device_error_bits() == 0
    assert np.array_equal(host_bits(b.k_cache), k_ref)
    assert np.array_equal(host_bits(b.v_cache), v_ref)


def test_shared_prefix_step_in_a_cuda_graph(cuda_device):
    """The shared-prefix step (copy-on-write, new tokens, shared plan, decode, merge)
    captured once and replayed gives bit-identical results to eager launches, and every
    replay meets the tolerance against the oracle."""
    b = workloads.c4_shared_prefix(device=cuda_device, prompts=3, samples=5, prefix=300,
                                   max_tail=60, num_blocks=500)
    host = b.host()
    k_ref, v_ref = oracle_caches_after_step(b, host)
    ref = oracle.paged_decode(host["q"], k_ref, v_ref, b.block_tables, b.context_lens, b.scale)
    dev = cuda_device
    bt = dev_i32(b.block_tables, dev)
    cl = dev_i32(b.context_lens, dev)
    gs = dev_i32(np.asarray(b.meta["group_start"]), dev)
    sb = dev_i32(np.asarray(b.meta["shared_blocks"]), dev)
    mcl = b.max_context_len
    ws = torch.empty(pkv.decode_shared_workspace_bytes(
        pkv.make_dims(b.num_seqs, b.num_q_heads, b.k_cache, b.max_blocks_per_seq), mcl),
        dtype=torch.uint8, device=dev)
    pairs = torch.from_numpy(b.cow_pairs).to(dev)
    seq, pos = dev_i32(b.new_seq, dev), dev_i32(b.new_pos, dev)
    slots = torch.empty(b.new_seq.shape[0], dtype=torch.int64, device=dev)
    out = torch.empty_like(b.q)

    def step():
        pkv.copy_blocks(b.k_cache, b.v_cache, pairs, validate=False)
        pkv.slot_mapping(bt, b.num_blocks, token_seq=seq, token_pos=pos, out=slots)
        pkv.reshape_and_cache(b.new_k, b.new_v, b.k_cache, b.v_cache, slots)
        plan = pkv.SharedDecodePlan(bt, cl, gs, sb, b.num_q_heads, b.k_cache,
                                    max_context_len=mcl, workspace_tensor=ws)
        plan.run(out, b.q, b.k_cache, b.v_cache, b.scale)

    step()
    torch.cuda.synchronize()
    eager = out.clone()
    s = torch.cuda.Stream(device=dev)
    s.wait_stream(torch.cuda.current_stream(dev))
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        step()
        torch.cuda.synchronize()
        out.zero_()
        with torch.cuda.graph(g, stream=s):
            step()
    torch.cuda.synchronize()
    for _ in range(3):
        out.zero_()
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(out.view(torch.int16), eager.view(torch.int16))
        check_close(out, ref, "bf16", "shared-prefix graph replay")
    assert pkv.device_error_bits() == 0
