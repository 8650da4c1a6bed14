"""Kernels chained on one stream with no host synchronization.

Every kernel of the library is a programmatic dependent launch: its CTAs may
start while the previous kernel drains, and each waits for that kernel before
touching memory it may have written (with KVQ_ATTN_INPUTS_READY the decode
reads q, the page table and the context lengths before that wait). A wait in
the wrong place shows up here as a decode that reads a half-written cache, a
write that overwrites pages a decode is still reading, or two decodes racing
on one workspace. The kernels are deterministic, so each chained result must
equal, bit for bit, the same call made with the device synchronized before
and after it.
"""
import numpy as np
import pytest
import torch

import bit_kv_cache_20_b200 as kvq
from bit_kv_cache_20_b200 import workloads

pytestmark = pytest.mark.gpu


def _setup(block):
    w = workloads.random_case(seed=41, B=2, Hq=32, Hkv=8, D=128, block=block,
                              context_lens=[8192, 5000])
    g = torch.Generator().manual_seed(42)
    # a second K/V set for the same slots (the chain alternates them)
    k2 = (torch.randn(w.k_new.shape, generator=g) * 3).to(torch.bfloat16)
    v2 = (torch.randn(w.v_new.shape, generator=g) * 3).to(torch.bfloat16)
    dev = torch.device("cuda")
    sets = [(w.k_new.to(dev), w.v_new.to(dev)), (k2.to(dev), v2.to(dev))]
    slots = torch.as_tensor(w.slots_new).to(dev)
    pool = kvq.alloc_cache(w.num_pages, w.Hkv, w.D)
    q = w.q.to(dev)
    pt = torch.as_tensor(w.page_table).to(dev)
    cl = torch.as_tensor(w.context_lens).to(dev)
    ws = kvq.alloc_workspace(kvq.attn_workspace_size(w.B, w.Hq, w.Hkv, w.D, w.num_pages,
                                                     w.max_pages, block))
    return w, sets, slots, pool, q, pt, cl, ws


@pytest.mark.parametrize("block", [0, 128])
def test_write_decode_chain_matches_synchronized_calls(block):
    w, sets, slots, pool, q, pt, cl, ws = _setup(block)
    cache, scales, zeros = pool

    def write(i):
        k, v = sets[i]
        kvq.kv_quant_write(k, v, slots, cache, scales, zeros, block)

    def decode(out, ready):
        kvq.paged_decode_attn_int4(q, cache, scales, zeros, pt, cl, out, block, ws, inputs_ready=ready)

    ref = []
    for i in range(2):
        out = torch.empty((w.B, w.Hq, w.D), device="cuda")
        torch.cuda.synchronize()
        write(i)
        torch.cuda.synchronize()
        decode(out, False)
        torch.cuda.synchronize()
        ref.append(out.cpu())
    assert not torch.equal(ref[0], ref[1]), "the two K/V sets must give different outputs"

    order = [0, 1, 0, 1, 1, 0]
    outs = [torch.full((w.B, w.Hq, w.D), float("nan"), device="cuda") for _ in order]
    torch.cuda.synchronize()
    for i, out in zip(order, outs):
        write(i)        # overwrites every page the previous decode read
        decode(out, True)
    torch.cuda.synchronize()
    assert kvq.get_device_error() == 0
    for j, (i, out) in enumerate(zip(order, outs)):
        assert torch.equal(out.cpu(), ref[i]), f"chained step {j} (set {i}) differs"
    assert int(torch.count_nonzero(ws)) == 0


def test_back_to_back_decodes_share_one_workspace():
    w, sets, slots, pool, q, pt, cl, ws = _setup(128)
    cache, scales, zeros = pool
    kvq.kv_quant_write(*sets[0], slots, cache, scales, zeros, 128)
    ref = torch.empty((w.B, w.Hq, w.D), device="cuda")
    torch.cuda.synchronize()
    kvq.paged_decode_attn_int4(q, cache, scales, zeros, pt, cl, ref, 128, ws)
    torch.cuda.synchronize()
    outs = [torch.full((w.B, w.Hq, w.D), float("nan"), device="cuda") for _ in range(6)]
    for j, out in enumerate(outs):
        kvq.paged_decode_attn_int4(q, cache, scales, zeros, pt, cl, out, 128, ws,
                                   inputs_ready=bool(j % 2))
    torch.cuda.synchronize()
    assert kvq.get_device_error() == 0
    for j, out in enumerate(outs):
        assert torch.equal(out, ref), f"decode {j} of the chain differs"
    assert int(torch.count_nonzero(ws)) == 0
