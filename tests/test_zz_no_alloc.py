"""The allocation-free decode entry point (paged_decode_attn_int4_static_ws).

It serves callers that cannot allocate device memory - a plug-in whose host
runtime owns all GPU memory through its own pool, or a path where an
allocation's implicit device synchronization is not acceptable: its split-K
scratch is a fixed array inside the library instead of a caller-provided
workspace. Through the C ABI this checks, on two calls in a row, that it gives
the regular entry point's output (allocated workspace) within the parity
tolerance, that it matches the oracle, that the array is left all zero, and
that a per-sequence plan (host copy of the context lengths) and a GQA-8 shape
fit in the array. The file is collected last so that a run stopping at the
first failure has already run everything else; it sets up all its own state,
so it also passes alone in a fresh process.
"""
import numpy as np
import pytest
import torch

import bit_kv_cache_20_b200 as kvq
from bit_kv_cache_20_b200 import _lib, workloads

pytestmark = pytest.mark.gpu

TOL = 2e-3


def _pool(w):
    cache, scales, zeros = kvq.alloc_cache(w.num_pages, w.Hkv, w.D)
    kvq.kv_quant_write(w.k_new.cuda(), w.v_new.cuda(), torch.as_tensor(w.slots_new).cuda(),
                       cache, scales, zeros, w.block)
    return cache, scales, zeros


def _case(name):
    if name == "two-sequences":
        return workloads.random_case(seed=31, B=2, Hq=16, Hkv=4, D=128, block=128, context_lens=[3000, 777]), None
    if name == "llama3-8b-32k":
        return workloads.make("llama3-8b-32k"), None
    if name == "gqa8-per-sequence-plan":
        w = workloads.random_case(seed=33, B=4, Hq=64, Hkv=8, D=128, block=128,
                                  context_lens=[9000, 1200, 4000, 64])
        return w, np.asarray(w.context_lens, np.int32)
    raise ValueError(name)


@pytest.mark.parametrize("case", ["two-sequences", "llama3-8b-32k", "gqa8-per-sequence-plan"])
def test_static_workspace_matches_the_allocating_entry_point(orc, case):
    w, host = _case(case)
    need = kvq.attn_workspace_size(w.B, w.Hq, w.Hkv, w.D, w.num_pages, w.max_pages, w.block,
                                   host_lengths=host is not None)
    assert need > 0, "the case must use split-K scratch"
    cache, scales, zeros = _pool(w)
    q = w.q.cuda()
    pt = torch.as_tensor(w.page_table).cuda()
    cl = torch.as_tensor(w.context_lens).cuda()

    ref = torch.empty((w.B, w.Hq, w.D), dtype=torch.float32, device="cuda")
    kvq.paged_decode_attn_int4(q, cache, scales, zeros, pt, cl, ref, w.block, kvq.alloc_workspace(need),
                               context_lens_host=host)
    outs = []
    for _ in range(2):
        out = torch.full((w.B, w.Hq, w.D), float("nan"), dtype=torch.float32, device="cuda")
        kvq.paged_decode_attn_int4_static_ws(q, cache, scales, zeros, pt, cl, out, w.block,
                                             context_lens_host=host)
        outs.append(out)
    assert kvq.get_device_error() == 0
    # every word the calls wrote was read and cleared again
    assert _lib.lib().kvq_static_workspace_nonzero() == 0
    ref_h = ref.cpu().numpy()
    for i, out in enumerate(outs):
        err = float(np.abs(out.cpu().numpy() - ref_h).max())
        print(f"{case}: static-scratch call {i + 1}: max|diff| vs allocating call = {err:.3e}")
        assert err <= TOL
    # against the oracle on the same dequantized cache (sampled query heads
    # for the large cases)
    c = cache.cpu().numpy().reshape(-1)
    s = scales.cpu().view(torch.int16).numpy().view(np.uint16).reshape(-1)
    z = zeros.cpu().view(torch.int16).numpy().view(np.uint16).reshape(-1)
    qb = workloads.bf16_bits(w.q)
    rng = np.random.default_rng(5)
    pairs = [(int(rng.integers(w.B)), int(rng.integers(w.Hq))) for _ in range(6)]
    got = outs[1].cpu().numpy()
    for n, hq in pairs:
        r = orc.decode_one(qb, c, s, z, w.page_table, w.context_lens, n, hq, w.Hkv, w.block, w.num_pages, 0.0)
        err = float(np.abs(got[n, hq] - r).max())
        print(f"{case}: n={n} hq={hq}: max|err| vs oracle = {err:.3e}")
        assert err <= TOL
