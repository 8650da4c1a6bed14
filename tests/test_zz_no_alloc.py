"""The allocation-free decode entry point (paged_decode_attn_int4_static_ws).

It serves callers that cannot allocate device memory: its split-K scratch is
a fixed array inside the library instead of a caller-provided workspace. This
checks, through the C ABI, that two calls in a row give the same output as the
regular entry point with an allocated workspace (within the parity tolerance).
The file is collected last so that a run stopping at the first failure has
already run everything else; it sets up all its own state, so it also passes
alone in a fresh process.
"""
import numpy as np
import pytest
import torch

import bit_kv_cache_20_b200 as kvq
from bit_kv_cache_20_b200 import workloads

pytestmark = pytest.mark.gpu

TOL = 2e-3


def _pool(w):
    cache, scales, zeros = kvq.alloc_cache(w.num_pages, w.Hkv, w.D)
    kvq.kv_quant_write(w.k_new.cuda(), w.v_new.cuda(), torch.as_tensor(w.slots_new).cuda(),
                       cache, scales, zeros, w.block)
    return cache, scales, zeros


@pytest.mark.parametrize("case", ["two-sequences", "llama3-8b-32k"])
def test_static_workspace_matches_the_allocating_entry_point(case):
    if case == "two-sequences":
        w = workloads.random_case(seed=31, B=2, Hq=16, Hkv=4, D=128, block=128,
                                  context_lens=[3000, 777])
    else:
        w = workloads.make("llama3-8b-32k")
    need = kvq.attn_workspace_size(w.B, w.Hq, w.Hkv, w.D, w.num_pages, w.max_pages, w.block)
    assert need > 0, "the case must use split-K scratch"
    cache, scales, zeros = _pool(w)
    q = w.q.cuda()
    pt = torch.as_tensor(w.page_table).cuda()
    cl = torch.as_tensor(w.context_lens).cuda()

    ref = torch.empty((w.B, w.Hq, w.D), dtype=torch.float32, device="cuda")
    kvq.paged_decode_attn_int4(q, cache, scales, zeros, pt, cl, ref, w.block,
                               kvq.alloc_workspace(need))
    outs = []
    for _ in range(2):
        out = torch.full((w.B, w.Hq, w.D), float("nan"), dtype=torch.float32, device="cuda")
        kvq.paged_decode_attn_int4_static_ws(q, cache, scales, zeros, pt, cl, out, w.block)
        outs.append(out)
    assert kvq.get_device_error() == 0
    ref_h = ref.cpu().numpy()
    for i, out in enumerate(outs):
        err = float(np.abs(out.cpu().numpy() - ref_h).max())
        print(f"{case}: static-scratch call {i + 1}: max|diff| vs allocating call = {err:.3e}")
        assert err <= TOL
