"""The failure path of the bounded waits, on the GPU without a fault: a wait
on a condition that nothing completes (an mbarrier nobody arrives on; the
split-merge poll of a word that stays zero) runs out, the kernel records
KVQ_ERR_TIMEOUT and returns, the host reads the status, and the context stays
usable for the next call."""
import time

import numpy as np
import pytest
import torch

import bit_kv_cache_20_b200 as kvq
from bit_kv_cache_20_b200 import workloads

pytestmark = pytest.mark.gpu

KVQ_ERR_TIMEOUT = 5


@pytest.mark.parametrize("which", [0, 1])
def test_bounded_wait_runs_out_and_is_reported(orc, which):
    assert kvq.get_device_error() == 0
    t0 = time.monotonic()
    kvq.selftest_bounded_wait(which)
    assert kvq.get_device_error() == KVQ_ERR_TIMEOUT
    assert time.monotonic() - t0 < 60
    assert kvq.get_device_error() == 0  # read and cleared

    # the context still works: a write and a decode match the oracle
    import oracle
    w = workloads.make("tiny")
    cache, scales, zeros = kvq.alloc_cache(w.num_pages, w.Hkv, w.D)
    kvq.kv_quant_write(w.k_new.cuda(), w.v_new.cuda(), torch.as_tensor(w.slots_new).cuda(), cache, scales,
                       zeros, w.block)
    out = torch.empty((w.B, w.Hq, w.D), dtype=torch.float32, device="cuda")
    ws = kvq.alloc_workspace(kvq.attn_workspace_size(w.B, w.Hq, w.Hkv, w.D, w.num_pages, w.max_pages, w.block))
    kvq.paged_decode_attn_int4(w.q.cuda(), cache, scales, zeros, torch.as_tensor(w.page_table).cuda(),
                               torch.as_tensor(w.context_lens).cuda(), out, w.block, ws)
    assert kvq.get_device_error() == 0
    c = cache.cpu().numpy().reshape(-1)
    s = scales.cpu().view(torch.int16).numpy().view(np.uint16).reshape(-1)
    z = zeros.cpu().view(torch.int16).numpy().view(np.uint16).reshape(-1)
    ref = oracle.decode_attn(workloads.bf16_bits(w.q), c, s, z, w.page_table, w.context_lens, w.Hkv, w.block,
                             w.num_pages)
    assert float(np.abs(out.cpu().numpy().astype(np.float64) - ref).max()) <= 2e-3


def test_selftest_rejects_an_unknown_wait():
    with pytest.raises(kvq.KVQError):
        kvq.selftest_bounded_wait(2)
