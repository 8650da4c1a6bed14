"""The decode while another stream's kernel holds almost every SM.

A decode launch that splits a (sequence, kv head) across CTAs merges their
partial results inside the same launch: merger CTAs poll for the partials of
the other splits, so those splits must get to run. Nothing guarantees that
all CTAs of a launch are resident at once when other kernels hold SMs. Here a
kernel on a second stream keeps all but two SMs for 0.4 s - longer than a
merge poll's bound (~0.27 s) - while the decode is launched: mergers that
find splits of their group not yet started hand their rows over to the
group's last-started CTA and exit, so the decode completes on the two free
SMs, matches the oracle and records no device error. A call right after, on
an idle GPU, must give the same output and leave the workspace all zero.
"""
import time

import numpy as np
import pytest
import torch

import bit_kv_cache_20_b200 as kvq
from bit_kv_cache_20_b200 import workloads

pytestmark = pytest.mark.gpu

TOL = 2e-3


@pytest.mark.parametrize("case", ["uniform-plan", "per-sequence-plan"])
def test_decode_correct_while_another_stream_holds_sms(orc, case):
    if case == "uniform-plan":
        w = workloads.random_case(seed=41, B=1, Hq=32, Hkv=8, D=128, block=128, context_lens=[8192])
        host = None
    else:
        w = workloads.random_case(seed=42, B=3, Hq=16, Hkv=4, D=128, block=64,
                                  context_lens=[6000, 300, 2500])
        host = np.asarray(w.context_lens, np.int32)
    cache, scales, zeros = kvq.alloc_cache(w.num_pages, w.Hkv, w.D)
    kvq.kv_quant_write(w.k_new.cuda(), w.v_new.cuda(), torch.as_tensor(w.slots_new).cuda(), cache, scales,
                       zeros, w.block)
    need = kvq.attn_workspace_size(w.B, w.Hq, w.Hkv, w.D, w.num_pages, w.max_pages, w.block,
                                   host_lengths=host is not None)
    assert need > 0, "the case must split a (sequence, kv head) and merge"
    ws = kvq.alloc_workspace(need)
    q, pt, cl = w.q.cuda(), torch.as_tensor(w.page_table).cuda(), torch.as_tensor(w.context_lens).cuda()
    torch.cuda.synchronize()
    c = cache.cpu().numpy().reshape(-1)
    s = scales.cpu().view(torch.int16).numpy().view(np.uint16).reshape(-1)
    z = zeros.cpu().view(torch.int16).numpy().view(np.uint16).reshape(-1)
    ref = orc.decode_attn(workloads.bf16_bits(w.q), c, s, z, w.page_table, w.context_lens, w.Hkv, w.block,
                          w.num_pages)

    sms = torch.cuda.get_device_properties(0).multi_processor_count
    hog, main = torch.cuda.Stream(), torch.cuda.Stream()
    outs = []
    for busy in (True, False):
        out = torch.full((w.B, w.Hq, w.D), float("nan"), dtype=torch.float32, device="cuda")
        t0 = time.monotonic()
        if busy:
            kvq.selftest_occupy(sms - 2, 400_000, stream=hog)
            time.sleep(0.02)  # the holder is resident before the decode is launched
        kvq.paged_decode_attn_int4(q, cache, scales, zeros, pt, cl, out, w.block, ws, stream=main,
                                   context_lens_host=host)
        main.synchronize()
        t_dec = time.monotonic() - t0
        hog.synchronize()
        assert kvq.get_device_error(main) == 0
        err = float(np.abs(out.cpu().numpy().astype(np.float64) - ref).max())
        print(f"{case} busy={busy}: decode done after {t_dec * 1e3:.1f} ms, max|err| = {err:.3e}")
        assert err <= TOL
        outs.append(out)
    assert torch.equal(outs[0], outs[1])
    assert int(ws.count_nonzero()) == 0


def test_occupy_hook_rejects_bad_arguments():
    with pytest.raises(kvq.KVQError):
        kvq.selftest_occupy(0, 10)
    with pytest.raises(kvq.KVQError):
        kvq.selftest_occupy(1, 2_000_000)
