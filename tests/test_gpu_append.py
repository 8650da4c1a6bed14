"""paged_decode_append_attn_int4 (CUDA, through the C ABI) against the oracle.

The fused step stores each sequence's new token and attends over contexts
that include it. Checked: the stored rows against the oracle's rotation and
quantization of the new tokens (the write bar: codes exact except within the
rounding of a code boundary, s and z within one fp16 ulp), and the output
against the fp64 oracle reading the cache as the call left it (the decode
bar, 2e-3), so the attention must have used exactly the rows it stored.
"""
import numpy as np
import pytest
import torch

import bit_kv_cache_20_b200 as kvq
from bit_kv_cache_20_b200 import workloads
from test_gpu_decode import assert_close
from test_gpu_write import CANARY, Pool, check_tokens

pytestmark = pytest.mark.gpu


def _split_last(w):
    """Token indices (into k_new / slots_new) of every sequence's last token
    and of all the others."""
    ends = np.cumsum(w.context_lens.astype(np.int64))
    last = ends - 1
    rest = np.setdiff1d(np.arange(int(ends[-1])), last)
    return last, rest


def _run(orc, w, b, host_lens=False, slots_override=None, out_dtype=torch.float32, signs=None):
    last, rest = _split_last(w)
    pool = Pool(w.num_pages, w.Hkv, w.D)
    slots = torch.as_tensor(w.slots_new)
    if rest.size:
        kvq.kv_quant_write(w.k_new[rest].cuda(), w.v_new[rest].cuda(), slots[rest].cuda(),
                           pool.cache, pool.scales, pool.zeros, b, hadamard_signs=signs)
    step_slots = slots[last].clone() if slots_override is None else torch.as_tensor(slots_override)
    pt = torch.as_tensor(w.page_table).cuda()
    cl = torch.as_tensor(w.context_lens).cuda()
    out = torch.full((w.B, w.Hq, w.D), 7.0, dtype=out_dtype, device="cuda")
    ws = kvq.alloc_workspace(kvq.attn_workspace_size(w.B, w.Hq, w.Hkv, w.D, w.num_pages, w.max_pages, b,
                                                     host_lengths=host_lens))
    kvq.paged_decode_append_attn_int4(
        w.q.cuda(), w.k_new[last].contiguous().cuda(), w.v_new[last].contiguous().cuda(),
        step_slots.to(torch.int64).cuda(), pool.cache, pool.scales, pool.zeros, pt, cl, out, b, ws,
        context_lens_host=w.context_lens if host_lens else None, hadamard_signs=signs)
    torch.cuda.synchronize()
    return pool, last, step_slots.numpy(), out.float().cpu().numpy().astype(np.float64), ws


def _oracle(orc, w, pool, b, signs=None):
    c, s, z = pool.host()
    return orc.decode_attn(workloads.bf16_bits(w.q), c.reshape(-1), s, z, w.page_table, w.context_lens,
                           w.Hkv, b, w.num_pages, signs=signs)


@pytest.mark.parametrize("b", [0, 64, 128])
@pytest.mark.parametrize("G", [4, 8])
def test_append_stores_and_attends_like_the_oracle(orc, b, G):
    ctx = [1, 16, 17, 33, 250, 900, 4000]
    w = workloads.random_case(seed=61 + b + G, B=len(ctx), Hq=2 * G, Hkv=2, D=128, block=b, context_lens=ctx)
    pool, last, step_slots, got, ws = _run(orc, w, b)
    assert kvq.get_device_error() == 0
    check_tokens(orc, pool, w.k_new, w.v_new, w.slots_new, b, tokens=last)
    assert_close(got, _oracle(orc, w, pool, b), f"append b={b} G={G}")
    assert int(torch.count_nonzero(ws)) == 0


@pytest.mark.parametrize("host_lens", [False, True])
def test_append_long_context_many_splits(orc, host_lens):
    """One long sequence is split over many CTAs; only the one holding the
    last page stores and patches the new token."""
    ctx = [32768 - 5, 3000]
    w = workloads.random_case(seed=63, B=2, Hq=32, Hkv=8, D=128, block=128, context_lens=ctx)
    pool, last, step_slots, got, _ = _run(orc, w, 128, host_lens=host_lens)
    assert kvq.get_device_error() == 0
    check_tokens(orc, pool, w.k_new, w.v_new, w.slots_new, 128, tokens=last)
    rng = np.random.default_rng(64)
    c, s, z = pool.host()
    for n, h in [(0, 0), (0, 31), (1, 5)] + [(int(a), int(b_)) for a, b_ in zip(rng.integers(0, 2, 4),
                                                                             rng.integers(0, 32, 4))]:
        ref = orc.decode_one(workloads.bf16_bits(w.q), c.reshape(-1), s, z, w.page_table, w.context_lens,
                             n, h, w.Hkv, 128, w.num_pages)
        assert_close(got[n, h], ref, f"long n={n} hq={h}")


def test_append_slot_minus_one_and_a_mismatched_slot(orc):
    """-1: nothing is stored for that sequence and it is decoded as it stands.
    A slot that is not the sequence's last position: not stored, reported."""
    ctx = [40, 70, 100]
    w = workloads.random_case(seed=65, B=3, Hq=8, Hkv=2, D=64, block=32, context_lens=ctx)
    last, _ = _split_last(w)
    good = np.asarray(w.slots_new)[last]
    slots = good.copy()
    slots[0] = -1
    slots[2] = good[2] ^ 1  # the neighbouring offset in the same page
    pool, _, _, got, _ = _run(orc, w, 32, slots_override=slots)
    assert kvq.get_device_error() == 3
    c, s, z = pool.host()
    for n in (0, 2):  # the cache still holds the canary at the skipped rows
        page, off = divmod(int(good[n]), 16)
        for h in range(w.Hkv):
            for kv in range(2):
                row = ((page * w.Hkv + h) * 2 + kv) * 16 + off
                assert np.all(c[row] == CANARY), (n, h, kv)
    check_tokens(orc, pool, w.k_new, w.v_new, w.slots_new, 32, tokens=[last[1]])
    ref = _oracle(orc, w, pool, 32)
    assert_close(got[1], ref[1], "appended sequence")


def test_append_with_randomized_hadamard_signs(orc):
    ctx = [700, 18, 4100]
    w = workloads.random_case(seed=66, B=len(ctx), Hq=16, Hkv=4, D=128, block=64, context_lens=ctx)
    sig = workloads.random_signs(67, 128)
    pool, last, _, got, _ = _run(orc, w, 64, signs=sig)
    assert kvq.get_device_error() == 0
    check_tokens(orc, pool, w.k_new, w.v_new, w.slots_new, 64, tokens=last, signs=sig)
    assert_close(got, _oracle(orc, w, pool, 64, signs=sig), "append with signs")
