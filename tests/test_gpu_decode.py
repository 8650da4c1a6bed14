"""Parity of paged_decode_attn_int4 (CUDA, through the C ABI) with the oracle.

The oracle reads the cache bytes the CUDA write produced, so write-path
differences cannot leak into this check. Bar: fp32 output within 2e-3
max-abs of the fp64 oracle; bf16 output equal to the round-to-nearest bf16 of
the fp32 output; guard regions around `out` untouched; a workspace reused
without clearing gives the same result.
"""
import dataclasses

import numpy as np
import pytest
import torch

import bit_kv_cache_20_b200 as kvq
from bit_kv_cache_20_b200 import workloads

pytestmark = pytest.mark.gpu

TOL = 2e-3
GUARD = 1024


def build_cache(w, b=None):
    b = w.block if b is None else b
    cache, scales, zeros = kvq.alloc_cache(w.num_pages, w.Hkv, w.D)
    for k, v, s in ((w.k_prior, w.v_prior, w.slots_prior), (w.k_new, w.v_new, w.slots_new)):
        if k.shape[0]:
            kvq.kv_quant_write(k.cuda(), v.cuda(), torch.as_tensor(s).cuda(), cache, scales, zeros, b)
    assert kvq.get_device_error() == 0
    return cache, scales, zeros


def host_cache(cache, scales, zeros):
    return (cache.cpu().numpy().reshape(-1),
            scales.cpu().view(torch.int16).numpy().view(np.uint16).reshape(-1),
            zeros.cpu().view(torch.int16).numpy().view(np.uint16).reshape(-1))


def gpu_decode(w, pool, b=None, out_dtype=torch.float32, softmax_scale=0.0, ws=None,
               page_table=None, ctx=None, host_lens=None):
    b = w.block if b is None else b
    cache, scales, zeros = pool
    pt = torch.as_tensor(w.page_table if page_table is None else page_table).cuda()
    cl = torch.as_tensor(w.context_lens if ctx is None else ctx).cuda()
    n = w.B * w.Hq * w.D
    big = torch.full((n + 2 * GUARD,), 7.0, dtype=out_dtype, device="cuda")
    out = big[GUARD:GUARD + n].view(w.B, w.Hq, w.D)
    if ws is None:
        nbytes = kvq.attn_workspace_size(w.B, w.Hq, w.Hkv, w.D, w.num_pages, pt.shape[1], b,
                                         host_lengths=host_lens is not None)
        ws = kvq.alloc_workspace(nbytes)
    kvq.paged_decode_attn_int4(w.q.cuda(), cache, scales, zeros, pt, cl, out, b, ws,
                               softmax_scale=softmax_scale, context_lens_host=host_lens)
    torch.cuda.synchronize()
    g = big.cpu()
    assert torch.all(g[:GUARD] == 7.0) and torch.all(g[GUARD + n:] == 7.0), "out guard overwritten"
    return out.float().cpu().numpy().astype(np.float64), ws


def oracle_out(orc, w, pool, b=None, softmax_scale=0.0, pairs=None):
    b = w.block if b is None else b
    c, s, z = host_cache(*pool)
    qb = workloads.bf16_bits(w.q)
    if pairs is None:
        return orc.decode_attn(qb, c, s, z, w.page_table, w.context_lens, w.Hkv, b, w.num_pages,
                               softmax_scale)
    return {(n, hq): orc.decode_one(qb, c, s, z, w.page_table, w.context_lens, n, hq, w.Hkv, b,
                                    w.num_pages, softmax_scale) for n, hq in pairs}


def assert_close(got, ref, label):
    err = float(np.abs(got - ref).max()) if ref.size else 0.0
    print(f"{label}: max|err| = {err:.3e} (max|ref| = {float(np.abs(ref).max(initial=0)):.3e})")
    assert err <= TOL, (label, err)


def test_decode_tiny_config(orc):
    w = workloads.make("tiny")
    pool = build_cache(w)
    got, ws = gpu_decode(w, pool)
    assert_close(got, oracle_out(orc, w, pool), "tiny")


@pytest.mark.parametrize("D,b", [(64, 0), (64, 32), (64, 64), (128, 0), (128, 32), (128, 64), (128, 128)])
@pytest.mark.parametrize("G", [1, 2, 4, 8])
def test_decode_random_shapes(orc, D, b, G):
    # contexts: empty, a single token, page boundary -1/0/+1, several pages,
    # and enough pages for several splits
    ctx = [0, 1, 15, 16, 17, 33, 250, 1000]
    w = workloads.random_case(seed=D * 3 + b + G, B=len(ctx), Hq=2 * G, Hkv=2, D=D, block=b,
                              context_lens=ctx, extra_pages=3)
    pool = build_cache(w)
    got, ws = gpu_decode(w, pool)
    ref = oracle_out(orc, w, pool)
    assert_close(got, ref, f"D={D} b={b} G={G}")
    assert np.all(got[0] == 0.0), "empty context must give zero output"


def test_decode_single_split_path(orc):
    # enough (sequence, kv head) pairs that each is one CTA (no workspace)
    w = workloads.random_case(seed=21, B=64, Hq=32, Hkv=8, D=128, block=64,
                              context_lens=list(np.arange(64) * 7 + 1), extra_pages=0)
    assert kvq.attn_workspace_size(w.B, w.Hq, w.Hkv, w.D, w.num_pages, w.max_pages, 64) == 0
    pool = build_cache(w)
    got, _ = gpu_decode(w, pool)
    assert_close(got, oracle_out(orc, w, pool), "single split")


def test_decode_full_size_llama3_8b_32k(orc):
    # the benchmark's decode launch: 1 sequence of 32768 tokens, 32 q heads
    w = workloads.make("llama3-8b-32k")
    pool = build_cache(w)
    got, _ = gpu_decode(w, pool)
    ref = oracle_out(orc, w, pool)
    assert_close(got, ref, "llama3-8b-32k")
    got16, _ = gpu_decode(w, pool, out_dtype=torch.bfloat16)
    ref16 = torch.from_numpy(got.astype(np.float32)).to(torch.bfloat16).float().numpy()
    assert np.array_equal(got16.astype(np.float32), ref16)


def test_decode_llama2_70b_b8_sampled(orc):
    w = workloads.make("llama2-70b-b8")
    pool = build_cache(w)
    got, _ = gpu_decode(w, pool)
    rng = np.random.default_rng(2)
    pairs = [(int(n), int(h)) for n, h in zip(rng.integers(0, w.B, 12), rng.integers(0, w.Hq, 12))]
    ref = oracle_out(orc, w, pool, pairs=pairs)
    for (n, h), r in ref.items():
        assert_close(got[n, h], r, f"llama2-70b-b8 n={n} hq={h}")


def test_decode_serving_b64_sampled(orc):
    w = workloads.make("serving-b64")
    pool = build_cache(w)
    got, _ = gpu_decode(w, pool)
    rng = np.random.default_rng(3)
    pairs = [(int(n), int(h)) for n, h in zip(rng.integers(0, w.B, 16), rng.integers(0, w.Hq, 16))]
    for (n, h), r in oracle_out(orc, w, pool, pairs=pairs).items():
        assert_close(got[n, h], r, f"serving-b64 n={n} hq={h}")


@pytest.mark.parametrize("b", [0, 32, 64, 128])
def test_decode_stress_lognormal_contexts_sampled(orc, b):
    w = workloads.make("stress-b256", block=b, batch=24)
    pool = build_cache(w, b)
    got, _ = gpu_decode(w, pool, b)
    rng = np.random.default_rng(4 + b)
    pairs = [(int(n), int(h)) for n, h in zip(rng.integers(0, w.B, 10), rng.integers(0, w.Hq, 10))]
    for (n, h), r in oracle_out(orc, w, pool, b, pairs=pairs).items():
        assert_close(got[n, h], r, f"stress b={b} n={n} hq={h}")


def test_decode_explicit_softmax_scale_and_bf16(orc):
    w = workloads.random_case(seed=8, B=3, Hq=8, Hkv=2, D=128, block=64, context_lens=[70, 3, 400])
    pool = build_cache(w)
    got, _ = gpu_decode(w, pool, softmax_scale=0.05)
    assert_close(got, oracle_out(orc, w, pool, softmax_scale=0.05), "softmax_scale=0.05")
    got16, _ = gpu_decode(w, pool, out_dtype=torch.bfloat16, softmax_scale=0.05)
    ref16 = torch.from_numpy(got.astype(np.float32)).to(torch.bfloat16).float().numpy()
    assert np.array_equal(got16.astype(np.float32), ref16)


def test_decode_deterministic_and_workspace_left_zeroed():
    """Repeated calls on one workspace give identical outputs, and each call
    leaves every workspace word at zero: partial results are stored
    bit-inverted and a merger takes a non-zero word as written, so a stale
    word would be merged in place of the next call's value."""
    w = workloads.random_case(seed=9, B=2, Hq=16, Hkv=4, D=128, block=128, context_lens=[3000, 777])
    pool = build_cache(w)
    a, ws = gpu_decode(w, pool)
    assert ws.numel() > 16, "the case must use partial results"
    assert int(torch.count_nonzero(ws)) == 0
    for _ in range(3):
        b_, ws = gpu_decode(w, pool, ws=ws)
        assert np.array_equal(a, b_)
        assert int(torch.count_nonzero(ws)) == 0


@pytest.mark.parametrize("host", [False, True])
@pytest.mark.parametrize("ctx,Hq,Hkv", [([40000 - 7], 8, 2), ([36001, 2000], 8, 2), ([1, 17, 900], 8, 2),
                                        ([60000] + [16] * 39, 8, 8)])
def test_decode_counts_every_page_once(ctx, Hq, Hkv, host):
    """q = 0 makes the softmax uniform, and on a plain INT4 cache a constant V
    row c is stored exactly (s = 0, z = c). With c = a different integer per
    page, the output is the mean page value over the context: a page skipped
    or counted twice by the split plan moves it by ~16 |c - mean| / ctx, far
    above fp32 rounding. In the last case 320 (sequence, kv head) pairs leave
    at most 3 splits per pair on 148 SMs, so a split of the long sequence
    holds more pages than the kernel keeps page ids for in shared memory."""
    B = len(ctx)
    w = workloads.random_case(seed=31, B=B, Hq=Hq, Hkv=Hkv, D=128, block=0, context_lens=ctx)
    vals = []
    for n in range(B):
        pos = np.arange(ctx[n])
        vals.append(((pos // 16) % 97 - 48).astype(np.float64))
    c = torch.as_tensor(np.concatenate(vals), dtype=torch.bfloat16)
    v_new = c[:, None, None].expand(-1, w.Hkv, w.D).contiguous()
    w = dataclasses.replace(w, v_new=v_new, q=torch.zeros_like(w.q))
    pool = build_cache(w)
    got, _ = gpu_decode(w, pool, host_lens=np.asarray(ctx, np.int32) if host else None)
    for n in range(B):
        ref = vals[n].mean()
        err = float(np.abs(got[n] - ref).max())
        assert err <= 1e-5 * max(1.0, abs(ref)), (ctx, n, err)


def test_decode_bad_page_id_and_long_context_are_reported(orc):
    w = workloads.random_case(seed=10, B=2, Hq=4, Hkv=2, D=64, block=32, context_lens=[40, 20])
    pool = build_cache(w)
    pt = w.page_table.copy()
    pt[0, 1] = w.num_pages + 5
    gpu_decode(w, pool, page_table=pt)
    assert kvq.get_device_error() == 3
    ctx = w.context_lens.copy()
    ctx[1] = w.max_pages * 16 + 1
    gpu_decode(w, pool, ctx=ctx)
    assert kvq.get_device_error() == 3
    assert kvq.get_device_error() == 0


def test_decode_rejects_missing_workspace():
    w = workloads.random_case(seed=12, B=1, Hq=8, Hkv=2, D=128, block=128, context_lens=[4000])
    need = kvq.attn_workspace_size(w.B, w.Hq, w.Hkv, w.D, w.num_pages, w.max_pages, 128)
    assert need > 0
    pool = build_cache(w)
    out = torch.empty((1, 8, 128), device="cuda")
    with pytest.raises(kvq.KVQError):
        kvq.paged_decode_attn_int4(w.q.cuda(), *pool, torch.as_tensor(w.page_table).cuda(),
                                   torch.as_tensor(w.context_lens).cuda(), out, 128,
                                   kvq.alloc_workspace(need - 16))


@pytest.mark.parametrize("case", ["mixed-g4", "mixed-g8", "many-short"])
def test_decode_per_sequence_plan_matches_oracle(orc, case):
    """With the host copy of the context lengths the launch is planned per
    sequence: long sequences get several splits, short ones one CTA, the
    longest start first, and a batch with more (sequence, head) pairs than
    resident CTAs runs in several waves."""
    if case == "mixed-g4":
        ctx = [1, 17, 900, 4000, 12000, 0, 250, 33, 20000, 5]
        w = workloads.random_case(seed=51, B=len(ctx), Hq=32, Hkv=8, D=128, block=64, context_lens=ctx)
    elif case == "mixed-g8":
        ctx = [30000, 100, 7000, 16, 2500]
        w = workloads.random_case(seed=52, B=len(ctx), Hq=64, Hkv=8, D=128, block=128, context_lens=ctx)
    else:
        rng = np.random.default_rng(53)
        ctx = [int(x) for x in rng.integers(1, 3000, size=300)]
        ctx[7] = 9000
        w = workloads.random_case(seed=53, B=len(ctx), Hq=8, Hkv=2, D=64, block=32, context_lens=ctx)
    pool = build_cache(w)
    got, _ = gpu_decode(w, pool, host_lens=np.asarray(ctx, np.int32))
    if w.B <= 16:
        assert_close(got, oracle_out(orc, w, pool), case)
    else:
        rng = np.random.default_rng(54)
        pairs = [(7, 0)] + [(int(n), int(h)) for n, h in zip(rng.integers(0, w.B, 20), rng.integers(0, w.Hq, 20))]
        for (n, h), r in oracle_out(orc, w, pool, pairs=pairs).items():
            assert_close(got[n, h], r, f"{case} n={n} hq={h}")


@pytest.mark.parametrize("factor", [0.5, 2.0])
def test_decode_out_of_date_host_lengths_stay_correct(orc, factor):
    """A host copy that no longer matches the device lengths (the plan of a
    captured graph replayed a step later) changes only the balance: shorter
    host lengths make the kernel re-split the affected sequences itself."""
    ctx = [9000, 300, 17, 4100]
    w = workloads.random_case(seed=55, B=len(ctx), Hq=32, Hkv=8, D=128, block=128, context_lens=ctx)
    pool = build_cache(w)
    host = np.maximum((np.asarray(ctx) * factor).astype(np.int32), 1)
    got, _ = gpu_decode(w, pool, host_lens=host)
    assert_close(got, oracle_out(orc, w, pool), f"host lengths x{factor}")
    assert kvq.get_device_error() == 0


def test_decode_ignores_garbage_past_the_context(orc):
    """Rows of a sequence's last page past its context may hold anything (a
    freed sequence's data, never-written memory): filled here with NaN scales
    and offsets and random code bytes, they must not reach the output."""
    ctx = [1, 17, 250, 31]
    w = workloads.random_case(seed=71, B=len(ctx), Hq=16, Hkv=2, D=128, block=64, context_lens=ctx)
    cache, scales, zeros = kvq.alloc_cache(w.num_pages, w.Hkv, w.D)
    g = torch.Generator(device="cuda").manual_seed(72)
    cache.copy_(torch.randint(0, 256, cache.shape, generator=g, device="cuda", dtype=torch.int32).to(torch.uint8))
    scales.view(torch.int16).fill_(0x7E00)  # fp16 NaN
    zeros.view(torch.int16).fill_(0x7E00)
    pool = (cache, scales, zeros)
    kvq.kv_quant_write(w.k_new.cuda(), w.v_new.cuda(), torch.as_tensor(w.slots_new).cuda(), *pool, w.block)
    got, _ = gpu_decode(w, pool)
    assert np.all(np.isfinite(got))
    assert_close(got, oracle_out(orc, w, pool), "garbage past the context")


@pytest.mark.parametrize("D,b,G", [(64, 32, 4), (128, 64, 8), (128, 128, 4)])
def test_decode_randomized_hadamard_signs(orc, D, b, G):
    """q rotated by R = H_b diag(sigma)/sqrt(b), the output by R^T, over a
    cache written with the same signs; several splits (long context)."""
    ctx = [5000, 33, 1]
    w = workloads.random_case(seed=91 + D + b + G, B=len(ctx), Hq=2 * G, Hkv=2, D=D, block=b, context_lens=ctx)
    sig = workloads.random_signs(92 + D, D)
    cache, scales, zeros = kvq.alloc_cache(w.num_pages, w.Hkv, w.D)
    kvq.kv_quant_write(w.k_new.cuda(), w.v_new.cuda(), torch.as_tensor(w.slots_new).cuda(), cache, scales,
                       zeros, b, hadamard_signs=sig)
    pool = (cache, scales, zeros)
    pt = torch.as_tensor(w.page_table).cuda()
    cl = torch.as_tensor(w.context_lens).cuda()
    out = torch.empty((w.B, w.Hq, w.D), device="cuda")
    ws = kvq.alloc_workspace(kvq.attn_workspace_size(w.B, w.Hq, w.Hkv, w.D, w.num_pages, w.max_pages, b))
    kvq.paged_decode_attn_int4(w.q.cuda(), cache, scales, zeros, pt, cl, out, b, ws, hadamard_signs=sig)
    got = out.cpu().numpy().astype(np.float64)
    c, s_, z_ = host_cache(*pool)
    ref = orc.decode_attn(workloads.bf16_bits(w.q), c, s_, z_, w.page_table, w.context_lens, w.Hkv, b,
                          w.num_pages, signs=sig)
    assert_close(got, ref, f"signs D={D} b={b} G={G}")
