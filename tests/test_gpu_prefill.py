"""Chunked-prefill attention (CUDA, tcgen05, through the C ABI) against the
oracle: every query of a chunk is the oracle's decode over the context up to
and including its own position (a pinned routine, composed, not retyped).
Bar: 2e-3 max-abs (fp32 output), as for the decode."""
import numpy as np
import pytest
import torch

import bit_kv_cache_20_b200 as kvq
from bit_kv_cache_20_b200 import workloads
from test_gpu_decode import assert_close, host_cache

pytestmark = pytest.mark.gpu


def _case(seed, ctx, qlen, Hq, Hkv, b, signs=None, D=128):
    w = workloads.random_case(seed=seed, B=len(ctx), Hq=Hq, Hkv=Hkv, D=D, block=b, context_lens=ctx)
    cache, scales, zeros = kvq.alloc_cache(w.num_pages, w.Hkv, w.D)
    kvq.kv_quant_write(w.k_new.cuda(), w.v_new.cuda(), torch.as_tensor(w.slots_new).cuda(), cache, scales,
                       zeros, b, hadamard_signs=signs)
    g = torch.Generator().manual_seed(seed + 1)
    qstart = np.concatenate([[0], np.cumsum(qlen)]).astype(np.int32)
    q = (torch.randn((int(qstart[-1]), Hq, D), generator=g) / 8).to(torch.bfloat16)
    out = torch.full(q.shape, 7.0, dtype=torch.float32, device="cuda")
    kvq.paged_prefill_attn_int4(q.cuda(), cache, scales, zeros, torch.as_tensor(w.page_table).cuda(),
                                torch.as_tensor(w.context_lens).cuda(), torch.as_tensor(qstart).cuda(),
                                int(max(qlen)), out, b, hadamard_signs=signs)
    torch.cuda.synchronize()
    assert kvq.get_device_error() == 0
    # oracle: query token i of sequence n = a decode over positions 0 .. its own
    rows_n = np.repeat(np.arange(len(ctx)), qlen)
    pos = np.concatenate([np.arange(c - l, c) for c, l in zip(ctx, qlen)])
    c, s, z = host_cache(cache, scales, zeros)
    ref = orc_decode(q, c, s, z, w.page_table[rows_n], (pos + 1).astype(np.int32), Hkv, b, w.num_pages, signs)
    return out.cpu().numpy().astype(np.float64), ref


def orc_decode(q, c, s, z, pt, ctx, Hkv, b, num_pages, signs):
    import oracle
    return oracle.decode_attn(workloads.bf16_bits(q), c, s, z, pt, ctx, Hkv, b, num_pages, signs=signs)


@pytest.mark.parametrize("G", [1, 2, 4, 8])
@pytest.mark.parametrize("b", [0, 64, 128])
def test_prefill_matches_the_oracle(orc, G, b):
    # chunks: 1 token, a ragged tile, exactly one tile of 128 / G tokens, several tiles;
    # prior contexts from empty to several blocks of 64
    ctx = [1, 70, 128 // G + 1000, 300]
    qlen = [1, 17, 128 // G, 300]
    got, ref = _case(100 + G + b, ctx, qlen, Hq=2 * G, Hkv=2, b=b)
    assert_close(got, ref, f"prefill G={G} b={b}")


@pytest.mark.parametrize("b", [0, 32, 64])
def test_prefill_head_dim_64(orc, b):
    ctx = [1, 70, 1000 + 32, 300]
    qlen = [1, 17, 32, 300]
    sig = workloads.random_signs(9, 64) if b else None
    got, ref = _case(140 + b, ctx, qlen, Hq=8, Hkv=2, b=b, signs=sig, D=64)
    assert_close(got, ref, f"prefill D=64 b={b}")


def test_prefill_long_context_and_signs(orc):
    ctx = [5000, 40]
    qlen = [200, 40]
    sig = workloads.random_signs(7, 128)
    got, ref = _case(120, ctx, qlen, Hq=16, Hkv=4, b=128, signs=sig)
    assert_close(got, ref, "prefill long context with signs")


@pytest.mark.parametrize("bad", ["context_shorter_than_chunk", "chunk_longer_than_max_q_len"])
def test_prefill_out_of_range_sequence_is_reported_and_left_unwritten(orc, bad):
    # sequence 1 is invalid; sequence 0 must still match the oracle
    ctx, qlen = [300, 64], [32, 64]
    w = workloads.random_case(seed=131, B=2, Hq=8, Hkv=2, D=128, block=128, context_lens=ctx)
    cache, scales, zeros = kvq.alloc_cache(w.num_pages, w.Hkv, w.D)
    kvq.kv_quant_write(w.k_new.cuda(), w.v_new.cuda(), torch.as_tensor(w.slots_new).cuda(), cache, scales,
                       zeros, 128)
    cl = np.array(ctx, np.int32)
    max_q = 64
    if bad == "context_shorter_than_chunk":
        cl[1] = 30
    else:
        max_q = 32   # one tile of 32 query tokens (G = 4); sequence 1's chunk of 64 needs two
    qstart = np.array([0, 32, 96], np.int32)
    q = (torch.randn((96, 8, 128), generator=torch.Generator().manual_seed(3)) / 8).to(torch.bfloat16)
    out = torch.full(q.shape, 7.0, dtype=torch.float32, device="cuda")
    kvq.paged_prefill_attn_int4(q.cuda(), cache, scales, zeros, torch.as_tensor(w.page_table).cuda(),
                                torch.as_tensor(cl).cuda(), torch.as_tensor(qstart).cuda(), max_q, out, 128)
    assert kvq.get_device_error() == 3  # KVQ_ERR_OUT_OF_RANGE
    got = out.cpu().numpy().astype(np.float64)
    assert (got[32:] == 7.0).all(), "the invalid sequence's rows must stay unwritten"
    c, s, z = host_cache(cache, scales, zeros)
    pos = np.arange(268, 300)
    ref = orc_decode(q[:32], c, s, z, w.page_table[np.zeros(32, int)], (pos + 1).astype(np.int32), 2, 128,
                     w.num_pages, None)
    assert_close(got[:32], ref, "prefill valid sequence beside an invalid one")


def test_prefill_bf16_output_is_the_rounded_fp32_output(orc):
    ctx, qlen = [600, 90], [130, 90]
    w = workloads.random_case(seed=150, B=2, Hq=8, Hkv=2, D=128, block=64, context_lens=ctx)
    cache, scales, zeros = kvq.alloc_cache(w.num_pages, w.Hkv, w.D)
    kvq.kv_quant_write(w.k_new.cuda(), w.v_new.cuda(), torch.as_tensor(w.slots_new).cuda(), cache, scales,
                       zeros, 64)
    qstart = torch.tensor([0, 130, 220], dtype=torch.int32).cuda()
    q = (torch.randn((220, 8, 128), generator=torch.Generator().manual_seed(4)) / 8).to(torch.bfloat16).cuda()
    args = (cache, scales, zeros, torch.as_tensor(w.page_table).cuda(), torch.as_tensor(w.context_lens).cuda(),
            qstart, 130)
    o32 = torch.empty(q.shape, dtype=torch.float32, device="cuda")
    o16 = torch.empty(q.shape, dtype=torch.bfloat16, device="cuda")
    kvq.paged_prefill_attn_int4(q, *args, o32, 64)
    kvq.paged_prefill_attn_int4(q, *args, o16, 64)
    assert kvq.get_device_error() == 0
    assert torch.equal(o16, o32.to(torch.bfloat16))


def test_prefill_ignores_garbage_past_the_context(orc):
    """Rows of a sequence's last page past its context may hold anything
    (filled here with NaN scales and offsets and random code bytes); they
    must not reach the output."""
    ctx, qlen = [250, 31, 100], [60, 31, 1]
    w = workloads.random_case(seed=160, B=3, Hq=8, Hkv=2, D=128, block=64, context_lens=ctx)
    cache, scales, zeros = kvq.alloc_cache(w.num_pages, w.Hkv, w.D)
    g = torch.Generator(device="cuda").manual_seed(161)
    cache.copy_(torch.randint(0, 256, cache.shape, generator=g, device="cuda", dtype=torch.int32).to(torch.uint8))
    scales.view(torch.int16).fill_(0x7E00)  # fp16 NaN
    zeros.view(torch.int16).fill_(0x7E00)
    kvq.kv_quant_write(w.k_new.cuda(), w.v_new.cuda(), torch.as_tensor(w.slots_new).cuda(), cache, scales,
                       zeros, 64)
    qstart = np.concatenate([[0], np.cumsum(qlen)]).astype(np.int32)
    q = (torch.randn((int(qstart[-1]), 8, 128), generator=torch.Generator().manual_seed(162)) / 8).to(torch.bfloat16)
    out = torch.empty(q.shape, dtype=torch.float32, device="cuda")
    kvq.paged_prefill_attn_int4(q.cuda(), cache, scales, zeros, torch.as_tensor(w.page_table).cuda(),
                                torch.as_tensor(w.context_lens).cuda(), torch.as_tensor(qstart).cuda(),
                                max(qlen), out, 64)
    assert kvq.get_device_error() == 0
    got = out.cpu().numpy().astype(np.float64)
    assert np.all(np.isfinite(got))
    rows_n = np.repeat(np.arange(3), qlen)
    pos = np.concatenate([np.arange(c - l, c) for c, l in zip(ctx, qlen)])
    c, s, z = host_cache(cache, scales, zeros)
    ref = orc_decode(q, c, s, z, w.page_table[rows_n], (pos + 1).astype(np.int32), 2, 64, w.num_pages, None)
    assert_close(got, ref, "prefill with garbage past the context")


def test_prefill_bad_page_id_is_reported(orc):
    ctx, qlen = [100, 40], [30, 40]
    w = workloads.random_case(seed=170, B=2, Hq=4, Hkv=2, D=64, block=32, context_lens=ctx)
    cache, scales, zeros = kvq.alloc_cache(w.num_pages, w.Hkv, w.D)
    kvq.kv_quant_write(w.k_new.cuda(), w.v_new.cuda(), torch.as_tensor(w.slots_new).cuda(), cache, scales,
                       zeros, 32)
    pt = w.page_table.copy()
    pt[0, 2] = w.num_pages + 5
    qstart = torch.tensor([0, 30, 70], dtype=torch.int32).cuda()
    q = (torch.randn((70, 4, 64), generator=torch.Generator().manual_seed(171)) / 8).to(torch.bfloat16).cuda()
    out = torch.empty(q.shape, dtype=torch.float32, device="cuda")
    kvq.paged_prefill_attn_int4(q, cache, scales, zeros, torch.as_tensor(pt).cuda(),
                                torch.as_tensor(w.context_lens).cuda(), qstart, 40, out, 32)
    assert kvq.get_device_error() == 3  # KVQ_ERR_OUT_OF_RANGE
    assert kvq.get_device_error() == 0
    assert np.all(np.isfinite(out.cpu().numpy()))


def test_prefill_bench_workload_sampled(orc):
    """The call bench.py times (llama3-8b-32k: the last 2048 tokens of the
    32768-token context as one chunk, bf16 queries drawn as there), with 8
    query tokens (all 32 heads) checked one by one against the oracle."""
    import bench
    w = workloads.make("llama3-8b-32k")
    cache, scales, zeros = kvq.alloc_cache(w.num_pages, w.Hkv, w.D)
    kvq.kv_quant_write(w.k_new.cuda(), w.v_new.cuda(), torch.as_tensor(w.slots_new).cuda(), cache, scales,
                       zeros, w.block)
    L = min(bench.PREFILL_CHUNK, int(w.context_lens[0]))
    g = torch.Generator().manual_seed(w.cfg.seed + 7)
    q = (torch.randn((L, w.Hq, w.D), generator=g) / 8).to(torch.bfloat16)
    out = torch.empty(q.shape, dtype=torch.float32, device="cuda")
    kvq.paged_prefill_attn_int4(q.cuda(), cache, scales, zeros, torch.as_tensor(w.page_table).cuda(),
                                torch.as_tensor(w.context_lens).cuda(),
                                torch.tensor([0, L], dtype=torch.int32, device="cuda"), L, out, w.block)
    assert kvq.get_device_error() == 0
    ctx = int(w.context_lens[0])
    rows = np.array([0, 1, 31, 32, 777, 1500, L - 2, L - 1])
    pos = ctx - L + rows
    c, s, z = host_cache(cache, scales, zeros)
    ref = orc_decode(q[rows], c, s, z, np.repeat(w.page_table, len(rows), axis=0), (pos + 1).astype(np.int32),
                     w.Hkv, w.block, w.num_pages, None)
    assert_close(out.cpu().numpy().astype(np.float64)[rows], ref, "prefill, bench workload, sampled rows")
