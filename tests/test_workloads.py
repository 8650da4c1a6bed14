"""The synthetic inputs follow the stated recipe: the shapes of each config,
scattered pages that every sequence owns exclusively, slots that follow the
page table, lognormal(0, 1) token norms, x10 K outlier channels, q ~ N(0,1)/8,
and the context-length distributions of the serving and stress configs."""
import numpy as np
import torch

from bit_kv_cache_20_b200 import workloads


def test_shapes_of_the_named_configs():
    want = {  # batch, Hq, Hkv, D, block, outliers
        "tiny": (1, 4, 2, 64, 32, 2),
        "llama3-8b-32k": (1, 32, 8, 128, 128, 4),
        "serving-b64": (64, 32, 8, 128, 64, 4),
        "llama2-70b-b8": (8, 64, 8, 128, 128, 4),
        "stress-b256": (256, 32, 8, 128, 128, 4),
    }
    for name, (B, Hq, Hkv, D, b, no) in want.items():
        c = workloads.CONFIGS[name]
        assert (c.batch, c.num_q_heads, c.num_kv_heads, c.head_dim, c.block, c.n_outliers) == (B, Hq, Hkv, D, b, no)
    assert workloads.CONFIGS["tiny"].context == 64
    assert workloads.CONFIGS["llama3-8b-32k"].context == 32768
    assert workloads.CONFIGS["llama2-70b-b8"].context == 32768


def _check_pages_and_slots(w):
    used = np.concatenate([w.page_table[n, :(int(c) + 15) // 16] for n, c in enumerate(w.context_lens)])
    # exactly the pages the contexts need, each owned by one sequence, scattered
    assert sorted(used.tolist()) == list(range(w.num_pages))
    if w.num_pages > 16:
        assert not np.array_equal(used, np.arange(w.num_pages))
    # every written position sits at its page-table slot
    pos_new = np.concatenate([np.arange(int(p), int(c)) for p, c in zip(w.prior_lens, w.context_lens)])
    seq_new = np.concatenate([np.full(int(c) - int(p), n) for n, (p, c) in
                              enumerate(zip(w.prior_lens, w.context_lens))])
    want = w.page_table[seq_new, pos_new // 16].astype(np.int64) * 16 + pos_new % 16
    assert np.array_equal(np.asarray(w.slots_new), want)


def test_llama3_8b_32k_inputs_follow_the_recipe():
    w = workloads.make("llama3-8b-32k")
    assert w.k_new.shape == (32768, 8, 128) and w.k_new.dtype == torch.bfloat16
    assert w.q.shape == (1, 32, 128)
    _check_pages_and_slots(w)
    v = w.v_new.float()
    # per-token rms over all heads and channels ~ m = exp(N(0, 1))
    log_m = torch.log(v.pow(2).mean(dim=(1, 2)).sqrt()).numpy()
    assert abs(log_m.mean()) < 0.05 and abs(log_m.std() - 1.0) < 0.05
    # K: 4 outlier channels per head, x10 the others' rms
    k = w.k_new.float()
    rms = k.pow(2).mean(dim=0).sqrt().numpy()  # [Hkv, D]
    for h in range(8):
        out = np.asarray(w.outlier_channels[h])
        assert len(out) == 4
        rest = np.setdiff1d(np.arange(128), out)
        ratio = rms[h, out].mean() / rms[h, rest].mean()
        assert 9.0 < ratio < 11.0, ratio
    # q ~ N(0, 1) / 8
    assert abs(float(w.q.float().std()) - 0.125) < 0.01


def test_serving_and_stress_context_lengths():
    g = torch.Generator().manual_seed(workloads.CONFIGS["serving-b64"].seed)
    ctx, prior = workloads._context_lengths(workloads.CONFIGS["serving-b64"], g)
    assert len(ctx) == 64
    assert prior.min() >= 1024 and prior.max() <= 8192
    assert np.array_equal(ctx, prior + 2048)
    g = torch.Generator().manual_seed(workloads.CONFIGS["stress-b256"].seed)
    ctx, prior = workloads._context_lengths(workloads.CONFIGS["stress-b256"], g)
    assert len(ctx) == 256 and ctx.min() >= 1 and ctx.max() <= 32768 and not prior.any()
    assert 1400 < np.median(ctx) < 3000  # median 2048, lognormal sigma 1


def test_small_configs_are_reproducible_and_consistent():
    a, b = workloads.make("tiny"), workloads.make("tiny")
    assert torch.equal(a.k_new, b.k_new) and torch.equal(a.q, b.q)
    assert np.array_equal(a.page_table, b.page_table)
    _check_pages_and_slots(a)
    r = workloads.random_case(seed=3, B=3, Hq=8, Hkv=2, D=64, block=32, context_lens=[1, 17, 40])
    _check_pages_and_slots(r)
