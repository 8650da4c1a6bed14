"""Seeded synthetic workloads for the rotated-INT4 paged KV cache.

This module only draws inputs; it holds none of the method's arithmetic, and
both the CUDA path and the CPU oracle consume what it returns.

The shapes follow the serving workloads the pages speak of (SAW-INT4 Abstract:
latency-sensitive small batches and high-concurrency serving; the news
article's Llama-2-70B 32K-token table; OScaR/OSCAR's reasoning traces of up to
32K tokens). The value distributions follow OScaR's Token Norm Imbalance
(forum summary, section "Root Cause: Token Norm Imbalance"): per-token norms
vary widely, drawn here as lognormal(0, 1); K additionally carries a few x10
outlier channels per head.

Recipe (fixed order of draws from one torch CPU generator seeded per config):
  1. context lengths (only for configs whose lengths are random);
  2. per kv head, the K outlier channels: randperm(D)[:n_outliers];
  3. the page pool permutation: randperm(total_pages);
  4. q ~ N(0,1)/8, shape [B, Hq, D];
  5. K and V rows of the already-cached ("prior") tokens, then of the new
     tokens, each in chunks: m = exp(N(0,1)) per token, x = N(0,1) * m
     (K then V per chunk); K's outlier channels x10; all cast to bf16.
The pool holds exactly the pages the contexts need; sequence n takes the next
ceil(ctx_n/16) entries of the permutation, so pages are scattered.
"""
from __future__ import annotations

import dataclasses
import math
from typing import List, Optional

import numpy as np
import torch

PAGE = 16


@dataclasses.dataclass(frozen=True)
class Config:
    name: str
    batch: int
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    block: int
    seed: int
    n_outliers: int
    context: Optional[int] = None         # fixed context length for every sequence
    prior_range: Optional[tuple] = None   # (lo, hi) uniform prior length; new tokens appended
    new_tokens: int = 0                   # tokens appended after the prior part
    lognormal_median: Optional[int] = None  # lognormal(sigma=1) context lengths
    context_cap: int = 32768
    description: str = ""


CONFIGS = {
    "tiny": Config("tiny", 1, 4, 2, 64, 32, 0, 2, context=64,
                   description="1 seq, 2 KV / 4 Q heads, head_dim 64, 64 tokens, block 32"),
    "llama3-8b-32k": Config("llama3-8b-32k", 1, 32, 8, 128, 128, 1, 4, context=32768,
                            description="Llama-3-8B-shaped layer, batch 1, context 32768, block 128"),
    "serving-b64": Config("serving-b64", 64, 32, 8, 128, 64, 2, 4, prior_range=(1024, 8192),
                          new_tokens=2048,
                          description="batch 64, prior contexts U{1K..8K}, 2048 new tokens each, block 64"),
    "llama2-70b-b8": Config("llama2-70b-b8", 8, 64, 8, 128, 128, 3, 4, context=32768,
                            description="Llama-2-70B-shaped layer (GQA 8), batch 8, context 32768, block 128"),
    "stress-b256": Config("stress-b256", 256, 32, 8, 128, 128, 4, 4, lognormal_median=2048,
                          description="batch 256, lognormal contexts (median 2K, cap 32K), block swept"),
}


@dataclasses.dataclass
class Workload:
    cfg: Config
    block: int
    context_lens: np.ndarray   # int32 [B]
    prior_lens: np.ndarray     # int32 [B]  tokens cached before the write under test
    page_table: np.ndarray     # int32 [B, max_pages]
    num_pages: int
    q: torch.Tensor            # bf16 [B, Hq, D]
    k_prior: torch.Tensor      # bf16 [sum(prior), Hkv, D]
    v_prior: torch.Tensor
    slots_prior: np.ndarray    # int64 [sum(prior)]
    k_new: torch.Tensor        # bf16 [sum(ctx - prior), Hkv, D]
    v_new: torch.Tensor
    slots_new: np.ndarray      # int64 [sum(ctx - prior)]
    outlier_channels: List[np.ndarray]

    @property
    def max_pages(self) -> int:
        return int(self.page_table.shape[1])

    @property
    def B(self) -> int:
        return self.cfg.batch

    @property
    def Hq(self) -> int:
        return self.cfg.num_q_heads

    @property
    def Hkv(self) -> int:
        return self.cfg.num_kv_heads

    @property
    def D(self) -> int:
        return self.cfg.head_dim

    @property
    def tokens_written(self) -> int:
        return int(self.k_new.shape[0])

    @property
    def tokens_cached(self) -> int:
        return int(self.context_lens.sum())


def _context_lengths(cfg: Config, g: torch.Generator):
    B = cfg.batch
    if cfg.context is not None:
        ctx = np.full(B, cfg.context, np.int64)
        prior = np.zeros(B, np.int64)
    elif cfg.prior_range is not None:
        lo, hi = cfg.prior_range
        prior = torch.randint(lo, hi + 1, (B,), generator=g).numpy().astype(np.int64)
        ctx = prior + cfg.new_tokens
    else:
        z = torch.randn(B, generator=g, dtype=torch.float64).numpy()
        ctx = np.clip(np.rint(cfg.lognormal_median * np.exp(z)), 1, cfg.context_cap).astype(np.int64)
        prior = np.zeros(B, np.int64)
    return ctx.astype(np.int32), prior.astype(np.int32)


def _draw_rows(g: torch.Generator, n: int, Hkv: int, D: int, outliers, chunk: int = 1 << 16):
    k = torch.empty((n, Hkv, D), dtype=torch.bfloat16)
    v = torch.empty((n, Hkv, D), dtype=torch.bfloat16)
    for s in range(0, n, chunk):
        c = min(chunk, n - s)
        mk = torch.exp(torch.randn(c, generator=g))
        kc = torch.randn((c, Hkv, D), generator=g) * mk[:, None, None]
        for h in range(Hkv):
            kc[:, h, torch.as_tensor(outliers[h])] *= 10.0
        mv = torch.exp(torch.randn(c, generator=g))
        vc = torch.randn((c, Hkv, D), generator=g) * mv[:, None, None]
        k[s:s + c] = kc.to(torch.bfloat16)
        v[s:s + c] = vc.to(torch.bfloat16)
    return k, v


def make(name: str, block: Optional[int] = None, batch: Optional[int] = None,
         context: Optional[int] = None, seed: Optional[int] = None) -> Workload:
    """Draw the named workload. `block`, `batch`, `context` and `seed`
    override the config's values (used by parity tests to cut sizes)."""
    cfg = CONFIGS[name]
    if batch is not None or context is not None or seed is not None:
        cfg = dataclasses.replace(
            cfg,
            batch=batch if batch is not None else cfg.batch,
            context=context if context is not None else cfg.context,
            seed=seed if seed is not None else cfg.seed,
        )
    b = cfg.block if block is None else block
    g = torch.Generator().manual_seed(cfg.seed)
    ctx, prior = _context_lengths(cfg, g)
    B, Hkv, D = cfg.batch, cfg.num_kv_heads, cfg.head_dim
    outliers = [torch.randperm(D, generator=g)[: cfg.n_outliers].numpy() for _ in range(Hkv)]
    pages_per_seq = [(int(c) + PAGE - 1) // PAGE for c in ctx]
    total_pages = int(sum(pages_per_seq))
    perm = torch.randperm(max(total_pages, 1), generator=g).numpy().astype(np.int32)
    max_pages = max(1, max(pages_per_seq) if pages_per_seq else 1)
    page_table = np.zeros((B, max_pages), np.int32)
    off = 0
    for n, npg in enumerate(pages_per_seq):
        page_table[n, :npg] = perm[off: off + npg]
        off += npg
    q = (torch.randn((B, cfg.num_q_heads, D), generator=g) / 8.0).to(torch.bfloat16)

    def slots(lo_pos, hi_pos):
        out = []
        for n in range(B):
            pos = np.arange(lo_pos[n], hi_pos[n], dtype=np.int64)
            out.append(page_table[n, pos // PAGE].astype(np.int64) * PAGE + pos % PAGE)
        return np.concatenate(out) if out else np.zeros(0, np.int64)

    zeros_b = np.zeros(B, np.int64)
    slots_prior = slots(zeros_b, prior)
    slots_new = slots(prior, ctx)
    k_prior, v_prior = _draw_rows(g, int(prior.sum()), Hkv, D, outliers)
    k_new, v_new = _draw_rows(g, int((ctx - prior).sum()), Hkv, D, outliers)
    return Workload(cfg, b, ctx, prior, page_table, max(total_pages, 1), q, k_prior, v_prior,
                    slots_prior, k_new, v_new, slots_new, outliers)


def random_case(seed: int, B: int, Hq: int, Hkv: int, D: int, block: int,
                context_lens, n_outliers: int = 2, extra_pages: int = 0,
                skip_fraction: float = 0.0) -> Workload:
    """A small workload with explicit shapes (parity tests): arbitrary context
    lengths, a pool with `extra_pages` unused pages, and a fraction of new
    tokens whose slot is -1 (skipped by the write)."""
    cfg = Config(f"random-{seed}", B, Hq, Hkv, D, block, seed, n_outliers, context=0)
    g = torch.Generator().manual_seed(seed)
    ctx = np.asarray(context_lens, np.int32)
    prior = np.zeros(B, np.int32)
    outliers = [torch.randperm(D, generator=g)[:n_outliers].numpy() for _ in range(Hkv)]
    pages_per_seq = [(int(c) + PAGE - 1) // PAGE for c in ctx]
    total_pages = int(sum(pages_per_seq)) + extra_pages
    perm = torch.randperm(max(total_pages, 1), generator=g).numpy().astype(np.int32)
    max_pages = max(1, max(pages_per_seq) if pages_per_seq else 1)
    page_table = np.zeros((B, max_pages), np.int32)
    off = 0
    for n, npg in enumerate(pages_per_seq):
        page_table[n, :npg] = perm[off: off + npg]
        off += npg
    q = (torch.randn((B, Hq, D), generator=g) / 8.0).to(torch.bfloat16)
    out = []
    for n in range(B):
        pos = np.arange(0, ctx[n], dtype=np.int64)
        out.append(page_table[n, pos // PAGE].astype(np.int64) * PAGE + pos % PAGE)
    slots_new = np.concatenate(out) if out else np.zeros(0, np.int64)
    if skip_fraction > 0 and slots_new.size:
        drop = torch.rand(slots_new.size, generator=g).numpy() < skip_fraction
        slots_new = np.where(drop, -1, slots_new)
    k_new, v_new = _draw_rows(g, int(ctx.sum()), Hkv, D, outliers)
    empty = torch.empty((0, Hkv, D), dtype=torch.bfloat16)
    return Workload(cfg, block, ctx, prior, page_table, max(total_pages, 1), q, empty, empty,
                    np.zeros(0, np.int64), k_new, v_new, slots_new, outliers)


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    """The uint16 bit patterns of a bf16 tensor (for the oracle)."""
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def page_count(context_lens) -> int:
    return int(sum(math.ceil(int(c) / PAGE) for c in context_lens))


def random_signs(seed: int, D: int) -> np.ndarray:
    """A seeded randomized-Hadamard sign vector: D booleans, True = negate
    that channel before the transform."""
    g = torch.Generator().manual_seed(seed)
    return (torch.rand(D, generator=g) < 0.5).numpy()


def oscar_rows(w: Workload):
    """The rows of a workload arranged for the OScaR layout, where a page is
    quantized whole: each sequence's full pages as write groups of 16 rows
    (k, v bf16 [16 P, Hkv, D], page ids int32 [P] from its page table), and
    its last ctx % 16 rows as the bf16 unfinished page k_tail, v_tail
    [B, Hkv, 16, D] (rows past the tail zero)."""
    B, Hkv, D = w.B, w.Hkv, w.D
    ks, vs, ids = [], [], []
    k_tail = torch.zeros((B, Hkv, PAGE, D), dtype=torch.bfloat16)
    v_tail = torch.zeros((B, Hkv, PAGE, D), dtype=torch.bfloat16)
    op = on = 0
    for n in range(B):
        npr, ctx = int(w.prior_lens[n]), int(w.context_lens[n])
        k = torch.cat([w.k_prior[op:op + npr], w.k_new[on:on + ctx - npr]])
        v = torch.cat([w.v_prior[op:op + npr], w.v_new[on:on + ctx - npr]])
        op += npr
        on += ctx - npr
        full = ctx // PAGE
        ks.append(k[:full * PAGE])
        vs.append(v[:full * PAGE])
        ids.append(w.page_table[n, :full].astype(np.int32))
        tail = ctx - full * PAGE
        k_tail[n, :, :tail] = k[full * PAGE:].transpose(0, 1)
        v_tail[n, :, :tail] = v[full * PAGE:].transpose(0, 1)
    return (torch.cat(ks), torch.cat(vs), np.concatenate(ids) if ids else np.zeros(0, np.int32),
            k_tail, v_tail)
