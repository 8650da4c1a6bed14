"""Parity of kv_quant_write (CUDA, through the C ABI) with the CPU oracle.

Bar: s and z within one fp16 ulp and identical when b = 0; every code equal to
the oracle's quantization of its rotated row under the kernel's (s, z), except
elements whose quotient sits within the fp32-butterfly rounding band of a
half-integer (counted; at most 1e-5 of the elements); placement exact; bytes
of unwritten rows, and guard regions around every buffer, untouched.
"""
import numpy as np
import pytest
import torch

import bit_kv_cache_20_b200 as kvq
from bit_kv_cache_20_b200 import workloads
from helpers import compare_write_rows

pytestmark = pytest.mark.gpu

CANARY = 0xA5
SZ_CANARY = 0x7E00   # fp16 NaN pattern
GUARD = 4096


def guarded(numel, dtype, fill):
    """A tensor with GUARD bytes of known pattern before and after it."""
    el = torch.empty(0, dtype=dtype).element_size()
    g = GUARD // el
    big = torch.empty(numel + 2 * g, dtype=dtype, device="cuda")
    big.view(torch.uint8).fill_(fill & 0xFF) if dtype == torch.uint8 else big.view(torch.int16).fill_(fill)
    return big, big[g:g + numel]


def check_guards(big, numel, dtype, fill):
    el = torch.empty(0, dtype=dtype).element_size()
    g = GUARD // el
    a = big.cpu()
    if dtype == torch.uint8:
        assert torch.all(a[:g] == fill) and torch.all(a[g + numel:] == fill)
    else:
        iv = a.view(torch.int16)
        assert torch.all(iv[:g] == fill) and torch.all(iv[g + numel:] == fill)


class Pool:
    def __init__(self, P, Hkv, D):
        self.P, self.Hkv, self.D = P, Hkv, D
        n_rows = P * Hkv * 2 * 16
        self.cache_big, c = guarded(n_rows * D // 2, torch.uint8, CANARY)
        self.s_big, s = guarded(n_rows, torch.float16, SZ_CANARY)
        self.z_big, z = guarded(n_rows, torch.float16, SZ_CANARY)
        self.cache = c.view(P, Hkv, 2, 16, D // 2)
        self.scales = s.view(P, Hkv, 2, 16)
        self.zeros = z.view(P, Hkv, 2, 16)
        self.n_rows = n_rows

    def host(self):
        torch.cuda.synchronize()
        return (self.cache.cpu().numpy().reshape(-1, self.D // 2),
                self.scales.cpu().view(torch.int16).numpy().view(np.uint16).reshape(-1),
                self.zeros.cpu().view(torch.int16).numpy().view(np.uint16).reshape(-1))

    def check_guards(self):
        check_guards(self.cache_big, self.n_rows * self.D // 2, torch.uint8, CANARY)
        check_guards(self.s_big, self.n_rows, torch.float16, SZ_CANARY)
        check_guards(self.z_big, self.n_rows, torch.float16, SZ_CANARY)


def gpu_write(pool, k, v, slots, b):
    kvq.kv_quant_write(k.cuda(), v.cuda(), torch.as_tensor(slots, dtype=torch.int64).cuda(),
                       pool.cache, pool.scales, pool.zeros, b)
    assert kvq.get_device_error() == 0


def check_tokens(orc, pool, k, v, slots, b, tokens=None, written_rows=None, signs=None):
    """Compare the rows of `tokens` (default: all) with the oracle."""
    cache, scales, zeros = pool.host()
    kb = workloads.bf16_bits(k)
    vb = workloads.bf16_bits(v)
    T, Hkv, D = kb.shape
    tokens = np.arange(T) if tokens is None else np.asarray(tokens)
    tokens = tokens[np.asarray(slots)[tokens] >= 0]
    rows, ys, xs = [], [], []
    for t in tokens:
        page, off = divmod(int(slots[t]), 16)
        for h in range(Hkv):
            for kv, src in enumerate((kb, vb)):
                rows.append(((page * Hkv + h) * 2 + kv) * 16 + off)
                ys.append(orc.rotate_row(src[t, h], b, signs=signs))
                xs.append(src[t, h].view(np.int16).astype(np.int32) << 16)
    rows = np.asarray(rows, np.int64)
    x_rows = np.asarray(xs, np.int32).view(np.float32).astype(np.float64) if xs else np.zeros((0, D))
    stats = compare_write_rows(orc, np.asarray(ys, np.float32).reshape(-1, D), x_rows.reshape(-1, D), b,
                               cache[rows], scales[rows], zeros[rows], D)
    assert stats["code_mismatch_near_boundary"] <= max(1e-5 * stats["elements"], 0), stats
    if written_rows is not None:
        mask = np.zeros(scales.size, bool)
        mask[written_rows] = True
        assert np.all(cache[~mask] == CANARY)
        assert np.all(scales[~mask] == SZ_CANARY) and np.all(zeros[~mask] == SZ_CANARY)
    pool.check_guards()
    return stats


def all_rows(slots, Hkv):
    out = []
    for s in slots:
        if s < 0:
            continue
        page, off = divmod(int(s), 16)
        for h in range(Hkv):
            for kv in range(2):
                out.append(((page * Hkv + h) * 2 + kv) * 16 + off)
    return np.asarray(out, np.int64)


def test_write_tiny_config(orc):
    w = workloads.make("tiny")
    pool = Pool(w.num_pages, w.Hkv, w.D)
    gpu_write(pool, w.k_new, w.v_new, w.slots_new, w.block)
    check_tokens(orc, pool, w.k_new, w.v_new, w.slots_new, w.block,
                 written_rows=all_rows(w.slots_new, w.Hkv))


@pytest.mark.parametrize("D,b", [(64, 0), (64, 32), (64, 64), (128, 0), (128, 32), (128, 64), (128, 128)])
@pytest.mark.parametrize("Hkv,ctx", [(1, [1]), (2, [31, 33]), (8, [100, 17, 5, 64])])
def test_write_random_shapes(orc, D, b, Hkv, ctx):
    w = workloads.random_case(seed=D + b + Hkv, B=len(ctx), Hq=Hkv, Hkv=Hkv, D=D, block=b,
                              context_lens=ctx, extra_pages=2, skip_fraction=0.15)
    pool = Pool(w.num_pages, Hkv, D)
    gpu_write(pool, w.k_new, w.v_new, w.slots_new, b)
    check_tokens(orc, pool, w.k_new, w.v_new, w.slots_new, b, written_rows=all_rows(w.slots_new, Hkv))


def test_write_many_tiles_with_ragged_tail(orc):
    # several warp tiles per head and a partial last tile, all blocks
    for b in (0, 32, 64, 128):
        w = workloads.random_case(seed=70 + b, B=3, Hq=8, Hkv=4, D=128, block=b,
                                  context_lens=[300, 129, 577], extra_pages=1)
        pool = Pool(w.num_pages, 4, 128)
        gpu_write(pool, w.k_new, w.v_new, w.slots_new, b)
        check_tokens(orc, pool, w.k_new, w.v_new, w.slots_new, b,
                     written_rows=all_rows(w.slots_new, 4))


def test_write_full_size_llama3_8b_32k_sampled(orc):
    # the benchmark's write launch: 32768 tokens x 8 kv heads, block 128
    w = workloads.make("llama3-8b-32k")
    pool = Pool(w.num_pages, w.Hkv, w.D)
    gpu_write(pool, w.k_new, w.v_new, w.slots_new, w.block)
    rng = np.random.default_rng(0)
    sample = np.sort(rng.choice(w.tokens_written, 768, replace=False))
    stats = check_tokens(orc, pool, w.k_new, w.v_new, w.slots_new, w.block, tokens=sample)
    print("llama3-8b-32k write sample:", stats)
    # every slot of the pool was written (the pool holds exactly the context)
    _, scales, zeros = pool.host()
    assert not np.any(scales == SZ_CANARY) and not np.any(zeros == SZ_CANARY)


def test_write_degenerate_rows(orc):
    T, Hkv, D = 6, 1, 128
    x = torch.zeros((T, Hkv, D))
    x[1] = 0.3                                               # constant, off the fp16 grid
    x[2] = 0.5                                               # constant, on the grid
    x[3, 0] = -1.0 + (torch.arange(D) % 16) / 8.0            # on the INT4 grid
    x[4] = torch.linspace(-1e-6, 1e-6, D)                    # fp16 subnormal step
    x[5] = torch.linspace(-3000.0, 3000.0, D)                # large magnitude
    k = x.to(torch.bfloat16)
    v = (-x).to(torch.bfloat16)
    slots = np.arange(T, dtype=np.int64) * 3                 # scattered offsets in 2 pages
    for b in (0, 32, 64, 128):
        pool = Pool(2, Hkv, D)
        gpu_write(pool, k, v, slots, b)
        check_tokens(orc, pool, k, v, slots, b, written_rows=all_rows(slots, Hkv))


def test_write_zero_tokens_is_a_no_op():
    pool = Pool(1, 1, 64)
    e = torch.empty((0, 1, 64), dtype=torch.bfloat16, device="cuda")
    kvq.kv_quant_write(e, e, torch.empty(0, dtype=torch.int64, device="cuda"), pool.cache,
                       pool.scales, pool.zeros, 32)
    cache, scales, _ = pool.host()
    assert np.all(cache == CANARY) and np.all(scales == SZ_CANARY)


def test_write_out_of_range_slot_is_skipped_and_reported(orc):
    w = workloads.random_case(seed=5, B=1, Hq=2, Hkv=2, D=64, block=32, context_lens=[20])
    slots = w.slots_new.copy()
    slots[3] = w.num_pages * 16          # one past the pool
    slots[7] = -5                        # negative but not the skip marker
    pool = Pool(w.num_pages, 2, 64)
    kvq.kv_quant_write(w.k_new.cuda(), w.v_new.cuda(), torch.as_tensor(slots).cuda(), pool.cache,
                       pool.scales, pool.zeros, 32)
    assert kvq.get_device_error() == 3   # KVQ_ERR_OUT_OF_RANGE
    assert kvq.get_device_error() == 0   # read-and-clear
    good = slots.copy()
    good[[3, 7]] = -1
    check_tokens(orc, pool, w.k_new, w.v_new, good, 32, written_rows=all_rows(good, 2))


def test_write_is_deterministic():
    w = workloads.random_case(seed=11, B=2, Hq=8, Hkv=8, D=128, block=128, context_lens=[200, 90])
    outs = []
    for _ in range(2):
        pool = Pool(w.num_pages, 8, 128)
        gpu_write(pool, w.k_new, w.v_new, w.slots_new, 128)
        outs.append(pool.host())
    for a, b in zip(*outs):
        assert np.array_equal(a, b)


def test_write_prior_then_append(orc):
    # serving shape cut to 6 sequences: prior contexts written first, then
    # 2048 appended tokens per sequence continue the same pages
    w = workloads.make("serving-b64", batch=6)
    pool = Pool(w.num_pages, w.Hkv, w.D)
    gpu_write(pool, w.k_prior, w.v_prior, w.slots_prior, w.block)
    gpu_write(pool, w.k_new, w.v_new, w.slots_new, w.block)
    rng = np.random.default_rng(1)
    check_tokens(orc, pool, w.k_prior, w.v_prior, w.slots_prior, w.block,
                 tokens=rng.choice(w.k_prior.shape[0], 200, replace=False))
    check_tokens(orc, pool, w.k_new, w.v_new, w.slots_new, w.block,
                 tokens=rng.choice(w.tokens_written, 200, replace=False))


@pytest.mark.parametrize("D,b", [(64, 32), (64, 64), (128, 64), (128, 128)])
def test_write_randomized_hadamard_signs(orc, D, b):
    """R = H_b diag(sigma) / sqrt(b) with seeded random signs: the tensor-core
    operand carries the signs; codes, s and z against the oracle's signed
    rotation."""
    w = workloads.random_case(seed=81 + D + b, B=2, Hq=4, Hkv=2, D=D, block=b, context_lens=[300, 77])
    sig = workloads.random_signs(82 + b, D)
    pool = Pool(w.num_pages, w.Hkv, D)
    kvq.kv_quant_write(w.k_new.cuda(), w.v_new.cuda(), torch.as_tensor(w.slots_new).cuda(),
                       pool.cache, pool.scales, pool.zeros, b, hadamard_signs=sig)
    assert kvq.get_device_error() == 0
    check_tokens(orc, pool, w.k_new, w.v_new, w.slots_new, b, signs=sig)
    # the signs matter: the unsigned rotation stores other codes
    plain = Pool(w.num_pages, w.Hkv, D)
    kvq.kv_quant_write(w.k_new.cuda(), w.v_new.cuda(), torch.as_tensor(w.slots_new).cuda(),
                       plain.cache, plain.scales, plain.zeros, b)
    assert not np.array_equal(pool.host()[0], plain.host()[0])
