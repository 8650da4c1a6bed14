"""Parity of the OScaR variant (kv_quant_write_oscar, paged_decode_attn_oscar,
CUDA through the C ABI) with the CPU oracle.

The variant (OScaR forum summary, "The OScaR Framework": V^ = Quant(S (R V));
OScaR abstract: per-channel K quantization, Token Norm Imbalance, INT2): K
rows rotated, scaled to unit norm per token (the fp16 norm stored), quantized
per channel over each 16-token page; V rotated, quantized per token; the
unfinished last page of a sequence kept in bf16.

Bar, write: b = 0 - every byte of the codes, norms and (s, z) identical to the
oracle's. b > 0 (the kernel rotates with an fp32 butterfly, the oracle in
fp64): token norms and every (s, z) within one fp16 ulp; every code equal to
the oracle's decision on its own rotated values under the kernel's (n, s, z),
except within the butterfly's rounding band of a half-integer, where the two
differ by one. Placement exact; pages and bytes outside the written ones, and
guards, untouched.
Bar, decode: max |GPU - oracle| <= 2e-3 over the same cache (the kernel's
error is fp32 accumulation and the fp16 hi + lo splits of q~ * s and p * s,
about 2^-20 relative per term; the outputs are O(1)).
"""
import math

import numpy as np
import pytest
import torch

import bit_kv_cache_20_b200 as kvq
from bit_kv_cache_20_b200 import workloads
from helpers import f16_bits_to_float, f16_ordinal

pytestmark = pytest.mark.gpu

TOL = 2e-3
CANARY = 0x5A
H_CANARY = 0x7E00  # fp16 NaN pattern


def gpu_pool(P, Hkv, D):
    cache, kmeta, tmeta = kvq.alloc_oscar_cache(P, Hkv, D)
    cache.fill_(CANARY)
    kmeta.view(torch.int16).fill_(H_CANARY)
    tmeta.view(torch.int16).fill_(H_CANARY)
    return cache, kmeta, tmeta


def host(pool):
    torch.cuda.synchronize()
    c, km, tm = pool
    return (c.cpu().numpy(), km.cpu().view(torch.int16).numpy().view(np.uint16),
            tm.cpu().view(torch.int16).numpy().view(np.uint16))


def write_both(orc, w, b, pool_pages=None):
    k, v, ids, k_tail, v_tail = workloads.oscar_rows(w)
    P = w.num_pages if pool_pages is None else pool_pages
    pool = gpu_pool(P, w.Hkv, w.D)
    if ids.size:
        kvq.kv_quant_write_oscar(k.cuda(), v.cuda(), torch.as_tensor(ids).cuda(), *pool, b)
    assert kvq.get_device_error() == 0
    kb, vb = workloads.bf16_bits(k), workloads.bf16_bits(v)
    ora = orc.oscar_write(kb, vb, ids, P, b) if ids.size else orc.oscar_alloc(P, w.Hkv, w.D)
    return pool, ora, (k, v, ids, k_tail, v_tail)


def unpack2(codes, D):
    b = np.asarray(codes, np.uint8)
    return np.stack([(b >> (2 * i)) & 3 for i in range(4)], axis=-1).reshape(b.shape[:-1] + (D,))


def butterfly_bound(x_rows, b):
    """Bound on |fp32 butterfly - exact rotation| per row (log2(b) + 2
    roundings of at most 2^-24 times the block's sum of |x|, / sqrt(b))."""
    n, D = x_rows.shape
    blocks = np.abs(x_rows).reshape(n, D // b, b).sum(axis=2).max(axis=1)
    return (math.log2(b) + 2) * 2.0 ** -24 * blocks / math.sqrt(b)


def check_codes(orc, vals, s_bits, z_bits, gpu_codes, win):
    """gpu_codes against the oracle's decision on vals under (s, z); a
    mismatch must sit within win (in code units) of a half-integer and be off
    by one. Returns the number of such mismatches."""
    ref = orc.oscar_codes_given(vals, s_bits, z_bits)
    bad = np.nonzero(ref != gpu_codes)[0]
    if bad.size:
        s = np.float32(f16_bits_to_float(s_bits))
        z = np.float32(f16_bits_to_float(z_bits))
        qt = (vals[bad] - z).astype(np.float64) * np.float64(np.float32(1.0) / s)
        dist = np.abs(qt - (np.floor(qt) + 0.5))
        assert np.all(dist <= win), (bad, qt, win)
        assert np.all(np.abs(ref[bad].astype(int) - gpu_codes[bad].astype(int)) == 1)
    return int(bad.size)


def compare_oscar_write(orc, gpu, ora, k, v, ids, b):
    gc, gk, gt = gpu
    oc, ok, ot = ora
    P, Hkv, _, _, Dq = gc.shape
    D = 4 * Dq
    written = np.zeros(P, bool)
    written[ids] = True
    # pages that no group names stay as they were
    assert np.all(gc[~written] == CANARY)
    assert np.all(gk[~written] == H_CANARY) and np.all(gt[~written] == H_CANARY)
    if b == 0:
        assert np.array_equal(gc[written], oc[written])
        assert np.array_equal(f16_ordinal(gk[written]), f16_ordinal(ok[written]))
        assert np.array_equal(f16_ordinal(gt[written]), f16_ordinal(ot[written]))
        return {"mismatch": 0}
    kb, vb = workloads.bf16_bits(k), workloads.bf16_bits(v)
    mism = 0
    for g, page in enumerate(ids):
        for h in range(Hkv):
            xk = kb[16 * g:16 * g + 16, h]
            xv = vb[16 * g:16 * g + 16, h]
            yk = np.stack([orc.rotate_row(xk[t], b) for t in range(16)])
            yv = np.stack([orc.rotate_row(xv[t], b) for t in range(16)])
            bk = butterfly_bound(f16_free(xk), b)
            bv = butterfly_bound(f16_free(xv), b)
            # K: token norms within one ulp; u from the oracle's rotation and the kernel's norm
            kn_g, kn_o = gt[page, h, 0], ot[page, h, 0]
            assert np.abs(f16_ordinal(kn_g) - f16_ordinal(kn_o)).max() <= 1, (g, h)
            n = f16_bits_to_float(kn_g)
            with np.errstate(divide="ignore", invalid="ignore"):
                u = np.where(n[:, None] > 0, (yk.astype(np.float64) / n[:, None]), 0.0).astype(np.float32)
                err_u = np.where(n > 0, bk / n, 0.0) + 3 * 2.0 ** -24
            _, ks_o, kz_o = orc.oscar_quant_channels(u)
            ks_g, kz_g = gk[page, h, 0], gk[page, h, 1]
            assert np.abs(f16_ordinal(ks_g) - f16_ordinal(ks_o)).max() <= 1, (g, h)
            assert np.abs(f16_ordinal(kz_g) - f16_ordinal(kz_o)).max() <= 1, (g, h)
            kcodes = unpack2(gc[page, h, 0], D)
            for c in range(D):
                s = f16_bits_to_float(ks_g[c])
                win = (err_u.max() / s if s > 0 else 0.0) + 2.0 ** -19
                mism += check_codes(orc, u[:, c].copy(), int(ks_g[c]), int(kz_g[c]), kcodes[:, c], win)
            # V: per token, the INT4 path's rule with top 3
            vs_g, vz_g = gt[page, h, 1], gt[page, h, 2]
            assert np.abs(f16_ordinal(vs_g) - f16_ordinal(ot[page, h, 1])).max() <= 1, (g, h)
            assert np.abs(f16_ordinal(vz_g) - f16_ordinal(ot[page, h, 2])).max() <= 1, (g, h)
            vcodes = unpack2(gc[page, h, 1], D)
            for t in range(16):
                s = f16_bits_to_float(vs_g[t])
                win = ((bv[t] + 2.0 ** -24 * np.abs(yv[t]).max()) / s if s > 0 else 0.0) + 2.0 ** -19
                mism += check_codes(orc, yv[t], int(vs_g[t]), int(vz_g[t]), vcodes[t], win)
    total = 2 * ids.size * Hkv * 16 * D
    assert mism <= max(8, 1e-4 * total), (mism, total)
    return {"mismatch": mism, "elements": total}


def f16_free(x_bits):
    """bf16 bits -> fp64 values."""
    return (np.asarray(x_bits, np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def gpu_decode(w, pool, rows, b, out_dtype=torch.float32, softmax_scale=0.0):
    _, _, ids, k_tail, v_tail = rows
    full_pages = max(1, int(max((int(c) // 16 for c in w.context_lens), default=1)))
    pt = torch.as_tensor(np.ascontiguousarray(w.page_table[:, :full_pages])).cuda()
    cl = torch.as_tensor(w.context_lens).cuda()
    out = torch.full((w.B, w.Hq, w.D), 7.0, dtype=out_dtype, device="cuda")
    nb = kvq.oscar_workspace_size(w.B, w.Hq, w.Hkv, w.D, w.num_pages if pool is None else pool[0].shape[0],
                                  pt.shape[1], b)
    ws = torch.full((nb,), 0xEE, dtype=torch.uint8, device="cuda")  # contents need not be zero
    kvq.paged_decode_attn_oscar(w.q.cuda(), *pool, pt, cl, k_tail.cuda(), v_tail.cuda(), out, b, ws,
                                softmax_scale=softmax_scale)
    torch.cuda.synchronize()
    assert kvq.get_device_error() == 0
    return out.float().cpu().numpy().astype(np.float64), pt.cpu().numpy()


def oracle_decode(orc, w, pool_host, rows, pt, b, softmax_scale=0.0, pairs=None):
    _, _, _, k_tail, v_tail = rows
    qb = workloads.bf16_bits(w.q)
    ktb, vtb = workloads.bf16_bits(k_tail), workloads.bf16_bits(v_tail)
    if pairs is None:
        return orc.oscar_decode_attn(qb, *pool_host, pt, w.context_lens, ktb, vtb, b, softmax_scale)
    return {(n, hq): orc.oscar_decode_one(qb, *pool_host, pt, w.context_lens, ktb, vtb, n, hq, b,
                                          softmax_scale) for n, hq in pairs}


def assert_close(got, ref, label):
    err = float(np.abs(got - ref).max()) if ref.size else 0.0
    print(f"{label}: max|err| = {err:.3e} (max|ref| = {float(np.abs(ref).max(initial=0)):.3e})")
    assert err <= TOL, (label, err)


# ---------------------------------------------------------------------------
# write
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("b", [0, 32, 64, 128])
def test_oscar_write_matches_oracle(orc, b):
    # 3 sequences, 13 full pages in all, a pool with unused pages
    w = workloads.random_case(100 + b, 3, 8, 4, 128, b, [40, 133, 31], n_outliers=3, extra_pages=5)
    pool, ora, rows = write_both(orc, w, b)
    k, v, ids, _, _ = rows
    res = compare_oscar_write(orc, host(pool), ora, k, v, ids, b)
    print("write", b, res)


def test_oscar_write_edge_rows(orc):
    """Zero tokens (norm 0, u = 0), a constant token (V s = 0),
    huge and tiny norms side by side, outlier channels: bit-exact at b = 0."""
    g = torch.Generator().manual_seed(7)
    k = torch.randn((32, 2, 128), generator=g)
    v = torch.randn((32, 2, 128), generator=g)
    k[0] = 0.0
    k[1, 0] = 3.0
    v[2] = 0.25
    k[3] *= 1e4
    k[4] *= 1e-4
    k[5:16, 1, 7] *= 100.0
    k, v = k.to(torch.bfloat16), v.to(torch.bfloat16)
    ids = np.array([3, 1], np.int32)
    pool = gpu_pool(5, 2, 128)
    kvq.kv_quant_write_oscar(k.cuda(), v.cuda(), torch.as_tensor(ids).cuda(), *pool, 0)
    assert kvq.get_device_error() == 0
    ora = orc.oscar_write(workloads.bf16_bits(k), workloads.bf16_bits(v), ids, 5, 0)
    compare_oscar_write(orc, host(pool), ora, k, v, ids, 0)
    gc, gk, gt = host(pool)
    assert gt[3, 0, 0, 0] == 0                                  # the zero token: norm 0,
    K, _ = orc.oscar_dequant_page(gc, gk, gt, 3, 0)
    assert np.all(K[0] == 0.0)                                  # so its dequantized row is 0


def test_oscar_write_bad_page_id_skips_group(orc):
    g = torch.Generator().manual_seed(9)
    k = torch.randn((48, 2, 128), generator=g).to(torch.bfloat16)
    v = torch.randn((48, 2, 128), generator=g).to(torch.bfloat16)
    ids = np.array([0, 9, 2], np.int32)  # 9 is outside a 4-page pool
    pool = gpu_pool(4, 2, 128)
    kvq.kv_quant_write_oscar(k.cuda(), v.cuda(), torch.as_tensor(ids).cuda(), *pool, 64)
    torch.cuda.synchronize()
    assert kvq.get_device_error() == 3  # KVQ_ERR_OUT_OF_RANGE
    assert kvq.get_device_error() == 0
    keep = np.array([0, 2], np.int32)
    rows = torch.cat([k[0:16], k[32:48]]), torch.cat([v[0:16], v[32:48]])
    ora = orc.oscar_write(workloads.bf16_bits(rows[0]), workloads.bf16_bits(rows[1]), keep, 4, 64)
    compare_oscar_write(orc, host(pool), ora, rows[0], rows[1], keep, 64)


# ---------------------------------------------------------------------------
# decode
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("b,G", [(0, 1), (128, 1), (64, 2), (128, 4), (32, 4), (0, 4)])
def test_oscar_decode_matches_oracle(orc, b, G):
    Hkv = 4
    # lengths: tail only, exact pages, tails of 1 and 15, an empty sequence, several splits
    ctx = [7, 64, 161, 0, 1423, 303]
    w = workloads.random_case(300 + b + G, len(ctx), G * Hkv, Hkv, 128, b, ctx, n_outliers=2, extra_pages=3)
    pool, _, rows = write_both(orc, w, b)
    got, pt = gpu_decode(w, pool, rows, b)
    ref = oracle_decode(orc, w, host(pool), rows, pt, b)
    assert_close(got, ref, f"oscar decode b={b} G={G}")
    assert np.all(got[3] == 0.0)  # the empty sequence


def test_oscar_decode_bf16_out_and_scale(orc):
    ctx = [500, 37]
    w = workloads.random_case(41, 2, 8, 4, 128, 128, ctx)
    pool, _, rows = write_both(orc, w, 128)
    got, pt = gpu_decode(w, pool, rows, 128, out_dtype=torch.bfloat16, softmax_scale=0.2)
    ref = oracle_decode(orc, w, host(pool), rows, pt, 128, softmax_scale=0.2)
    # bf16 output: rounding to bf16 adds up to 2^-9 relative
    err = np.abs(got - ref) - 2.0 ** -8 * np.abs(ref)
    assert float(err.max()) <= TOL


def test_oscar_decode_full_size_sampled(orc):
    """The 32768-token, 8-kv-head, 32-query-head step (one sequence, all
    pages full): every output against the oracle."""
    b = 128
    w = workloads.make("llama3-8b-32k", block=b)
    pool, _, rows = write_both(orc, w, b)
    got, pt = gpu_decode(w, pool, rows, b)
    pairs = [(0, hq) for hq in (0, 5, 13, 31)]
    ref = oracle_decode(orc, w, host(pool), rows, pt, b, pairs=pairs)
    for (n, hq), r in ref.items():
        assert_close(got[n, hq], r, f"full size (n={n}, hq={hq})")


def test_oscar_write_full_size_sampled_pages(orc):
    """The full 32768-token write; sampled pages compared with the oracle."""
    b = 128
    w = workloads.make("llama3-8b-32k", block=b)
    k, v, ids, _, _ = workloads.oscar_rows(w)
    pool = gpu_pool(w.num_pages, w.Hkv, w.D)
    kvq.kv_quant_write_oscar(k.cuda(), v.cuda(), torch.as_tensor(ids).cuda(), *pool, b)
    assert kvq.get_device_error() == 0
    gc, gk, gt = host(pool)
    pick = np.array([0, 1, 777, ids.size - 1])
    sel_rows = np.concatenate([np.arange(16 * g, 16 * g + 16) for g in pick])
    ks, vs = k[sel_rows], v[sel_rows]
    ora = orc.oscar_write(workloads.bf16_bits(ks), workloads.bf16_bits(vs), ids[pick], w.num_pages, b)
    mask = np.zeros(w.num_pages, bool)
    mask[ids[pick]] = True
    sub = (np.where(mask[:, None, None, None, None], gc, CANARY).astype(np.uint8),
           np.where(mask[:, None, None, None], gk, H_CANARY).astype(np.uint16),
           np.where(mask[:, None, None, None], gt, H_CANARY).astype(np.uint16))
    compare_oscar_write(orc, sub, ora, ks, vs, ids[pick], b)


def test_oscar_argument_errors():
    cache, kmeta, tmeta = kvq.alloc_oscar_cache(4, 2, 128)
    q = torch.zeros((1, 16, 128), dtype=torch.bfloat16, device="cuda")  # G = 8: not built
    pt = torch.zeros((1, 2), dtype=torch.int32, device="cuda")
    cl = torch.full((1,), 20, dtype=torch.int32, device="cuda")
    tail = torch.zeros((1, 2, 16, 128), dtype=torch.bfloat16, device="cuda")
    out = torch.zeros((1, 16, 128), dtype=torch.float32, device="cuda")
    ws = torch.zeros(1 << 20, dtype=torch.uint8, device="cuda")
    with pytest.raises(kvq.KVQError) as e:
        kvq.paged_decode_attn_oscar(q, cache, kmeta, tmeta, pt, cl, tail, tail, out, 128, ws)
    assert e.value.status == 2
    q = torch.zeros((1, 4, 128), dtype=torch.bfloat16, device="cuda")
    out = torch.zeros((1, 4, 128), dtype=torch.float32, device="cuda")
    with pytest.raises(kvq.KVQError) as e:
        kvq.paged_decode_attn_oscar(q, cache, kmeta, tmeta, pt, cl, tail, tail, out, 128, ws[:16])
    assert e.value.status == 4
    with pytest.raises(kvq.KVQError) as e:
        kvq.paged_decode_attn_oscar(q, cache, kmeta, tmeta, pt, cl, tail, tail, out, 48, ws)
    assert e.value.status == 2


def test_oscar_decode_out_of_range_inputs(orc):
    """A page id outside the pool skips that page and records
    KVQ_ERR_OUT_OF_RANGE; a context length above the table's capacity is
    clamped (and recorded); the rest of the batch is unaffected."""
    ctx = [90, 50]
    w = workloads.random_case(61, 2, 4, 2, 128, 64, ctx)
    pool, _, rows = write_both(orc, w, 64)
    good, pt = gpu_decode(w, pool, rows, 64)
    # sequence 1: a bad id in its page table
    bad_pt = pt.copy()
    bad_pt[1, 1] = w.num_pages + 5
    _, _, ids, k_tail, v_tail = rows
    out = torch.zeros((w.B, w.Hq, w.D), dtype=torch.float32, device="cuda")
    nb = kvq.oscar_workspace_size(w.B, w.Hq, w.Hkv, w.D, w.num_pages, pt.shape[1], 64)
    ws = torch.zeros(nb, dtype=torch.uint8, device="cuda")
    kvq.paged_decode_attn_oscar(w.q.cuda(), *pool, torch.as_tensor(bad_pt).cuda(),
                                torch.as_tensor(w.context_lens).cuda(), k_tail.cuda(), v_tail.cuda(), out, 64, ws)
    torch.cuda.synchronize()
    assert kvq.get_device_error() == 3
    assert kvq.get_device_error() == 0
    got = out.cpu().numpy()
    assert np.array_equal(got[0], good[0].astype(np.float32))  # sequence 0 untouched
    # a context length beyond max_pages * 16 + 15 is clamped to it
    big = np.array(ctx, np.int32)
    big[0] = pt.shape[1] * 16 + 100
    kvq.paged_decode_attn_oscar(w.q.cuda(), *pool, torch.as_tensor(pt).cuda(), torch.as_tensor(big).cuda(),
                                k_tail.cuda(), v_tail.cuda(), out, 64, ws)
    torch.cuda.synchronize()
    assert kvq.get_device_error() == 3
    assert np.all(np.isfinite(out.cpu().numpy()))


def test_oscar_empty_calls():
    cache, kmeta, tmeta = kvq.alloc_oscar_cache(2, 2, 128)
    e = torch.zeros((0, 2, 128), dtype=torch.bfloat16, device="cuda")
    kvq.kv_quant_write_oscar(e, e, torch.zeros(0, dtype=torch.int32, device="cuda"), cache, kmeta, tmeta, 128)
    q = torch.zeros((0, 4, 128), dtype=torch.bfloat16, device="cuda")
    tail = torch.zeros((0, 2, 16, 128), dtype=torch.bfloat16, device="cuda")
    out = torch.zeros((0, 4, 128), dtype=torch.float32, device="cuda")
    ws = torch.zeros(16, dtype=torch.uint8, device="cuda")
    kvq.paged_decode_attn_oscar(q, cache, kmeta, tmeta, torch.zeros((0, 1), dtype=torch.int32, device="cuda"),
                                torch.zeros(0, dtype=torch.int32, device="cuda"), tail, tail, out, 128, ws)
    torch.cuda.synchronize()
    assert kvq.get_device_error() == 0


def test_oscar_write_full_size_plain_bit_exact(orc):
    """The full 32768-token write at b = 0: every byte of every page-head
    equal to the oracle's."""
    w = workloads.make("llama3-8b-32k", block=0)
    k, v, ids, _, _ = workloads.oscar_rows(w)
    pool = gpu_pool(w.num_pages, w.Hkv, w.D)
    kvq.kv_quant_write_oscar(k.cuda(), v.cuda(), torch.as_tensor(ids).cuda(), *pool, 0)
    assert kvq.get_device_error() == 0
    ora = orc.oscar_write(workloads.bf16_bits(k), workloads.bf16_bits(v), ids, w.num_pages, 0)
    compare_oscar_write(orc, host(pool), ora, k, v, ids, 0)


def test_oscar_decode_batched_gqa4(orc):
    """Eight sequences of mixed lengths (tails of every size, one sequence
    shorter than a page) in one call, GQA 4, b = 64, bf16 and fp32 out."""
    ctx = [3000, 17, 1024, 2500, 15, 777, 4096, 1601]
    w = workloads.random_case(77, len(ctx), 32, 8, 128, 64, ctx, n_outliers=4)
    pool, _, rows = write_both(orc, w, 64)
    got, pt = gpu_decode(w, pool, rows, 64)
    ref = oracle_decode(orc, w, host(pool), rows, pt, 64)
    assert_close(got, ref, "oscar decode batched")
    got16, _ = gpu_decode(w, pool, rows, 64, out_dtype=torch.bfloat16)
    assert float((np.abs(got16 - ref) - 2.0 ** -8 * np.abs(ref)).max()) <= TOL
    # deterministic: a second call (fresh workspace holding other bytes) is identical
    again, _ = gpu_decode(w, pool, rows, 64)
    assert np.array_equal(again, got)
