"""Pins of the CPU oracle against what the pages and the mathematics fix.

No page prints a worked example, so the oracle is pinned by hand-derived
fixtures (tests/golden/), library routines it must agree with (numpy's float16,
scipy's Sylvester Hadamard and softmax), closed forms, invariants and brute
force. Each check is chosen so a plausible slip (a dropped 1/sqrt(b), a
transposed or reordered Hadamard, round-to-nearest where a directed rounding
is defined, floor instead of round, a swapped nibble, a missing query or output
rotation, a wrong page index) fails at least one of them.
"""
import math

import numpy as np
import pytest
import scipy.linalg
import scipy.special
import torch

from helpers import golden, parse_bytes

BLOCKS = [32, 64, 128]


def blockdiag_hadamard(D, b):
    if b == 0:
        return np.eye(D)
    H = scipy.linalg.hadamard(b).astype(np.float64) / math.sqrt(b)
    return scipy.linalg.block_diag(*([H] * (D // b)))


def tni_rows(rng, n, D, outliers=2):
    """Rows with lognormal per-token norms and a few x10 channels (bf16 bits)."""
    x = rng.standard_normal((n, D)) * np.exp(rng.standard_normal((n, 1)))
    x[:, rng.choice(D, outliers, replace=False)] *= 10
    t = torch.from_numpy(x.astype(np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16), t.to(torch.float64).numpy()


def f16(bits):
    return float(np.array([bits], np.uint16).view(np.float16)[0])


# ----------------------------------------------------------------------------
# number formats
# ----------------------------------------------------------------------------

def test_half_to_double_matches_numpy_all_patterns(orc):
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ref = bits.view(np.float16).astype(np.float64)
    got = np.array([orc.half_to_double(int(b)) for b in bits])
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])


def test_bf16_to_double_matches_torch(orc):
    bits = np.arange(0, 65536, 7, dtype=np.uint32).astype(np.uint16)
    ref = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    got = np.array([orc.bf16_to_double(int(b)) for b in bits])
    nan = np.isnan(ref)
    assert np.array_equal(got[~nan], ref[~nan])


def _half_values(rng):
    mags = np.concatenate([
        rng.uniform(0, 6e-5, 300),             # subnormal range
        np.exp(rng.uniform(-12, 11.1, 3000)),   # normal range
        rng.uniform(65000, 70000, 100),         # around the overflow threshold
        [0.0, 5.96e-8, 2.98e-8, 65504.0, 65519.99, 65520.0, 1.0, 1.0 + 2 ** -11],
    ])
    return np.concatenate([mags, -mags])


@pytest.mark.filterwarnings("ignore::RuntimeWarning")
def test_half_round_nearest_matches_numpy(orc):
    rng = np.random.default_rng(1)
    for x in _half_values(rng):
        ref = np.array([x], np.float64).astype(np.float16).view(np.uint16)[0]
        assert orc.half_round_nearest(x) == ref, x


@pytest.mark.filterwarnings("ignore::RuntimeWarning")
def test_half_directed_roundings_bracket(orc):
    rng = np.random.default_rng(2)
    for x in _half_values(rng):
        dn, up = orc.half_round_down(x), orc.half_round_up(x)
        vd, vu = f16(dn), f16(up)
        assert vd <= x <= vu
        if vd == x:
            assert vu == x
        else:
            # adjacent binary16 values: nothing representable strictly between
            assert np.nextafter(np.float16(vd), np.float16(np.inf)) == np.float16(vu)
        rn = f16(orc.half_round_nearest(x))
        assert rn in (vd, vu) or abs(x) >= 65520


# ----------------------------------------------------------------------------
# rotation
# ----------------------------------------------------------------------------

@pytest.mark.parametrize("b", [2, 4, 8, 32, 64, 128])
def test_hadamard_is_sylvester_and_orthogonal(orc, b):
    H = orc.hadamard(b).astype(np.int64)
    assert np.array_equal(H @ H.T, b * np.eye(b, dtype=np.int64))
    assert np.array_equal(H, scipy.linalg.hadamard(b))
    # recursive construction [[H, H], [H, -H]] from order 1
    R = np.array([[1]])
    while R.shape[0] < b:
        R = np.block([[R, R], [R, -R]])
    assert np.array_equal(H, R)
    assert np.array_equal(H @ np.ones(b, np.int64), b * np.eye(b, dtype=np.int64)[0])


@pytest.mark.parametrize("b", BLOCKS)
@pytest.mark.parametrize("D", [64, 128])
def test_rotate_matches_dense_library_hadamard(orc, b, D):
    if b > D:
        pytest.skip("block larger than the head")
    rng = np.random.default_rng(b + D)
    for _ in range(20):
        x = rng.standard_normal(D) * np.exp(rng.standard_normal())
        y = orc.rotate_f64(x, b)
        ref = blockdiag_hadamard(D, b) @ x
        assert np.allclose(y, ref, rtol=1e-13, atol=1e-13 * np.abs(x).max())
        assert math.isclose(np.linalg.norm(y), np.linalg.norm(x), rel_tol=1e-12)
        assert np.allclose(orc.rotate_f64(y, b), x, rtol=1e-12, atol=1e-12 * np.abs(x).max())


@pytest.mark.parametrize("b", [0] + BLOCKS)
def test_rotate_row_is_one_fp32_rounding(orc, b):
    rng = np.random.default_rng(7 + b)
    bits, xd = tni_rows(rng, 50, 128)
    for i in range(bits.shape[0]):
        y = orc.rotate_row(bits[i], b)
        ref = blockdiag_hadamard(128, b) @ xd[i]
        # one rounding of the exact value: within half an fp32 ulp (+ fp64 noise)
        ulp = np.spacing(np.abs(ref).astype(np.float32)).astype(np.float64)
        assert np.all(np.abs(y.astype(np.float64) - ref) <= 0.5 * ulp + 1e-12 * np.abs(ref).max())
        rel = abs(np.linalg.norm(y.astype(np.float64)) / np.linalg.norm(xd[i]) - 1)
        assert rel <= 1e-6


def test_rotate_b0_is_identity(orc):
    rng = np.random.default_rng(3)
    bits, xd = tni_rows(rng, 5, 64)
    for i in range(5):
        assert np.array_equal(orc.rotate_row(bits[i], 0).astype(np.float64), xd[i])


# ----------------------------------------------------------------------------
# quantization: worked examples
# ----------------------------------------------------------------------------

def _golden_row(fx):
    D = int(fx["D"])
    x = np.zeros(D, np.float32)
    spec = fx["x"]
    if spec.startswith("8 * e_"):
        x[int(spec.split("_")[1])] = 8.0
    else:
        x[:] = [-1 + (c % 16) / 8 for c in range(D)]
    bits = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(torch.from_numpy(x).to(torch.bfloat16).float().numpy(), x)
    return D, int(fx["block"]), bits


@pytest.mark.parametrize("name", ["quant_grid_b0_d64.txt", "rotate_onehot0_b64_d128.txt",
                                  "rotate_onehot1_b64_d128.txt"])
def test_golden_quantized_rows(orc, name):
    fx = golden(name)
    D, b, bits = _golden_row(fx)
    y = orc.rotate_row(bits, b)
    codes, s, z = orc.quantize_row(y)
    assert s == int(fx["s_bits"], 16)
    assert z == int(fx["z_bits"], 16)
    assert list(orc.pack_row(codes)) == parse_bytes(fx["packed"])
    # the same row placed in a one-page pool
    k = bits.reshape(1, 1, D)
    cache, scales, zeros, _ = orc.quant_write(k, k, np.array([3], np.int64), 1, b)
    assert list(cache[3 * D // 2: 4 * D // 2]) == parse_bytes(fx["packed"])
    assert scales[3] == s and zeros[3] == z


def test_golden_placement_offsets(orc):
    fx = golden("placement.txt")
    Hkv, D = int(fx["Hkv"]), int(fx["D"])
    for case in fx["case"]:
        page, h, kv, off, row, byte = (int(t) for t in case.split())
        assert orc.scale_offset(page, Hkv, h, kv, off) == row
        assert orc.cache_row_offset(page, Hkv, D, h, kv, off) == byte


# ----------------------------------------------------------------------------
# quantization: properties
# ----------------------------------------------------------------------------

def _rows(orc, seed, n=200, D=128, b=128):
    rng = np.random.default_rng(seed)
    bits, _ = tni_rows(rng, n, D)
    return [orc.rotate_row(bits[i], b) for i in range(n)]


@pytest.mark.parametrize("b", [0] + BLOCKS)
def test_scale_zero_definition_against_numpy_float16(orc, b):
    for y in _rows(orc, 11 + b, b=b):
        codes, s, z = orc.quantize_row(y)
        mn, mx = float(y.min()), float(y.max())
        zf, sf = f16(z), f16(s)
        # z: the largest binary16 value not above the row minimum
        assert zf <= mn < float(np.nextafter(np.float16(zf), np.float16(np.inf)))
        # s: the smallest binary16 step that reaches the row maximum
        assert 15 * sf + zf >= mx
        if s > 0:
            sp = float(np.nextafter(np.float16(sf), np.float16(0)))
            assert 15 * sp + zf < mx


@pytest.mark.parametrize("b", [0] + BLOCKS)
def test_roundtrip_error_within_half_step(orc, b):
    # |y - (code*s + z)| <= s/2 up to the two fp32 roundings of the quotient
    # (each <= 2^-24 relative on a value <= 15): slack 15 * 2^-23 steps.
    for y in _rows(orc, 21 + b, b=b):
        codes, s, z = orc.quantize_row(y)
        xhat = orc.dequant_row(orc.pack_row(codes), y.size, s, z)
        err = np.abs(y.astype(np.float64) - xhat)
        assert np.all(err <= f16(s) * (0.5 + 15 * 2 ** -23))
        assert codes.max() <= 15


def test_exact_roundtrip_on_the_grid(orc):
    rng = np.random.default_rng(5)
    for _ in range(50):
        k = np.concatenate([rng.permutation(16) for _ in range(8)])  # every code in each row
        x = (-1.0 + k / 8.0).astype(np.float32)                     # z = -1, s = 2^-3
        bits = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
        y = orc.rotate_row(bits, 0)
        codes, s, z = orc.quantize_row(y)
        assert (f16(s), f16(z)) == (0.125, -1.0)
        assert np.array_equal(codes, k)
        assert np.array_equal(orc.dequant_row(orc.pack_row(codes), 128, s, z), x.astype(np.float64))


def test_constant_rows(orc):
    # on the fp16 grid: s = 0, every code 0, exact
    codes, s, z = orc.quantize_row(np.full(64, 0.5, np.float32))
    assert s == 0 and f16(z) == 0.5 and codes.max() == 0
    # off the grid: z falls below, the error stays within s/2
    y = np.full(64, np.float32(0.3), np.float32)
    codes, s, z = orc.quantize_row(y)
    xhat = orc.dequant_row(orc.pack_row(codes), 64, s, z)
    assert s > 0 and f16(z) < 0.3
    assert np.all(np.abs(xhat - float(y[0])) <= f16(s) / 2 * (1 + 1e-6))


@pytest.mark.parametrize("j", [-3, 2, 5])
def test_power_of_two_token_scaling_leaves_codes(orc, j):
    # OScaR (forum summary, "The OScaR Framework"): V^ = Quant(S.(R.V)) with a
    # per-token scale S. Under token-wise min/max quantization a power-of-two S
    # changes only s and z (by the same factor), never the codes.
    for y in _rows(orc, 31, n=100, b=64):
        if np.abs(y).max() * 2.0 ** j > 60000 or np.abs(y).max() * 2.0 ** j < 1:
            continue
        c1, s1, z1 = orc.quantize_row(y)
        c2, s2, z2 = orc.quantize_row((y * np.float32(2.0 ** j)).astype(np.float32))
        assert np.array_equal(c1, c2)
        assert f16(s2) == f16(s1) * 2.0 ** j and f16(z2) == f16(z1) * 2.0 ** j


def test_codes_are_the_nearest_level_brute_force(orc):
    for y in _rows(orc, 41, n=100, b=32):
        codes, s, z = orc.quantize_row(y)
        levels = f16(z) + np.arange(16) * f16(s)
        dist = np.abs(y.astype(np.float64)[:, None] - levels[None, :])
        best = dist.argmin(axis=1)
        srt = np.sort(dist, axis=1)
        clear = (srt[:, 1] - srt[:, 0]) > 1e-5 * f16(s)   # not a near-tie
        assert np.array_equal(codes[clear], best[clear])


def test_nibble_order_and_pack_roundtrip(orc):
    codes = np.tile(np.arange(16, dtype=np.uint8), 4)
    packed = orc.pack_row(codes)
    assert packed[0] == 0x10 and packed[7] == 0xFE  # low nibble = even channel
    assert np.array_equal(orc.unpack_row(packed, 64), codes)


def test_quant_write_placement_and_untouched_bytes(orc):
    from bit_kv_cache_20_b200 import workloads
    w = workloads.random_case(seed=9, B=3, Hq=4, Hkv=2, D=64, block=32,
                              context_lens=[5, 16, 37], extra_pages=2, skip_fraction=0.2)
    kb, vb = workloads.bf16_bits(w.k_new).reshape(-1, 2, 64), workloads.bf16_bits(w.v_new).reshape(-1, 2, 64)
    P, Hkv, D = w.num_pages, 2, 64
    cache = np.full(P * Hkv * 2 * 16 * D // 2, 0xA5, np.uint8)
    scales = np.full(P * Hkv * 2 * 16, 0x7E00, np.uint16)
    zeros = np.full(P * Hkv * 2 * 16, 0x7E00, np.uint16)
    orc.quant_write(kb, vb, w.slots_new, P, 32, cache, scales, zeros)
    written_bytes = np.zeros(cache.size, bool)
    written_rows = np.zeros(scales.size, bool)
    for t, slot in enumerate(w.slots_new):
        if slot < 0:
            continue
        page, off = divmod(int(slot), 16)
        for h in range(Hkv):
            for kv, src in enumerate((kb, vb)):
                codes, s, z = orc.quantize_row(orc.rotate_row(src[t, h], 32))
                o = orc.cache_row_offset(page, Hkv, D, h, kv, off)
                assert np.array_equal(cache[o:o + D // 2], orc.pack_row(codes))
                r = orc.scale_offset(page, Hkv, h, kv, off)
                assert scales[r] == s and zeros[r] == z
                written_bytes[o:o + D // 2] = True
                written_rows[r] = True
    assert np.all(cache[~written_bytes] == 0xA5)
    assert np.all(scales[~written_rows] == 0x7E00) and np.all(zeros[~written_rows] == 0x7E00)
    assert written_rows.sum() == 4 * (w.slots_new >= 0).sum()


def test_quant_write_rejects_slots_outside_the_pool(orc):
    k = np.zeros((2, 1, 64), np.uint16)
    with pytest.raises(ValueError):
        orc.quant_write(k, k, np.array([0, 16], np.int64), 1, 0)
    with pytest.raises(ValueError):
        orc.quant_write(k, k, np.array([0, -2], np.int64), 1, 0)


# ----------------------------------------------------------------------------
# attention
# ----------------------------------------------------------------------------

def textbook_attention(q, K, V, scale):
    p = scipy.special.softmax(scale * (K @ q))
    return p @ V


def test_attention_two_token_closed_form(orc):
    fx = golden("attn_two_tokens.txt")
    D = int(fx["D"])
    P = 3
    k = np.zeros((2, 1, D), np.float32)
    v = np.zeros((2, 1, D), np.float32)
    k[0, 0, 0] = 1.875
    v[0, 0, 1] = 1.875
    v[1, 0, 2] = 1.875
    to_bits = lambda a: torch.from_numpy(a).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    q = np.zeros((1, 1, D), np.float32)
    q[0, 0, 0] = 8.0
    # positions 0 and 1 of the sequence sit on page 2 of a 3-page pool
    slots = np.array([2 * 16 + 0, 2 * 16 + 1], np.int64)
    cache, scales, zeros, _ = orc.quant_write(to_bits(k), to_bits(v), slots, P, 0)
    page_table = np.array([[2]], np.int32)
    out = orc.decode_attn(to_bits(q), cache, scales, zeros, page_table, np.array([2], np.int32),
                          Hkv=1, b=0, num_pages=P)[0, 0]
    p0 = 1.0 / (1.0 + math.exp(-1.875))
    ref = np.zeros(D)
    ref[1] = 1.875 * p0
    ref[2] = 1.875 * (1 - p0)
    assert np.allclose(out, ref, rtol=0, atol=1e-14)


@pytest.mark.parametrize("b", BLOCKS)
def test_attention_rotation_invariance(orc, b):
    # attention computed in the rotated space (q rotated, rows rotated, output
    # rotated back) equals plain attention: R is orthogonal and R^T = R.
    rng = np.random.default_rng(b)
    D, n = 128, 37
    for _ in range(5):
        q = rng.standard_normal(D) / 8
        K = rng.standard_normal((n, D)) * np.exp(rng.standard_normal((n, 1)))
        V = rng.standard_normal((n, D)) * np.exp(rng.standard_normal((n, 1)))
        R = blockdiag_hadamard(D, b)
        got = orc.attn_rows(q, K @ R.T, V @ R.T, b, 1 / math.sqrt(D))
        ref = textbook_attention(q, K, V, 1 / math.sqrt(D))
        assert np.allclose(got, ref, rtol=1e-11, atol=1e-11 * np.abs(ref).max())


def test_attention_special_cases(orc):
    rng = np.random.default_rng(4)
    D, b = 64, 32
    R = blockdiag_hadamard(D, b)
    # one token: the output is that token's value, back in the original basis
    q = rng.standard_normal(D)
    K = rng.standard_normal((1, D))
    V = rng.standard_normal((1, D))
    assert np.allclose(orc.attn_rows(q, K, V, b, 0.125), R @ V[0], atol=1e-13)
    # q = 0: uniform weights, the output is the mean value
    K = rng.standard_normal((9, D))
    V = rng.standard_normal((9, D))
    assert np.allclose(orc.attn_rows(np.zeros(D), K, V, b, 0.125), R @ V.mean(axis=0), atol=1e-13)
    # no tokens: zero output
    assert np.array_equal(orc.attn_rows(q, np.zeros((0, D)), np.zeros((0, D)), b, 0.125), np.zeros(D))


def test_attention_matches_fp32_textbook_on_unquantized_rows(orc):
    rng = np.random.default_rng(6)
    D, n, b = 64, 12, 32
    R = blockdiag_hadamard(D, b)
    q = (rng.standard_normal(D) / 8).astype(np.float32)
    K = rng.standard_normal((n, D)).astype(np.float32)
    V = rng.standard_normal((n, D)).astype(np.float32)
    Kr, Vr = (K.astype(np.float64) @ R.T), (V.astype(np.float64) @ R.T)
    got = orc.attn_rows(q.astype(np.float64), Kr, Vr, b, 0.125)
    logits = (K @ q) * np.float32(0.125)
    p = np.exp(logits - logits.max())
    ref32 = (p / p.sum()) @ V
    assert np.allclose(got, ref32, rtol=0, atol=1e-5)


def test_paged_decode_equals_gathered_rows(orc):
    from bit_kv_cache_20_b200 import workloads
    w = workloads.random_case(seed=3, B=3, Hq=8, Hkv=2, D=64, block=32,
                              context_lens=[1, 17, 40], extra_pages=3)
    kb = workloads.bf16_bits(w.k_new).reshape(-1, 2, 64)
    vb = workloads.bf16_bits(w.v_new).reshape(-1, 2, 64)
    qb = workloads.bf16_bits(w.q).reshape(3, 8, 64)
    cache, scales, zeros, _ = orc.quant_write(kb, vb, w.slots_new, w.num_pages, 32)
    out = orc.decode_attn(qb, cache, scales, zeros, w.page_table, w.context_lens, 2, 32, w.num_pages)
    start = np.concatenate([[0], np.cumsum(w.context_lens)])
    for n in range(3):
        for hq in range(8):
            h = hq // 4
            rows = []
            for kv, src in enumerate((kb, vb)):
                xs = []
                for t in range(start[n], start[n + 1]):
                    codes, s, z = orc.quantize_row(orc.rotate_row(src[t, h], 32))
                    xs.append(orc.dequant_row(orc.pack_row(codes), 64, s, z))
                rows.append(np.array(xs))
            qd = np.array([orc.bf16_to_double(int(x)) for x in qb[n, hq]])
            ref = orc.attn_rows(qd, rows[0], rows[1], 32, 1 / 8)
            assert np.allclose(out[n, hq], ref, rtol=0, atol=1e-13)


def test_quantization_moves_each_logit_within_the_step_bound(orc):
    # |(Rq).(k^ - Rk)| <= sum_c |(Rq)_c| * s/2 per token (round-trip bound),
    # checked on the oracle's own rows against the unquantized rotated rows.
    rng = np.random.default_rng(8)
    bits, xd = tni_rows(rng, 64, 128)
    q = rng.standard_normal(128) / 8
    qr = orc.rotate_f64(q, 64)
    for i in range(64):
        y = orc.rotate_row(bits[i], 64)
        codes, s, z = orc.quantize_row(y)
        khat = orc.dequant_row(orc.pack_row(codes), 128, s, z)
        exact = orc.rotate_f64(xd[i], 64)
        gap = abs(qr @ (khat - exact))
        assert gap <= np.abs(qr).sum() * f16(s) * (0.5 + 1e-5) + 1e-6 * np.abs(qr).sum() * np.abs(exact).max()


# --- randomized Hadamard: R = H_b diag(sigma) / sqrt(b) ------------------------

def _random_sign_vector(D, seed):
    return np.random.default_rng(seed).integers(0, 2, D).astype(bool)


@pytest.mark.parametrize("b,D", [(32, 64), (64, 128), (128, 128)])
def test_signed_rotation_columns_closed_form(orc, b, D):
    """R e_i = sigma_i * (column i of H_b within i's block) / sqrt(b), with
    H_b[j][i] = (-1)^popcount(i & j): a sign applied after the transform, or
    to the wrong index, fails here."""
    sig = _random_sign_vector(D, 3 * b + D)
    for i in range(D):
        e = np.zeros(D)
        e[i] = 1.0
        y = orc.rotate_f64(e, b, signs=sig)
        blk, ii = (i // b) * b, i % b
        ref = np.zeros(D)
        for j in range(b):
            ref[blk + j] = (-1.0 if bin(ii & j).count("1") % 2 else 1.0) / math.sqrt(b)
        ref *= -1.0 if sig[i] else 1.0
        assert np.array_equal(y, ref) or np.allclose(y, ref, rtol=0, atol=1e-15), i


@pytest.mark.parametrize("b,D", [(32, 64), (64, 128), (128, 128)])
def test_signed_rotation_is_orthogonal_and_unrotate_is_its_transpose(orc, b, D):
    sig = _random_sign_vector(D, b + D)
    rng = np.random.default_rng(b)
    for i in range(D):  # R^T R = I on every basis vector
        e = np.zeros(D)
        e[i] = 1.0
        assert np.allclose(orc.unrotate_f64(orc.rotate_f64(e, b, signs=sig), b, signs=sig), e,
                           rtol=0, atol=1e-14)
    for _ in range(20):
        x = rng.standard_normal(D) * 10
        y = orc.rotate_f64(x, b, signs=sig)
        assert abs(np.linalg.norm(y) / np.linalg.norm(x) - 1) < 1e-12
        # <R x, z> = <x, R^T z> for a second vector
        z = rng.standard_normal(D)
        assert abs(y @ z - x @ orc.unrotate_f64(z, b, signs=sig)) < 1e-10 * np.linalg.norm(x) * np.linalg.norm(z)


def test_zero_sign_mask_is_the_plain_rotation(orc):
    from bit_kv_cache_20_b200 import workloads
    rng = np.random.default_rng(8)
    x = rng.standard_normal(128)
    xb = workloads.bf16_bits(torch.from_numpy(x.astype(np.float32)).to(torch.bfloat16))
    for b in (32, 64, 128):
        assert np.array_equal(orc.rotate_f64(x, b, signs=np.zeros(128, bool)), orc.rotate_f64(x, b))
        assert np.array_equal(orc.rotate_row(xb, b, signs=np.zeros(128, bool)), orc.rotate_row(xb, b))


@pytest.mark.parametrize("b", [32, 128])
def test_attention_invariance_with_random_signs(orc, b):
    """Attention in the randomized-rotated space (q by R, rows by R, output
    back by R^T) equals plain attention."""
    rng = np.random.default_rng(50 + b)
    D, n = 128, 29
    sig = _random_sign_vector(D, 60 + b)
    R = blockdiag_hadamard(D, b) @ np.diag(np.where(sig, -1.0, 1.0))
    for _ in range(4):
        q = rng.standard_normal(D) / 8
        K = rng.standard_normal((n, D)) * np.exp(rng.standard_normal((n, 1)))
        V = rng.standard_normal((n, D)) * np.exp(rng.standard_normal((n, 1)))
        got = orc.attn_rows(q, K @ R.T, V @ R.T, b, 1 / math.sqrt(D), signs=sig)
        ref = textbook_attention(q, K, V, 1 / math.sqrt(D))
        assert np.allclose(got, ref, rtol=1e-11, atol=1e-11 * np.abs(ref).max())


def test_quant_write_with_signs_rotates_each_row(orc):
    """The write's placement with signs: each stored row is the quantization
    of that row's signed rotation."""
    from bit_kv_cache_20_b200 import workloads
    rng = np.random.default_rng(9)
    T, Hkv, D, b = 5, 2, 128, 64
    sig = _random_sign_vector(D, 10)
    k = workloads.bf16_bits(torch.from_numpy(rng.standard_normal((T, Hkv, D)).astype(np.float32)).to(torch.bfloat16))
    v = workloads.bf16_bits(torch.from_numpy(rng.standard_normal((T, Hkv, D)).astype(np.float32)).to(torch.bfloat16))
    slots = np.array([3, 17, 0, 40, 31], np.int64)
    cache, scales, zeros, _ = orc.quant_write(k, v, slots, 4, b, signs=sig)
    for t in range(T):
        page, off = divmod(int(slots[t]), 16)
        for h in range(Hkv):
            for kv, src in enumerate((k, v)):
                codes, s_, z_ = orc.quantize_row(orc.rotate_row(src[t, h], b, signs=sig))
                row = ((page * Hkv + h) * 2 + kv) * 16 + off
                assert np.array_equal(cache.reshape(-1, D // 2)[row], orc.pack_row(codes))
                assert scales[row] == s_ and zeros[row] == z_
