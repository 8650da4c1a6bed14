"""Pins of the OScaR oracle (V^ = Quant(S (R V)); OScaR forum summary, "The
OScaR Framework"; OScaR abstract: per-channel K quantization, Token Norm
Imbalance, INT2) against what the definitions and the mathematics fix, not
against a retyped formula:

- the INT2 (s, z) rule against numpy float16 neighbours;
- the token norm against numpy's norm rounded by numpy to float16;
- the per-channel quantizer: exact round trip on the INT2 grid, every element
  within s/2 of its level, brute-force nearest level;
- Omni-Token Scaling: scaling a token by a power of two leaves every code and
  every per-channel (s, z) unchanged and scales only its stored norm;
- V token-wise: exact round trip of grid rows;
- the decode: a context of fewer than 16 tokens (all in the unfinished bf16
  page) is textbook softmax attention on the bf16 rows; full pages give
  textbook attention on the oracle's own dequantized rows rotated back with
  scipy's Hadamard matrix; placement leaves other pages untouched.
"""
import numpy as np
import pytest
import scipy.linalg
import torch

import oracle


def _bf16(x):
    return torch.from_numpy(np.asarray(x, np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def _bf16_val(bits):
    return (np.asarray(bits, np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def _h16(bits):
    return np.asarray(bits, np.uint16).view(np.float16).astype(np.float64)


def _unpack2(codes, D):
    b = np.asarray(codes, np.uint8)
    return np.stack([(b >> (2 * i)) & 3 for i in range(4)], axis=-1).reshape(b.shape[:-1] + (D,))


def test_int2_scale_zero_rule_against_float16_neighbours():
    rng = np.random.default_rng(1)
    for _ in range(400):
        a, c = np.sort(rng.standard_normal(2) * 10.0 ** rng.integers(-3, 3, 2))
        s, z = oracle.scale_zero_levels(np.float32(a), np.float32(c), 3)
        zf, sf = _h16(z), _h16(s)
        up = np.nextafter(np.float16(zf), np.float16(np.inf)).astype(np.float64)
        assert zf <= np.float32(a) < up                      # z: largest fp16 <= min
        assert 3 * sf + zf >= np.float32(c)                  # covers the max ...
        if s > 0:
            prev = _h16(s - 1)
            assert 3 * prev + zf < np.float32(c)             # ... and is the smallest that does


def test_token_norm_is_the_fp16_rounded_l2_norm():
    rng = np.random.default_rng(2)
    for _ in range(50):
        y = (rng.standard_normal(128) * np.exp(rng.standard_normal())).astype(np.float32)
        n, u = oracle.oscar_token_norm(y)
        ref = np.float16(np.linalg.norm(y.astype(np.float64)))
        assert n == ref.view(np.uint16)
        S = np.float32(1.0) / np.float32(ref)                       # numpy's fp32 quotient
        assert np.array_equal(u, (y.astype(np.float64) * np.float64(S)).astype(np.float32))
        # the scaled row has unit norm up to the fp16 rounding of n (2^-11)
        assert abs(np.linalg.norm(u.astype(np.float64)) - 1.0) <= 2.0 ** -11 + 2.0 ** -20
    n, u = oracle.oscar_token_norm(np.zeros(64, np.float32))
    assert n == 0 and not u.any()
    # a norm above the fp16 range saturates at 65504
    n, u = oracle.oscar_token_norm(np.full(128, 7000.0, np.float32))
    assert n == 0x7BFF and np.allclose(u, 7000.0 / 65504.0, rtol=2.0 ** -22)


def test_per_channel_round_trip_on_the_int2_grid():
    rng = np.random.default_rng(3)
    D = 128
    s = (2.0 ** rng.integers(-6, -1, D)).astype(np.float64)       # fp16-exact steps
    z = -np.round(rng.uniform(0, 1, D) * 64) / 64                  # fp16-exact offsets
    codes = rng.integers(0, 4, (16, D))
    codes[0], codes[1] = 0, 3                                      # every channel spans 0..3
    u = (z + codes * s).astype(np.float32)
    got, ks, kz = oracle.oscar_quant_channels(u)
    assert np.array_equal(_unpack2(got, D), codes)
    assert np.array_equal(_h16(ks), s) and np.array_equal(_h16(kz), z)


def test_per_channel_error_bound_and_nearest_level():
    rng = np.random.default_rng(4)
    D = 128
    u = (rng.standard_normal((16, D)) * rng.lognormal(0, 1, (16, 1))).astype(np.float32)
    got, ks, kz = oracle.oscar_quant_channels(u)
    c = _unpack2(got, D)
    s, z = _h16(ks), _h16(kz)
    uhat = z + c * s
    assert np.all(np.abs(uhat - u) <= s / 2 * (1 + 1e-6) + 1e-30)
    levels = z[None, :, None] + np.arange(4)[None, None, :] * s[None, :, None]   # [1, D, 4]
    dist = np.abs(levels - u[:, :, None].astype(np.float64))
    best = dist.min(axis=2)
    assert np.all(np.abs(uhat - u) <= best + 2e-6 * s)


@pytest.mark.parametrize("b", [0, 64, 128])
def test_omni_token_scaling_leaves_codes_unchanged(b):
    rng = np.random.default_rng(5 + b)
    D = 128
    k = rng.standard_normal((16, D)) * rng.lognormal(0, 1, (16, 1))
    k[:, 7] *= 10.0
    v = rng.standard_normal((16, D))
    base = oracle.oscar_quant_page(_bf16(k), _bf16(v), b)
    shift = rng.integers(-4, 5, 16)
    ks = k * (2.0 ** shift)[:, None]                               # per-token power-of-two factors
    scaled = oracle.oscar_quant_page(_bf16(ks), _bf16(v), b)
    for key in ("kcodes", "ks", "kz", "vcodes", "vs", "vz"):
        assert np.array_equal(base[key], scaled[key]), key
    assert np.array_equal(_h16(scaled["kn"]), _h16(base["kn"]) * 2.0 ** shift)


def test_value_rows_round_trip_on_the_int2_grid():
    rng = np.random.default_rng(6)
    D = 64
    codes = rng.integers(0, 4, (16, D))
    codes[:, 0], codes[:, 1] = 0, 3
    v = -1.0 + codes / 8.0                                         # bf16-exact grid rows
    out = oracle.oscar_quant_page(_bf16(np.ones((16, D))), _bf16(v), 0)
    assert np.array_equal(_unpack2(out["vcodes"], D), codes)
    assert np.all(_h16(out["vs"]) == 0.125) and np.all(_h16(out["vz"]) == -1.0)


def _case(seed, ctx, Hkv=2, Hq=4, D=64, b=32):
    rng = np.random.default_rng(seed)
    B = len(ctx)
    full = [c // 16 for c in ctx]
    npages = sum(full) + 2
    perm = rng.permutation(npages).astype(np.int32)
    pt = np.zeros((B, max(1, max(full))), np.int32)
    off = 0
    for n, f in enumerate(full):
        pt[n, :f] = perm[off:off + f]
        off += f
    T = sum(full) * 16
    k = rng.standard_normal((T, Hkv, D)) * rng.lognormal(0, 1, (T, 1, 1))
    v = rng.standard_normal((T, Hkv, D))
    ids = np.concatenate([pt[n, :f] for n, f in enumerate(full)]) if T else np.zeros(0, np.int32)
    pool = oracle.oscar_write(_bf16(k), _bf16(v), ids, npages, b)
    kt = _bf16(rng.standard_normal((B, Hkv, 16, D)))
    vt = _bf16(rng.standard_normal((B, Hkv, 16, D)))
    q = _bf16(rng.standard_normal((B, Hq, D)) / 4)
    return dict(pool=pool, pt=pt, ctx=np.asarray(ctx, np.int32), kt=kt, vt=vt, q=q, ids=ids, npages=npages,
                Hkv=Hkv, Hq=Hq, D=D, b=b)


def _softmax_attn(q, K, V, scale):
    lg = (K @ q) * scale
    p = np.exp(lg - lg.max())
    return (p / p.sum()) @ V


def test_decode_of_a_short_context_is_textbook_attention_on_the_bf16_rows():
    c = _case(7, [5, 15])
    out = oracle.oscar_decode_attn(c["q"], *c["pool"], c["pt"], c["ctx"], c["kt"], c["vt"], c["b"])
    G = c["Hq"] // c["Hkv"]
    for n, L in enumerate(c["ctx"]):
        for hq in range(c["Hq"]):
            h = hq // G
            ref = _softmax_attn(_bf16_val(c["q"][n, hq]), _bf16_val(c["kt"][n, h, :L]),
                                _bf16_val(c["vt"][n, h, :L]), 1 / np.sqrt(c["D"]))
            assert np.allclose(out[n, hq], ref, rtol=0, atol=1e-12)


def test_decode_with_full_pages_is_attention_on_the_dequantized_rows():
    c = _case(8, [16 * 5 + 3, 32], b=32)
    cache, kmeta, tmeta = c["pool"]
    out = oracle.oscar_decode_attn(c["q"], cache, kmeta, tmeta, c["pt"], c["ctx"], c["kt"], c["vt"], c["b"])
    D, b = c["D"], c["b"]
    R = scipy.linalg.block_diag(*[scipy.linalg.hadamard(b) / np.sqrt(b)] * (D // b))
    G = c["Hq"] // c["Hkv"]
    for n, L in enumerate(c["ctx"]):
        f, t = L // 16, L % 16
        for hq in range(c["Hq"]):
            h = hq // G
            Ks, Vs = [], []
            for p in range(f):
                K, V = oracle.oscar_dequant_page(cache, kmeta, tmeta, int(c["pt"][n, p]), h)
                Ks.append(K @ R)                                    # back to the original space (R = R^T)
                Vs.append(V @ R)
            Ks.append(_bf16_val(c["kt"][n, h, :t]))
            Vs.append(_bf16_val(c["vt"][n, h, :t]))
            ref = _softmax_attn(_bf16_val(c["q"][n, hq]), np.concatenate(Ks), np.concatenate(Vs), 1 / np.sqrt(D))
            assert np.allclose(out[n, hq], ref, rtol=0, atol=1e-10)


def test_write_places_pages_and_leaves_the_others_untouched():
    c = _case(9, [48, 16])
    cache, kmeta, tmeta = c["pool"]
    used = set(int(i) for i in c["ids"])
    for p in range(c["npages"]):
        if p not in used:
            assert not cache[p].any() and not kmeta[p].any() and not tmeta[p].any()
        else:
            assert tmeta[p, :, 0].all()                            # every token norm written
