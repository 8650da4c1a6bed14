"""CPU oracle of the rotated-INT4 paged KV cache (test infrastructure).

Only the test suite, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` leg
of ``bench.py`` may import this package. It wraps ``kvq_oracle.c`` (plain C,
fp64) with numpy marshalling; it never imports the CUDA package.

The arithmetic is in ``kvq_oracle.c``; see its header for the pages it
follows and the readings it takes.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "kvq_oracle.c")
_LIB = os.path.join(_HERE, "libkvq_oracle.so")

_lib = None


def build(force: bool = False) -> str:
    """Compile kvq_oracle.c into libkvq_oracle.so next to it (gcc, OpenMP)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["gcc", "-O2", "-std=c11", "-fopenmp", "-shared", "-fPIC", _SRC, "-o", tmp, "-lm"]
        )
        os.replace(tmp, _LIB)
    return _LIB


def _p(dtype):
    return np.ctypeslib.ndpointer(dtype=dtype, flags="C_CONTIGUOUS")


def lib():
    global _lib
    if _lib is None:
        L = ctypes.CDLL(build())
        u16, u8, i8, f32, f64, i64, i32 = (np.uint16, np.uint8, np.int8, np.float32,
                                            np.float64, np.int64, np.int32)
        c_int, c_i64, c_d = ctypes.c_int, ctypes.c_int64, ctypes.c_double
        sig = {
            "oracle_bf16_to_double": (c_d, [ctypes.c_uint16]),
            "oracle_half_to_double": (c_d, [ctypes.c_uint16]),
            "oracle_half_round_down": (ctypes.c_uint16, [c_d]),
            "oracle_half_round_up": (ctypes.c_uint16, [c_d]),
            "oracle_half_round_nearest": (ctypes.c_uint16, [c_d]),
            "oracle_hadamard": (None, [c_int, _p(i8)]),
            "oracle_rotate_f64": (c_int, [_p(f64), c_int, c_int, _p(f64)]),
            "oracle_rotate_f64_signed": (c_int, [_p(f64), c_int, c_int, ctypes.c_void_p, _p(f64)]),
            "oracle_unrotate_f64_signed": (c_int, [_p(f64), c_int, c_int, ctypes.c_void_p, _p(f64)]),
            "oracle_rotate_row": (c_int, [_p(u16), c_int, c_int, _p(f32)]),
            "oracle_rotate_row_signed": (c_int, [_p(u16), c_int, c_int, ctypes.c_void_p, _p(f32)]),
            "oracle_scale_zero": (None, [ctypes.c_float, ctypes.c_float,
                                         ctypes.POINTER(ctypes.c_uint16),
                                         ctypes.POINTER(ctypes.c_uint16)]),
            "oracle_quantize_given": (None, [_p(f32), c_int, ctypes.c_uint16, ctypes.c_uint16, _p(u8)]),
            "oracle_quotient_given": (None, [_p(f32), c_int, ctypes.c_uint16, ctypes.c_uint16, _p(f64)]),
            "oracle_quantize_row": (None, [_p(f32), c_int, _p(u8), ctypes.POINTER(ctypes.c_uint16),
                                           ctypes.POINTER(ctypes.c_uint16)]),
            "oracle_pack_row": (None, [_p(u8), c_int, _p(u8)]),
            "oracle_unpack_row": (None, [_p(u8), c_int, _p(u8)]),
            "oracle_dequant_row": (None, [_p(u8), c_int, ctypes.c_uint16, ctypes.c_uint16, _p(f64)]),
            "oracle_cache_row_offset": (ctypes.c_size_t, [c_i64, c_int, c_int, c_int, c_int, c_int]),
            "oracle_scale_offset": (ctypes.c_size_t, [c_i64, c_int, c_int, c_int, c_int]),
            "oracle_quant_write": (c_int, [_p(u16), _p(u16), _p(i64), c_int, c_int, c_int, c_int,
                                           ctypes.c_void_p, c_i64, _p(u8), _p(u16), _p(u16),
                                           ctypes.c_void_p]),
            "oracle_attn_rows": (c_int, [_p(f64), _p(f64), _p(f64), c_int, c_int, c_int, ctypes.c_void_p,
                                         c_d, _p(f64)]),
            "oracle_decode_one": (c_int, [_p(u16), _p(u8), _p(u16), _p(u16), _p(i32), _p(i32),
                                          c_int, c_int, c_int, c_int, c_int, c_int, ctypes.c_void_p,
                                          c_int, c_i64, c_d, _p(f64)]),
            "oracle_decode_attn": (c_int, [_p(u16), _p(u8), _p(u16), _p(u16), _p(i32), _p(i32),
                                           c_int, c_int, c_int, c_int, c_int, ctypes.c_void_p, c_int,
                                           c_i64, c_d, _p(f64)]),
            "oracle_num_threads": (c_int, []),
            "oracle_set_num_threads": (None, [c_int]),
            "oracle_scale_zero_levels": (None, [ctypes.c_float, ctypes.c_float, c_int,
                                                ctypes.POINTER(ctypes.c_uint16),
                                                ctypes.POINTER(ctypes.c_uint16)]),
            "oracle_oscar_token_norm": (ctypes.c_uint16, [_p(f32), c_int, _p(f32)]),
            "oracle_oscar_codes_given": (None, [_p(f32), c_int, ctypes.c_uint16, ctypes.c_uint16, _p(u8)]),
            "oracle_oscar_quant_channels": (None, [_p(f32), c_int, _p(u8), _p(u16), _p(u16)]),
            "oracle_oscar_quant_page": (c_int, [_p(u16), _p(u16), c_int, c_int, _p(u8), _p(u8), _p(u16),
                                                _p(u16), _p(u16), _p(u16), _p(u16)]),
            "oracle_oscar_write": (c_int, [_p(u16), _p(u16), _p(i32), c_int, c_int, c_int, c_int, c_i64,
                                           _p(u8), _p(u16), _p(u16)]),
            "oracle_oscar_dequant_page": (None, [_p(u8), _p(u16), _p(u16), c_i64, c_int, c_int, c_int,
                                                 _p(f64), _p(f64)]),
            "oracle_oscar_decode_one": (c_int, [_p(u16), _p(u8), _p(u16), _p(u16), _p(i32), _p(i32),
                                                _p(u16), _p(u16), c_int, c_int, c_int, c_int, c_int, c_int,
                                                c_int, c_i64, c_d, _p(f64)]),
            "oracle_oscar_decode_attn": (c_int, [_p(u16), _p(u8), _p(u16), _p(u16), _p(i32), _p(i32),
                                                 _p(u16), _p(u16), c_int, c_int, c_int, c_int, c_int, c_int,
                                                 c_i64, c_d, _p(f64)]),
        }
        for name, (res, args) in sig.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


# --- number formats -------------------------------------------------------

def half_to_double(bits: int) -> float:
    return lib().oracle_half_to_double(int(bits))


def half_round_down(x: float) -> int:
    return lib().oracle_half_round_down(float(x))


def half_round_up(x: float) -> int:
    return lib().oracle_half_round_up(float(x))


def half_round_nearest(x: float) -> int:
    return lib().oracle_half_round_nearest(float(x))


def bf16_to_double(bits: int) -> float:
    return lib().oracle_bf16_to_double(int(bits))


# --- rotation -------------------------------------------------------------

def hadamard(b: int) -> np.ndarray:
    H = np.zeros(b * b, np.int8)
    lib().oracle_hadamard(b, H)
    return H.reshape(b, b)


def sign_mask(signs, D: int):
    """The 4-word sign mask of a per-channel +-1 vector (bit c set: channel c
    negated; a bool / 0-1 array of D entries, or 4 words), or None."""
    if signs is None:
        return None
    a = np.asarray(signs)
    if a.dtype == np.uint32 and a.shape == (4,):
        return np.ascontiguousarray(a)
    a = a.astype(bool).reshape(-1)
    assert a.size == D
    words = np.zeros(4, np.uint32)
    for c in np.nonzero(a)[0]:
        words[c // 32] |= np.uint32(1) << np.uint32(c % 32)
    return words


def _sp(mask):
    return None if mask is None else mask.ctypes.data


def rotate_f64(x, b: int, signs=None) -> np.ndarray:
    """y = R x, R = H_b diag(sigma) / sqrt(b) per block (sigma = +1 without signs)."""
    x = _c(x, np.float64)
    y = np.zeros_like(x)
    m = sign_mask(signs, x.size)
    rc = lib().oracle_rotate_f64_signed(x, x.size, b, _sp(m), y)
    assert rc == 0, rc
    return y


def unrotate_f64(x, b: int, signs=None) -> np.ndarray:
    """y = R^T x."""
    x = _c(x, np.float64)
    y = np.zeros_like(x)
    m = sign_mask(signs, x.size)
    rc = lib().oracle_unrotate_f64_signed(x, x.size, b, _sp(m), y)
    assert rc == 0, rc
    return y


def rotate_row(x_bf16_bits, b: int, signs=None) -> np.ndarray:
    x = _c(x_bf16_bits, np.uint16)
    y = np.zeros(x.size, np.float32)
    m = sign_mask(signs, x.size)
    rc = lib().oracle_rotate_row_signed(x, x.size, b, _sp(m), y)
    assert rc == 0, rc
    return y


# --- quantization ---------------------------------------------------------

def scale_zero(mn: float, mx: float):
    s, z = ctypes.c_uint16(), ctypes.c_uint16()
    lib().oracle_scale_zero(float(mn), float(mx), ctypes.byref(s), ctypes.byref(z))
    return s.value, z.value


def quantize_row(y):
    y = _c(y, np.float32)
    codes = np.zeros(y.size, np.uint8)
    s, z = ctypes.c_uint16(), ctypes.c_uint16()
    lib().oracle_quantize_row(y, y.size, codes, ctypes.byref(s), ctypes.byref(z))
    return codes, s.value, z.value


def quantize_given(y, s: int, z: int) -> np.ndarray:
    y = _c(y, np.float32)
    codes = np.zeros(y.size, np.uint8)
    lib().oracle_quantize_given(y, y.size, int(s), int(z), codes)
    return codes


def quotient_given(y, s: int, z: int) -> np.ndarray:
    y = _c(y, np.float32)
    q = np.zeros(y.size, np.float64)
    lib().oracle_quotient_given(y, y.size, int(s), int(z), q)
    return q


def pack_row(codes) -> np.ndarray:
    codes = _c(codes, np.uint8)
    out = np.zeros(codes.size // 2, np.uint8)
    lib().oracle_pack_row(codes, codes.size, out)
    return out


def unpack_row(packed, D: int) -> np.ndarray:
    packed = _c(packed, np.uint8)
    out = np.zeros(D, np.uint8)
    lib().oracle_unpack_row(packed, D, out)
    return out


def dequant_row(packed, D: int, s: int, z: int) -> np.ndarray:
    packed = _c(packed, np.uint8)
    out = np.zeros(D, np.float64)
    lib().oracle_dequant_row(packed, D, int(s), int(z), out)
    return out


def cache_row_offset(page: int, Hkv: int, D: int, h: int, kv: int, off: int) -> int:
    return lib().oracle_cache_row_offset(page, Hkv, D, h, kv, off)


def scale_offset(page: int, Hkv: int, h: int, kv: int, off: int) -> int:
    return lib().oracle_scale_offset(page, Hkv, h, kv, off)


def quant_write(k_bits, v_bits, slot_mapping, num_pages: int, b: int, cache=None,
                scales=None, zeros=None, want_y: bool = False, signs=None):
    """Rotate, quantize and place every row. k_bits/v_bits: uint16 [T, Hkv, D]
    bf16 bit patterns. Returns (cache, scales, zeros, y) where y is the fp32
    rotated rows [T, Hkv, 2, D] (or None). Buffers passed in are updated."""
    k = _c(k_bits, np.uint16)
    v = _c(v_bits, np.uint16)
    T, Hkv, D = k.shape
    sm = _c(slot_mapping, np.int64)
    if cache is None:
        cache = np.zeros(num_pages * Hkv * 2 * 16 * D // 2, np.uint8)
    if scales is None:
        scales = np.zeros(num_pages * Hkv * 2 * 16, np.uint16)
    if zeros is None:
        zeros = np.zeros(num_pages * Hkv * 2 * 16, np.uint16)
    assert cache.flags.c_contiguous and scales.flags.c_contiguous and zeros.flags.c_contiguous
    y = np.zeros((T, Hkv, 2, D), np.float32) if want_y else None
    m = sign_mask(signs, D)
    rc = lib().oracle_quant_write(k, v, sm, T, Hkv, D, b, _sp(m), num_pages,
                                  cache.reshape(-1), scales.reshape(-1), zeros.reshape(-1),
                                  y.ctypes.data if y is not None else None)
    if rc != 0:
        raise ValueError(f"oracle_quant_write returned {rc}")
    return cache, scales, zeros, y


# --- attention ------------------------------------------------------------

def attn_rows(q, Krot, Vrot, b: int, scale: float, signs=None) -> np.ndarray:
    q = _c(q, np.float64)
    D = q.size
    Krot = _c(Krot, np.float64).reshape(-1, D)
    Vrot = _c(Vrot, np.float64).reshape(-1, D)
    out = np.zeros(D, np.float64)
    m = sign_mask(signs, D)
    rc = lib().oracle_attn_rows(q, Krot.reshape(-1), Vrot.reshape(-1), Krot.shape[0], D, b, _sp(m),
                                float(scale), out)
    assert rc == 0, rc
    return out


def decode_attn(q_bits, cache, scales, zeros, page_table, context_lens, Hkv: int, b: int,
                num_pages: int, softmax_scale: float = 0.0, signs=None) -> np.ndarray:
    q = _c(q_bits, np.uint16)
    B, Hq, D = q.shape
    pt = _c(page_table, np.int32)
    cl = _c(context_lens, np.int32)
    out = np.zeros((B, Hq, D), np.float64)
    rc = lib().oracle_decode_attn(q.reshape(-1), _c(cache, np.uint8).reshape(-1),
                                  _c(scales, np.uint16).reshape(-1), _c(zeros, np.uint16).reshape(-1),
                                  pt.reshape(-1), cl, B, Hq, Hkv, D, b, _sp(sign_mask(signs, D)),
                                  pt.shape[1], num_pages, float(softmax_scale), out.reshape(-1))
    if rc != 0:
        raise ValueError(f"oracle_decode_attn returned {rc}")
    return out


def decode_one(q_bits, cache, scales, zeros, page_table, context_lens, n: int, hq: int,
               Hkv: int, b: int, num_pages: int, softmax_scale: float = 0.0, signs=None) -> np.ndarray:
    q = _c(q_bits, np.uint16)
    B, Hq, D = q.shape
    pt = _c(page_table, np.int32)
    out = np.zeros(D, np.float64)
    rc = lib().oracle_decode_one(q.reshape(-1), _c(cache, np.uint8).reshape(-1),
                                 _c(scales, np.uint16).reshape(-1), _c(zeros, np.uint16).reshape(-1),
                                 pt.reshape(-1), _c(context_lens, np.int32), n, hq, Hq, Hkv, D, b,
                                 _sp(sign_mask(signs, D)), pt.shape[1], num_pages, float(softmax_scale),
                                 out)
    if rc != 0:
        raise ValueError(f"oracle_decode_one returned {rc}")
    return out


def num_threads() -> int:
    return lib().oracle_num_threads()


def set_num_threads(n: int) -> None:
    """Threads of the oracle's OpenMP loops from now on (timing legs only)."""
    lib().oracle_set_num_threads(int(n))


# --- OScaR (forum summary, "The OScaR Framework": V^ = Quant(S (R V))) -------

OSCAR_TOP = 3  # INT2 codes 0..3


def scale_zero_levels(mn: float, mx: float, top: int):
    """(s, z) fp16 bits: z = largest fp16 <= mn, s = smallest fp16 >= 0 with
    top * s + z >= mx."""
    s_, z_ = ctypes.c_uint16(), ctypes.c_uint16()
    lib().oracle_scale_zero_levels(float(mn), float(mx), int(top), ctypes.byref(s_), ctypes.byref(z_))
    return int(s_.value), int(z_.value)


def oscar_token_norm(y):
    """(n fp16 bits, u fp32 row): the Omni-Token factor of a rotated row."""
    y = _c(y, np.float32)
    u = np.zeros_like(y)
    n = lib().oracle_oscar_token_norm(y, y.size, u)
    return int(n), u


def oscar_codes_given(u, s: int, z: int) -> np.ndarray:
    """INT2 codes (uint8, one per value) of the fp32 values u under the given
    (s, z) fp16 bits: round-half-even(fp32(u - z) * fp32(1/s)) in 0..3."""
    u = _c(u, np.float32)
    out = np.zeros(u.size, np.uint8)
    lib().oracle_oscar_codes_given(u.reshape(-1), u.size, int(s), int(z), out)
    return out.reshape(u.shape)


def oscar_quant_channels(u):
    """Per-channel INT2 quantization of 16 normalized rows u (fp32 [16, D]):
    (codes uint8 [16, D/4], ks, kz fp16 bits [D])."""
    u = _c(u, np.float32)
    D = u.shape[1]
    codes = np.zeros((16, D // 4), np.uint8)
    ks = np.zeros(D, np.uint16)
    kz = np.zeros(D, np.uint16)
    lib().oracle_oscar_quant_channels(u.reshape(-1), D, codes.reshape(-1), ks, kz)
    return codes, ks, kz


def oscar_quant_page(k_bits, v_bits, b: int):
    """One page-head: k_bits, v_bits uint16 [16, D] (bf16). Returns a dict of
    kcodes, vcodes (uint8 [16, D/4]), ks, kz (fp16 bits [D]), kn, vs, vz
    (fp16 bits [16])."""
    k = _c(k_bits, np.uint16)
    v = _c(v_bits, np.uint16)
    D = k.shape[1]
    out = {"kcodes": np.zeros((16, D // 4), np.uint8), "vcodes": np.zeros((16, D // 4), np.uint8),
           "ks": np.zeros(D, np.uint16), "kz": np.zeros(D, np.uint16), "kn": np.zeros(16, np.uint16),
           "vs": np.zeros(16, np.uint16), "vz": np.zeros(16, np.uint16)}
    rc = lib().oracle_oscar_quant_page(k.reshape(-1), v.reshape(-1), D, b, out["kcodes"].reshape(-1),
                                       out["vcodes"].reshape(-1), out["ks"], out["kz"], out["kn"], out["vs"],
                                       out["vz"])
    assert rc == 0, rc
    return out


def oscar_alloc(num_pages: int, Hkv: int, D: int):
    """Zeroed host OScaR pool: cache uint8 [pages][Hkv][2][16][D/4], kmeta
    fp16 bits [pages][Hkv][2][D] (K per-channel s, z), tmeta fp16 bits
    [pages][Hkv][3][16] (K token norm, V s, V z)."""
    return (np.zeros((num_pages, Hkv, 2, 16, D // 4), np.uint8), np.zeros((num_pages, Hkv, 2, D), np.uint16),
            np.zeros((num_pages, Hkv, 3, 16), np.uint16))


def oscar_write(k_bits, v_bits, page_ids, num_pages: int, b: int, pool=None):
    """Token group g (rows 16 g .. 16 g + 15 of k_bits, v_bits: uint16
    [T, Hkv, D]) fills page page_ids[g]. Returns (cache, kmeta, tmeta)."""
    k = _c(k_bits, np.uint16)
    v = _c(v_bits, np.uint16)
    T, Hkv, D = k.shape
    ids = _c(page_ids, np.int32)
    assert T == 16 * ids.size
    cache, kmeta, tmeta = pool if pool is not None else oscar_alloc(num_pages, Hkv, D)
    rc = lib().oracle_oscar_write(k.reshape(-1), v.reshape(-1), ids, ids.size, Hkv, D, b, num_pages,
                                  cache.reshape(-1), kmeta.reshape(-1), tmeta.reshape(-1))
    if rc != 0:
        raise ValueError(f"oracle_oscar_write returned {rc}")
    return cache, kmeta, tmeta


def oscar_dequant_page(cache, kmeta, tmeta, page: int, h: int):
    """Dequantized rotated K, V rows [16, D] (fp64) of one page-head."""
    P, Hkv, _, _, Dq = cache.shape
    D = 4 * Dq
    K = np.zeros((16, D), np.float64)
    V = np.zeros((16, D), np.float64)
    lib().oracle_oscar_dequant_page(_c(cache, np.uint8).reshape(-1), _c(kmeta, np.uint16).reshape(-1),
                                    _c(tmeta, np.uint16).reshape(-1), page, Hkv, D, h, K.reshape(-1),
                                    V.reshape(-1))
    return K, V


def oscar_decode_one(q_bits, cache, kmeta, tmeta, page_table, context_lens, k_tail_bits, v_tail_bits,
                     n: int, hq: int, b: int, softmax_scale: float = 0.0) -> np.ndarray:
    """One (sequence n, query head hq) of the OScaR decode, fp64 [D]."""
    q = _c(q_bits, np.uint16)
    B, Hq, D = q.shape
    P, Hkv = cache.shape[0], cache.shape[1]
    pt = _c(page_table, np.int32)
    out = np.zeros(D, np.float64)
    rc = lib().oracle_oscar_decode_one(q.reshape(-1), _c(cache, np.uint8).reshape(-1),
                                       _c(kmeta, np.uint16).reshape(-1), _c(tmeta, np.uint16).reshape(-1),
                                       pt.reshape(-1), _c(context_lens, np.int32),
                                       _c(k_tail_bits, np.uint16).reshape(-1),
                                       _c(v_tail_bits, np.uint16).reshape(-1), n, hq, Hq, Hkv, D, b,
                                       pt.shape[1], P, float(softmax_scale), out)
    if rc != 0:
        raise ValueError(f"oracle_oscar_decode_one returned {rc}")
    return out


def oscar_decode_attn(q_bits, cache, kmeta, tmeta, page_table, context_lens, k_tail_bits, v_tail_bits,
                      b: int, softmax_scale: float = 0.0) -> np.ndarray:
    """The OScaR decode: full pages from the INT2 pool, the last ctx % 16
    tokens of each sequence from k_tail / v_tail (uint16 [B, Hkv, 16, D]
    bf16). Returns fp64 [B, Hq, D]."""
    q = _c(q_bits, np.uint16)
    B, Hq, D = q.shape
    P, Hkv = cache.shape[0], cache.shape[1]
    pt = _c(page_table, np.int32)
    out = np.zeros((B, Hq, D), np.float64)
    rc = lib().oracle_oscar_decode_attn(q.reshape(-1), _c(cache, np.uint8).reshape(-1),
                                        _c(kmeta, np.uint16).reshape(-1), _c(tmeta, np.uint16).reshape(-1),
                                        pt.reshape(-1), _c(context_lens, np.int32),
                                        _c(k_tail_bits, np.uint16).reshape(-1),
                                        _c(v_tail_bits, np.uint16).reshape(-1), B, Hq, Hkv, D, b, pt.shape[1],
                                        P, float(softmax_scale), out.reshape(-1))
    if rc != 0:
        raise ValueError(f"oracle_oscar_decode_attn returned {rc}")
    return out
