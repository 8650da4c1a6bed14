"""Shared helpers for the test suite (fixture parsing, comparisons)."""
import os

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def golden(name):
    """Parse a tests/golden fixture: '# ...' comment lines, then 'key = value'
    lines; repeated keys collect into lists."""
    out = {}
    with open(os.path.join(ROOT, "tests", "golden", name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, val = (s.strip() for s in line.split("=", 1))
            if key in out:
                if not isinstance(out[key], list):
                    out[key] = [out[key]]
                out[key].append(val)
            else:
                out[key] = val
    return out


def parse_bytes(spec):
    """'10 32 FE' or 'FF*32 00*32' -> list of ints."""
    res = []
    for tok in spec.split():
        if "*" in tok:
            v, n = tok.split("*")
            res += [int(v, 16)] * int(n)
        else:
            res.append(int(tok, 16))
    return res


# ----------------------------------------------------------------------------
# comparison of the CUDA write path with the oracle
# ----------------------------------------------------------------------------
import math as _math

import numpy as _np


def f16_ordinal(bits):
    """binary16 patterns mapped to integers in value order (-0 and +0 -> 0)."""
    b = _np.asarray(bits, _np.uint16).astype(_np.int64)
    mag = b & 0x7FFF
    return _np.where(b & 0x8000, -mag, mag)


def f16_bits_to_float(bits):
    return _np.asarray(bits, _np.uint16).view(_np.float16).astype(_np.float64)


def write_window(x_rows, b, s_bits):
    """Per-row width (in code units) of the band around a rounding boundary in
    which the kernel's fp32 butterfly may legitimately land on the other code
    than the oracle's once-rounded fp64 rotation: the butterfly's rounding
    error bound (log2(b) + 1 roundings of at most 2^-24 times the block's sum
    of |x|, times 1/sqrt(b)), divided by the step s. Zero when b = 0: then
    the rotated row is the bf16 input itself on both sides."""
    if b == 0:
        return _np.zeros(x_rows.shape[0])
    n, D = x_rows.shape
    blocks = _np.abs(x_rows).reshape(n, D // b, b).sum(axis=2).max(axis=1)
    bound_y = (_math.log2(b) + 2) * 2.0 ** -24 * blocks / _math.sqrt(b)
    s = f16_bits_to_float(s_bits)
    with _np.errstate(divide="ignore", invalid="ignore"):
        w = _np.where(s > 0, bound_y / s, 0.0)
    return w + 2.0 ** -19


def compare_write_rows(orc, y_oracle, x_rows, b, gpu_packed, gpu_s, gpu_z, D):
    """Compare GPU rows (packed codes, s, z) with the oracle's rotated rows.

    Returns a dict of counts. Asserts: s and z within 1 fp16 ulp (identical
    when b = 0); every code equal to the oracle's quantization of its rotated
    row under the GPU's (s, z), except where the oracle's quotient lies within
    the rounding window of a half-integer."""
    n = y_oracle.shape[0]
    s_o = _np.zeros(n, _np.uint16)
    z_o = _np.zeros(n, _np.uint16)
    mism = near = 0
    win = write_window(x_rows, b, gpu_s)
    for i in range(n):
        codes_o, s_o[i], z_o[i] = orc.quantize_row(y_oracle[i])
    ds = _np.abs(f16_ordinal(s_o) - f16_ordinal(gpu_s))
    dz = _np.abs(f16_ordinal(z_o) - f16_ordinal(gpu_z))
    if b == 0:
        assert _np.array_equal(s_o, gpu_s) and _np.array_equal(z_o, gpu_z), "s/z differ with b = 0"
    assert ds.max(initial=0) <= 1 and dz.max(initial=0) <= 1, (ds.max(), dz.max())
    gpu_codes = _np.empty((n, D), _np.uint8)
    gpu_codes[:, 0::2] = gpu_packed & 15
    gpu_codes[:, 1::2] = gpu_packed >> 4
    for i in range(n):
        ref = orc.quantize_given(y_oracle[i], int(gpu_s[i]), int(gpu_z[i]))
        bad = _np.nonzero(ref != gpu_codes[i])[0]
        if bad.size:
            q = orc.quotient_given(y_oracle[i], int(gpu_s[i]), int(gpu_z[i]))[bad]
            dist = _np.abs(q - (_np.floor(q) + 0.5))
            assert _np.all(dist <= win[i]), (i, bad, q, win[i])
            assert _np.all(_np.abs(ref[bad].astype(int) - gpu_codes[i, bad].astype(int)) == 1)
            mism += bad.size
            near += bad.size
    return {"rows": n, "elements": n * D, "code_mismatch_near_boundary": mism,
            "s_ulp_diff": int((ds > 0).sum()), "z_ulp_diff": int((dz > 0).sum())}
