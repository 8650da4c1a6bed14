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
