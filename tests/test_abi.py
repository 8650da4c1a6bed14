"""The C-ABI library loads without a GPU, exports every entry point that
include/kvq.h declares, and rejects bad arguments on the host before it
touches a device (no compute call is made here)."""
import ctypes
import os
import re
import subprocess

import pytest

from helpers import ROOT

HEADER = os.path.join(ROOT, "include", "kvq.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:kvq_status|size_t|const char\s*\*|int32_t)\s+(\w+)\s*\(",
                                 text, flags=re.M)))


@pytest.fixture(scope="module")
def L():
    from bit_kv_cache_20_b200 import build, _lib
    build.build()
    return _lib.lib()


def test_header_declares_the_hot_path():
    names = declared_functions()
    for n in ("kv_quant_write", "paged_decode_attn_int4", "kvq_attn_workspace_size",
              "kvq_get_device_error", "kvq_status_string", "kvq_abi_version"):
        assert n in names


def test_library_exports_every_declared_symbol(L):
    from bit_kv_cache_20_b200 import _lib
    out = subprocess.run(["nm", "-D", "--defined-only", _lib.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(line.split()[-1] for line in out.splitlines() if line.strip())
    for name in declared_functions():
        assert name in exported, name
        assert getattr(L, name) is not None
    # the binding declares a prototype for each of them
    assert set(n for n, _, _ in _lib.SIGNATURES) == set(declared_functions())


def test_version_and_status_strings(L):
    assert L.kvq_abi_version() == 6
    assert L.kvq_status_string(0) == b"KVQ_OK"
    assert L.kvq_status_string(5) == b"KVQ_ERR_TIMEOUT"
    assert L.kvq_status_string(99) == b"KVQ_ERR_UNKNOWN"


FAKE = 1 << 20  # a 16-byte aligned non-null address; never dereferenced here


def write_call(L, desc, k=FAKE, v=FAKE, slots=FAKE, cache=FAKE, s=FAKE, z=FAKE, b=32):
    from bit_kv_cache_20_b200 import _lib
    P = ctypes.c_void_p
    return L.kv_quant_write(P(k), P(v), P(slots), None, P(cache), P(s), P(z), b,
                            ctypes.byref(desc) if desc is not None else None, None)


def test_write_argument_errors(L):
    from bit_kv_cache_20_b200._lib import WriteDesc
    assert write_call(L, None) == 1
    assert write_call(L, WriteDesc(4, 2, 96, 16, 4)) == 2          # head_dim
    assert write_call(L, WriteDesc(4, 2, 64, 16, 4), b=16) == 2     # block size
    assert write_call(L, WriteDesc(4, 2, 64, 16, 4), b=128) == 2    # block > head_dim
    assert write_call(L, WriteDesc(4, 2, 64, 8, 4)) == 1            # page size
    assert write_call(L, WriteDesc(-1, 2, 64, 16, 4)) == 1
    assert write_call(L, WriteDesc(4, 0, 64, 16, 4)) == 1
    assert write_call(L, WriteDesc(4, 2, 64, 16, 0)) == 1
    assert write_call(L, WriteDesc(4, 2, 64, 16, 4), k=0) == 1      # null
    assert write_call(L, WriteDesc(4, 2, 64, 16, 4), cache=FAKE + 8) == 1  # misaligned
    assert write_call(L, WriteDesc(0, 2, 64, 16, 4)) == 0           # nothing to do
    sg = ctypes.c_uint32 * 4
    assert write_call(L, WriteDesc(4, 2, 64, 16, 4, sg(0, 0, 2, 0)), b=64) == 1  # sign of channel 65 > D
    assert write_call(L, WriteDesc(4, 2, 64, 16, 4, sg(1, 0, 0, 0)), b=0) == 1   # signs without a rotation


def attn_call(L, desc, ws=None, ws_bytes=0, out=FAKE):
    P = ctypes.c_void_p
    return L.paged_decode_attn_int4(P(FAKE), P(FAKE), P(FAKE), P(FAKE), P(FAKE), P(FAKE), P(out),
                                    P(ws) if ws else None, ws_bytes,
                                    ctypes.byref(desc) if desc is not None else None, None)


def test_decode_argument_errors(L):
    from bit_kv_cache_20_b200._lib import AttnDesc
    ok = dict(batch=2, num_q_heads=8, num_kv_heads=2, head_dim=128, page_size=16, num_pages=10,
              max_pages_per_seq=5, hadamard_block=128, softmax_scale=0.0, out_dtype=0, flags=0,
              context_lens_host=None, hadamard_signs=(ctypes.c_uint32 * 4)(0, 0, 0, 0))

    def d(**kw):
        a = dict(ok)
        a.update(kw)
        return AttnDesc(*a.values())

    assert attn_call(L, None) == 1
    assert attn_call(L, d(num_q_heads=6, num_kv_heads=4)) == 1     # Hq not a multiple of Hkv
    assert attn_call(L, d(num_q_heads=32, num_kv_heads=2)) == 2    # GQA group 16
    assert attn_call(L, d(head_dim=96)) == 2
    assert attn_call(L, d(hadamard_block=48)) == 2
    assert attn_call(L, d(page_size=32)) == 1
    assert attn_call(L, d(softmax_scale=-1.0)) == 1
    assert attn_call(L, d(out_dtype=3)) == 1
    assert attn_call(L, d(flags=2)) == 1                            # unknown flag bit
    assert attn_call(L, d(hadamard_block=0, hadamard_signs=(ctypes.c_uint32 * 4)(1, 0, 0, 0))) == 1
    assert attn_call(L, d(head_dim=64, hadamard_block=64,
                          hadamard_signs=(ctypes.c_uint32 * 4)(0, 0, 1, 0))) == 1  # channel 64 of D = 64
    assert attn_call(L, d(max_pages_per_seq=0)) == 1
    assert attn_call(L, d(), out=FAKE + 2) == 1                     # fp32 out misaligned
    assert attn_call(L, d(batch=0)) == 0                            # nothing to do
    size_max = ctypes.c_size_t(-1).value
    assert L.kvq_attn_workspace_size(ctypes.byref(d(head_dim=96))) == size_max


def _desc(**kw):
    from bit_kv_cache_20_b200._lib import AttnDesc
    a = dict(batch=2, num_q_heads=8, num_kv_heads=2, head_dim=128, page_size=16, num_pages=10,
             max_pages_per_seq=5, hadamard_block=128, softmax_scale=0.0, out_dtype=0, flags=0,
             context_lens_host=None, hadamard_signs=(ctypes.c_uint32 * 4)(0, 0, 0, 0))
    a.update(kw)
    return AttnDesc(*a.values())


def append_call(L, desc, k=FAKE, v=FAKE, slots=FAKE):
    P = ctypes.c_void_p
    return L.paged_decode_append_attn_int4(P(FAKE), P(k), P(v), P(slots), P(FAKE), P(FAKE), P(FAKE),
                                           P(FAKE), P(FAKE), P(FAKE), None, 0,
                                           ctypes.byref(desc) if desc is not None else None, None)


def test_append_argument_errors(L):
    assert append_call(L, None) == 1
    assert append_call(L, _desc(), k=0) == 1                        # no new K
    assert append_call(L, _desc(), v=FAKE + 8) == 1                 # misaligned V
    assert append_call(L, _desc(), slots=FAKE + 4) == 1             # misaligned slot_mapping
    assert append_call(L, _desc(head_dim=96)) == 2                  # as the decode
    assert append_call(L, _desc(batch=0), k=0, v=0, slots=0) == 0   # nothing to do


def prefill_call(L, desc, max_q=64, q=FAKE, q_start=FAKE, out=FAKE):
    P = ctypes.c_void_p
    return L.paged_prefill_attn_int4(P(q), P(FAKE), P(FAKE), P(FAKE), P(FAKE), P(FAKE), P(q_start), max_q,
                                     P(out), ctypes.byref(desc) if desc is not None else None, None)


def test_prefill_argument_errors(L):
    assert prefill_call(L, None) == 1
    assert prefill_call(L, _desc(head_dim=96)) == 2                      # as the decode
    assert prefill_call(L, _desc(num_q_heads=32, num_kv_heads=2)) == 2   # GQA group 16
    assert prefill_call(L, _desc(hadamard_block=48)) == 2
    assert prefill_call(L, _desc(), max_q=-1) == 1
    assert prefill_call(L, _desc(), q_start=0) == 1                      # null
    assert prefill_call(L, _desc(), q=FAKE + 8) == 1                     # misaligned q
    assert prefill_call(L, _desc(out_dtype=1), out=FAKE + 1) == 1        # misaligned bf16 out
    assert prefill_call(L, _desc(batch=0)) == 0                          # nothing to do
    assert prefill_call(L, _desc(), max_q=0) == 0


def test_binding_fails_loudly_without_the_library(tmp_path, monkeypatch):
    from bit_kv_cache_20_b200 import _lib
    monkeypatch.setattr(_lib, "LIB_PATH", str(tmp_path / "missing.so"))
    monkeypatch.setattr(_lib, "_lib", None)
    with pytest.raises(ImportError):
        _lib.lib()
