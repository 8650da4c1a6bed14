"""ctypes view of libkvq.so (the C ABI in include/kvq.h). Argument marshalling
only; every step of the path runs in the library's kernels."""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libkvq.so")

KVQ_OK = 0
STATUS_NAMES = {
    0: "KVQ_OK", 1: "KVQ_ERR_INVALID_ARG", 2: "KVQ_ERR_UNSUPPORTED", 3: "KVQ_ERR_OUT_OF_RANGE",
    4: "KVQ_ERR_WORKSPACE", 5: "KVQ_ERR_TIMEOUT", 6: "KVQ_ERR_CUDA",
}


class WriteDesc(ctypes.Structure):
    _fields_ = [("num_tokens", ctypes.c_int32), ("num_kv_heads", ctypes.c_int32),
                ("head_dim", ctypes.c_int32), ("page_size", ctypes.c_int32),
                ("num_pages", ctypes.c_int32), ("hadamard_signs", ctypes.c_uint32 * 4)]


class AttnDesc(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int32), ("num_q_heads", ctypes.c_int32),
                ("num_kv_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
                ("page_size", ctypes.c_int32), ("num_pages", ctypes.c_int32),
                ("max_pages_per_seq", ctypes.c_int32), ("hadamard_block", ctypes.c_int32),
                ("softmax_scale", ctypes.c_float), ("out_dtype", ctypes.c_int32),
                ("flags", ctypes.c_int32), ("context_lens_host", ctypes.POINTER(ctypes.c_int32)),
                ("hadamard_signs", ctypes.c_uint32 * 4)]


class OscarWriteDesc(ctypes.Structure):
    _fields_ = [("num_groups", ctypes.c_int32), ("num_kv_heads", ctypes.c_int32),
                ("head_dim", ctypes.c_int32), ("num_pages", ctypes.c_int32)]


class OscarAttnDesc(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int32), ("num_q_heads", ctypes.c_int32),
                ("num_kv_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
                ("num_pages", ctypes.c_int32), ("max_pages_per_seq", ctypes.c_int32),
                ("hadamard_block", ctypes.c_int32), ("softmax_scale", ctypes.c_float),
                ("out_dtype", ctypes.c_int32)]


ATTN_INPUTS_READY = 1  # KVQ_ATTN_INPUTS_READY


class KVQError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {STATUS_NAMES.get(status, status)}")


_lib = None

# (name, restype, argtypes) of every entry point declared in include/kvq.h
SIGNATURES = [
    ("kv_quant_write", ctypes.c_int, [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                      ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int32,
                                      ctypes.POINTER(WriteDesc), ctypes.c_void_p]),
    ("kvq_attn_workspace_size", ctypes.c_size_t, [ctypes.POINTER(AttnDesc)]),
    ("paged_decode_attn_int4", ctypes.c_int, [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                              ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                              ctypes.c_void_p, ctypes.c_void_p, ctypes.c_size_t,
                                              ctypes.POINTER(AttnDesc), ctypes.c_void_p]),
    ("paged_decode_append_attn_int4", ctypes.c_int, [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                                     ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                                     ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                                     ctypes.c_void_p, ctypes.c_void_p, ctypes.c_size_t,
                                                     ctypes.POINTER(AttnDesc), ctypes.c_void_p]),
    ("paged_prefill_attn_int4", ctypes.c_int, [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                               ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                               ctypes.c_void_p, ctypes.c_int32, ctypes.c_void_p,
                                               ctypes.POINTER(AttnDesc), ctypes.c_void_p]),
    ("paged_decode_attn_int4_static_ws", ctypes.c_int, [ctypes.c_void_p, ctypes.c_void_p,
                                                        ctypes.c_void_p, ctypes.c_void_p,
                                                        ctypes.c_void_p, ctypes.c_void_p,
                                                        ctypes.c_void_p, ctypes.POINTER(AttnDesc),
                                                        ctypes.c_void_p]),
    ("kv_quant_write_oscar", ctypes.c_int, [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                            ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int32,
                                            ctypes.POINTER(OscarWriteDesc), ctypes.c_void_p]),
    ("kvq_oscar_workspace_size", ctypes.c_size_t, [ctypes.POINTER(OscarAttnDesc)]),
    ("paged_decode_attn_oscar", ctypes.c_int, [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                               ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                               ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                               ctypes.c_void_p, ctypes.c_size_t, ctypes.POINTER(OscarAttnDesc),
                                               ctypes.c_void_p]),
    ("kvq_get_device_error", ctypes.c_int, [ctypes.c_void_p]),
    ("kvq_selftest_bounded_wait", ctypes.c_int, [ctypes.c_int32, ctypes.c_void_p]),
    ("kvq_selftest_occupy", ctypes.c_int, [ctypes.c_int32, ctypes.c_int32, ctypes.c_void_p]),
    ("kvq_static_workspace_nonzero", ctypes.c_size_t, []),
    ("kvq_set_device", ctypes.c_int, [ctypes.c_int32]),
    ("kvq_status_string", ctypes.c_char_p, [ctypes.c_int32]),
    ("kvq_abi_version", ctypes.c_int32, []),
]


def lib():
    """Load libkvq.so; raise if it has not been built (there is no fallback)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(
                f"{LIB_PATH} is missing: build the CUDA library first "
                "(python -m bit_kv_cache_20_b200.build)")
        L = ctypes.CDLL(LIB_PATH)
        for name, res, args in SIGNATURES:
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def check(status: int, where: str) -> None:
    if status != KVQ_OK:
        raise KVQError(status, where)
