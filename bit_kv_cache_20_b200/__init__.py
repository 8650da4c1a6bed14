"""Rotated-INT4 paged KV cache for B200 (sm_100a).

Python binding of the C ABI in include/kvq.h: torch tensors in, pointers and
sizes out, the current CUDA stream by default. The two hot-path calls are

    kv_quant_write(k, v, slot_mapping, cache, scales, zeros, hadamard_block)
    paged_decode_attn_int4(q, cache, scales, zeros, page_table, context_lens,
                           out, hadamard_block)

Every step runs in the library's kernels; if libkvq.so is missing the calls
raise (there is no CPU or PyTorch fallback).
"""
from __future__ import annotations

import ctypes
from typing import Optional, Tuple

import numpy as np
import torch

from . import _lib
from ._lib import ATTN_INPUTS_READY, AttnDesc, KVQError, OscarAttnDesc, OscarWriteDesc, WriteDesc

PAGE_SIZE = 16

__all__ = [
    "PAGE_SIZE", "KVQError", "alloc_cache", "kv_quant_write", "paged_decode_attn_int4",
    "attn_workspace_size", "alloc_workspace", "get_device_error", "selftest_bounded_wait", "library_path",
    "paged_decode_attn_int4_static_ws", "paged_decode_append_attn_int4", "paged_prefill_attn_int4",
    "sign_words", "selftest_occupy", "alloc_oscar_cache", "kv_quant_write_oscar", "oscar_workspace_size",
    "paged_decode_attn_oscar",
]


def library_path() -> str:
    return _lib.LIB_PATH


def _stream_handle(stream) -> int:
    if stream is None:
        stream = torch.cuda.current_stream()
    return int(stream.cuda_stream) if hasattr(stream, "cuda_stream") else int(stream)


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _need(t: torch.Tensor, name: str, dtype) -> None:
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_cuda:
        raise ValueError(f"{name} must live on a CUDA device")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def alloc_cache(num_pages: int, num_kv_heads: int, head_dim: int,
                device="cuda") -> Tuple[torch.Tensor, torch.Tensor, torch.Tensor]:
    """Empty pool: cache uint8 [pages, Hkv, 2, 16, D/2], scales and zeros
    fp16 [pages, Hkv, 2, 16]."""
    cache = torch.zeros((num_pages, num_kv_heads, 2, PAGE_SIZE, head_dim // 2), dtype=torch.uint8,
                        device=device)
    scales = torch.zeros((num_pages, num_kv_heads, 2, PAGE_SIZE), dtype=torch.float16, device=device)
    zeros = torch.zeros_like(scales)
    return cache, scales, zeros


def _pool_shape(cache, scales, zeros):
    _need(cache, "cache", torch.uint8)
    _need(scales, "scales", torch.float16)
    _need(zeros, "zeros", torch.float16)
    if cache.dim() != 5 or cache.shape[2] != 2 or cache.shape[3] != PAGE_SIZE:
        raise ValueError("cache must be uint8 [num_pages, Hkv, 2, 16, D/2]")
    P, Hkv = int(cache.shape[0]), int(cache.shape[1])
    D = int(cache.shape[4]) * 2
    if tuple(scales.shape) != (P, Hkv, 2, PAGE_SIZE) or tuple(zeros.shape) != tuple(scales.shape):
        raise ValueError("scales/zeros must be fp16 [num_pages, Hkv, 2, 16]")
    return P, Hkv, D


def kv_quant_write(k: torch.Tensor, v: torch.Tensor, slot_mapping: torch.Tensor,
                   cache: torch.Tensor, scales: torch.Tensor, zeros: torch.Tensor,
                   hadamard_block: int, page_table: Optional[torch.Tensor] = None,
                   stream=None, hadamard_signs=None) -> None:
    """Rotate (block Hadamard), quantize (token-wise INT4) and store new K/V
    rows [T, Hkv, D] (bf16) at slot_mapping (int64 [T], -1 = skip).
    hadamard_signs: optional per-channel booleans for the randomized rotation
    H_b diag(sigma) / sqrt(b) (decode with the same signs)."""
    P, Hkv, D = _pool_shape(cache, scales, zeros)
    _need(k, "k", torch.bfloat16)
    _need(v, "v", torch.bfloat16)
    _need(slot_mapping, "slot_mapping", torch.int64)
    if k.dim() != 3 or tuple(k.shape[1:]) != (Hkv, D) or k.shape != v.shape:
        raise ValueError("k and v must be bf16 [T, Hkv, D] matching the cache")
    T = int(k.shape[0])
    if slot_mapping.numel() != T:
        raise ValueError("slot_mapping must hold one slot per token")
    desc = WriteDesc(T, Hkv, D, PAGE_SIZE, P, sign_words(hadamard_signs, D))
    st = _lib.lib().kv_quant_write(_ptr(k), _ptr(v), _ptr(slot_mapping), _ptr(page_table),
                                   _ptr(cache), _ptr(scales), _ptr(zeros), int(hadamard_block),
                                   ctypes.byref(desc), ctypes.c_void_p(_stream_handle(stream)))
    _lib.check(st, "kv_quant_write")


def sign_words(signs, head_dim: int):
    """The 4-word mask of a randomized-Hadamard sign vector: `signs` holds
    head_dim booleans (True negates that channel before the transform), or is
    None (no signs)."""
    words = (ctypes.c_uint32 * 4)(0, 0, 0, 0)
    if signs is None:
        return words
    a = np.asarray(signs.cpu() if isinstance(signs, torch.Tensor) else signs).astype(bool).reshape(-1)
    if a.size != head_dim:
        raise ValueError("hadamard_signs must hold one entry per channel")
    for c in np.nonzero(a)[0]:
        words[int(c) // 32] |= 1 << (int(c) % 32)
    return words


def _host_lengths(context_lens_host, batch):
    """int32 host array of the context lengths (kept alive by the caller) and
    its pointer, or (None, None)."""
    if context_lens_host is None:
        return None, None
    arr = np.ascontiguousarray(np.asarray(context_lens_host, dtype=np.int32))
    if arr.shape != (batch,):
        raise ValueError("context_lens_host must hold one length per sequence")
    return arr, arr.ctypes.data_as(ctypes.POINTER(ctypes.c_int32))


def _attn_desc(q, cache, scales, zeros, page_table, hadamard_block, softmax_scale, out_dtype,
               inputs_ready=False, lens_ptr=None, signs=None):
    P, Hkv, D = _pool_shape(cache, scales, zeros)
    if q.dim() != 3 or int(q.shape[2]) != D:
        raise ValueError("q must be bf16 [B, Hq, D]")
    B, Hq = int(q.shape[0]), int(q.shape[1])
    if page_table.dim() != 2 or int(page_table.shape[0]) != B:
        raise ValueError("page_table must be int32 [B, max_pages]")
    return AttnDesc(B, Hq, Hkv, D, PAGE_SIZE, P, int(page_table.shape[1]), int(hadamard_block),
                    float(softmax_scale), out_dtype, ATTN_INPUTS_READY if inputs_ready else 0,
                    lens_ptr, sign_words(signs, D))


def attn_workspace_size(batch: int, num_q_heads: int, num_kv_heads: int, head_dim: int,
                        num_pages: int, max_pages_per_seq: int, hadamard_block: int,
                        device=None, host_lengths: bool = False) -> int:
    """Bytes of workspace paged_decode_attn_int4 needs on `device` (default:
    torch's current CUDA device); with host_lengths, enough for calls that pass
    context_lens_host (a per-sequence plan), whatever the lengths."""
    L = _lib.lib()
    idx = None if device is None else torch.device(device).index
    dev = torch.cuda.current_device() if idx is None else idx
    _lib.check(L.kvq_set_device(int(dev)), "kvq_set_device")
    dummy = (ctypes.c_int32 * 1)(0)
    desc = AttnDesc(batch, num_q_heads, num_kv_heads, head_dim, PAGE_SIZE, num_pages,
                    max_pages_per_seq, hadamard_block, 0.0, 0, 0,
                    ctypes.cast(dummy, ctypes.POINTER(ctypes.c_int32)) if host_lengths else None)
    n = L.kvq_attn_workspace_size(ctypes.byref(desc))
    if n == ctypes.c_size_t(-1).value:
        raise KVQError(1, "kvq_attn_workspace_size (invalid shapes or no device)")
    return int(n)


def alloc_workspace(nbytes: int, device="cuda") -> torch.Tensor:
    """A zero-filled workspace (the decode call keeps it zero between calls)."""
    return torch.zeros(max(int(nbytes), 16), dtype=torch.uint8, device=device)


def paged_decode_attn_int4(q: torch.Tensor, cache: torch.Tensor, scales: torch.Tensor,
                           zeros: torch.Tensor, page_table: torch.Tensor,
                           context_lens: torch.Tensor, out: torch.Tensor, hadamard_block: int,
                           workspace: Optional[torch.Tensor] = None, softmax_scale: float = 0.0,
                           stream=None, inputs_ready: bool = False,
                           context_lens_host=None, hadamard_signs=None) -> None:
    """One decode step over the INT4 cache; out is fp32 or bf16 [B, Hq, D].
    inputs_ready: q, page_table and context_lens were not written by the
    kernel launched just before this call on the stream (KVQ_ATTN_INPUTS_READY),
    so the call may read them while that kernel finishes.
    context_lens_host: an optional host copy of the context lengths; the work
    is then split per sequence in proportion to its length (size the workspace
    with attn_workspace_size(..., host_lengths=True))."""
    _need(q, "q", torch.bfloat16)
    _need(page_table, "page_table", torch.int32)
    _need(context_lens, "context_lens", torch.int32)
    if out.dtype not in (torch.float32, torch.bfloat16):
        raise TypeError("out must be float32 or bfloat16")
    _need(out, "out", out.dtype)
    if tuple(out.shape) != tuple(q.shape):
        raise ValueError("out must have q's shape")
    lens_arr, lens_ptr = _host_lengths(context_lens_host, int(q.shape[0]) if q.dim() == 3 else -1)
    desc = _attn_desc(q, cache, scales, zeros, page_table, hadamard_block, softmax_scale,
                      0 if out.dtype == torch.float32 else 1, inputs_ready, lens_ptr, hadamard_signs)
    if context_lens.numel() != desc.batch:
        raise ValueError("context_lens must hold one length per sequence")
    L = _lib.lib()
    ws_ptr, ws_bytes = None, 0
    if workspace is not None:
        _need(workspace, "workspace", torch.uint8)
        ws_ptr, ws_bytes = _ptr(workspace), workspace.numel()
    st = L.paged_decode_attn_int4(_ptr(q), _ptr(cache), _ptr(scales), _ptr(zeros), _ptr(page_table),
                                  _ptr(context_lens), _ptr(out), ws_ptr, ws_bytes,
                                  ctypes.byref(desc), ctypes.c_void_p(_stream_handle(stream)))
    _lib.check(st, "paged_decode_attn_int4")


def selftest_occupy(ctas: int, microseconds: int, stream=None) -> None:
    """Test hook: `ctas` CTAs that each hold most of an SM's shared memory and
    end on their own after `microseconds`, launched on `stream`."""
    _lib.check(_lib.lib().kvq_selftest_occupy(int(ctas), int(microseconds),
                                              ctypes.c_void_p(_stream_handle(stream))),
               "kvq_selftest_occupy")


def paged_decode_append_attn_int4(q: torch.Tensor, k_new: torch.Tensor, v_new: torch.Tensor,
                                  slot_mapping: torch.Tensor, cache: torch.Tensor,
                                  scales: torch.Tensor, zeros: torch.Tensor,
                                  page_table: torch.Tensor, context_lens: torch.Tensor,
                                  out: torch.Tensor, hadamard_block: int,
                                  workspace: Optional[torch.Tensor] = None,
                                  softmax_scale: float = 0.0, stream=None,
                                  inputs_ready: bool = False, context_lens_host=None,
                                  hadamard_signs=None) -> None:
    """One decode step that first appends each sequence's new token: k_new,
    v_new bf16 [B, Hkv, D] are rotated, quantized and stored at slot_mapping
    (int64 [B], -1 = no new token), position context_lens - 1 of their
    sequence, and the attention runs over contexts that include them - one
    launch instead of kv_quant_write + paged_decode_attn_int4."""
    _need(q, "q", torch.bfloat16)
    _need(k_new, "k_new", torch.bfloat16)
    _need(v_new, "v_new", torch.bfloat16)
    _need(slot_mapping, "slot_mapping", torch.int64)
    _need(page_table, "page_table", torch.int32)
    _need(context_lens, "context_lens", torch.int32)
    if out.dtype not in (torch.float32, torch.bfloat16):
        raise TypeError("out must be float32 or bfloat16")
    _need(out, "out", out.dtype)
    if tuple(out.shape) != tuple(q.shape):
        raise ValueError("out must have q's shape")
    lens_arr, lens_ptr = _host_lengths(context_lens_host, int(q.shape[0]) if q.dim() == 3 else -1)
    desc = _attn_desc(q, cache, scales, zeros, page_table, hadamard_block, softmax_scale,
                      0 if out.dtype == torch.float32 else 1, inputs_ready, lens_ptr, hadamard_signs)
    if context_lens.numel() != desc.batch or slot_mapping.numel() != desc.batch:
        raise ValueError("context_lens and slot_mapping must hold one entry per sequence")
    if tuple(k_new.shape) != (desc.batch, desc.num_kv_heads, desc.head_dim) or k_new.shape != v_new.shape:
        raise ValueError("k_new and v_new must be bf16 [B, Hkv, D]")
    ws_ptr, ws_bytes = None, 0
    if workspace is not None:
        _need(workspace, "workspace", torch.uint8)
        ws_ptr, ws_bytes = _ptr(workspace), workspace.numel()
    st = _lib.lib().paged_decode_append_attn_int4(
        _ptr(q), _ptr(k_new), _ptr(v_new), _ptr(slot_mapping), _ptr(cache), _ptr(scales), _ptr(zeros),
        _ptr(page_table), _ptr(context_lens), _ptr(out), ws_ptr, ws_bytes, ctypes.byref(desc),
        ctypes.c_void_p(_stream_handle(stream)))
    _lib.check(st, "paged_decode_append_attn_int4")


def paged_prefill_attn_int4(q: torch.Tensor, cache: torch.Tensor, scales: torch.Tensor,
                            zeros: torch.Tensor, page_table: torch.Tensor, context_lens: torch.Tensor,
                            q_start: torch.Tensor, max_q_len: int, out: torch.Tensor, hadamard_block: int,
                            softmax_scale: float = 0.0, stream=None, hadamard_signs=None) -> None:
    """Chunked-prefill attention over the INT4 cache (head_dim 128): q, bf16
    [Tq, Hq, D], holds for sequence n the queries of its last
    q_start[n + 1] - q_start[n] context tokens (q_start int32 [B + 1]), which
    the cache already holds; each attends causally to its own position and
    everything before it. out: fp32 or bf16 [Tq, Hq, D]."""
    _need(q, "q", torch.bfloat16)
    _need(page_table, "page_table", torch.int32)
    _need(context_lens, "context_lens", torch.int32)
    _need(q_start, "q_start", torch.int32)
    if out.dtype not in (torch.float32, torch.bfloat16):
        raise TypeError("out must be float32 or bfloat16")
    _need(out, "out", out.dtype)
    if tuple(out.shape) != tuple(q.shape) or q.dim() != 3:
        raise ValueError("q and out must be [Tq, Hq, D]")
    P, Hkv, D = _pool_shape(cache, scales, zeros)
    B = int(context_lens.numel())
    if q_start.numel() != B + 1 or page_table.dim() != 2 or int(page_table.shape[0]) != B:
        raise ValueError("q_start must hold B + 1 offsets and page_table B rows")
    desc = AttnDesc(B, int(q.shape[1]), Hkv, D, PAGE_SIZE, P, int(page_table.shape[1]), int(hadamard_block),
                    float(softmax_scale), 0 if out.dtype == torch.float32 else 1, 0, None,
                    sign_words(hadamard_signs, D))
    st = _lib.lib().paged_prefill_attn_int4(
        _ptr(q), _ptr(cache), _ptr(scales), _ptr(zeros), _ptr(page_table), _ptr(context_lens),
        _ptr(q_start), int(max_q_len), _ptr(out), ctypes.byref(desc), ctypes.c_void_p(_stream_handle(stream)))
    _lib.check(st, "paged_prefill_attn_int4")


def paged_decode_attn_int4_static_ws(q: torch.Tensor, cache: torch.Tensor, scales: torch.Tensor,
                                     zeros: torch.Tensor, page_table: torch.Tensor,
                                     context_lens: torch.Tensor, out: torch.Tensor,
                                     hadamard_block: int, softmax_scale: float = 0.0,
                                     stream=None, context_lens_host=None, hadamard_signs=None) -> None:
    """paged_decode_attn_int4 for callers that must not allocate device memory
    (e.g. a plug-in whose host runtime owns all GPU memory): the split-K
    scratch is a fixed array inside the library, shared by every call on the
    device, so calls must not overlap on the GPU. The first call on a device
    looks up that array's address; make it before any stream capture."""
    _need(q, "q", torch.bfloat16)
    _need(page_table, "page_table", torch.int32)
    _need(context_lens, "context_lens", torch.int32)
    if out.dtype not in (torch.float32, torch.bfloat16):
        raise TypeError("out must be float32 or bfloat16")
    _need(out, "out", out.dtype)
    if tuple(out.shape) != tuple(q.shape):
        raise ValueError("out must have q's shape")
    lens_arr, lens_ptr = _host_lengths(context_lens_host, int(q.shape[0]) if q.dim() == 3 else -1)
    desc = _attn_desc(q, cache, scales, zeros, page_table, hadamard_block, softmax_scale,
                      0 if out.dtype == torch.float32 else 1, False, lens_ptr, hadamard_signs)
    if context_lens.numel() != desc.batch:
        raise ValueError("context_lens must hold one length per sequence")
    st = _lib.lib().paged_decode_attn_int4_static_ws(
        _ptr(q), _ptr(cache), _ptr(scales), _ptr(zeros), _ptr(page_table), _ptr(context_lens),
        _ptr(out), ctypes.byref(desc), ctypes.c_void_p(_stream_handle(stream)))
    _lib.check(st, "paged_decode_attn_int4_static_ws")


def selftest_bounded_wait(which: int, stream=None) -> None:
    """Run one of the library's bounded waits on a condition that nothing
    completes (0: an mbarrier wait, 1: the split-merge poll): it runs out
    within seconds and records KVQ_ERR_TIMEOUT (read it with
    get_device_error). For tests of the failure path."""
    _lib.check(_lib.lib().kvq_selftest_bounded_wait(int(which), ctypes.c_void_p(_stream_handle(stream))),
               "kvq_selftest_bounded_wait")


def get_device_error(stream=None) -> int:
    """Synchronize the stream and return (and clear) the device error word."""
    return int(_lib.lib().kvq_get_device_error(ctypes.c_void_p(_stream_handle(stream))))


# --- OScaR variant: INT2, K per channel after a per-token scale -------------

def alloc_oscar_cache(num_pages: int, num_kv_heads: int, head_dim: int, device="cuda"):
    """Empty OScaR pool: cache uint8 [pages, Hkv, 2, 16, D/4] (K then V
    codes), kmeta fp16 [pages, Hkv, 2, D] (K per-channel s, z), tmeta fp16
    [pages, Hkv, 3, 16] (K token norms, V s, V z)."""
    return (torch.zeros((num_pages, num_kv_heads, 2, PAGE_SIZE, head_dim // 4), dtype=torch.uint8, device=device),
            torch.zeros((num_pages, num_kv_heads, 2, head_dim), dtype=torch.float16, device=device),
            torch.zeros((num_pages, num_kv_heads, 3, PAGE_SIZE), dtype=torch.float16, device=device))


def _oscar_pool(cache, kmeta, tmeta):
    _need(cache, "cache", torch.uint8)
    _need(kmeta, "kmeta", torch.float16)
    _need(tmeta, "tmeta", torch.float16)
    if cache.dim() != 5 or cache.shape[2] != 2 or cache.shape[3] != PAGE_SIZE:
        raise ValueError("cache must be uint8 [num_pages, Hkv, 2, 16, D/4]")
    P, Hkv, D = int(cache.shape[0]), int(cache.shape[1]), 4 * int(cache.shape[4])
    if tuple(kmeta.shape) != (P, Hkv, 2, D) or tuple(tmeta.shape) != (P, Hkv, 3, PAGE_SIZE):
        raise ValueError("kmeta must be fp16 [pages, Hkv, 2, D] and tmeta fp16 [pages, Hkv, 3, 16]")
    return P, Hkv, D


def kv_quant_write_oscar(k: torch.Tensor, v: torch.Tensor, page_ids: torch.Tensor, cache: torch.Tensor,
                         kmeta: torch.Tensor, tmeta: torch.Tensor, hadamard_block: int, stream=None) -> None:
    """OScaR write: rows 16 g .. 16 g + 15 of k, v (bf16 [16 P, Hkv, D]) fill
    page page_ids[g] (int32 [P]) whole."""
    P, Hkv, D = _oscar_pool(cache, kmeta, tmeta)
    _need(k, "k", torch.bfloat16)
    _need(v, "v", torch.bfloat16)
    _need(page_ids, "page_ids", torch.int32)
    if k.dim() != 3 or tuple(k.shape[1:]) != (Hkv, D) or k.shape != v.shape or k.shape[0] != 16 * page_ids.numel():
        raise ValueError("k and v must be bf16 [16 * len(page_ids), Hkv, D] matching the pool")
    desc = OscarWriteDesc(int(page_ids.numel()), Hkv, D, P)
    st = _lib.lib().kv_quant_write_oscar(_ptr(k), _ptr(v), _ptr(page_ids), _ptr(cache), _ptr(kmeta), _ptr(tmeta),
                                         int(hadamard_block), ctypes.byref(desc),
                                         ctypes.c_void_p(_stream_handle(stream)))
    _lib.check(st, "kv_quant_write_oscar")


def oscar_workspace_size(batch: int, num_q_heads: int, num_kv_heads: int, head_dim: int, num_pages: int,
                         max_pages_per_seq: int, hadamard_block: int, device=None) -> int:
    L = _lib.lib()
    idx = None if device is None else torch.device(device).index
    _lib.check(L.kvq_set_device(int(torch.cuda.current_device() if idx is None else idx)), "kvq_set_device")
    desc = OscarAttnDesc(batch, num_q_heads, num_kv_heads, head_dim, num_pages, max_pages_per_seq,
                         hadamard_block, 0.0, 0)
    n = L.kvq_oscar_workspace_size(ctypes.byref(desc))
    if n == ctypes.c_size_t(-1).value:
        raise KVQError(1, "kvq_oscar_workspace_size (invalid shapes or no device)")
    return int(n)


def paged_decode_attn_oscar(q: torch.Tensor, cache: torch.Tensor, kmeta: torch.Tensor, tmeta: torch.Tensor,
                            page_table: torch.Tensor, context_lens: torch.Tensor, k_tail: torch.Tensor,
                            v_tail: torch.Tensor, out: torch.Tensor, hadamard_block: int,
                            workspace: torch.Tensor, softmax_scale: float = 0.0, stream=None) -> None:
    """OScaR decode step: full pages from the INT2 pool, each sequence's last
    context_lens % 16 tokens from k_tail / v_tail (bf16 [B, Hkv, 16, D])."""
    P, Hkv, D = _oscar_pool(cache, kmeta, tmeta)
    _need(q, "q", torch.bfloat16)
    _need(page_table, "page_table", torch.int32)
    _need(context_lens, "context_lens", torch.int32)
    _need(k_tail, "k_tail", torch.bfloat16)
    _need(v_tail, "v_tail", torch.bfloat16)
    _need(workspace, "workspace", torch.uint8)
    if out.dtype not in (torch.float32, torch.bfloat16):
        raise TypeError("out must be float32 or bfloat16")
    _need(out, "out", out.dtype)
    B, Hq = int(q.shape[0]), int(q.shape[1])
    if tuple(out.shape) != tuple(q.shape) or tuple(k_tail.shape) != (B, Hkv, PAGE_SIZE, D) or \
            k_tail.shape != v_tail.shape or page_table.dim() != 2 or int(page_table.shape[0]) != B:
        raise ValueError("shapes: q/out [B, Hq, D], k_tail/v_tail [B, Hkv, 16, D], page_table [B, max_pages]")
    desc = OscarAttnDesc(B, Hq, Hkv, D, P, int(page_table.shape[1]), int(hadamard_block), float(softmax_scale),
                         0 if out.dtype == torch.float32 else 1)
    st = _lib.lib().paged_decode_attn_oscar(
        _ptr(q), _ptr(cache), _ptr(kmeta), _ptr(tmeta), _ptr(page_table), _ptr(context_lens), _ptr(k_tail),
        _ptr(v_tail), _ptr(out), _ptr(workspace), workspace.numel(), ctypes.byref(desc),
        ctypes.c_void_p(_stream_handle(stream)))
    _lib.check(st, "paged_decode_attn_oscar")
