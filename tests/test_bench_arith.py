"""The benchmark's algorithmic-byte arithmetic, counted from the layouts
rather than from its own formulas: a byte budget built up buffer by buffer
for small shapes, and the traffic digests' insensitivity to comments."""
import pytest

import bench
from bit_kv_cache_20_b200 import workloads


def test_write_bytes_match_the_buffers():
    T, Hkv, D = 37, 3, 128
    k = v = T * Hkv * D * 2                      # bf16 K and V read
    codes = 2 * T * Hkv * (D // 2)               # two 4-bit codes per byte, K and V
    sz = 2 * 2 * T * Hkv * 2                     # fp16 s and z, K and V
    slots = T * 8                                # int64 slot per token
    assert bench.write_bytes(T, Hkv, D) == k + v + codes + sz + slots


def test_decode_bytes_match_the_buffers():
    ctx = [1, 16, 17, 40]
    B, Hq, Hkv, D = len(ctx), 8, 2, 64
    cached = sum(ctx) * Hkv * (2 * (D // 2) + 4 * 2)   # K and V codes, four fp16 s/z
    pages = sum((c + 15) // 16 for c in ctx) * 4        # int32 page-table entries read
    lens = B * 4
    q = B * Hq * D * 2
    out = B * Hq * D * 4
    assert bench.decode_bytes(ctx, B, Hq, Hkv, D, out_elem=4) == cached + pages + lens + q + out


def test_oscar_page_head_bytes_match_the_pools():
    D = 128
    codes = 2 * 16 * D // 4        # K then V, four 2-bit codes per byte
    kmeta = 2 * D * 2              # fp16 s and z per channel
    tmeta = 3 * 16 * 2             # fp16 norm, V s, V z per token
    assert bench.OSCAR_PAGE_HEAD_BYTES == codes + kmeta + tmeta == 1632


def test_llama3_step_bytes():
    w = workloads.make("llama3-8b-32k")
    assert bench.write_bytes(w.tokens_written, w.Hkv, w.D) == 170_131_456
    assert bench.decode_bytes(w.context_lens, w.B, w.Hq, w.Hkv, w.D, out_elem=2) == 35_676_164


def test_source_digest_ignores_comments():
    src = "int a; // one\n/* two\n three */ int b;\n"
    assert bench.strip_comments(src) == bench.strip_comments("int a;\n int b;\n")
    assert bench.strip_comments("int a;") != bench.strip_comments("int b;")


@pytest.mark.parametrize("kernel", sorted(bench.KERNEL_SOURCES))
def test_every_kernel_has_a_digest(kernel):
    d = bench.source_digest(kernel)
    assert len(d) == 16 and int(d, 16) >= 0
