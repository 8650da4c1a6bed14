#!/usr/bin/env python
"""Benchmark of the rotated-INT4 paged KV cache hot path on B200.

One step = one pass of the whole hot path over one batch of the
Llama-3-8B-shaped workload (8 KV / 32 Q heads, head_dim 128, one sequence of
32768 tokens, page 16, Hadamard block 128):
  kv_quant_write      - rotate + quantize + page all 32768 tokens' K and V;
  paged_decode_attn_int4 - one decode step over the 32768-token INT4 cache.
The metric is HBM GB/s of algorithmic bytes (the bytes the step must move at
minimum), whole job over all ranks.

L2 hygiene: the working sets rotate so no kernel reads data still resident in
L2: two K/V input sets (134 MB each, larger than L2) alternate, and the decode
of step i reads the cache written at step i-2 (six cache pools, 214 MB in
all), with more than 300 MB of traffic in between.

Besides the step, the JSON line carries:
  - each kernel timed alone, and a roofline object for each;
  - the plain-INT4 comparator (rotation overhead);
  - the randomized-sign rotation;
  - the decode step with a fused 1-token append;
  - a chunked prefill (the last 2048 context tokens as one chunk, L2 flushed
    before each launch);
  - an end-to-end figure through the public API with host buffers;
  - the SM clocks sampled during the timed regions;
  - the oracle's throughput on the host cores.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--config NAME] [--only write|decode|prefill] [--no-graph]
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

WORKLOAD = "llama3-8b-32k"


def parse_args(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--config", default=WORKLOAD)
    ap.add_argument("--block", type=int, default=None, help="override the Hadamard block (0 = plain INT4)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-plain", action="store_true")
    ap.add_argument("--no-graph", action="store_true",
                    help="time direct launches instead of CUDA graph replays (for profilers)")
    ap.add_argument("--only", choices=["write", "decode", "prefill", "oscar"], default=None,
                    help="time one kernel alone (profiling captures; oscar: the OScaR write and decode); "
                         "prints its line")
    ap.add_argument("--no-oscar", action="store_true", help="skip the OScaR variant's line")
    ap.add_argument("--e2e-steps", type=int, default=100)
    ap.add_argument("--no-configs", action="store_true",
                    help="skip the other workloads' write and decode lines")
    ap.add_argument("--launch-check", action="store_true",
                    help="start the ranks, count them over gloo on the CPU and print n_gpus (no GPU work)")
    return ap.parse_args(argv)


# ----------------------------------------------------------------------------
# algorithmic bytes (the minimum a launch must move)
# ----------------------------------------------------------------------------

def write_bytes(T, Hkv, D):
    """Per token-head: K and V read (2 x 2D bytes), codes written (2 x D/2),
    s and z written (4 x 2 bytes); per token: its 8-byte slot."""
    return T * Hkv * (5 * D + 8) + 8 * T


def decode_bytes(context_lens, B, Hq, Hkv, D, out_elem=2):
    """Per cached token-head: K and V codes (D bytes) + 4 fp16 s/z; per
    sequence: its page-table entries and context length; q (bf16) and out."""
    tok = int(sum(int(c) for c in context_lens))
    pages = int(sum((int(c) + 15) // 16 for c in context_lens))
    return tok * Hkv * (D + 8) + 4 * pages + 4 * B + B * Hq * D * 2 + B * Hq * D * out_elem


def rank_seed(base_seed, rank):
    """Weak scaling: every rank serves its own, independently drawn batch."""
    return base_seed + 1000 * rank


def aggregate_gbs(bytes_per_step, steps, world, max_ms):
    """Whole-job GB/s: the bytes all ranks moved over the slowest rank's time."""
    return bytes_per_step * steps * world / (max_ms / 1e3) / 1e9


KERNEL_SOURCES = {
    "kv_quant_write": ["kvq_write_tc.cuh", "kvq_write.cuh", "kvq_device.cuh"],
    "paged_decode_attn_int4": ["kvq_decode.cuh", "kvq_device.cuh"],
    "paged_prefill_attn_int4": ["kvq_prefill.cuh", "kvq_decode.cuh", "kvq_write_tc.cuh", "kvq_device.cuh"],
    "kv_quant_write_oscar": ["kvq_oscar.cuh", "kvq_decode.cuh", "kvq_device.cuh"],
    "paged_decode_attn_oscar": ["kvq_oscar.cuh", "kvq_decode.cuh", "kvq_device.cuh"],
}


def strip_comments(src):
    """C/C++ source without its // and /* */ comments and trailing blanks
    (string literals in these kernels hold no comment markers)."""
    import re
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    src = re.sub(r"//[^\n]*", "", src)
    return "\n".join(line.rstrip() for line in src.splitlines() if line.strip())


def source_digest(kernel):
    """Hash of one kernel's sources, comments excluded: a committed
    DRAM-traffic figure is valid only for the code it was captured from."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "bit_kv_cache_20_b200", "csrc")
    for name in KERNEL_SOURCES[kernel]:
        with open(os.path.join(csrc, name)) as f:
            h.update(name.encode() + strip_comments(f.read()).encode())
    return h.hexdigest()[:16]


def committed_traffic(kernel):
    """Per-launch DRAM bytes from profiles/traffic.json if it was captured
    from the current kernel sources, else None."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            t = json.load(f)
    except (OSError, ValueError):
        return None
    entry = t.get(kernel)
    if not entry or entry.get("source_digest") != source_digest(kernel):
        return None
    return entry.get("dram_bytes_per_launch")


def measured_peaks(key="hbm_gbs"):
    """(peak, "measured" | "fallback"): HBM GB/s, or with key="bf16_tflops"
    the dense bf16 tensor TFLOP/s (burst: the kernels it is used for are
    timed alone)."""
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p[key]), "measured"
    except (OSError, ValueError, KeyError):
        return (6650.0 if key == "hbm_gbs" else 1590.0), "fallback"


# chunked prefill: every sequence's last PREFILL_CHUNK context tokens (all of
# it when shorter) are one chunk of queries over the cache that holds them
PREFILL_CHUNK = 2048


def prefill_flops(context_lens, chunk, Hq, D):
    """Algorithmic FLOPs of a causal chunked prefill: query token i of a chunk
    of L at context c attends to c - L + i + 1 positions, and each (query
    head, position) pair costs 2D for q.k and 2D for p.v."""
    pairs = 0
    for c in context_lens:
        c = int(c)
        L = min(chunk, c)
        pairs += L * (c - L) + L * (L + 1) // 2
    return 4 * D * Hq * pairs


def prefill_run(step, launches, warm):
    """paged_prefill_attn_int4 over the cache of pool 0: each launch preceded
    by an L2 flush (a 256 MB write), timed alone with CUDA events on the
    launching stream. Returns (mean ms per launch, FLOPs per launch)."""
    import numpy as np
    import torch
    kvq, w, dev = step.kvq, step.w, step.dev
    lens = np.minimum(np.asarray(w.context_lens, np.int64), PREFILL_CHUNK)
    q_start = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    g = torch.Generator().manual_seed(w.cfg.seed + 7)
    q = (torch.randn((int(q_start[-1]), w.Hq, w.D), generator=g) / 8).to(torch.bfloat16).to(dev)
    out = torch.empty(q.shape, dtype=torch.bfloat16, device=dev)
    qs = torch.as_tensor(q_start).to(dev)
    c, s, z = step.pools[0]
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    max_q = int(lens.max())

    def launch():
        kvq.paged_prefill_attn_int4(q, c, s, z, step.pt, step.ctx, qs, max_q, out, step.b, stream=step.stream)

    total = 0.0
    with torch.cuda.stream(step.stream):
        for k in range(warm + launches):
            flush.zero_()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(step.stream)
            launch()
            e1.record(step.stream)
            e1.synchronize()
            if k >= warm:
                total += e0.elapsed_time(e1)
    if kvq.get_device_error(step.stream) != 0:
        raise RuntimeError("paged_prefill_attn_int4 recorded a device error")
    return total / launches, prefill_flops(w.context_lens, PREFILL_CHUNK, w.Hq, w.D)


def prefill_cpu_baseline(w, block, n_ctx=4096, n_q=64):
    """The oracle's attention for a chunk of `n_q` queries at the end of an
    `n_ctx`-token context of sequence 0 (its cache written by the oracle from
    the workload's first tokens, untimed), on the host cores. None when the
    workload's new tokens do not start with sequence 0's positions 0, 1, ..."""
    import numpy as np
    import torch
    import oracle
    from bit_kv_cache_20_b200 import workloads
    n = min(n_ctx, int(w.context_lens[0]), w.tokens_written)
    want = np.array([int(w.page_table[0][p // 16]) * 16 + p % 16 for p in range(n)], np.int64)
    if int(w.prior_lens[0]) != 0 or n < n_q or not np.array_equal(np.asarray(w.slots_new[:n]), want):
        return None
    cache, scales, zeros, _ = oracle.quant_write(workloads.bf16_bits(w.k_new[:n]), workloads.bf16_bits(w.v_new[:n]),
                                                 w.slots_new[:n], w.num_pages, block)
    g = torch.Generator().manual_seed(w.cfg.seed + 7)
    q = (torch.randn((n_q, w.Hq, w.D), generator=g) / 8).to(torch.bfloat16)
    ctx = np.arange(n - n_q + 1, n + 1).astype(np.int32)
    pt = np.repeat(np.asarray(w.page_table)[:1], n_q, axis=0)
    t0 = time.perf_counter()
    oracle.decode_attn(workloads.bf16_bits(q), cache, scales, zeros, pt, ctx, w.Hkv, block, w.num_pages)
    dt = time.perf_counter() - t0
    flops = 4 * w.D * w.Hq * int(ctx.sum())
    return {"value": round(flops / dt / 1e12, 6), "unit": "TFLOP/s", "cores": oracle.num_threads(),
            "kind": "oracle",
            "sample": f"{n_q} causal chunk queries x {w.Hq} heads at the end of a {n}-token context; "
                      f"{dt:.2f} s"}


def prefill_line(ms, flops):
    peak, src = measured_peaks("bf16_tflops")
    tf = flops / (ms / 1e3) / 1e12
    return {
        "what": f"chunked prefill: each sequence's last {PREFILL_CHUNK} context tokens (all when shorter) "
                "as queries, causal, over the INT4 cache; L2 flushed before each launch",
        "us": round(1e3 * ms, 1), "TFLOP/s": round(tf, 2),
        "roofline": {"kernel": "paged_prefill_attn_int4", "bound": "tensor", "achieved": round(tf, 2),
                     "peak": peak, "unit": "TFLOP/s", "frac": round(tf / peak, 4),
                     "traffic": committed_traffic("paged_prefill_attn_int4"),
                     "algorithmic_flops": flops,
                     "peak_source": "measured (MEASURED_PEAKS.json bf16_tflops, burst)" if src == "measured"
                     else "fallback 1.59 PFLOP/s"},
    }


# ----------------------------------------------------------------------------
# clocks during the timed region
# ----------------------------------------------------------------------------

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []          # (host monotonic time, csv line)
        self.window = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "20"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except OSError:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.monotonic(), line.strip()))

    def wait_first_sample(self, timeout=5.0):
        t_end = time.monotonic() + timeout
        while self.proc is not None and not self.lines and time.monotonic() < t_end:
            time.sleep(0.01)

    def mark(self, t0, t1):
        """The host-time window during which the GPU ran the timed steps."""
        self.window = (t0, t1)

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
        return False

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        lines = self.lines
        if self.window is not None:
            lines = [(t, l) for t, l in self.lines if self.window[0] <= t <= self.window[1]]
        for _, line in lines:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for name, val in zip(names, parts[5:9]):
                if val.lower() == "active":
                    reasons.add(name)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": mx, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# ----------------------------------------------------------------------------
# the CUDA arm
# ----------------------------------------------------------------------------

class Step:
    """Prepared C-ABI calls for one workload on one device, on a stream of its
    own. Timed regions replay a CUDA graph captured from those calls (what a
    serving loop does with its decode step), so the host's launch rate never
    gates the GPU: the kernels run back to back exactly as launched."""

    N_POOLS = 6

    def __init__(self, w, block, dev, graph=True, signs=None):
        import ctypes
        import numpy as np
        import torch
        import bit_kv_cache_20_b200 as kvq
        from bit_kv_cache_20_b200 import _lib

        self.torch, self.kvq, self.ct = torch, kvq, ctypes
        self.L = _lib.lib()
        self.w, self.b, self.dev, self.graph = w, block, dev, graph
        k0 = w.k_new.to(dev)
        v0 = w.v_new.to(dev)
        self.kv_sets = [(k0, v0), (k0.clone(), v0.clone())]
        self.slots = torch.as_tensor(w.slots_new).to(dev)
        self.pools = [kvq.alloc_cache(w.num_pages, w.Hkv, w.D, device=dev) for _ in range(self.N_POOLS)]
        self.q = w.q.to(dev)
        self.pt = torch.as_tensor(w.page_table).to(dev)
        self.ctx = torch.as_tensor(w.context_lens).to(dev)
        self.out = torch.empty((w.B, w.Hq, w.D), dtype=torch.bfloat16, device=dev)
        nbytes = kvq.attn_workspace_size(w.B, w.Hq, w.Hkv, w.D, w.num_pages, w.max_pages, block,
                                         host_lengths=True)
        self.ws = kvq.alloc_workspace(nbytes, device=dev)
        self.ws_bytes = self.ws.numel()
        self.stream = torch.cuda.Stream(dev)
        self.sh = ctypes.c_void_p(self.stream.cuda_stream)
        # randomized Hadamard: the same sign mask in both descriptors
        sw = kvq.sign_words(signs, w.D)
        self.wdesc = _lib.WriteDesc(w.tokens_written, w.Hkv, w.D, 16, w.num_pages, sw)
        # q, the page table and the context lengths are set up once, never
        # written by the write kernel that precedes each decode
        # with the host copy of the context lengths (a serving engine has it)
        # the work is split per sequence in proportion to its length
        self.lens_host = np.ascontiguousarray(w.context_lens, dtype=np.int32)
        self.adesc = _lib.AttnDesc(w.B, w.Hq, w.Hkv, w.D, 16, w.num_pages, w.max_pages, block, 0.0, 1,
                                   _lib.ATTN_INPUTS_READY,
                                   self.lens_host.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)), sw)
        P = ctypes.c_void_p
        self.write_args = []
        for i in range(self.N_POOLS):
            k, v = self.kv_sets[i % 2]
            c, s, z = self.pools[i]
            self.write_args.append((P(k.data_ptr()), P(v.data_ptr()), P(self.slots.data_ptr()), None,
                                    P(c.data_ptr()), P(s.data_ptr()), P(z.data_ptr()), block,
                                    ctypes.byref(self.wdesc), self.sh))
        self.attn_args = []
        for i in range(self.N_POOLS):
            c, s, z = self.pools[(i - 2) % self.N_POOLS]
            self.attn_args.append((P(self.q.data_ptr()), P(c.data_ptr()), P(s.data_ptr()), P(z.data_ptr()),
                                   P(self.pt.data_ptr()), P(self.ctx.data_ptr()), P(self.out.data_ptr()),
                                   P(self.ws.data_ptr()), self.ws_bytes, ctypes.byref(self.adesc), self.sh))
        # decode-append: each sequence's last context token is the step's
        # new token (rewritten in place every step, so every step does the
        # same work); separate = a 1-token-per-sequence write + the decode,
        # fused = one paged_decode_append_attn_int4 launch
        k1, v1, s1 = self.last_tokens(w)
        self.k1, self.v1, self.s1 = k1.to(dev), v1.to(dev), s1.to(dev)
        self.wdesc1 = _lib.WriteDesc(w.B, w.Hkv, w.D, 16, w.num_pages, sw)
        self.write1_args, self.app_args = [], []
        for i in range(self.N_POOLS):
            c, s, z = self.pools[(i - 2) % self.N_POOLS]
            self.write1_args.append((P(self.k1.data_ptr()), P(self.v1.data_ptr()), P(self.s1.data_ptr()), None,
                                     P(c.data_ptr()), P(s.data_ptr()), P(z.data_ptr()), block,
                                     ctypes.byref(self.wdesc1), self.sh))
            self.app_args.append((P(self.q.data_ptr()), P(self.k1.data_ptr()), P(self.v1.data_ptr()),
                                  P(self.s1.data_ptr()), P(c.data_ptr()), P(s.data_ptr()), P(z.data_ptr()),
                                  P(self.pt.data_ptr()), P(self.ctx.data_ptr()), P(self.out.data_ptr()),
                                  P(self.ws.data_ptr()), self.ws_bytes, ctypes.byref(self.adesc), self.sh))
        torch.cuda.synchronize(dev)  # allocations above ran on the default stream

    @staticmethod
    def last_tokens(w):
        """K, V ([B, Hkv, D]) and slot of every sequence's last context token,
        wherever the workload holds it (the step's new tokens or the prior
        context); a sequence with an empty context gets slot -1."""
        import numpy as np
        import torch
        where = {}
        for src, (k, v, slots) in enumerate(((w.k_prior, w.v_prior, w.slots_prior),
                                              (w.k_new, w.v_new, w.slots_new))):
            for i, sl in enumerate(np.asarray(slots).tolist()):
                if sl >= 0:
                    where[sl] = (src, i)
        k1 = torch.zeros((w.B, w.Hkv, w.D), dtype=torch.bfloat16)
        v1 = torch.zeros_like(k1)
        s1 = np.full(w.B, -1, np.int64)
        for n in range(w.B):
            c = int(w.context_lens[n])
            if c == 0:
                continue
            sl = int(w.page_table[n][(c - 1) // 16]) * 16 + (c - 1) % 16
            if sl not in where:
                continue
            src, i = where[sl]
            k, v = (w.k_prior, w.v_prior) if src == 0 else (w.k_new, w.v_new)
            k1[n], v1[n], s1[n] = k[i], v[i], sl
        return k1, v1, torch.as_tensor(s1)

    def write(self, i):
        st = self.L.kv_quant_write(*self.write_args[i % self.N_POOLS])
        if st:
            raise RuntimeError(f"kv_quant_write status {st}")

    def decode(self, i):
        st = self.L.paged_decode_attn_int4(*self.attn_args[i % self.N_POOLS])
        if st:
            raise RuntimeError(f"paged_decode_attn_int4 status {st}")

    def append_separate(self, i):
        st = self.L.kv_quant_write(*self.write1_args[i % self.N_POOLS])
        if st:
            raise RuntimeError(f"kv_quant_write status {st}")
        self.decode(i)

    def append_fused(self, i):
        st = self.L.paged_decode_append_attn_int4(*self.app_args[i % self.N_POOLS])
        if st:
            raise RuntimeError(f"paged_decode_append_attn_int4 status {st}")

    def fill_pools(self):
        for i in range(self.N_POOLS):
            self.write(i)
        self.torch.cuda.synchronize(self.dev)

    def capture(self, kinds, steps, start_index=0):
        """A CUDA graph of `steps` steps, each the calls named in `kinds`
        ("write", "decode") in that order, inputs and outputs rotating through
        the pools as in the direct calls. It is replayed once, untimed, so the
        first timed replay does not include the graph's upload."""
        torch = self.torch
        fns = [getattr(self, k) for k in kinds]
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=self.stream, capture_error_mode="thread_local"):
            for j in range(steps):
                for fn in fns:
                    fn(start_index + j)
        with torch.cuda.stream(self.stream):
            g.replay()
        self.stream.synchronize()
        return g

    def replay_ms(self, g):
        """Device time of one replay of `g` between two events on the stream."""
        torch = self.torch
        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(self.stream):
            t0.record(self.stream)
            g.replay()
            t1.record(self.stream)
        t1.synchronize()
        return t0.elapsed_time(t1)

    def direct_ms(self, kinds, steps, start_index=0):
        """The same launches issued directly on the stream between two events."""
        torch = self.torch
        fns = [getattr(self, k) for k in kinds]
        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        t0.record(self.stream)
        for j in range(steps):
            for fn in fns:
                fn(start_index + j)
        t1.record(self.stream)
        t1.synchronize()
        return t0.elapsed_time(t1)

    def run_ms(self, kinds, steps, start_index=0, rounds=1):
        """Device ms of `steps` steps of `kinds`: the median of `rounds`
        measurements (replays of one captured graph, or direct launches)."""
        if not self.graph:
            return statistics.median(self.direct_ms(kinds, steps, start_index) for _ in range(rounds))
        g = self.capture(kinds, steps, start_index)
        return statistics.median(self.replay_ms(g) for _ in range(rounds))

    def timed_only(self, kind, steps, start_index=0, rounds=1):
        """One kernel alone, `steps` back-to-back launches (inputs and outputs
        rotate through sets larger than L2). Returns the average ms per launch
        (median of `rounds` measurements)."""
        return self.run_ms((kind,), steps, start_index, rounds) / steps

    def timed(self, steps, start_index=0, rounds=3):
        """`steps` whole steps (write, then decode) back to back. Returns the
        total ms (median of `rounds` measurements)."""
        return self.run_ms(("write", "decode"), steps, start_index, rounds)


def e2e_run(w, block, dev, steps, warmup):
    """The same step through the public API with host inputs: each step copies
    K, V, the slot mapping, q, the page table and the context lengths from
    pinned host memory, runs both calls, and copies the output back."""
    import torch
    import bit_kv_cache_20_b200 as kvq

    host = {
        "k": w.k_new.pin_memory(), "v": w.v_new.pin_memory(),
        "slots": torch.as_tensor(w.slots_new).pin_memory(), "q": w.q.pin_memory(),
        "pt": torch.as_tensor(w.page_table).pin_memory(),
        "ctx": torch.as_tensor(w.context_lens).pin_memory(),
    }
    devb = {k: torch.empty_like(v, device=dev) for k, v in host.items()}
    out_d = torch.empty((w.B, w.Hq, w.D), dtype=torch.bfloat16, device=dev)
    out_h = torch.empty_like(out_d, device="cpu").pin_memory()
    cache, scales, zeros = kvq.alloc_cache(w.num_pages, w.Hkv, w.D, device=dev)
    ws = kvq.alloc_workspace(kvq.attn_workspace_size(w.B, w.Hq, w.Hkv, w.D, w.num_pages,
                                                     w.max_pages, block), device=dev)
    h2d = sum(t.numel() * t.element_size() for t in host.values())
    d2h = out_h.numel() * out_h.element_size()

    def step():
        for key in host:
            devb[key].copy_(host[key], non_blocking=True)
        kvq.kv_quant_write(devb["k"], devb["v"], devb["slots"], cache, scales, zeros, block)
        kvq.paged_decode_attn_int4(devb["q"], cache, scales, zeros, devb["pt"], devb["ctx"], out_d,
                                   block, ws)
        out_h.copy_(out_d, non_blocking=True)

    for _ in range(warmup):
        step()
    torch.cuda.synchronize(dev)
    s = torch.cuda.current_stream(dev)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(s)
    for _ in range(steps):
        step()
    b.record(s)
    b.synchronize()
    return a.elapsed_time(b), h2d, d2h


# ----------------------------------------------------------------------------
# the CPU oracle: the cpu_baseline leg and the reference arm
# ----------------------------------------------------------------------------

def oracle_sample(w, block, n_tokens):
    """Time the oracle on the first `n_tokens` tokens of the workload: write
    them (all kv heads, K and V), then one decode step of every query head
    over that n_tokens-long context. Returns (seconds, algorithmic bytes)."""
    import numpy as np
    import oracle
    from bit_kv_cache_20_b200 import workloads

    n = min(n_tokens, w.tokens_written)
    kb = workloads.bf16_bits(w.k_new[:n])
    vb = workloads.bf16_bits(w.v_new[:n])
    qb = workloads.bf16_bits(w.q)
    ctx = np.full(w.B, n // w.B, np.int32)
    t0 = time.perf_counter()
    cache, scales, zeros, _ = oracle.quant_write(kb, vb, w.slots_new[:n], w.num_pages, block)
    oracle.decode_attn(qb, cache, scales, zeros, w.page_table, ctx, w.Hkv, block, w.num_pages)
    dt = time.perf_counter() - t0
    nbytes = write_bytes(n, w.Hkv, w.D) + decode_bytes(ctx, w.B, w.Hq, w.Hkv, w.D)
    return dt, nbytes


def cpu_model():
    """The host CPU's model name (lscpu), or None."""
    try:
        out = subprocess.run(["lscpu"], capture_output=True, text=True, timeout=10).stdout
    except (OSError, subprocess.SubprocessError):
        return None
    for line in out.splitlines():
        if line.strip().startswith("Model name:"):
            return line.split(":", 1)[1].strip()
    return None


def cpu_baseline(w, block, n_tokens=32768, min_seconds=10.0, max_passes=20, single_tokens=2048):
    """The oracle on a bounded sample of the workload, repeated until it has
    run for `min_seconds` (at most `max_passes` passes), on all host cores;
    then once on a smaller sample with one thread."""
    import oracle
    passes, total_t, total_b = 0, 0.0, 0
    while passes < max_passes and total_t < min_seconds:
        dt, nbytes = oracle_sample(w, block, n_tokens)
        passes += 1
        total_t += dt
        total_b += nbytes
    cores = oracle.num_threads()
    oracle.set_num_threads(1)
    try:
        dt1, nb1 = oracle_sample(w, block, single_tokens)
    finally:
        oracle.set_num_threads(cores)
    n1 = min(single_tokens, w.tokens_written)
    return {"value": round(total_b / total_t / 1e9, 4), "unit": "GB/s", "cores": cores,
            "kind": "oracle", "cpu_model": cpu_model(),
            "sample": f"{passes} passes of: write of the first {min(n_tokens, w.tokens_written)} tokens "
                      f"(all kv heads, K and V) + one decode step of all {w.Hq} query heads over them; "
                      f"{total_t:.1f} s in all",
            "single_thread": {"value": round(nb1 / dt1 / 1e9, 5), "unit": "GB/s", "cores": 1,
                              "sample": f"write of the first {n1} tokens + one decode step over them; "
                                        f"{dt1:.1f} s"}}


REFERENCE_BUDGET_S = 120.0


def run_reference(args):
    """The oracle timed as it stands on the host cores, same metric/config."""
    import oracle
    from bit_kv_cache_20_b200 import workloads
    w = workloads.make(args.config, block=args.block)
    block = w.block
    warm = max(args.warmup, 0)
    # each step's sample is sized so that the whole run takes about
    # REFERENCE_BUDGET_S: 256 .. 4096 tokens, from a timed 1024-token sample
    dt_cal, _ = oracle_sample(w, block, 1024)
    per_step = REFERENCE_BUDGET_S / (max(args.steps, 1) + warm)
    n_tokens = max(256, min(4096, int(per_step / (dt_cal / 1024)) // 256 * 256))
    for _ in range(warm):
        oracle_sample(w, block, n_tokens)
    total_t, total_b = 0.0, 0
    for _ in range(args.steps):
        dt, nb = oracle_sample(w, block, n_tokens)
        total_t += dt
        total_b += nb
    value = total_b / total_t / 1e9
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": "GB/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": warm,
        "ms_per_step": round(1e3 * total_t / max(args.steps, 1), 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_block(w, block, not args.no_graph),
        "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": oracle.num_threads(),
                         "kind": "oracle",
                         "sample": f"per step: write of {n_tokens} tokens (all kv heads, K and V) + one "
                                   f"decode step of all {w.Hq} query heads over them"},
        "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    return line


METRIC = "fused rot+INT4 KV write & INT4 paged decode attn: HBM GB/s, % of peak"


def config_block(w, block, graph=True):
    timing = ("the K steps as one CUDA graph (replayed once untimed, then once between two events)"
              if graph else "the K steps launched directly, back to back between two events")
    return {
        "workload": w.cfg.name, "batch": w.B, "kv_heads": w.Hkv, "q_heads": w.Hq, "head_dim": w.D,
        "context": int(w.context_lens.max()), "written_tokens": w.tokens_written, "page": 16,
        "hadamard_block": block, "out_dtype": "bf16",
        "l2": "inputs larger than L2 rotate; decode reads a cache written two steps earlier",
        "timing": timing + "; each kernel's line: the same, that kernel alone, median of 3 rounds "
                           "in which the rotated, plain-INT4 and randomized-sign kernels take turns "
                           "(all writes before all decodes, each kind after an untimed pass)",
    }


# ----------------------------------------------------------------------------
# the other workloads: each kernel alone, at each Hadamard block and plain
# ----------------------------------------------------------------------------

SWEEP = (("serving-b64", None), ("llama2-70b-b8", None), ("stress-b256", (32, 64, 128)))


def config_sweep(dev, steps, warm, rank, world, max_over_ranks):
    """For every other workload: kv_quant_write and paged_decode_attn_int4
    alone (graph replays of `steps` back-to-back launches), at its Hadamard
    block(s) and at 0 (plain INT4), the blocks taking turns over three rounds
    (median of 3), with GB/s, the fraction of the HBM peak and the rotation
    overhead."""
    import torch
    from bit_kv_cache_20_b200 import workloads
    peak, _ = measured_peaks()
    out = {}
    for name, blocks in SWEEP:
        cfg = workloads.CONFIGS[name]
        w = workloads.make(name, seed=rank_seed(cfg.seed, rank))
        blocks = tuple(blocks or (w.block,))
        wb = write_bytes(w.tokens_written, w.Hkv, w.D)
        db = decode_bytes(w.context_lens, w.B, w.Hq, w.Hkv, w.D, out_elem=2)
        # every block's Step set up first, then three rounds in which the
        # blocks take turns: one block measured after the others would run
        # on a hotter, more power-capped GPU than the first. All writes come
        # before all decodes: a decode timed right after a burst of the
        # tensor-core write (b > 0) would start at the lower clock that
        # burst leaves, one after the CUDA-core write (b = 0) would not
        sts = {}
        for b in (0,) + blocks:
            sts[b] = Step(w, b, dev, graph=True)
            sts[b].fill_pools()
            sts[b].timed_only("write", warm)
            sts[b].timed_only("decode", warm)
        # Each kind starts with an untimed pass over every block (the clock
        # settles at that kind's power level), and the block order rotates
        # from round to round, so that no block always follows the heaviest
        ms = {b: ([], []) for b in sts}
        order = list(sts)
        with ClockSampler(dev.index if dev.index is not None else 0) as clocks:
            clocks.wait_first_sample()
            t0 = time.monotonic()
            for kind in (0, 1):
                kname = ("write", "decode")[kind]
                for b in order:
                    sts[b].timed_only(kname, steps, start_index=warm)
                for r in range(3):
                    for b in order[r % len(order):] + order[:r % len(order)]:
                        ms[b][kind].append(sts[b].timed_only(kname, steps, start_index=warm))
            clocks.mark(t0, time.monotonic())
        times = {b: (max_over_ranks(statistics.median(ms[b][0])), max_over_ranks(statistics.median(ms[b][1])))
                 for b in sts}
        del sts
        torch.cuda.empty_cache()

        def line(b):
            wr, de = times[b]
            w_gbs, d_gbs = wb * world / (wr / 1e3) / 1e9, db * world / (de / 1e3) / 1e9
            entry = {"write_us": round(1e3 * wr, 2), "write_GB/s": round(w_gbs, 1),
                     "write_frac": round(w_gbs / (peak * world), 4),
                     "decode_us": round(1e3 * de, 2), "decode_GB/s": round(d_gbs, 1),
                     "decode_frac": round(d_gbs / (peak * world), 4)}
            if b != 0:
                entry["rotation_overhead"] = {"kv_quant_write": round(wr / times[0][0] - 1, 4),
                                              "paged_decode_attn_int4": round(de / times[0][1] - 1, 4)}
            return entry

        out[name] = {"batch": w.B, "kv_heads": w.Hkv, "q_heads": w.Hq, "head_dim": w.D,
                     "context_tokens": int(w.context_lens.sum()), "written_tokens": w.tokens_written,
                     "write_bytes": wb, "decode_bytes": db,
                     "blocks": {str(b): line(b) for b in (0,) + blocks}, "clocks": clocks.summary()}
        del w
    return out


# ----------------------------------------------------------------------------
# the OScaR variant (INT2: per-token norm scaling, K per channel) on the same
# workload: each kernel alone, graph replays of back-to-back launches
# ----------------------------------------------------------------------------

OSCAR_PAGE_HEAD_BYTES = 2 * 16 * 128 // 4 + 2 * 2 * 128 + 3 * 2 * 16   # codes + K (s, z) + (n, V s, V z)


def oscar_run(w, block, dev, steps, warm, max_over_ranks):
    """kv_quant_write_oscar and paged_decode_attn_oscar on the workload's
    full pages (each sequence's unfinished last page stays bf16 and is read
    by the decode), each alone: a CUDA graph of `steps` launches rotating
    through pools larger than L2, median of 3 replays."""
    import numpy as np
    import torch
    import bit_kv_cache_20_b200 as kvq
    from bit_kv_cache_20_b200 import workloads
    k, v, ids, k_tail, v_tail = workloads.oscar_rows(w)
    P = int(ids.size)
    pool_bytes = max(P * w.Hkv * OSCAR_PAGE_HEAD_BYTES, 1)
    n_pools = int(min(16, max(2, -(-300_000_000 // pool_bytes))))
    pools = [kvq.alloc_oscar_cache(w.num_pages, w.Hkv, w.D, device=dev) for _ in range(n_pools)]
    kc, vc, idc = k.to(dev), v.to(dev), torch.as_tensor(ids).to(dev)
    full = max(1, int(max(int(c) // 16 for c in w.context_lens)))
    pt = torch.as_tensor(np.ascontiguousarray(w.page_table[:, :full])).to(dev)
    cl = torch.as_tensor(w.context_lens).to(dev)
    q, ktc, vtc = w.q.to(dev), k_tail.to(dev), v_tail.to(dev)
    out = torch.empty((w.B, w.Hq, w.D), dtype=torch.bfloat16, device=dev)
    ws = torch.empty(kvq.oscar_workspace_size(w.B, w.Hq, w.Hkv, w.D, w.num_pages, full, block, device=dev),
                     dtype=torch.uint8, device=dev)
    stream = torch.cuda.Stream(dev)
    for pool in pools:
        kvq.kv_quant_write_oscar(kc, vc, idc, *pool, block)
    torch.cuda.synchronize(dev)

    def graph_ms(fn):
        with torch.cuda.stream(stream):
            for j in range(warm):
                fn(j)
        stream.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream, capture_error_mode="thread_local"):
            for j in range(steps):
                fn(warm + j)
        with torch.cuda.stream(stream):
            g.replay()
        stream.synchronize()
        ts = []
        for _ in range(3):
            t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            with torch.cuda.stream(stream):
                t0.record(stream)
                g.replay()
                t1.record(stream)
            t1.synchronize()
            ts.append(t0.elapsed_time(t1) / steps)
        del g
        return statistics.median(ts)

    def wr(j):
        kvq.kv_quant_write_oscar(kc, vc, idc, *pools[j % n_pools], block, stream=stream)

    def de(j):
        kvq.paged_decode_attn_oscar(q, *pools[j % n_pools], pt, cl, ktc, vtc, out, block, ws, stream=stream)

    wr_ms = max_over_ranks(graph_ms(wr))
    de_ms = max_over_ranks(graph_ms(de))
    assert kvq.get_device_error() == 0
    tails = int(sum(int(c) % 16 for c in w.context_lens))
    wbytes = P * w.Hkv * (16 * w.D * 2 * 2 + OSCAR_PAGE_HEAD_BYTES)
    dbytes = P * w.Hkv * OSCAR_PAGE_HEAD_BYTES + tails * w.Hkv * w.D * 2 * 2 + 2 * w.B * w.Hq * w.D * 2
    peak, _ = measured_peaks()
    w_gbs, d_gbs = wbytes / (wr_ms / 1e3) / 1e9, dbytes / (de_ms / 1e3) / 1e9
    del pools, kc, vc, ws
    torch.cuda.empty_cache()
    return {
        "what": "OScaR: R, then each K token scaled to unit norm (fp16 norm kept), K INT2 per channel over "
                "each 16-token page, V INT2 per token; the unfinished last page in bf16",
        "hadamard_block": block, "pages": P, "bytes_per_page_head": OSCAR_PAGE_HEAD_BYTES,
        "timing": f"each kernel alone: a CUDA graph of {steps} launches over {n_pools} pools (larger than "
                  "L2), median of 3 replays",
        "kernels": {
            "kv_quant_write_oscar": {"us": round(1e3 * wr_ms, 3), "GB/s": round(w_gbs, 1),
                                     "algorithmic_bytes": wbytes, "frac": round(w_gbs / peak, 4),
                                     "traffic": committed_traffic("kv_quant_write_oscar")},
            "paged_decode_attn_oscar": {"us": round(1e3 * de_ms, 3), "GB/s": round(d_gbs, 1),
                                        "algorithmic_bytes": dbytes, "frac": round(d_gbs / peak, 4),
                                        "traffic": committed_traffic("paged_decode_attn_oscar"),
                                        "launches": 2},
        },
    }


# ----------------------------------------------------------------------------
# main
# ----------------------------------------------------------------------------

def free_port():
    import socket
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        return sk.getsockname()[1]


def launch_local_ranks(n, argv):
    """`python bench.py --gpus N` without torchrun: start N ranks of this
    script on this node (RANK / LOCAL_RANK / WORLD_SIZE / MASTER_* set), one
    per GPU; rank 0 prints the line. Returns the worst exit code."""
    env = dict(os.environ, WORLD_SIZE=str(n), MASTER_ADDR="127.0.0.1", MASTER_PORT=str(free_port()))
    procs = [subprocess.Popen([sys.executable, os.path.abspath(__file__)] + list(argv),
                              env=dict(env, RANK=str(r), LOCAL_RANK=str(r))) for r in range(n)]
    return max(p.wait() for p in procs)


def launch_check(rank, world):
    """Count the ranks over gloo (CPU) and print what the line would report."""
    import datetime
    import torch
    import torch.distributed as dist
    t = torch.ones(1)
    if world > 1:
        dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
        dist.all_reduce(t)
    if rank == 0:
        print(json.dumps({"launch_check": True, "n_gpus": world, "ranks_seen": int(t.item())}), flush=True)
    if world > 1:
        dist.destroy_process_group()
    return 0


def reduce_max(x, world, device):
    """Max of a per-rank scalar over all ranks (the job's time is the slowest
    rank's)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def main(argv=None):
    argv = sys.argv[1:] if argv is None else list(argv)
    args = parse_args(argv)
    if args.gpus > 1 and "WORLD_SIZE" not in os.environ:
        return launch_local_ranks(args.gpus, argv)
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.launch_check:
        return launch_check(rank, world)
    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args)), flush=True)
        return 0

    import datetime
    import torch
    import torch.distributed as dist
    from bit_kv_cache_20_b200 import workloads

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=180), device_id=dev)
    warm = max(args.warmup, 3)
    cfg = workloads.CONFIGS[args.config]
    # weak scaling: every rank serves its own batch (its own seed)
    w = workloads.make(args.config, block=args.block, seed=rank_seed(cfg.seed, rank))
    block = w.block
    wb = write_bytes(w.tokens_written, w.Hkv, w.D)
    db = decode_bytes(w.context_lens, w.B, w.Hq, w.Hkv, w.D, out_elem=2)

    def barrier():
        torch.cuda.synchronize(dev)
        if world > 1:
            dist.barrier()

    def max_over_ranks(x):
        return reduce_max(x, world, dev)

    if args.only == "oscar":
        line = oscar_run(w, block, dev, args.steps, warm, max_over_ranks)
        if rank == 0:
            print(json.dumps({"only": "oscar", **line, "config": config_block(w, block)}), flush=True)
        if world > 1:
            dist.destroy_process_group()
        return 0
    step = Step(w, block, dev, graph=not args.no_graph)
    step.fill_pools()
    if args.only == "prefill":
        ms_pf, fl = prefill_run(step, args.steps, warm)
        ms_pf = max_over_ranks(ms_pf)
        if rank == 0:
            print(json.dumps({"only": "prefill", **prefill_line(ms_pf, fl * world), "launches": args.steps,
                              "config": config_block(w, block, not args.no_graph)}), flush=True)
        if world > 1:
            dist.destroy_process_group()
        return 0
    if args.only:
        step.timed_only(args.only, warm)
        barrier()
        mean = step.timed_only(args.only, args.steps, start_index=warm)
        barrier()
        if rank == 0:
            nb = wb if args.only == "write" else db
            print(json.dumps({"only": args.only, "us": round(1e3 * mean, 3),
                              "GB/s": round(nb / (mean / 1e3) / 1e9, 2), "launches": args.steps,
                              "config": config_block(w, block, not args.no_graph)}), flush=True)
        if world > 1:
            dist.destroy_process_group()
        return 0
    # the plain-INT4 comparator (block 0) on the same workload; its kernels are
    # timed in alternation with the rotated ones, so that drifting clocks or
    # power cannot bias the rotation overhead
    p = None
    if not args.no_plain and block != 0:
        p = Step(w, 0, dev, graph=not args.no_graph)
        p.fill_pools()
    # randomized Hadamard (a seeded sign mask) on the same workload
    r = None
    if not args.no_plain and block != 0:
        r = Step(w, block, dev, graph=not args.no_graph, signs=workloads.random_signs(cfg.seed + 11, w.D))
        r.fill_pools()
    rounds = 3
    with ClockSampler(local) as clocks:
        clocks.wait_first_sample()
        step.timed(warm)                    # warm-up steps (untimed)
        if p is not None:
            p.timed(warm)
        barrier()
        t_host0 = time.monotonic()
        total_ms = step.timed(args.steps, start_index=warm)
        barrier()
        p_total = p.timed(args.steps, start_index=warm) if p is not None else None
        barrier()
        # each kernel alone, back to back, for its own line: the median of
        # `rounds` measurements. Rotated, plain and randomized-sign variants
        # take turns, their order rotating from round to round; all writes
        # come first, then all decodes, each kind after an untimed pass of
        # every variant, so that no decode is timed right after a burst of
        # the power-hungrier tensor-core write and the clock it leaves
        ms = {k: [] for k in ("write", "decode", "p_write", "p_decode", "r_write", "r_decode",
                              "append_separate", "append_fused")}
        variants = [("", step)] + ([("p_", p)] if p is not None else []) + ([("r_", r)] if r is not None else [])
        for kind in ("write", "decode"):
            for _, obj in variants:
                obj.timed_only(kind, args.steps, start_index=warm)
                barrier()
            for rd in range(rounds):
                k0 = rd % len(variants)
                for pre, obj in variants[k0:] + variants[:k0]:
                    ms[pre + kind].append(obj.timed_only(kind, args.steps, start_index=warm))
                    barrier()
        # decode with a 1-token append per sequence: two launches or one
        for rd in range(rounds):
            for kind in (("append_separate", "append_fused") if rd % 2 == 0 else ("append_fused", "append_separate")):
                ms[kind].append(step.timed_only(kind, args.steps, start_index=warm))
                barrier()
        t_host1 = time.monotonic()
        clocks.mark(t_host0, t_host1)
    barrier()
    total_ms = max_over_ranks(total_ms)
    wr_ms = max_over_ranks(statistics.median(ms["write"]))
    de_ms = max_over_ranks(statistics.median(ms["decode"]))
    ap_sep_ms = max_over_ranks(statistics.median(ms["append_separate"]))
    ap_fus_ms = max_over_ranks(statistics.median(ms["append_fused"]))

    plain = None
    if p is not None:
        p_total = max_over_ranks(p_total)
        p_wr_ms = max_over_ranks(statistics.median(ms["p_write"]))
        p_de_ms = max_over_ranks(statistics.median(ms["p_decode"]))
        plain = {
            "hadamard_block": 0,
            "kernels": {"kv_quant_write": "kvq_write_kernel<D> (CUDA cores, no rotation) vs the rotated "
                                          "kvq_write_tc_kernel<D, b> (tcgen05 rotation)",
                        "paged_decode_attn_int4": "kvq_decode_kernel with b = 0 (the same template, "
                                                  "rotations compiled out)"},
            "kv_quant_write_us": round(1e3 * p_wr_ms, 3),
            "paged_decode_attn_int4_us": round(1e3 * p_de_ms, 3),
            "ms_per_step": round(p_total / args.steps, 5),
            "rotation_overhead": {
                "kv_quant_write": round(wr_ms / p_wr_ms - 1, 4),
                "paged_decode_attn_int4": round(de_ms / p_de_ms - 1, 4),
                "step": round(total_ms / p_total - 1, 4),
            },
        }
        del p
    randomized = None
    if r is not None:
        r_wr_ms = max_over_ranks(statistics.median(ms["r_write"]))
        r_de_ms = max_over_ranks(statistics.median(ms["r_decode"]))
        randomized = {
            "what": "R = H_b diag(sigma) / sqrt(b), a seeded sign mask in both descriptors",
            "kv_quant_write_us": round(1e3 * r_wr_ms, 3),
            "paged_decode_attn_int4_us": round(1e3 * r_de_ms, 3),
            "vs_plain_rotation": {"kv_quant_write": round(r_wr_ms / wr_ms - 1, 4),
                                  "paged_decode_attn_int4": round(r_de_ms / de_ms - 1, 4)},
        }
        del r

    # chunked prefill (a row beside the step, not part of it): a few launches
    pf_ms, pf_flops = prefill_run(step, 3, 1)
    pf_ms = max_over_ranks(pf_ms)
    del step
    torch.cuda.empty_cache()

    # the OScaR variant on the same workload (not part of the step)
    oscar = None if args.no_oscar else oscar_run(w, block, dev, min(args.steps, 50), warm, max_over_ranks)

    # the other workloads, each kernel alone (not part of the step)
    configs = None
    if not args.no_configs:
        configs = config_sweep(dev, min(args.steps, 50), warm, rank, world, max_over_ranks)

    e2e = None
    if not args.no_e2e:
        e_steps = max(1, min(args.steps, args.e2e_steps))
        e_ms, h2d, d2h = e2e_run(w, block, dev, e_steps, warm)
        e_ms = max_over_ranks(e_ms)
        e2e = {"value": round(aggregate_gbs(wb + db, e_steps, world, e_ms), 3), "unit": "GB/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
               "ms_per_step": round(e_ms / e_steps, 4), "steps": e_steps}

    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return 0

    peak, peak_src = measured_peaks()
    value = aggregate_gbs(wb + db, args.steps, world, total_ms)
    w_gbs = wb / (wr_ms / 1e3) / 1e9
    d_gbs = db / (de_ms / 1e3) / 1e9
    line = {
        "metric": METRIC, "value": round(value, 3), "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": warm, "ms_per_step": round(total_ms / args.steps, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "fp32",
        "data": "synthetic", "config": config_block(w, block, not args.no_graph),
        "pct_of_peak": round(100 * value / (peak * world), 2),
        "roofline": {"kernel": "kv_quant_write", "bound": "hbm", "achieved": round(w_gbs, 2),
                     "peak": peak, "unit": "GB/s", "frac": round(w_gbs / peak, 4),
                     "traffic": committed_traffic("kv_quant_write"),
                     "algorithmic_bytes": wb, "peak_source": f"{peak_src} (MEASURED_PEAKS.json hbm_gbs)"
                     if peak_src == "measured" else "fallback 6.65 TB/s"},
        "roofline_decode": {"kernel": "paged_decode_attn_int4", "bound": "hbm", "achieved": round(d_gbs, 2),
                            "peak": peak, "unit": "GB/s", "frac": round(d_gbs / peak, 4),
                            "traffic": committed_traffic("paged_decode_attn_int4"),
                            "algorithmic_bytes": db},
        "kernels": {
            "kv_quant_write": {"us": round(1e3 * wr_ms, 3), "GB/s": round(w_gbs, 2),
                               "tokens_per_s": round(w.tokens_written / (wr_ms / 1e3), 1)},
            "paged_decode_attn_int4": {"us": round(1e3 * de_ms, 3), "GB/s": round(d_gbs, 2),
                                       "decode_steps_x_batch_per_s": round(w.B / (de_ms / 1e3), 1),
                                       "cached_tokens_per_s": round(w.tokens_cached / (de_ms / 1e3), 1)},
        },
        "plain_int4": plain,
        "randomized_hadamard": randomized,
        "decode_append": {
            "what": "each sequence's new token stored, then a decode step over contexts that include it",
            "separate_us": round(1e3 * ap_sep_ms, 3),  # kv_quant_write (B tokens) + paged_decode_attn_int4
            "fused_us": round(1e3 * ap_fus_ms, 3),     # paged_decode_append_attn_int4
        },
        "prefill": prefill_line(pf_ms, pf_flops * world),
        "oscar": oscar,
        "configs": configs,
        "e2e": e2e,
        "clocks": clocks.summary(),
        "gpu_launches": 2 * args.steps,
    }
    if not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(w, block)
        line["prefill"]["cpu_baseline"] = prefill_cpu_baseline(w, block)
    print(json.dumps(line), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
