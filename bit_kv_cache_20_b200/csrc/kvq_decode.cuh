// kvq_decode.cuh - split-K paged decode attention over the rotated INT4 cache.
//
// SAW-INT4 (Abstract): attention is computed by the kernel that reads the
// quantized paged cache, with no separate dequantization pass. The rotation R is orthogonal and its own inverse, so the kernel
// rotates q once, runs attention in the rotated space directly on the codes,
// and rotates the output back: out = R sum_t p_t v^_t.
//
// 8 warps per CTA. A CTA serves HG kv heads (HG = 1, 2 or 4) over one
// contiguous range of one sequence's pages; warp w works for head w % HG and
// takes every (8/HG)-th page of the range. Grid: (split, kv-head group,
// sequence) with the same number of splits for every sequence, or, when the
// host passed its copy of the context lengths, (kv-head group, item) over a
// per-sequence item table (splits in proportion to length, longest first).
// The CTAs that take part in split merges are all resident at once. Each warp streams its own pages into a private
// ring of kWarpRing page slots in shared memory with 16-byte cp.async copies
// (the codes of one (page, head) are 16*D contiguous bytes; its 32 scales and
// 32 zeros 64 B each), kWarpRing - 1 pages ahead of the one it computes on.
// (Measured on B200 with this page layout: per-warp cp.async streams reach the
// bandwidth of a contiguous read; a single issuing thread with 1-D bulk copies
// and mbarriers stayed near a third of it.)
//
// Per page (16 tokens) and kv head, on the tensor cores, with the GQA group of
// up to 4 query heads as 8 columns:
//   QK (mma.m16n8k32, u8 x s8 -> s32, exact):
//        S^T[16 tokens x 8] = codes[16 tokens x D] * Q8^T[D x 8]
//   PV (mma.m16n8k16, f16 -> f32):
//        O^T[D x 8]        += codes^T[D x 16 tokens] * Phl^T[16 tokens x 8]
// QK takes the code bytes as they are: byte & 0x0F is the low code, byte &
// 0xF0 the high code times 16, each product summed in its own accumulator.
// q~ enters as three int8 limbs per element, q~ = sigma (q0 + q1 / 256 +
// q2 / 32768) with sigma = max|q~| / 127 per query head (error <= 2^-16 sigma;
// with two limbs the logit error, ~sigma / 512 times |k|, reached 1.7e-3 of
// output on keys with x10 outlier channels and large token norms); columns
// are (head, limb 0 / 1) in one 8-column tile and (head, limb 2) in the even
// columns of a second. PV needs floating
// weights: p * s_v enters as an fp16 "hi" and "lo" part (hi + lo keeps ~22
// bits) and the codes as exact normal fp16 values c * 2^-9: a byte holding a
// code in its low nibble, read as e4m3, is exactly c * 2^-9 (subnormal e4m3
// for c < 8, normal fp16 after the conversion), so one cvt turns two bytes
// into an A-operand register and the epilogue multiplies by 2^9. Subnormal
// fp16 operands are avoided on purpose - small products built from them lost
// precision in the tensor-core accumulation (a systematic bias of ~2^-13
// relative, measured on B200). QK leaves a thread the logits of 2 tokens for one query head; PV
// wants 4 tokens of one column, so 4 warp shuffles move the weights across.
// Dequantization is folded into per-token scalars:
//   logit_t = s_t * (q~ . code_t) + z_t * sum(q~)
//   o_rot   = (sum_t p_t s_t code_t + sum_t p_t z_t) / sum_t p_t
// with an online softmax in base 2 (log2 e folded into q~) that rescales only
// when the running maximum grows. q is rotated once per CTA in shared memory.
//
// With one split per (sequence, head group) the CTA rotates its output back
// and writes it; otherwise every split writes a partial result (O + Z, M, L)
// to the workspace in a self-validating encoding, and the first few splits
// each gather, merge, rotate back and write some of the group's query rows
// (details at the merge below).
#pragma once

#include <climits>

#include "kvq_device.cuh"

namespace kvq {

constexpr int kMaxPlanItems = 1024;  // (sequence, split) entries of a per-sequence plan

struct AttnParams {
  const uint16_t* q;          // bf16 [B][Hq][D]
  const uint8_t* cache;       // [pages][Hkv][2][16][D/2]
  const uint16_t* scales;     // fp16 [pages][Hkv][2][16]
  const uint16_t* zeros;
  const int32_t* page_table;  // [B][max_pages]
  const int32_t* ctx_lens;    // [B]
  void* out;                  // [B][Hq][D] fp32 or bf16
  uint32_t* ws_part;          // [slots][Hkv][G][D + 4]: ~bits of O + Z, M, L; a hand-over
                              // word; 1 unused. Zero between calls
  int B, Hq, Hkv, G;
  int num_pages, max_pages;
  int n_splits, pages_per_split;
  int out_bf16;
  float qmul;                 // c_b * softmax_scale * log2(e)
  float cb;                   // c_b (output rotation), 1 for plain INT4
  uint32_t signs[4];          // randomized Hadamard signs (bit c: channel c), as written
  int inputs_ready;           // q, page_table, ctx_lens not written by the previous kernel
  // Decode-append (slots_new != nullptr): sequence n's new token, k_new /
  // v_new bf16 [B][Hkv][D], is quantized and stored at slots_new[n] (-1: none)
  // as position ctx_lens[n] - 1 of the sequence, through cache_w, scales_w,
  // zeros_w (the same buffers as cache, scales, zeros).
  const uint16_t* k_new;
  const uint16_t* v_new;
  const int64_t* slots_new;
  uint8_t* cache_w;
  uint16_t* scales_w;
  uint16_t* zeros_w;
  // Per-sequence plan (n_items > 0; grid = (Hkv / HG, n_items)): item i is
  // x = sequence | split << 16 | splits << 24, y = first partial slot of the
  // sequence | pages per split << 16. Otherwise the grid is (n_splits,
  // Hkv / HG, B) with pages_per_split pages each and slot n * n_splits + split.
  int n_items;
  uint2 items[kMaxPlanItems];
};

// Warps per CTA: 8 for up to 4 query heads per kv head (two CTAs per SM);
// 12 for 8 query heads, whose doubled accumulators leave room for one CTA per
// SM only, so that SM still runs 12 page streams to hide each warp's
// per-page dependency chain.
__host__ __device__ constexpr int attn_warps(int nc) { return nc == 2 ? 12 : 8; }
constexpr int kWarpRing = 4;        // page slots per warp
constexpr int kMaxSplits = 128;
constexpr int kMaxPids = 1024;      // page ids of a CTA's range kept in shared memory
// states of a partial-result row's word D + 2 (zero: not written yet)
constexpr uint32_t kRowWritten = 1u;
constexpr uint32_t kRowHandedOver = 2u;
constexpr float kHead = 3.0f;        // log2 headroom of the lazy softmax reference
constexpr float kBigScale = 8188.0f; // 65504 / 2^kHead: larger V scales force p <= 1

// Shared memory of one decode CTA serving HG kv heads with NC column tiles
// (4 query heads each).
template <int D, int HG, int NC>
struct AttnSmem {
  static constexpr int kWarps = attn_warps(NC);
  static constexpr int kSlotBytes = 16 * D + 128;               // codes + 32 scales + 32 zeros
  static constexpr int kRingBytes = kWarps * kWarpRing * kSlotBytes;
  static constexpr int kRows = HG * 4 * NC;                     // query rows (G padded to 4 NC)
  // per-warp result: O[4 NC rows][D], then (m, l, zs, unused) per row
  static constexpr int kResFloats = 4 * NC * (D + 4);
  static constexpr int kOffRes = kRingBytes;
  static constexpr int kOffQ = kOffRes + kWarps * kResFloats * 4;  // float [kRows][D]
  static constexpr int kOffQInfo = kOffQ + kRows * D * 4;       // float [kRows][4]: scale, sum
  static constexpr int kOffQ8 = kOffQInfo + kRows * 16;         // int8 [kRows][3 limbs][D], B order
  static constexpr int kOffPid = kOffQ8 + kRows * 3 * D;
  // decode-append: per (kv head of the CTA, K|V) the new token's packed row,
  // then its fp16 scale and zero
  static constexpr int kAppRow = D / 2 + 16;
  static constexpr int kOffApp = kOffPid + kMaxPids * 4;
  // split-merge control words (see the merge at the end)
  static constexpr int kOffCtl = (kOffApp + HG * 2 * kAppRow + 15) / 16 * 16;
  static constexpr int kTotal = kOffCtl + 16;
};

template <int N>
__device__ __forceinline__ void lds_words(const uint8_t* src, uint32_t (&w)[N]) {
  if constexpr (N == 4) {
    const uint4 t = *reinterpret_cast<const uint4*>(src);
    w[0] = t.x; w[1] = t.y; w[2] = t.z; w[3] = t.w;
  } else if constexpr (N == 2) {
    const uint2 t = *reinterpret_cast<const uint2*>(src);
    w[0] = t.x; w[1] = t.y;
  } else {
    w[0] = *reinterpret_cast<const uint32_t*>(src);
  }
}

// fp16 pair of (x0, x1): the "hi" rounding, or with `lo` the remainder
// fp16(x - hi) of each.
__device__ __forceinline__ uint32_t hilo_pair(float x0, float x1, bool lo) {
  const __half2 h = __floats2half2_rn(x0, x1);
  const float2 hf = __half22float2(h);
  const __half2 l = __floats2half2_rn(__fsub_rn(x0, hf.x), __fsub_rn(x1, hf.y));
  const uint32_t hu = *reinterpret_cast<const uint32_t*>(&h), lu = *reinterpret_cast<const uint32_t*>(&l);
  return lo ? lu : hu;
}

__device__ __forceinline__ void store_out(const AttnParams& p, size_t idx, float v) {
  if (p.out_bf16)
    reinterpret_cast<__nv_bfloat16*>(p.out)[idx] = __float2bfloat16_rn(v);
  else
    reinterpret_cast<float*>(p.out)[idx] = v;
}

// Fast Walsh-Hadamard transform (blocks of BLK, Sylvester natural order:
// y_i = sum_j (-1)^popcount(i & j) x_j) of one row of D values spread over a
// warp, lane l holding elements [E l, E l + E), E = D / 32. Stages shorter than
// E stay in the thread; the others pair lanes l and l ^ (len / E).
template <int D, int BLK>
__device__ __forceinline__ void warp_fwht(float (&v)[D / 32], int lane) {
  constexpr int E = D / 32;
#pragma unroll
  for (int len = 1; len < E && len < BLK; len <<= 1) {
#pragma unroll
    for (int i = 0; i < E; ++i) {
      if ((i & len) == 0) {
        const float a = v[i], b = v[i + len];
        v[i] = a + b;
        v[i + len] = a - b;
      }
    }
  }
#pragma unroll
  for (int len = E; len < BLK; len <<= 1) {
    const int m = len / E;
    const bool upper = (lane & m) != 0;
#pragma unroll
    for (int i = 0; i < E; ++i) {
      const float other = __shfl_xor_sync(0xffffffffu, v[i], m);
      v[i] = upper ? (other - v[i]) : (v[i] + other);
    }
  }
}


// Randomized Hadamard: negate the lane's elements (channels E lane + e) whose
// sign bit is set. R = H_b diag(sigma) / sqrt(b): applied before the
// transform to rotate, after it for R^T.
template <int D>
__device__ __forceinline__ void apply_signs(float (&v)[D / 32], const uint32_t (&sg)[4], int lane) {
  constexpr int E = D / 32;
#pragma unroll
  for (int e = 0; e < E; ++e) {
    const int c = E * lane + e;
    v[e] = __uint_as_float(__float_as_uint(v[e]) ^ (((sg[c >> 5] >> (c & 31)) & 1u) << 31));
  }
}

template <int D, int BLK, int HG, int NC, bool APP>
__global__ void __launch_bounds__(32 * attn_warps(NC), NC == 1 ? 2 : 1)
    kvq_decode_kernel(const __grid_constant__ AttnParams p) {
  using S = AttnSmem<D, HG, NC>;
  constexpr int kAttnWarps = S::kWarps;
  constexpr int kAttnThreads = 32 * kAttnWarps;
  constexpr int NSUB = kAttnWarps / HG;  // warps per head
  constexpr int R = kWarpRing;
  constexpr int SLOT = S::kSlotBytes;
  constexpr int KW = D / 32;   // K-row words per thread (QK)
  constexpr int KM = KW / 2;   // QK MMAs per nibble half (32 codes of a row each)
  constexpr int VW = D / 64;   // V-row words per thread (PV)
  constexpr int MT = D / 16;   // PV m-tiles (16 channels each)
  constexpr int NR = 4 * NC;   // query rows per head, padded
  constexpr int E = D / 32;    // row elements per lane in warp-level row work
  extern __shared__ __align__(128) uint8_t smem[];
  float* res = reinterpret_cast<float*>(smem + S::kOffRes);
  float* qs = reinterpret_cast<float*>(smem + S::kOffQ);
  float* qinfo = reinterpret_cast<float*>(smem + S::kOffQInfo);
  int8_t* q8 = reinterpret_cast<int8_t*>(smem + S::kOffQ8);
  int* pids = reinterpret_cast<int*>(smem + S::kOffPid);

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2, tig = lane & 3;
  const int hw = warp % HG, sub = warp / HG;
  int n, split, ns, slot_base, pps, hgi;
  if (p.n_items > 0) {
    const uint2 it = p.items[blockIdx.y];
    hgi = blockIdx.x;
    n = it.x & 0xFFFF;
    split = (it.x >> 16) & 0xFF;
    ns = it.x >> 24;
    slot_base = it.y & 0xFFFF;
    pps = it.y >> 16;
  } else {
    split = blockIdx.x;
    hgi = blockIdx.y;
    n = blockIdx.z;
    ns = p.n_splits;
    slot_base = n * ns;
    pps = p.pages_per_split;
  }
  const int G = p.G;
  const unsigned FULL = 0xffffffffu;
  // Split-merge control words: [0] a merger's hand-over decision (0 none yet,
  // 3 being taken, 1 kept every row, 2 handed rows over), [1] rows handed
  // over by this CTA, [2] rows handed over to this CTA.
  uint32_t* sctl = reinterpret_cast<uint32_t*>(smem + S::kOffCtl);

  // The launch may overlap the previous kernel on the stream (programmatic
  // dependent launch). By default everything waits for it here; with
  // inputs_ready the page ids, context length and q are read and q is
  // rotated first, and the wait comes before the first cache read.
  const bool early = p.inputs_ready != 0;
  if (!early) {
    pdl_wait();
    pdl_launch_dependents();
  }

  // Page ids of the split's range (the page-table row is max_pages long, so
  // they are read before the context length is known), the context length,
  // and the query rows of the CTA's heads (fp32, rows >= G zero).
  int p_begin = split * pps;
  const int32_t* pt_row = p.page_table + (size_t)n * p.max_pages + p_begin;
  for (int i = tid; i < min(p_begin + pps, p.max_pages) - p_begin && i < kMaxPids; i += kAttnThreads)
    pids[i] = pt_row[i];
  int ctx = p.ctx_lens[n];
  long long app_slot = -1;
  if constexpr (APP) app_slot = p.slots_new[n];
  for (int i = tid; i < S::kRows * (D / 8); i += kAttnThreads) {
    const int row = i / (D / 8), c8 = i % (D / 8);
    const int hh = row / NR, r = row % NR;
    float v[8];
    if (r < G) {
      const uint4 u = *reinterpret_cast<const uint4*>(
          p.q + ((size_t)n * p.Hq + (size_t)(hgi * HG + hh) * G + r) * D + 8 * c8);
      const uint32_t w4[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        v[2 * e] = __uint_as_float(w4[e] << 16);
        v[2 * e + 1] = __uint_as_float(w4[e] & 0xffff0000u);
      }
    } else {
#pragma unroll
      for (int e = 0; e < 8; ++e) v[e] = 0.0f;
    }
    float4* dst = reinterpret_cast<float4*>(qs + row * D + 8 * c8);
    dst[0] = make_float4(v[0], v[1], v[2], v[3]);
    dst[1] = make_float4(v[4], v[5], v[6], v[7]);
  }
  const int cap = p.max_pages * 16;
  if (ctx < 0 || ctx > cap) {
    if (tid == 0) record_error(KVQ_ERR_OUT_OF_RANGE);
    ctx = ctx < 0 ? 0 : cap;
  }
  const int n_pages = (ctx + 15) >> 4;
  if (n_pages > ns * pps) {
    // only a per-sequence plan made from host lengths shorter than these:
    // re-split so that every page is still covered once
    pps = (n_pages + ns - 1) / ns;
    p_begin = split * pps;
    pt_row = p.page_table + (size_t)n * p.max_pages + p_begin;
    for (int i = tid; i < min(p_begin + pps, p.max_pages) - p_begin && i < kMaxPids; i += kAttnThreads)
      pids[i] = pt_row[i];
  }
  const int npg = max(min(p_begin + pps, n_pages) - p_begin, 0);
  if (tid < 4) sctl[tid] = 0;
  __syncthreads();

  // Decode-append: the CTA whose range holds position ctx - 1 owns the new
  // token; its slot must be that position's (page-table entry, offset).
  int app_t = -1, app_off = 0;  // the token's page within the range, and row
  if (APP && app_slot >= 0) {
    const int tn = ctx - 1, pl = tn >> 4;
    if (tn >= 0 && pl >= p_begin && pl < p_begin + npg) {
      const int t = pl - p_begin;
      const int id = (t < kMaxPids) ? pids[t] : pt_row[t];
      if (app_slot < (long long)p.num_pages * 16 && (app_slot >> 4) == id && (int)(app_slot & 15) == (tn & 15)) {
        app_t = t;
        app_off = tn & 15;
      } else if (tid == 0) {
        record_error(KVQ_ERR_OUT_OF_RANGE);
      }
    } else if (tn < 0 && tid == 0) {
      record_error(KVQ_ERR_OUT_OF_RANGE);  // a new token for an empty context
    }
  }

  // ---- this warp's page stream: pages sub, sub + NSUB, ... of head hw -----
  // fetch(k) copies the warp's k-th page into ring slot k % R (one commit
  // group per call, empty past the end); bit k % R of `valid` says whether
  // the slot holds a page. Lane l copies 16-byte chunks l, l + 32, ... of the
  // codes; lanes 0..3 one chunk of the scales, lanes 4..7 of the zeros.
  uint8_t* ring = smem + warp * (R * SLOT);
  const uint32_t ring_lane = smem_addr(ring) + lane * 16;
  const size_t head_off = (size_t)hgi * HG + hw;
  const uint8_t* code_lane = p.cache + head_off * (16 * D) + lane * 16;
  const uint16_t* sz_lane = (lane < 4 ? p.scales : p.zeros) + head_off * 32 + (lane & 3) * 8;
  const size_t code_page = (size_t)p.Hkv * (16 * D);  // bytes per page
  const size_t sz_page = (size_t)p.Hkv * 32;          // fp16 per page
  uint32_t valid = 0;
  auto fetch_t = [&](int k, int t) {
    const int slot = k % R;
    bool ok = false;
    if (t < npg) {
      const int id = (t < kMaxPids) ? pids[t] : pt_row[t];
      ok = id >= 0 && id < p.num_pages;
      if (ok) {
        const uint8_t* src = code_lane + (size_t)id * code_page;
        const uint32_t dst = ring_lane + slot * SLOT;
#pragma unroll
        for (int j = 0; j < D / 32; ++j) cp_async_16(dst + 512 * j, src + 512 * j);
        cp_async_16_if(dst + 16 * D, sz_lane + (size_t)id * sz_page, lane < 8);
      } else if (lane == 0) {
        record_error(KVQ_ERR_OUT_OF_RANGE);
      }
    }
    valid = ok ? (valid | (1u << slot)) : (valid & ~(1u << slot));
    cp_async_commit();
  };
  auto fetch = [&](int k) { fetch_t(k, sub + k * NSUB); };
  // ---- q~ = R q * (softmax_scale * log2 e) -----------------------------------
  // One warp per row. Limbs, with a = q~ / sigma and sigma = max|q~| / 127:
  // q0 = rint(a), r1 = 256 (a - q0), q1 = rint(r1), q2 = rint(128 (r1 - q1))
  // (every step exact in fp32; |q1|, |q2| <= 64 except at exact ties, where
  // the +-127 clamp costs at most sigma / 32768). They are stored in B-fragment
  // order: element 8w + j goes to byte tig*8KW + ((m*2 + (j&1))*2 + h)*4 +
  // (j>>1) of its limb's array, w = KW*tig + 2m + h, so that thread tig reads
  // its fragments as 8KW contiguous bytes.
  auto prep_q = [&]() {
    for (int row = warp; row < S::kRows; row += kAttnWarps) {
      const float* rp = qs + row * D;
      float v[E];
#pragma unroll
      for (int e = 0; e < E; ++e) v[e] = rp[E * lane + e];
      if constexpr (BLK > 0) {
        apply_signs<D>(v, p.signs, lane);
        warp_fwht<D, BLK>(v, lane);
      }
      float amax = 0.0f, sum = 0.0f;
#pragma unroll
      for (int e = 0; e < E; ++e) {
        v[e] *= p.qmul;
        amax = fmaxf(amax, fabsf(v[e]));
        sum += v[e];
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        amax = fmaxf(amax, __shfl_xor_sync(FULL, amax, o));
        sum += __shfl_xor_sync(FULL, sum, o);
      }
      const float sigma = amax / 127.0f;
      const float inv = (amax > 0.0f) ? 127.0f / amax : 0.0f;
      if (lane == 0) {
        qinfo[row * 4 + 0] = sigma * (1.0f / 16.0f);
        qinfo[row * 4 + 1] = sum;
      }
      int8_t* l0 = q8 + row * 3 * D;
      int8_t* l1 = l0 + D;
      int8_t* l2 = l1 + D;
#pragma unroll
      for (int e = 0; e < E; ++e) {
        const int el = E * lane + e, w = el >> 3, j = el & 7;
        const int tw = w / KW, rw = w % KW;
        const int off = tw * (8 * KW) + (((rw >> 1) * 2 + (j & 1)) * 2 + (rw & 1)) * 4 + (j >> 1);
        const float a = __fmul_rn(v[e], inv);
        const float q0 = rintf(a);
        const float r1 = __fmul_rn(__fsub_rn(a, q0), 256.0f);
        const float q1 = fminf(fmaxf(rintf(r1), -127.0f), 127.0f);
        const float q2 = fminf(fmaxf(rintf(__fmul_rn(__fsub_rn(r1, q1), 128.0f)), -127.0f), 127.0f);
        l0[off] = (int8_t)(int)q0;
        l1[off] = (int8_t)(int)q1;
        l2[off] = (int8_t)(int)q2;
      }
    }
    __syncthreads();
  };
  // Decode-append, in the owner CTA: warp 2 hh + kv rotates, quantizes and
  // packs the new token's K (kv = 0) or V row of head hh exactly as
  // kv_quant_write defines it (z = RD16(min y), s = the smallest fp16 with
  // 15 s + z >= max y, code = rint(fp32(y - z) * fp32(1/s))), stores it in the
  // cache and keeps a copy in shared memory; the warp that computes on that
  // page patches its copy of the page with it (the cp.async copy may predate
  // the store), so the attention sees the row as stored.
  auto append = [&]() {
    if (!APP || app_t < 0 || warp >= 2 * HG) return;
    const int hh = warp >> 1, kv = warp & 1;
    const size_t head = (size_t)hgi * HG + hh;
    const uint16_t* src = (kv ? p.v_new : p.k_new) + ((size_t)n * p.Hkv + head) * D + E * lane;
    float v[E];
#pragma unroll
    for (int e = 0; e < E; ++e) v[e] = bf16_bits_to_float(src[e]);
    if constexpr (BLK > 0) {
      apply_signs<D>(v, p.signs, lane);
      warp_fwht<D, BLK>(v, lane);
    }
    float mn = v[0], mx = v[0];
#pragma unroll
    for (int e = 1; e < E; ++e) {
      mn = fminf(mn, v[e]);
      mx = fmaxf(mx, v[e]);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      mn = fminf(mn, __shfl_xor_sync(FULL, mn, o));
      mx = fmaxf(mx, __shfl_xor_sync(FULL, mx, o));
    }
    mn = __fmul_rn(mn, p.cb);  // y = fp32(H x) * c_b is monotone in H x
    mx = __fmul_rn(mx, p.cb);
    const __half zh = __float2half_rd(mn);
    const float zf = __half2float(zh);
    const float dz = __fsub_ru(mx, zf);
    const float need = __fmul_ru(dz, 0.0666666701f);  // RU(1/15): a candidate at most one step high
    unsigned short sbits = __half_as_ushort(__float2half_ru(need));
    if (sbits != 0 && sbits < 0x7C00) {  // one fp16 step lower may still cover max y (exact fp32 test)
      const unsigned short pb = (unsigned short)(sbits - 1);
      if (__fmul_rn(15.0f, __half2float(__ushort_as_half(pb))) >= dz) sbits = pb;
    }
    const float sf = __half2float(__ushort_as_half(sbits));
    const float inv = (sf > 0.0f) ? __frcp_rn(sf) : 0.0f;
    uint32_t packed = 0;  // E codes, two per byte, low nibble first
#pragma unroll
    for (int e = 0; e < E; ++e) {
      const float y = __fmul_rn(v[e], p.cb);
      const uint32_t code = __float_as_uint(__fmaf_rn(__fsub_rn(y, zf), inv, 8388608.0f)) & 0xFu;
      packed |= code << (4 * e);
    }
    const long long row = (((app_slot >> 4) * p.Hkv + (long long)head) * 2 + kv) * 16 + app_off;
    uint8_t* sdst = smem + S::kOffApp + (hh * 2 + kv) * S::kAppRow;
    if constexpr (E == 4) {
      *reinterpret_cast<uint16_t*>(p.cache_w + row * (D / 2) + 2 * lane) = (uint16_t)packed;
      *reinterpret_cast<uint16_t*>(sdst + 2 * lane) = (uint16_t)packed;
    } else {
      p.cache_w[row * (D / 2) + lane] = (uint8_t)packed;
      sdst[lane] = (uint8_t)packed;
    }
    if (lane == 0) {
      p.scales_w[row] = sbits;
      p.zeros_w[row] = __half_as_ushort(zh);
      reinterpret_cast<uint16_t*>(sdst + D / 2)[0] = sbits;
      reinterpret_cast<uint16_t*>(sdst + D / 2)[1] = __half_as_ushort(zh);
    }
  };
  static_assert(E == 2 || E == 4, "row elements per lane");

  if (early) {
    prep_q();    // overlaps the previous kernel's last CTAs
    pdl_wait();  // the cache (and the workspace) may be what that kernel wrote
    pdl_launch_dependents();
#pragma unroll
    for (int k = 0; k < R - 1; ++k) fetch(k);
    append();
    if (APP && app_t >= 0) __syncthreads();  // the shared copy of the new rows
  } else {
#pragma unroll
    for (int k = 0; k < R - 1; ++k) fetch(k);
    append();
    prep_q();    // while the first pages land (ends with a barrier)
  }

  // B fragments of QK. Tile 0: column g is limb g&1 of query row 4c + g/2 of
  // head hw; tile 1: column g is limb 2 of that row for even g, zero for odd.
  // MMA (m, half) of thread tig: b0 = bytes of k-group tig, b1 of k-group
  // 4 + tig; their codes are the low (half 0) or high (half 1) nibbles of K
  // words KW*tig + 2m (b0) and KW*tig + 2m + 1 (b1). With one column tile
  // they stay in registers; with two they are read from shared memory for
  // every page (registers for a third CTA-wide warp group instead).
  const uint8_t* qfb[NC];
#pragma unroll
  for (int c = 0; c < NC; ++c)
    qfb[c] = reinterpret_cast<const uint8_t*>(q8 + (hw * NR + 4 * c + (g >> 1)) * 3 * D) + tig * (8 * KW);
  auto qfrag = [&](int c, int m, uint4& f4, uint4& h4) {
    f4 = *reinterpret_cast<const uint4*>(qfb[c] + (g & 1) * D + 16 * m);
    h4 = (g & 1) ? make_uint4(0u, 0u, 0u, 0u) : *reinterpret_cast<const uint4*>(qfb[c] + 2 * D + 16 * m);
  };
  constexpr int NCR = NC == 1 ? 1 : 0;  // column tiles whose fragments stay in registers
  uint4 bqf[NCR > 0 ? NCR : 1][KM], bqh[NCR > 0 ? NCR : 1][KM];
#pragma unroll
  for (int c = 0; c < NCR; ++c)
#pragma unroll
    for (int m = 0; m < KM; ++m) qfrag(c, m, bqf[c][m], bqh[c][m]);
  // this thread's QK results belong to query row 4c + tig of head hw
  float qsc[NC], qsm[NC];
  bool hv[NC];
#pragma unroll
  for (int c = 0; c < NC; ++c) {
    const int row = hw * NR + 4 * c + tig;
    qsc[c] = qinfo[row * 4 + 0];
    qsm[c] = qinfo[row * 4 + 1];
    hv[c] = 4 * c + tig < G;
  }
  // PV B fragments: column g wants tokens 2tig, 2tig+1 (held by lanes
  // 8tig + g/2 and 8tig + 4 + g/2 as their token g) and 2tig+8, 2tig+9 (the
  // same lanes' token g+8)
  const int la = 8 * tig + (g >> 1), lb = la + 4;

  float o[NC][MT][4];
#pragma unroll
  for (int c = 0; c < NC; ++c)
#pragma unroll
    for (int i = 0; i < MT; ++i) o[c][i][0] = o[c][i][1] = o[c][i][2] = o[c][i][3] = 0.0f;
  float m_run[NC], l_run[NC], zs_run[NC];
#pragma unroll
  for (int c = 0; c < NC; ++c) {
    m_run[c] = hv[c] ? -INFINITY : 0.0f;  // padding rows: p = exp2(-inf - 0) = 0
    l_run[c] = 0.0f;
    zs_run[c] = 0.0f;
  }
  const int tok_base = p_begin * 16;

  for (int k = 0; sub + k * NSUB < npg; ++k) {
    const int t = sub + k * NSUB;
    fetch(k + R - 1);
    cp_async_wait<R - 1>();  // page k has landed (this lane's copies)
    __syncwarp();            // ... and every other lane's
    if ((valid >> (k % R)) & 1u) {
      if (APP && t == app_t) {
        // the new token's rows replace this page's copy of that position
        uint8_t* pg = ring + (k % R) * SLOT;
        const uint8_t* a = smem + S::kOffApp + hw * 2 * S::kAppRow;  // K row, then V row
        constexpr int CH = D / 32;  // 16-byte chunks of a packed row
        if (lane < 2 * CH) {
          const int kvp = lane / CH, c = lane % CH;
          *reinterpret_cast<uint4*>(pg + kvp * 8 * D + app_off * (D / 2) + 16 * c) =
              *reinterpret_cast<const uint4*>(a + kvp * S::kAppRow + 16 * c);
        } else if (lane < 2 * CH + 2) {
          const int kvp = lane - 2 * CH;
          const uint16_t* sz = reinterpret_cast<const uint16_t*>(a + kvp * S::kAppRow + D / 2);
          reinterpret_cast<uint16_t*>(pg + 16 * D)[16 * kvp + app_off] = sz[0];
          reinterpret_cast<uint16_t*>(pg + 16 * D + 64)[16 * kvp + app_off] = sz[1];
        }
        __syncwarp();
      }
      const uint8_t* kb = ring + (k % R) * SLOT;  // K block [16][D/2], then V block
      const uint8_t* vb = kb + 8 * D;
      const __half* scl = reinterpret_cast<const __half*>(kb + 16 * D);       // 16 K, then 16 V scales
      const __half* zer = reinterpret_cast<const __half*>(kb + 16 * D + 64);  // zeros, likewise

      // QK: A = code bytes of tokens g (rows 0..7) and g+8 (rows 8..15)
      uint32_t ka[KW], kc[KW];
      lds_words<KW>(kb + g * (D / 2) + tig * (4 * KW), ka);
      lds_words<KW>(kb + (g + 8) * (D / 2) + tig * (4 * KW), kc);
      int accl[NC][4], acch[NC][4], accl2[NC][4], acch2[NC][4];
#pragma unroll
      for (int m = 0; m < KM; ++m) {
        const uint32_t x0 = ka[2 * m], x1 = ka[2 * m + 1], y0 = kc[2 * m], y1 = kc[2 * m + 1];
        const uint32_t al[4] = {x0 & 0x0F0F0F0Fu, y0 & 0x0F0F0F0Fu, x1 & 0x0F0F0F0Fu, y1 & 0x0F0F0F0Fu};
        const uint32_t ah[4] = {x0 & 0xF0F0F0F0u, y0 & 0xF0F0F0F0u, x1 & 0xF0F0F0F0u, y1 & 0xF0F0F0F0u};
#pragma unroll
        for (int c = 0; c < NC; ++c) {
          uint4 f4, h4;
          if constexpr (NCR > 0) {
            f4 = bqf[c][m];
            h4 = bqh[c][m];
          } else {
            qfrag(c, m, f4, h4);
          }
          if (m == 0) {
            mma_u8s8_16832_z(accl[c], al, f4.x, f4.y);
            mma_u8s8_16832_z(acch[c], ah, f4.z, f4.w);
            mma_u8s8_16832_z(accl2[c], al, h4.x, h4.y);
            mma_u8s8_16832_z(acch2[c], ah, h4.z, h4.w);
          } else {
            mma_u8s8_16832(accl[c], al, f4.x, f4.y);
            mma_u8s8_16832(acch[c], ah, f4.z, f4.w);
            mma_u8s8_16832(accl2[c], al, h4.x, h4.y);
            mma_u8s8_16832(acch2[c], ah, h4.z, h4.w);
          }
        }
      }
      const float sk0 = __half2float(scl[g]), sk1 = __half2float(scl[g + 8]);
      const float zk0 = __half2float(zer[g]), zk1 = __half2float(zer[g + 8]);
      float sv0 = __half2float(scl[16 + g]), sv1 = __half2float(scl[24 + g]);
      float zv0 = __half2float(zer[16 + g]), zv1 = __half2float(zer[24 + g]);
      const int tok = tok_base + 16 * t;
      const bool tail = tok + 16 > ctx;
      const bool sv_big = fmaxf(sv0, sv1) > kBigScale;
      if (tail) {
        // rows past the context may hold anything, NaN scales included: they
        // get p = 0 below, and V scale and offset 0 so that 0 * garbage
        // cannot reach the sums
        if (tok + g >= ctx) sv0 = zv0 = 0.0f;
        if (tok + g + 8 >= ctx) sv1 = zv1 = 0.0f;
      }

      uint32_t bp[NC][2];
#pragma unroll
      for (int c = 0; c < NC; ++c) {
        // logits (base 2) of tokens g and g+8 for query row 4c + tig
        // X_l = 16 S_l = 16 acc_lo + acc_hi of limb l, an integer below 2^22
        // in magnitude (exact in fp32); q~ . code = sigma / 16 (X_0 + X_1 / 256
        // + X_2 / 32768), summed in fp32
        const float T0 = fmaf(fmaf((float)(accl2[c][0] * 16 + acch2[c][0]), 1.0f / 128.0f,
                                   (float)(accl[c][1] * 16 + acch[c][1])),
                              1.0f / 256.0f, (float)(accl[c][0] * 16 + acch[c][0]));
        const float T1 = fmaf(fmaf((float)(accl2[c][2] * 16 + acch2[c][2]), 1.0f / 128.0f,
                                   (float)(accl[c][3] * 16 + acch[c][3])),
                              1.0f / 256.0f, (float)(accl[c][2] * 16 + acch[c][2]));
        float lg0 = fmaf(T0 * qsc[c], sk0, zk0 * qsm[c]);
        float lg1 = fmaf(T1 * qsc[c], sk1, zk1 * qsm[c]);
        if (!hv[c]) lg0 = lg1 = -INFINITY;
        if (tail) {
          if (tok + g >= ctx) lg0 = -INFINITY;
          if (tok + g + 8 >= ctx) lg1 = -INFINITY;
        }
        // lazy online softmax: p = exp2(logit - m) with m the reference the
        // sums are kept in; it moves only when a logit exceeds m + kHead
        // (or a huge V scale could overflow the fp16 weight), so most pages
        // need neither a max reduction nor a rescale
        const bool need = (lg0 > m_run[c] + kHead) || (lg1 > m_run[c] + kHead) || sv_big;
        if (__any_sync(FULL, need)) {
          float pm = fmaxf(lg0, lg1);
          pm = fmaxf(pm, __shfl_xor_sync(FULL, pm, 4));
          pm = fmaxf(pm, __shfl_xor_sync(FULL, pm, 8));
          pm = fmaxf(pm, __shfl_xor_sync(FULL, pm, 16));
          const bool big = __any_sync(FULL, sv_big);
          const float mn = (pm > m_run[c] + kHead || (big && pm > m_run[c])) ? pm : m_run[c];
          const float alpha = fast_exp2(m_run[c] - mn);
#pragma unroll
          for (int i = 0; i < MT; ++i) {
            o[c][i][0] *= alpha; o[c][i][1] *= alpha; o[c][i][2] *= alpha; o[c][i][3] *= alpha;
          }
          l_run[c] *= alpha;
          zs_run[c] *= alpha;
          m_run[c] = mn;
        }
        const float p0 = fast_exp2(lg0 - m_run[c]);
        const float p1 = fast_exp2(lg1 - m_run[c]);
        l_run[c] += p0 + p1;
        zs_run[c] = fmaf(p0, zv0, fmaf(p1, zv1, zs_run[c]));
        const float P0 = p0 * sv0, P1 = p1 * sv1;
        // move p*s_v to the PV B layout (4 tokens of column g)
        const float q0 = __shfl_sync(FULL, P0, la), q1 = __shfl_sync(FULL, P0, lb);
        const float q2 = __shfl_sync(FULL, P1, la), q3 = __shfl_sync(FULL, P1, lb);
        bp[c][0] = hilo_pair(q0, q1, g & 1);
        bp[c][1] = hilo_pair(q2, q3, g & 1);
      }

      // PV: A = codes^T; rows g / g+8 of m-tile 4u+j are channels
      // 8cb + {0,1,4,5}[j] / 8cb + {2,3,6,7}[j] (cb = VW g + u); k-slots
      // 2tig, 2tig+1, 2tig+8, 2tig+9 are those tokens
      uint32_t va[VW], vb2[VW], vc[VW], vd[VW];
      lds_words<VW>(vb + (2 * tig) * (D / 2) + g * (4 * VW), va);
      lds_words<VW>(vb + (2 * tig + 1) * (D / 2) + g * (4 * VW), vb2);
      lds_words<VW>(vb + (2 * tig + 8) * (D / 2) + g * (4 * VW), vc);
      lds_words<VW>(vb + (2 * tig + 9) * (D / 2) + g * (4 * VW), vd);
#pragma unroll
      for (int u = 0; u < VW; ++u) {
        // bytes [tok0.b0, tok1.b0, tok0.b1, tok1.b1] (and b2, b3); a code in a
        // byte's low nibble, read as e4m3, is exactly code * 2^-9
        const uint32_t x0 = prmt(va[u], vb2[u], 0x5140), x1 = prmt(va[u], vb2[u], 0x7362);
        const uint32_t y0 = prmt(vc[u], vd[u], 0x5140), y1 = prmt(vc[u], vd[u], 0x7362);
        auto cv = [](uint32_t x, uint32_t& lo, uint32_t& hi) {
          asm("{\n .reg .b16 a, b;\n mov.b32 {a, b}, %2;\n cvt.rn.f16x2.e4m3x2 %0, a;\n"
              " cvt.rn.f16x2.e4m3x2 %1, b;\n}\n" : "=r"(lo), "=r"(hi) : "r"(x));
        };
        uint32_t m0[4], m1[4], m2[4], m3[4];
        cv(x0 & 0x0F0F0F0Fu, m0[0], m0[1]);
        cv((x0 >> 4) & 0x0F0F0F0Fu, m1[0], m1[1]);
        cv(y0 & 0x0F0F0F0Fu, m0[2], m0[3]);
        cv((y0 >> 4) & 0x0F0F0F0Fu, m1[2], m1[3]);
        cv(x1 & 0x0F0F0F0Fu, m2[0], m2[1]);
        cv((x1 >> 4) & 0x0F0F0F0Fu, m3[0], m3[1]);
        cv(y1 & 0x0F0F0F0Fu, m2[2], m2[3]);
        cv((y1 >> 4) & 0x0F0F0F0Fu, m3[2], m3[3]);
#pragma unroll
        for (int c = 0; c < NC; ++c) {
          mma_f16_16816(o[c][4 * u + 0], m0, bp[c][0], bp[c][1]);
          mma_f16_16816(o[c][4 * u + 1], m1, bp[c][0], bp[c][1]);
          mma_f16_16816(o[c][4 * u + 2], m2, bp[c][0], bp[c][1]);
          mma_f16_16816(o[c][4 * u + 3], m3, bp[c][0], bp[c][1]);
        }
      }
    }
    __syncwarp();  // the slot is read out before a later fetch refills it
  }
  cp_async_wait<0>();

  // ---- per-warp result: O[row][channel], (m, l, zs) per row -----------------
#pragma unroll
  for (int c = 0; c < NC; ++c) {
#pragma unroll
    for (int o2 = 4; o2 < 32; o2 <<= 1) {
      l_run[c] += __shfl_xor_sync(FULL, l_run[c], o2);
      zs_run[c] += __shfl_xor_sync(FULL, zs_run[c], o2);
    }
  }
  {
    float* mine = res + warp * S::kResFloats;
#pragma unroll
    for (int c = 0; c < NC; ++c) {
      float* orow = mine + (4 * c + tig) * D;
#pragma unroll
      for (int u = 0; u < VW; ++u) {
        const int cb = VW * g + u;
        const float* t0 = o[c][4 * u];
        const float* t1 = o[c][4 * u + 1];
        const float* t2 = o[c][4 * u + 2];
        const float* t3 = o[c][4 * u + 3];
        // hi + lo columns; the codes entered as c * 2^-9
        float4* dst = reinterpret_cast<float4*>(orow + 8 * cb);
        dst[0] = make_float4((t0[0] + t0[1]) * 512.0f, (t1[0] + t1[1]) * 512.0f, (t0[2] + t0[3]) * 512.0f,
                             (t1[2] + t1[3]) * 512.0f);
        dst[1] = make_float4((t2[0] + t2[1]) * 512.0f, (t3[0] + t3[1]) * 512.0f, (t2[2] + t2[3]) * 512.0f,
                             (t3[2] + t3[3]) * 512.0f);
      }
      if (g == 0) {
        float* ml = mine + NR * D + (4 * c + tig) * 4;
        ml[0] = m_run[c];
        ml[1] = l_run[c];
        ml[2] = zs_run[c];
      }
    }
  }
  __syncthreads();

  // ---- merge the NSUB warps of each head: output rows or a partial result --
  const bool single = ns == 1;
  for (int e = tid; e < HG * G * (D / 4); e += kAttnThreads) {
    const int hh = e / (G * (D / 4)), r = (e / (D / 4)) % G, c4 = 4 * (e % (D / 4));
    float mw[NSUB];
    float M = -INFINITY;
#pragma unroll
    for (int s2 = 0; s2 < NSUB; ++s2) {
      mw[s2] = res[(hh + HG * s2) * S::kResFloats + NR * D + r * 4];
      M = fmaxf(M, mw[s2]);
    }
    float4 O = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
    float L = 0.0f, Z = 0.0f;
    if (M != -INFINITY) {
#pragma unroll
      for (int s2 = 0; s2 < NSUB; ++s2) {
        const float* sl = res + (hh + HG * s2) * S::kResFloats;
        const float wgt = (mw[s2] == -INFINITY) ? 0.0f : fast_exp2(mw[s2] - M);
        const float4 v = *reinterpret_cast<const float4*>(sl + r * D + c4);
        O.x = fmaf(wgt, v.x, O.x);
        O.y = fmaf(wgt, v.y, O.y);
        O.z = fmaf(wgt, v.z, O.z);
        O.w = fmaf(wgt, v.w, O.w);
        L = fmaf(wgt, sl[NR * D + r * 4 + 1], L);
        Z = fmaf(wgt, sl[NR * D + r * 4 + 2], Z);
      }
    }
    if (single) {
      const float inv = (L > 0.0f) ? 1.0f / L : 0.0f;
      *reinterpret_cast<float4*>(qs + (hh * NR + r) * D + c4) =
          make_float4((O.x + Z) * inv, (O.y + Z) * inv, (O.z + Z) * inv, (O.w + Z) * inv);
    } else {
      // the split's partial result, every word stored as ~bits (see below)
      uint32_t* dst = p.ws_part + ((((size_t)slot_base + split) * p.Hkv + hgi * HG + hh) * G + r) * (D + 4);
      *reinterpret_cast<uint4*>(dst + c4) = make_uint4(~__float_as_uint(O.x + Z), ~__float_as_uint(O.y + Z),
                                                       ~__float_as_uint(O.z + Z), ~__float_as_uint(O.w + Z));
      if (c4 == 0) {
        *reinterpret_cast<uint2*>(dst + D) = make_uint2(~__float_as_uint(M), ~__float_as_uint(L));
        // mark the row written; a merger may have handed the row to this
        // split meanwhile (see the split merge)
        if (atomicExch(dst + D + 2, kRowWritten) == kRowHandedOver) atomicOr(&sctl[2], 1u << (hh * G + r));
      }
    }
  }

  if (!single) {
    __syncthreads();  // the rows handed over to this split are known
    // ---- split merge: CTA j < K merges query rows j, j + K, ... ------------
    // Each 32-bit word of a partial result is stored as ~bits(x). fp32
    // arithmetic never yields the bits 0xFFFFFFFF (a NaN payload it does not
    // produce), so no stored word is zero, and a zero word of the zero-filled
    // workspace means that split has not written it yet. A merger polls the
    // words of its rows in L2 until none is zero - no fence or ticket between
    // writer and reader, each word validates itself - folds them and zeroes
    // them again for the next call.
    //
    // The splits a merger waits for have to get to run, and nothing
    // guarantees that all CTAs of a launch are resident at once (other
    // streams' kernels may hold SMs). So a merger never waits for long on a
    // split that has not written: after a while it hands its rows over to
    // such a split through a compare-and-swap of that split's row word D + 2
    // (0 -> handed over) and exits. Every split, when it writes a row of its
    // partial result, exchanges that word for "written"; finding "handed
    // over", it merges the row itself once its partial is written. The word
    // changes once either way, so each row is merged exactly once, and a CTA
    // only ever waits for splits that have written (their stores are in
    // flight) or hands over and leaves.
    const int rows = HG * G;
    const int K = min(rows, ns);
    uint32_t todo = sctl[2];  // rows handed over to this split
    if (split < K)
      for (int rr = split; rr < rows; rr += K) todo |= 1u << rr;
    if (todo == 0u) return;
    // Merge of one row: warp w takes splits w, w + 8, ...; lane l the output
    // float4 l. Each warp folds its splits into a running (max, l, acc), all
    // loads of a round (up to 8 splits) issued before any is used; the warps'
    // states are then combined through shared memory.
    constexpr int kRowBatch = 8;
    constexpr uint32_t kHandOverRounds = 256;  // polls (~0.2 ms) before a merger hands over
    float* mred = reinterpret_cast<float*>(smem);            // [kAttnWarps] (the rings are free)
    float4* ored = reinterpret_cast<float4*>(smem + 64);     // [kAttnWarps][32]
    float* lred = reinterpret_cast<float*>(smem + 64 + kAttnWarps * 32 * 16);  // [kAttnWarps]
    static_assert(64 + kAttnWarps * 32 * 16 + kAttnWarps * 4 <= S::kRingBytes, "row-merge scratch fits in the rings");
    const size_t sstride = (size_t)p.Hkv * G * (D + 4);  // between consecutive slots
    uint32_t* row0 = p.ws_part + ((size_t)slot_base * p.Hkv + (size_t)hgi * HG) * G * (D + 4);
    const int first = __ffs(todo) - 1;  // the hand-over window is this row's poll
    for (uint32_t rest = todo; rest != 0u; rest &= rest - 1u) {
      const int rr = __ffs(rest) - 1;
      if ((sctl[1] >> rr) & 1u) continue;  // handed over
      const int hh = rr / G, r = rr % G;
      uint32_t* base = row0 + (size_t)rr * (D + 4);
      float mw = -INFINITY, L = 0.0f;
      float4 acc = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
      for (int s0 = warp; s0 < ns; s0 += kAttnWarps * kRowBatch) {
        uint4 v[kRowBatch];
        uint2 ml[kRowBatch];
        for (uint32_t rounds = 0;; ++rounds) {
          bool ok = true;
          uint32_t miss = 0u;  // this lane's splits (bit k) with a word not written
#pragma unroll
          for (int k = 0; k < kRowBatch; ++k) {
            const int s2 = s0 + k * kAttnWarps;
            v[k] = make_uint4(1u, 1u, 1u, 1u);
            ml[k] = make_uint2(1u, 1u);
            if (s2 < ns) {
              if (lane < D / 4) v[k] = ld_relaxed_gpu_v4(base + s2 * sstride + 4 * lane);
              ml[k] = ld_relaxed_gpu_v2(base + s2 * sstride + D);
            }
            const bool okk = v[k].x && v[k].y && v[k].z && v[k].w && ml[k].x && ml[k].y;
            ok = ok && okk;
            miss |= okk ? 0u : 1u << k;
          }
          if (__all_sync(FULL, ok)) break;
          if (rounds >= kMaxSpinRounds) {
            if (lane == 0) record_error(KVQ_ERR_TIMEOUT);
            break;
          }
          if (rounds == kHandOverRounds && rr == first) {
            const uint32_t wmiss = __reduce_or_sync(FULL, miss);
            if (lane == 0 && wmiss != 0u && atomicCAS(&sctl[0], 0u, 3u) == 0u) {
              // this warp decides for the CTA: hand every row of `todo` to
              // one split that has not written; a row whose word already
              // says "written" stays here (that split's stores are landing)
              const int sj = s0 + (__ffs(wmiss) - 1) * kAttnWarps;
              uint32_t gone = 0u;
              for (uint32_t t2 = todo; t2 != 0u; t2 &= t2 - 1u) {
                const int r2 = __ffs(t2) - 1;
                if (atomicCAS(row0 + (size_t)sj * sstride + (size_t)r2 * (D + 4) + D + 2, 0u, kRowHandedOver) == 0u)
                  gone |= 1u << r2;
              }
              atomicOr(&sctl[1], gone);
              atomicExch(&sctl[0], gone ? 2u : 1u);
            }
          }
          if (__shfl_sync(FULL, lane == 0 ? (*reinterpret_cast<volatile uint32_t*>(&sctl[1]) >> rr) & 1u : 0u, 0))
            break;  // the row was handed over
          __nanosleep(64);
        }
        __syncwarp();
        if ((*reinterpret_cast<volatile uint32_t*>(&sctl[1]) >> rr) & 1u) break;  // handed over: the words stay
        float mb = mw;
#pragma unroll
        for (int k = 0; k < kRowBatch; ++k)
          if (s0 + k * kAttnWarps < ns) mb = fmaxf(mb, __uint_as_float(~ml[k].x));
        if (mb == -INFINITY) continue;
        const float a0 = (mw == -INFINITY) ? 0.0f : fast_exp2(mw - mb);
        acc.x *= a0; acc.y *= a0; acc.z *= a0; acc.w *= a0;
        L *= a0;
#pragma unroll
        for (int k = 0; k < kRowBatch; ++k) {
          const float mk = __uint_as_float(~ml[k].x);
          if (s0 + k * kAttnWarps >= ns || mk == -INFINITY) continue;
          const float wgt = fast_exp2(mk - mb);
          acc.x = fmaf(wgt, __uint_as_float(~v[k].x), acc.x);
          acc.y = fmaf(wgt, __uint_as_float(~v[k].y), acc.y);
          acc.z = fmaf(wgt, __uint_as_float(~v[k].z), acc.z);
          acc.w = fmaf(wgt, __uint_as_float(~v[k].w), acc.w);
          L = fmaf(wgt, __uint_as_float(~ml[k].y), L);
        }
        mw = mb;
      }
      if (lane == 0) {
        mred[warp] = mw;
        lred[warp] = L;
      }
      if (lane < D / 4) ored[warp * 32 + lane] = acc;
      __syncthreads();
      if ((sctl[1] >> rr) & 1u) continue;  // this row went to another split
      // the row's words are all read: zero them (and its word D + 2) for the
      // next call
      for (int s2 = warp; s2 < ns; s2 += kAttnWarps) {
        if (lane < D / 4) *reinterpret_cast<uint4*>(base + s2 * sstride + 4 * lane) = make_uint4(0u, 0u, 0u, 0u);
        if (lane == 0) *reinterpret_cast<uint4*>(base + s2 * sstride + D) = make_uint4(0u, 0u, 0u, 0u);
      }
      if (warp == 0) {
        float M = mred[0];
#pragma unroll
        for (int w2 = 1; w2 < kAttnWarps; ++w2) M = fmaxf(M, mred[w2]);
        float Lt = 0.0f;
        float4 sum = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
        if (M != -INFINITY) {
#pragma unroll
          for (int w2 = 0; w2 < kAttnWarps; ++w2) {
            if (mred[w2] == -INFINITY) continue;
            const float f = fast_exp2(mred[w2] - M);
            Lt = fmaf(f, lred[w2], Lt);
            if (lane < D / 4) {
              const float4 x = ored[w2 * 32 + lane];
              sum.x = fmaf(f, x.x, sum.x);
              sum.y = fmaf(f, x.y, sum.y);
              sum.z = fmaf(f, x.z, sum.z);
              sum.w = fmaf(f, x.w, sum.w);
            }
          }
        }
        const float inv = (Lt > 0.0f) ? 1.0f / Lt : 0.0f;
        if (lane < D / 4)
          *reinterpret_cast<float4*>(qs + (hh * NR + r) * D + 4 * lane) =
              make_float4(sum.x * inv, sum.y * inv, sum.z * inv, sum.w * inv);
      }
      __syncthreads();
    }
    // rotate back the merged rows (one warp per row) and store
    const uint32_t done = todo & ~sctl[1];
    int nth = 0;
    for (uint32_t rest = done; rest != 0u; rest &= rest - 1u, ++nth) {
      if (nth % kAttnWarps != warp) continue;
      const int rr = __ffs(rest) - 1;
      const int hh = rr / G, r = rr % G;
      const float* rp = qs + (hh * NR + r) * D;
      float v[E];
#pragma unroll
      for (int e2 = 0; e2 < E; ++e2) v[e2] = rp[E * lane + e2];
      if constexpr (BLK > 0) {
        warp_fwht<D, BLK>(v, lane);
        apply_signs<D>(v, p.signs, lane);
      }
      const size_t o_base = ((size_t)n * p.Hq + (size_t)(hgi * HG + hh) * G + r) * D + E * lane;
#pragma unroll
      for (int e2 = 0; e2 < E; ++e2) store_out(p, o_base + e2, BLK > 0 ? v[e2] * p.cb : v[e2]);
    }
    return;
  }
  __syncthreads();

  // ---- rotate back (one warp per query row) and store ---------------------
  for (int rr = warp; rr < HG * G; rr += kAttnWarps) {
    const int hh = rr / G, r = rr % G;
    const float* rp = qs + (hh * NR + r) * D;
    float v[E];
#pragma unroll
    for (int e2 = 0; e2 < E; ++e2) v[e2] = rp[E * lane + e2];
    if constexpr (BLK > 0) {
      warp_fwht<D, BLK>(v, lane);
      apply_signs<D>(v, p.signs, lane);
    }
    const size_t o_base = ((size_t)n * p.Hq + (size_t)(hgi * HG + hh) * G + r) * D + E * lane;
#pragma unroll
    for (int e2 = 0; e2 < E; ++e2) store_out(p, o_base + e2, BLK > 0 ? v[e2] * p.cb : v[e2]);
  }
}

}  // namespace kvq
