// kvq_decode.cuh - split-K paged decode attention over the rotated INT4 cache.
//
// SAW-INT4 (Abstract): "fused attention execution" over the quantized paged
// cache. The rotation R is orthogonal and its own inverse, so the kernel
// rotates q once, runs attention in the rotated space directly on the codes,
// and rotates the output back: out = R sum_t p_t v^_t.
//
// Grid (split, kv-head group, sequence), 4 warps per CTA. A CTA serves HG kv
// heads (HG = 4, 2 or 1, dividing Hkv); warp w works for head w % HG. Because
// the cache is laid out [page][kv head][K|V][token][D/2], the HG heads of one
// page are one contiguous block: each page costs the CTA three 1-D bulk
// copies (TMA engine) - HG*16*D code bytes, HG*64 B of scales, HG*64 B of
// zeros - into a CTA-wide ring of stages (a stage = two pages), completing on
// one mbarrier per stage. The last warp done with a stage refills it.
//
// Per page, on the tensor cores (mma.m16n8k16, f16 in, f32 accumulate):
//   QK: S[16 rows x 16 tokens] = Qhl[16 x D] * codes^T
//   PV: O[16 rows x D]        += Phl[16 x 16 tokens] * codes
// A rows 0..7 carry the fp16 "hi" part of up to 8 query heads (the GQA group)
// and rows 8..15 the "lo" remainder (x = hi + lo keeps ~22 bits), so one MMA
// does both halves. The 4-bit codes enter as exact normal fp16 values c (or
// 16c for a nibble at bits 4..7, compensated by 1/16 on the other operand or
// in the epilogue); subnormal fp16 operands are avoided on purpose - small
// products built from them lost precision in the tensor-core accumulation (a
// systematic bias of ~2^-13 relative, measured on B200). Dequantization is
// folded into per-token scalars:
//   logit_t = s_t * (q~ . code_t) + z_t * sum(q~)
//   o_rot   = (sum_t p_t s_t code_t + sum_t p_t z_t) / sum_t p_t
// with an online softmax in base 2 (log2 e folded into q~) that rescales only
// when the running maximum grows. q is rotated and the output rotated back in
// registers: each thread holds a contiguous D/4-channel slice of one query
// row, and the butterfly stages that cross slices use warp shuffles.
//
// The splits of one (sequence, head group) form thread-block clusters (up to
// 8 CTAs) that merge through distributed shared memory into the cluster's
// first CTA. With one cluster per (sequence, head group) that CTA writes the
// output; otherwise each cluster writes a partial result to the workspace and
// kvq_decode_combine_kernel (chained by programmatic dependent launch) merges
// them and rotates back.
#pragma once

#include <climits>

#include "kvq_device.cuh"

namespace kvq {

struct AttnParams {
  const uint16_t* q;          // bf16 [B][Hq][D]
  const uint8_t* cache;       // [pages][Hkv][2][16][D/2]
  const uint16_t* scales;     // fp16 [pages][Hkv][2][16]
  const uint16_t* zeros;
  const int32_t* page_table;  // [B][max_pages]
  const int32_t* ctx_lens;    // [B]
  void* out;                  // [B][Hq][D] fp32 or bf16
  float* ws_part;             // [B][Hkv][n_parts][G][D + 2]: O + Z, then M, L
  int B, Hq, Hkv, G;
  int num_pages, max_pages;
  int n_splits, pages_per_split;
  int cluster_size;           // CTAs per cluster along the split axis
  int n_parts;                // n_splits / cluster_size
  int out_bf16;
  float qmul;                 // c_b * softmax_scale * log2(e)
  float cb;                   // c_b (output rotation), 1 for plain INT4
};

constexpr int kAttnWarps = 4;
constexpr int kAttnThreads = kAttnWarps * 32;
constexpr int kMaxSplits = 256;
constexpr int kMaxParts = 64;
constexpr int kMaxCluster = 8;
constexpr int kMaxPids = 1024;   // page ids of a CTA's range kept in shared memory

template <int D>
struct AttnSmem {
  static constexpr int kHeadPageBytes = 16 * D + 128;       // codes + 32 scales + 32 zeros
  static constexpr int kRingBytes = 24 * kHeadPageBytes;    // 12/HG stages of 2 pages x HG heads
  // per-warp result slot (overlays the ring once every copy has landed):
  // O[8 rows][D], then (m, l, zs, unused) per row
  static constexpr int kSlotFloats = 8 * D + 8 * 4;
  static constexpr int kSlotBytes = kAttnWarps * kSlotFloats * 4;
  static constexpr int kUnionBytes = kRingBytes > kSlotBytes ? kRingBytes : kSlotBytes;
  static constexpr int kOffPid = kUnionBytes;
  static constexpr int kOffBar = kOffPid + kMaxPids * 4;
  static constexpr int kOffCnt = kOffBar + 12 * 8;
  static constexpr int kOffFlag = kOffCnt + 12 * 4;
  static constexpr int kTotal = kOffFlag + 12 * 4;
};

// Fast Walsh-Hadamard transform (blocks of BLK, Sylvester natural order) of a
// row spread over the 4 lanes of a quad: lane tig holds channels
// [C*tig, C*tig + C). Stages shorter than C stay in the thread; the longer
// ones pair lanes tig and tig ^ (len / C).
template <int C, int BLK>
__device__ __forceinline__ void quad_fwht(float (&v)[C], int tig) {
#pragma unroll
  for (int len = 1; len < C && len < BLK; len <<= 1) {
#pragma unroll
    for (int i = 0; i < C; ++i) {
      if ((i & len) == 0) {
        const float a = v[i], b = v[i + len];
        v[i] = a + b;
        v[i + len] = a - b;
      }
    }
  }
#pragma unroll
  for (int len = C; len < BLK; len <<= 1) {
    const int m = len / C;
    const bool upper = (tig & m) != 0;
#pragma unroll
    for (int i = 0; i < C; ++i) {
      const float other = __shfl_xor_sync(0xffffffffu, v[i], m);
      v[i] = upper ? (other - v[i]) : (v[i] + other);
    }
  }
}

// hi/lo fp16 pair of two floats, packed as the A fragment wants them.
__device__ __forceinline__ void split_pair(float x0, float x1, uint32_t& hi, uint32_t& lo) {
  const __half2 h = __floats2half2_rn(x0, x1);
  const float2 hf = __half22float2(h);
  const __half2 l = __floats2half2_rn(__fsub_rn(x0, hf.x), __fsub_rn(x1, hf.y));
  hi = *reinterpret_cast<const uint32_t*>(&h);
  lo = *reinterpret_cast<const uint32_t*>(&l);
}

__device__ __forceinline__ void store_out(const AttnParams& p, size_t idx, float v) {
  if (p.out_bf16)
    reinterpret_cast<__nv_bfloat16*>(p.out)[idx] = __float2bfloat16_rn(v);
  else
    reinterpret_cast<float*>(p.out)[idx] = v;
}

// Merge of the n_parts partial results of one (sequence, kv head, query row)
// and inverse rotation. Grid (G, Hkv, B), D threads (one per channel).
template <int D, int BLK>
__global__ void __launch_bounds__(D) kvq_decode_combine_kernel(const AttnParams p) {
  __shared__ float sm_m[kMaxParts], sm_w[kMaxParts], sm_row[D];
  __shared__ float sm_L;
  asm volatile("griddepcontrol.wait;\n" ::: "memory");  // the partials are complete
  const int r = blockIdx.x, h = blockIdx.y, n = blockIdx.z, c = threadIdx.x;
  const int np = p.n_parts, G = p.G;
  const size_t stride = (size_t)G * (D + 2);
  const float* base = p.ws_part + (((size_t)n * p.Hkv + h) * np * G + r) * (D + 2);
  for (int s = c; s < np; s += D) {
    sm_m[s] = __ldcg(base + s * stride + D);
    sm_w[s] = __ldcg(base + s * stride + D + 1);
  }
  __syncthreads();
  if (c < 32) {
    float M = -INFINITY;
    for (int s = c; s < np; s += 32) M = fmaxf(M, sm_m[s]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
    float L = 0.0f;
    for (int s = c; s < np; s += 32) {
      const float e = (sm_m[s] == -INFINITY) ? 0.0f : fast_exp2(sm_m[s] - M);
      L += e * sm_w[s];
      sm_w[s] = e;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) L += __shfl_xor_sync(0xffffffffu, L, o);
    if (c == 0) sm_L = L;
  }
  __syncthreads();
  // all partials of this channel in flight at once, 16 at a time
  float acc = 0.0f;
  for (int s0 = 0; s0 < np; s0 += 16) {
    float v[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) v[j] = (s0 + j < np) ? __ldcg(base + (size_t)(s0 + j) * stride + c) : 0.0f;
#pragma unroll
    for (int j = 0; j < 16; ++j)
      if (s0 + j < np) acc = fmaf(sm_w[s0 + j], v[j], acc);
  }
  sm_row[c] = (sm_L > 0.0f) ? acc / sm_L : 0.0f;
  __syncthreads();
  if constexpr (BLK > 0) {
#pragma unroll 1
    for (int len = 1; len < BLK; len <<= 1) {
      float v = 0.0f;
      if ((c & len) == 0) v = sm_row[c] + sm_row[c + len];
      else v = sm_row[c - len] - sm_row[c];
      __syncthreads();
      sm_row[c] = v;
      __syncthreads();
    }
  }
  const float val = (BLK > 0) ? sm_row[c] * p.cb : sm_row[c];
  store_out(p, ((size_t)n * p.Hq + (size_t)h * G + r) * D + c, val);
}

template <int D, int BLK, int HG>
__global__ void __launch_bounds__(kAttnThreads, 3) kvq_decode_kernel(const AttnParams p) {
  using S = AttnSmem<D>;
  constexpr int W = D / 32;    // code words of one token row per thread (QK)
  constexpr int WP = D / 64;   // code words of one token row per thread group (PV)
  constexpr int NT = D / 8;    // PV n-tiles
  constexpr int KS = D / 16;   // QK k-steps
  constexpr int C = D / 4;     // channels of one query row per thread
  constexpr int NSUB = kAttnWarps / HG;  // warps per head
  constexpr int NST = 12 / HG;           // ring stages (a multiple of NSUB)
  constexpr int HPB = S::kHeadPageBytes;
  constexpr int PGB = HG * HPB;          // one page of HG heads
  constexpr int STB = 2 * PGB;           // one stage = two pages
  static_assert(NST * STB == S::kRingBytes, "ring size");
  extern __shared__ __align__(128) uint8_t smem[];
  int* pids = reinterpret_cast<int*>(smem + S::kOffPid);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S::kOffBar);
  int* cnt = reinterpret_cast<int*>(smem + S::kOffCnt);
  int* sflags = reinterpret_cast<int*>(smem + S::kOffFlag);

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2, tig = lane & 3;
  const int hw = warp % HG, sub = warp / HG;
  const int split = blockIdx.x, hg = blockIdx.y, n = blockIdx.z;
  const int h = hg * HG + hw;
  const int G = p.G;
  const unsigned FULL = 0xffffffffu;

  // let a dependent combine kernel get scheduled early; it waits for this grid
  asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory");

  int ctx = p.ctx_lens[n];
  const int cap = p.max_pages * 16;
  if (ctx < 0 || ctx > cap) {
    if (tid == 0) record_error(KVQ_ERR_OUT_OF_RANGE);
    ctx = ctx < 0 ? 0 : cap;
  }
  const int n_pages = (ctx + 15) >> 4;
  const int p_begin = split * p.pages_per_split;
  const int p_end = min(p_begin + p.pages_per_split, n_pages);
  const int npg = max(p_end - p_begin, 0);
  const int n_tasks = (npg + 1) / 2;
  const int32_t* pt_row = p.page_table + (size_t)n * p.max_pages + p_begin;

  for (int i = tid; i < npg && i < kMaxPids; i += kAttnThreads) pids[i] = pt_row[i];
  if (tid == 0) {
    for (int st = 0; st < NST; ++st) {
      mbar_init(smem_addr(&bars[st]), 1);
      cnt[st] = 0;
    }
    mbar_init_fence();
  }
  __syncthreads();

  // Fill stage t % NST with task t (pages 2t, 2t+1 of the range); one thread.
  auto issue = [&](int t) {
    const int st = t % NST;
    const uint32_t bar = smem_addr(&bars[st]);
    const uint32_t dst = smem_addr(smem + st * STB);
    int ids[2];
    bool ok[2];
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      const int i = 2 * t + j;
      ids[j] = (i < npg) ? (i < kMaxPids ? pids[i] : pt_row[i]) : INT_MIN;
      ok[j] = ids[j] >= 0 && ids[j] < p.num_pages;
      if (ids[j] != INT_MIN && !ok[j]) record_error(KVQ_ERR_OUT_OF_RANGE);
    }
    sflags[st] = (ok[0] ? 1 : 0) | (ok[1] ? 2 : 0);
    const uint32_t bytes = (ok[0] ? PGB : 0) + (ok[1] ? PGB : 0);
    if (bytes == 0) {
      mbar_arrive(bar);
      return;
    }
    mbar_arrive_expect_tx(bar, bytes);
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      if (!ok[j]) continue;
      const size_t ph = (size_t)ids[j] * p.Hkv + (size_t)hg * HG;  // first page-head of the group
      const uint32_t d = dst + j * PGB;
      bulk_g2s(d, p.cache + ph * (16 * D), HG * 16 * D, bar);
      bulk_g2s(d + HG * 16 * D, p.scales + ph * 32, HG * 64, bar);
      bulk_g2s(d + HG * 16 * D + HG * 64, p.zeros + ph * 32, HG * 64, bar);
    }
  };
  if (tid == 0)
    for (int t = 0; t < NST && t < n_tasks; ++t) issue(t);

  // ---- q~ = R q * (softmax_scale * log2 e), in registers -------------------
  // Thread (g, tig) holds query row g (query head h*G + g) channels
  // [C tig, C tig + C); rows >= G are zero.
  float qv[C];
  if (g < G) {
    const uint4* src = reinterpret_cast<const uint4*>(p.q + ((size_t)n * p.Hq + (size_t)h * G + g) * D + C * tig);
#pragma unroll
    for (int i = 0; i < C / 8; ++i) {
      const uint4 u = src[i];
      const uint32_t w4[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        qv[8 * i + 2 * e] = __uint_as_float(w4[e] << 16);
        qv[8 * i + 2 * e + 1] = __uint_as_float(w4[e] & 0xffff0000u);
      }
    }
  } else {
#pragma unroll
    for (int i = 0; i < C; ++i) qv[i] = 0.0f;
  }
  if constexpr (BLK > 0) quad_fwht<C, BLK>(qv, tig);
  float amax = 0.0f, qsum = 0.0f;
#pragma unroll
  for (int i = 0; i < C; ++i) {
    qv[i] *= p.qmul;
    amax = fmaxf(amax, fabsf(qv[i]));
    qsum += qv[i];
  }
  amax = fmaxf(amax, __shfl_xor_sync(FULL, amax, 1));
  amax = fmaxf(amax, __shfl_xor_sync(FULL, amax, 2));
  qsum += __shfl_xor_sync(FULL, qsum, 1);
  qsum += __shfl_xor_sync(FULL, qsum, 2);
  // power-of-two prescale so the largest |q~| lands in [2^13, 2^14): both the
  // hi and lo fp16 parts stay normal
  int kexp = (amax > 0.0f) ? 13 - ilogbf(amax) : 0;
  kexp = max(-100, min(100, kexp));
  const float up = ldexpf(1.0f, kexp);
  const float acc_to_true = ldexpf(1.0f, -kexp);

  // A fragments of QK. k-step 2u takes channel pairs (8m, 8m+4), (8m+2, 8m+6)
  // of word m = W tig + u; k-step 2u+1 takes (8m+1, 8m+5), (8m+3, 8m+7) whose
  // codes arrive x16, so its q~ is divided by 16.
  uint32_t aq[KS][4];
#pragma unroll
  for (int u = 0; u < W; ++u) {
#pragma unroll
    for (int t = 0; t < 2; ++t) {
      const float f = t ? up * 0.0625f : up;
      split_pair(qv[8 * u + t] * f, qv[8 * u + t + 4] * f, aq[2 * u + t][0], aq[2 * u + t][1]);
      split_pair(qv[8 * u + t + 2] * f, qv[8 * u + t + 6] * f, aq[2 * u + t][2], aq[2 * u + t][3]);
    }
  }

  // ---- page stream: this warp takes tasks sub, sub + NSUB, ... -------------
  float o[NT][4];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) o[nt][0] = o[nt][1] = o[nt][2] = o[nt][3] = 0.0f;
  float m_run = -INFINITY, l_run = 0.0f, zs_run = 0.0f;

  for (int t = sub; t < n_tasks; t += NSUB) {
    const int st = t % NST;
    const bool waited = mbar_wait_bounded(smem_addr(&bars[st]), (t / NST) & 1);
    if (!__all_sync(FULL, waited)) break;
    const int fl = sflags[st];
    const uint8_t* stg = smem + st * STB;
    const int tok0 = (p_begin + 2 * t) * 16;  // first token of the task

#pragma unroll
    for (int pg = 0; pg < 2; ++pg) {
      if (!((fl >> pg) & 1)) continue;
      const uint8_t* kb = stg + pg * PGB + hw * (16 * D);              // K block, then V block
      const uint8_t* sz = stg + pg * PGB + HG * 16 * D + hw * 64;      // 16 K then 16 V scales
      const uint8_t* zz = stg + pg * PGB + HG * 16 * D + HG * 64 + hw * 64;
      const int tp = tok0 + 16 * pg;

      // QK on the codes: n-tile nt = token rows 8nt + g
      float acc[2][4];
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) {
        acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.0f;
        const uint8_t* row = kb + (8 * nt + g) * (D / 2) + tig * (4 * W);
        uint32_t wk[W];
        if constexpr (W == 4) {
          const uint4 t4 = *reinterpret_cast<const uint4*>(row);
          wk[0] = t4.x; wk[1] = t4.y; wk[2] = t4.z; wk[3] = t4.w;
        } else {
          const uint2 t2 = *reinterpret_cast<const uint2*>(row);
          wk[0] = t2.x; wk[1] = t2.y;
        }
#pragma unroll
        for (int u = 0; u < W; ++u) {
          const uint32_t w = wk[u], w8 = wk[u] >> 8;
          mma_f16_16816(acc[nt], aq[2 * u], codes_to_half2<false>(w), codes_to_half2<false>(w8));
          mma_f16_16816(acc[nt], aq[2 * u + 1], codes_to_half2<true>(w), codes_to_half2<true>(w8));
        }
      }
      // logits (base 2) of tokens 2tig, 2tig+1 (nt 0) and 2tig+8, 2tig+9 (nt 1)
      const float2 skA = __half22float2(reinterpret_cast<const __half2*>(sz)[tig]);
      const float2 skB = __half22float2(reinterpret_cast<const __half2*>(sz)[tig + 4]);
      const float2 zkA = __half22float2(reinterpret_cast<const __half2*>(zz)[tig]);
      const float2 zkB = __half22float2(reinterpret_cast<const __half2*>(zz)[tig + 4]);
      float lg[4];
      lg[0] = fmaf((acc[0][0] + acc[0][2]) * acc_to_true, skA.x, zkA.x * qsum);
      lg[1] = fmaf((acc[0][1] + acc[0][3]) * acc_to_true, skA.y, zkA.y * qsum);
      lg[2] = fmaf((acc[1][0] + acc[1][2]) * acc_to_true, skB.x, zkB.x * qsum);
      lg[3] = fmaf((acc[1][1] + acc[1][3]) * acc_to_true, skB.y, zkB.y * qsum);
      const int t0 = tp + 2 * tig;
      if (t0 >= ctx) lg[0] = -INFINITY;
      if (t0 + 1 >= ctx) lg[1] = -INFINITY;
      if (t0 + 8 >= ctx) lg[2] = -INFINITY;
      if (t0 + 9 >= ctx) lg[3] = -INFINITY;

      // online softmax, rescaling only when the running maximum grows
      float pm = fmaxf(fmaxf(lg[0], lg[1]), fmaxf(lg[2], lg[3]));
      pm = fmaxf(pm, __shfl_xor_sync(FULL, pm, 1));
      pm = fmaxf(pm, __shfl_xor_sync(FULL, pm, 2));
      if (pm > m_run) {
        const float alpha = fast_exp2(m_run - pm);
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          o[nt][0] *= alpha; o[nt][1] *= alpha; o[nt][2] *= alpha; o[nt][3] *= alpha;
        }
        l_run *= alpha;
        zs_run *= alpha;
        m_run = pm;
      }
      const float2 svA = __half22float2(reinterpret_cast<const __half2*>(sz + 32)[tig]);
      const float2 svB = __half22float2(reinterpret_cast<const __half2*>(sz + 32)[tig + 4]);
      const float2 zvA = __half22float2(reinterpret_cast<const __half2*>(zz + 32)[tig]);
      const float2 zvB = __half22float2(reinterpret_cast<const __half2*>(zz + 32)[tig + 4]);
      const float sv[4] = {svA.x, svA.y, svB.x, svB.y};
      const float zv[4] = {zvA.x, zvA.y, zvB.x, zvB.y};
      float pv[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float pr = (lg[j] == -INFINITY) ? 0.0f : fast_exp2(lg[j] - m_run);
        l_run += pr;
        pv[j] = (pr > 0.0f) ? pr * sv[j] : 0.0f;
        zs_run += (pr > 0.0f) ? pr * zv[j] : 0.0f;
      }
      uint32_t ap[4];
      split_pair(pv[0], pv[1], ap[0], ap[1]);
      split_pair(pv[2], pv[3], ap[2], ap[3]);

      // PV on the codes: B = code pairs of token rows (2tig, 2tig+1),
      // (2tig+8, 2tig+9); thread group g supplies channels [g*NT, g*NT + NT)
      const uint8_t* vb = kb + 8 * D;
      uint32_t wv[4][WP];
      const int rows_v[4] = {2 * tig, 2 * tig + 1, 2 * tig + 8, 2 * tig + 9};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const uint8_t* row = vb + rows_v[j] * (D / 2) + g * (4 * WP);
        if constexpr (WP == 2) {
          const uint2 t2 = *reinterpret_cast<const uint2*>(row);
          wv[j][0] = t2.x; wv[j][1] = t2.y;
        } else {
          wv[j][0] = *reinterpret_cast<const uint32_t*>(row);
        }
      }
#pragma unroll
      for (int u = 0; u < WP; ++u) {
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const uint32_t sel = k | (k << 4) | ((4 + k) << 8) | ((4 + k) << 12);
          const uint32_t x01 = prmt(wv[0][u], wv[1][u], sel);
          const uint32_t x23 = prmt(wv[2][u], wv[3][u], sel);
          mma_f16_16816(o[8 * u + 2 * k], ap, codes_to_half2<false>(x01), codes_to_half2<false>(x23));
          mma_f16_16816(o[8 * u + 2 * k + 1], ap, codes_to_half2<true>(x01), codes_to_half2<true>(x23));
        }
      }
    }
    // release the stage; the last of its HG consumer warps refills it
    __syncwarp();
    if (lane == 0) {
      const int old = atomicAdd(&cnt[st], 1);
      if (old == HG - 1) {
        cnt[st] = 0;
        if (t + NST < n_tasks) issue(t + NST);
      }
    }
  }
  // (a warp whose wait ran out stops early; the error word records it)

  // ---- per-warp result: O slice of row g, (m, l, zs) -----------------------
  l_run += __shfl_xor_sync(FULL, l_run, 1);
  l_run += __shfl_xor_sync(FULL, l_run, 2);
  zs_run += __shfl_xor_sync(FULL, zs_run, 1);
  zs_run += __shfl_xor_sync(FULL, zs_run, 2);
  float ov[C];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    const float sc = (nt & 1) ? 0.0625f : 1.0f;  // odd n-tiles carried 16c
    ov[nt] = (o[nt][0] + o[nt][2]) * sc;          // channel C tig + nt
    ov[NT + nt] = (o[nt][1] + o[nt][3]) * sc;     // channel C tig + NT + nt
  }

  // Merge (m, l, zs, O) sources into this thread's registers.
  auto merge_in = [&](float ms, float ls, float zss, const float* os) {
    const float M = fmaxf(m_run, ms);
    if (M == -INFINITY) return;
    const float a = (m_run == -INFINITY) ? 0.0f : fast_exp2(m_run - M);
    const float b = (ms == -INFINITY) ? 0.0f : fast_exp2(ms - M);
#pragma unroll
    for (int i = 0; i < C; ++i) ov[i] = ov[i] * a + os[i] * b;
    l_run = l_run * a + ls * b;
    zs_run = zs_run * a + zss * b;
    m_run = M;
  };

  __syncthreads();  // every copy has landed and been consumed: slots may overlay the ring
  float* slots = reinterpret_cast<float*>(smem);
  auto put_local = [&](float* slot) {
#pragma unroll
    for (int i = 0; i < C; ++i) slot[g * D + C * tig + i] = ov[i];
    if (tig == 0) {
      slot[8 * D + 4 * g] = m_run;
      slot[8 * D + 4 * g + 1] = l_run;
      slot[8 * D + 4 * g + 2] = zs_run;
    }
  };
  auto take = [&](const float* slot) {
    float os[C];
#pragma unroll
    for (int i = 0; i < C; ++i) os[i] = slot[g * D + C * tig + i];
    merge_in(slot[8 * D + 4 * g], slot[8 * D + 4 * g + 1], slot[8 * D + 4 * g + 2], os);
  };
  if constexpr (NSUB > 1) {
    // warps that shared a head hand their results to warp hw
    if (sub > 0) put_local(slots + warp * S::kSlotFloats);
    __syncthreads();
    if (sub == 0)
      for (int j = 1; j < NSUB; ++j) take(slots + (hw + HG * j) * S::kSlotFloats);
    __syncthreads();
  }
  const int cs = p.cluster_size;
  if (cs > 1) {
    // The cluster's CTAs merge into its first CTA along a binary tree: at
    // level r, CTA rank + 2^r pushes its result into level-r buffer of CTA
    // rank (remote shared-memory stores, fire and forget); after one cluster
    // barrier the receiver merges it from its own shared memory.
    constexpr int kPay = kAttnWarps * S::kSlotFloats;
    static_assert(3 * kPay * 4 <= S::kUnionBytes, "three merge buffers must fit in the ring");
    const int rank = (int)cluster_ctarank();
    cluster_sync_all();  // every CTA of the cluster is past its page loop
    int level = 0;
    for (int stride = 1; stride < cs; stride <<= 1, ++level) {
      float* buf = slots + level * kPay + hw * S::kSlotFloats;
      const int rel = rank % (2 * stride);
      if (rel == stride && sub == 0) {
        const uint32_t to = (uint32_t)(rank - stride);
#pragma unroll
        for (int i = 0; i < C; i += 4)
          st_dsmem_v4(buf + g * D + C * tig + i, to, ov[i], ov[i + 1], ov[i + 2], ov[i + 3]);
        if (tig == 0) st_dsmem_v4(buf + 8 * D + 4 * g, to, m_run, l_run, zs_run, 0.0f);
      }
      cluster_sync_all();
      if (rel == 0 && rank + stride < cs && sub == 0) take(buf);
    }
    if (rank != 0) return;
  }
  if (sub != 0) return;

  if (p.n_parts == 1) {
    const float inv_l = (l_run > 0.0f) ? 1.0f / l_run : 0.0f;
#pragma unroll
    for (int i = 0; i < C; ++i) ov[i] = (l_run > 0.0f) ? (ov[i] + zs_run) * inv_l : 0.0f;
    if constexpr (BLK > 0) {
      quad_fwht<C, BLK>(ov, tig);
#pragma unroll
      for (int i = 0; i < C; ++i) ov[i] *= p.cb;
    }
    if (g < G) {
      const size_t o_base = ((size_t)n * p.Hq + (size_t)h * G + g) * D + C * tig;
#pragma unroll
      for (int i = 0; i < C; ++i) store_out(p, o_base + i, ov[i]);
    }
  } else if (g < G) {
    const int part = split / cs;
    float* dst = p.ws_part + ((((size_t)n * p.Hkv + h) * p.n_parts + part) * G + g) * (D + 2);
#pragma unroll
    for (int i = 0; i < C; ++i) dst[C * tig + i] = ov[i] + zs_run;
    if (tig == 0) {
      dst[D] = m_run;
      dst[D + 1] = l_run;
    }
  }
}

}  // namespace kvq
