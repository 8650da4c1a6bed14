// kvq_decode.cuh - split-K paged decode attention over the rotated INT4 cache.
//
// SAW-INT4 (Abstract): "fused attention execution" over the quantized paged
// cache. The rotation R is orthogonal and its own inverse, so the kernel
// rotates q once, runs attention in the rotated space directly on the codes,
// and rotates the output back: out = R sum_t p_t v^_t.
//
// Grid (split, kv head, sequence); 4 warps per CTA. Each warp streams its
// pages (page p_begin + warp + 4 i) through a private ring of bulk copies
// (TMA engine, 1-D, completing on an mbarrier): 16*D code bytes (K block then
// V block) plus 64 B of scales and 64 B of zeros per page.
//
// Per page, on the tensor cores (mma.m16n8k16, f16 in, f32 accumulate):
//   rows 0..7 of the A operand = the "hi" fp16 part of up to 8 query heads,
//   rows 8..15 = their "lo" part (x = hi + lo keeps ~22 bits), so one MMA
//   carries both halves and GQA groups up to 8 share one K/V stream.
//   QK:  S[16 x 16 tokens] = Qhl[16 x D] * codes^T       (k = channels)
//   PV:  O[16 x D]        += Phl[16 x 16 tokens] * codes  (k = tokens)
//   The 4-bit codes enter the MMA as exact normal fp16 values c (or 16c for a
//   nibble at bits 4..7, compensated by a factor 1/16 on the other operand or
//   in the epilogue). Subnormal fp16 operands are avoided on purpose: small
//   products built from them lost precision in the tensor-core accumulation
//   (a systematic bias of ~2^-13 relative, measured on B200).
//   Dequantization is folded into the per-token scalars:
//     logit_t = s_t * (q~ . code_t) + z_t * sum(q~)
//     o_rot   = (sum_t p_t s_t code_t + sum_t p_t z_t) / sum_t p_t
// Online softmax in base 2 (log2 e folded into q~). Warps merge in shared
// memory; splits merge through a workspace, the last CTA to arrive (atomic
// ticket) combining them and applying the inverse rotation.
#pragma once

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
  float* ws_part;             // [B][Hkv][splits][G][D + 2]
  int* ws_count;              // [B][Hkv]
  int B, Hq, Hkv, G;
  int num_pages, max_pages;
  int n_splits, pages_per_split;
  int out_bf16;
  float qmul;                 // c_b * softmax_scale * log2(e)
  float cb;                   // c_b (output rotation), 1 for plain INT4
};

constexpr int kAttnWarps = 4;
constexpr int kAttnThreads = kAttnWarps * 32;
constexpr int kStages = 4;
constexpr int kMaxSplits = 64;

template <int D>
struct AttnSmem {
  static constexpr int kCodeBytes = 16 * D;             // K block + V block of one page-head
  static constexpr int kStageBytes = kCodeBytes + 128;  // + 32 scales + 32 zeros (fp16)
  static constexpr int kRingBytes = kAttnWarps * kStages * kStageBytes;
  // per-warp merge area (overlays the ring after the page loop)
  static constexpr int kMergeFloatsPerWarp = 8 * D + 3 * 8;
  static constexpr int kMergeBytes = kAttnWarps * kMergeFloatsPerWarp * 4;
  static constexpr int kUnionBytes = kRingBytes > kMergeBytes ? kRingBytes : kMergeBytes;
  static constexpr int kQBytes = 8 * D * 4;             // q / output rows, fp32
  static constexpr int kWeightBytes = (2 * 8 * kMaxSplits + 8) * 4;  // split maxima/weights, sums, per-head L
  static constexpr int kBarBytes = kAttnWarps * kStages * 8;
  static constexpr int kFlagBytes = kAttnWarps * kStages * 4 + 16;
  static constexpr int kOffQ = kUnionBytes;
  static constexpr int kOffW = kOffQ + kQBytes;
  static constexpr int kOffBar = kOffW + kWeightBytes;
  static constexpr int kOffFlag = kOffBar + kBarBytes;
  static constexpr int kTotal = kOffFlag + kFlagBytes;
};

// In-place FWHT of rows [0, nrows) of an fp32 [8][D] shared array, blocks of
// BLK channels; the whole CTA takes part.
template <int D, int BLK>
__device__ __forceinline__ void smem_fwht_rows(float* rows, int nrows) {
#pragma unroll 1
  for (int len = 1; len < BLK; len <<= 1) {
    for (int idx = threadIdx.x; idx < nrows * (D / 2); idx += kAttnThreads) {
      const int r = idx / (D / 2), pi = idx % (D / 2);
      const int i = (pi / len) * (2 * len) + (pi % len);
      float* row = rows + r * D;
      const float a = row[i], b = row[i + len];
      row[i] = a + b;
      row[i + len] = a - b;
    }
    __syncthreads();
  }
}

template <int D, int BLK>
__global__ void __launch_bounds__(kAttnThreads, 3) kvq_decode_kernel(const AttnParams p) {
  using S = AttnSmem<D>;
  constexpr int W = D / 32;   // code words of one token row per thread (QK)
  constexpr int KS = D / 16;  // QK k-steps
  constexpr int WP = D / 64;  // code words of one token row per thread group (PV)
  constexpr int NT = D / 8;   // PV n-tiles
  extern __shared__ __align__(128) uint8_t smem[];
  float* qs = reinterpret_cast<float*>(smem + S::kOffQ);
  float* wts = reinterpret_cast<float*>(smem + S::kOffW);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S::kOffBar);
  int* flags = reinterpret_cast<int*>(smem + S::kOffFlag);

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2, tig = lane & 3;
  const int split = blockIdx.x, h = blockIdx.y, n = blockIdx.z;
  const int G = p.G;
  const unsigned FULL = 0xffffffffu;

  int ctx = p.ctx_lens[n];
  const int cap = p.max_pages * 16;
  if (ctx < 0 || ctx > cap) {
    if (tid == 0) record_error(KVQ_ERR_OUT_OF_RANGE);
    ctx = ctx < 0 ? 0 : cap;
  }
  const int n_pages = (ctx + 15) >> 4;
  const int p_begin = split * p.pages_per_split;
  const int p_end = min(p_begin + p.pages_per_split, n_pages);

  if (lane == 0) {
    for (int s = 0; s < kStages; ++s) mbar_init(smem_addr(&bars[warp * kStages + s]), 1);
    mbar_init_fence();
  }

  // ---- q~ = R q * (softmax_scale * log2 e), rows >= G are zero ------------
  for (int i = tid; i < 8 * D; i += kAttnThreads) {
    const int r = i / D, c = i % D;
    qs[i] = (r < G) ? bf16_bits_to_float(p.q[((size_t)n * p.Hq + (size_t)h * G + r) * D + c]) : 0.0f;
  }
  __syncthreads();
  if constexpr (BLK > 0) smem_fwht_rows<D, BLK>(qs, G);

  // Thread (g, tig) holds head g's channels [8W tig, 8W tig + 8W).
  float qv[8 * W];
  float amax = 0.0f, qsum = 0.0f;
#pragma unroll
  for (int i = 0; i < 8 * W; ++i) {
    qv[i] = qs[g * D + 8 * W * tig + i] * p.qmul;
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
      __half h0, l0, h1, l1, h2, l2, h3, l3;
      split_half(qv[8 * u + t] * f, h0, l0);
      split_half(qv[8 * u + t + 4] * f, h1, l1);
      split_half(qv[8 * u + t + 2] * f, h2, l2);
      split_half(qv[8 * u + t + 6] * f, h3, l3);
      aq[2 * u + t][0] = pack_half2(h0, h1);
      aq[2 * u + t][1] = pack_half2(l0, l1);
      aq[2 * u + t][2] = pack_half2(h2, h3);
      aq[2 * u + t][3] = pack_half2(l2, l3);
    }
  }
  __syncthreads();  // barrier init visible; qs free for reuse later

  // ---- page stream ---------------------------------------------------------
  const int my_first = p_begin + warp;
  const int n_my = (my_first < p_end) ? (p_end - my_first + kAttnWarps - 1) / kAttnWarps : 0;
  uint8_t* ring = smem + warp * kStages * S::kStageBytes;
  const uint32_t ring_s = smem_addr(ring);
  const uint32_t bar0 = smem_addr(&bars[warp * kStages]);
  int* wflags = flags + warp * kStages;
  const int32_t* pt_row = p.page_table + (size_t)n * p.max_pages;

  int pid_base = 0;
  int pid_reg = (lane < n_my) ? pt_row[my_first + lane * kAttnWarps] : 0;
  auto issue = [&](int i) {  // called by all lanes, i increasing by one
    if (i - pid_base >= 32) {
      pid_base += 32;
      const int j = pid_base + lane;
      pid_reg = (j < n_my) ? pt_row[my_first + j * kAttnWarps] : 0;
    }
    const int pid = __shfl_sync(FULL, pid_reg, i - pid_base);
    if (lane == 0) {
      const int st = i % kStages;
      const uint32_t bar = bar0 + st * 8;
      const uint32_t dst = ring_s + st * S::kStageBytes;
      if (pid >= 0 && pid < p.num_pages) {
        wflags[st] = 1;
        const size_t ph = (size_t)pid * p.Hkv + h;
        mbar_arrive_expect_tx(bar, S::kStageBytes);
        bulk_g2s(dst, p.cache + ph * S::kCodeBytes, S::kCodeBytes, bar);
        bulk_g2s(dst + S::kCodeBytes, p.scales + ph * 32, 64, bar);
        bulk_g2s(dst + S::kCodeBytes + 64, p.zeros + ph * 32, 64, bar);
      } else {
        wflags[st] = 0;
        record_error(KVQ_ERR_OUT_OF_RANGE);
        mbar_arrive(bar);
      }
    }
  };

  const int pre = min(n_my, kStages);
  for (int i = 0; i < pre; ++i) issue(i);
  int issued = pre, consumed = 0;

  float o[NT][4];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) o[nt][0] = o[nt][1] = o[nt][2] = o[nt][3] = 0.0f;
  float m_run = -INFINITY, l_run = 0.0f, zs_run = 0.0f;
  bool ok = true;

  for (int i = 0; i < n_my; ++i) {
    const int st = i % kStages;
    const bool waited = mbar_wait_bounded(bar0 + st * 8, (i / kStages) & 1);
    if (!__all_sync(FULL, waited)) { ok = false; break; }
    consumed = i + 1;
    const uint8_t* stg = ring + st * S::kStageBytes;
    const bool valid = wflags[st] != 0;
    const int page_base = (my_first + i * kAttnWarps) * 16;
    const uint8_t* kb = stg;
    const uint8_t* vb = stg + 8 * D;
    const __half2* sk2 = reinterpret_cast<const __half2*>(stg + S::kCodeBytes);
    const __half2* sv2 = sk2 + 8;
    const __half2* zk2 = reinterpret_cast<const __half2*>(stg + S::kCodeBytes + 64);
    const __half2* zv2 = zk2 + 8;

    // QK on the codes: token rows g and 8 + g
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

    // logits (base 2) of this thread's tokens 2tig, 2tig+1, 2tig+8, 2tig+9
    const float2 skA = __half22float2(sk2[tig]), skB = __half22float2(sk2[tig + 4]);
    const float2 zkA = __half22float2(zk2[tig]), zkB = __half22float2(zk2[tig + 4]);
    const int t0 = page_base + 2 * tig;
    float lg[4];
    lg[0] = fmaf((acc[0][0] + acc[0][2]) * acc_to_true, skA.x, zkA.x * qsum);
    lg[1] = fmaf((acc[0][1] + acc[0][3]) * acc_to_true, skA.y, zkA.y * qsum);
    lg[2] = fmaf((acc[1][0] + acc[1][2]) * acc_to_true, skB.x, zkB.x * qsum);
    lg[3] = fmaf((acc[1][1] + acc[1][3]) * acc_to_true, skB.y, zkB.y * qsum);
    if (!valid || t0 >= ctx) lg[0] = -INFINITY;
    if (!valid || t0 + 1 >= ctx) lg[1] = -INFINITY;
    if (!valid || t0 + 8 >= ctx) lg[2] = -INFINITY;
    if (!valid || t0 + 9 >= ctx) lg[3] = -INFINITY;

    // online softmax, rescaling only when the running maximum grows
    float pm = fmaxf(fmaxf(lg[0], lg[1]), fmaxf(lg[2], lg[3]));
    pm = fmaxf(pm, __shfl_xor_sync(FULL, pm, 1));
    pm = fmaxf(pm, __shfl_xor_sync(FULL, pm, 2));
    if (pm > m_run) {
      const float alpha = exp2f(m_run - pm);
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        o[nt][0] *= alpha; o[nt][1] *= alpha; o[nt][2] *= alpha; o[nt][3] *= alpha;
      }
      l_run *= alpha;
      zs_run *= alpha;
      m_run = pm;
    }
    const float2 svA = __half22float2(sv2[tig]), svB = __half22float2(sv2[tig + 4]);
    const float2 zvA = __half22float2(zv2[tig]), zvB = __half22float2(zv2[tig + 4]);
    const float sv[4] = {svA.x, svA.y, svB.x, svB.y};
    const float zv[4] = {zvA.x, zvA.y, zvB.x, zvB.y};
    __half ph[4], pl[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float pr = (lg[j] == -INFINITY) ? 0.0f : exp2f(lg[j] - m_run);
      l_run += pr;
      const float pv = (pr > 0.0f) ? pr * sv[j] : 0.0f;
      zs_run += (pr > 0.0f) ? pr * zv[j] : 0.0f;
      split_half(pv, ph[j], pl[j]);
    }
    const uint32_t ap[4] = {pack_half2(ph[0], ph[1]), pack_half2(pl[0], pl[1]),
                            pack_half2(ph[2], ph[3]), pack_half2(pl[2], pl[3])};

    // PV on the codes: thread group g supplies channels [g*NT, g*NT + NT)
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
    __syncwarp();
    if (issued < n_my) { issue(issued); ++issued; }
  }
  if (!ok) {
    // a copy never completed: give the ones still outstanding a bounded wait
    for (int i = consumed; i < issued; ++i) mbar_wait_bounded(bar0 + (i % kStages) * 8, (i / kStages) & 1);
  }

  // ---- merge the four warps ------------------------------------------------
  l_run += __shfl_xor_sync(FULL, l_run, 1);
  l_run += __shfl_xor_sync(FULL, l_run, 2);
  zs_run += __shfl_xor_sync(FULL, zs_run, 1);
  zs_run += __shfl_xor_sync(FULL, zs_run, 2);
  __syncthreads();  // every warp is past its ring: the merge area may overlay it
  float* mrg = reinterpret_cast<float*>(smem);
  {
    float* mw = mrg + warp * S::kMergeFloatsPerWarp;
    if (g < G) {
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        const float sc = (nt & 1) ? 0.0625f : 1.0f;  // odd n-tiles carried 16c
        mw[g * D + (2 * tig) * NT + nt] = (o[nt][0] + o[nt][2]) * sc;
        mw[g * D + (2 * tig + 1) * NT + nt] = (o[nt][1] + o[nt][3]) * sc;
      }
      if (tig == 0) {
        mw[8 * D + g] = m_run;
        mw[8 * D + 8 + g] = l_run;
        mw[8 * D + 16 + g] = zs_run;
      }
    }
  }
  __syncthreads();
  float* part = nullptr;
  if (p.n_splits > 1)
    part = p.ws_part + ((((size_t)n * p.Hkv + h) * p.n_splits + split) * G) * (D + 2);
  for (int idx = tid; idx < G * D; idx += kAttnThreads) {
    const int r = idx / D, c = idx % D;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kAttnWarps; ++w) M = fmaxf(M, mrg[w * S::kMergeFloatsPerWarp + 8 * D + r]);
    float O = 0.0f, L = 0.0f, Z = 0.0f;
    if (M != -INFINITY) {
#pragma unroll
      for (int w = 0; w < kAttnWarps; ++w) {
        const float* mw = mrg + w * S::kMergeFloatsPerWarp;
        const float mwr = mw[8 * D + r];
        if (mwr == -INFINITY) continue;
        const float e = exp2f(mwr - M);
        O += mw[r * D + c] * e;
        L += mw[8 * D + 8 + r] * e;
        Z += mw[8 * D + 16 + r] * e;
      }
    }
    if (p.n_splits == 1) {
      qs[r * D + c] = (L > 0.0f) ? (O + Z) / L : 0.0f;
    } else {
      part[r * (D + 2) + c] = O + Z;
      if (c == 0) {
        part[r * (D + 2) + D] = M;
        part[r * (D + 2) + D + 1] = L;
      }
    }
  }

  // ---- merge the splits: the last CTA of this (sequence, kv head) ----------
  if (p.n_splits > 1) {
    __threadfence();
    __syncthreads();
    int* s_last = flags + kAttnWarps * kStages;
    if (tid == 0) {
      const int prev = atomicAdd(&p.ws_count[(size_t)n * p.Hkv + h], 1);
      *s_last = (prev == p.n_splits - 1);
    }
    __syncthreads();
    if (!*s_last) return;
    __threadfence();
    const float* base = p.ws_part + (((size_t)n * p.Hkv + h) * p.n_splits) * G * (D + 2);
    const int ns = p.n_splits;
    float* lsp = wts + 8 * kMaxSplits;   // per (head, split) sums
    float* Lr = wts + 16 * kMaxSplits;   // per head total
    // every (head, split) maximum and sum, loaded in parallel
    for (int idx = tid; idx < G * ns; idx += kAttnThreads) {
      const int r = idx % G, s = idx / G;
      const float* src = base + ((size_t)s * G + r) * (D + 2) + D;
      wts[r * kMaxSplits + s] = __ldcg(src);
      lsp[r * kMaxSplits + s] = __ldcg(src + 1);
    }
    __syncthreads();
    // per head: the global maximum, the split weights and the total sum (one warp per head)
    for (int r = warp; r < G; r += kAttnWarps) {
      float M = -INFINITY;
      for (int s = lane; s < ns; s += 32) M = fmaxf(M, wts[r * kMaxSplits + s]);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(FULL, M, o));
      float L = 0.0f;
      for (int s = lane; s < ns; s += 32) {
        const float ms = wts[r * kMaxSplits + s];
        const float e = (ms == -INFINITY) ? 0.0f : exp2f(ms - M);
        wts[r * kMaxSplits + s] = e;
        L += e * lsp[r * kMaxSplits + s];
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) L += __shfl_xor_sync(FULL, L, o);
      if (lane == 0) Lr[r] = L;
    }
    __syncthreads();
    // weighted sum over splits; independent loads, several in flight
    for (int idx = tid; idx < G * D; idx += kAttnThreads) {
      const int r = idx / D, c = idx % D;
      const float* src = base + (size_t)r * (D + 2) + c;
      const size_t stride = (size_t)G * (D + 2);
      float acc0 = 0.0f, acc1 = 0.0f, acc2 = 0.0f, acc3 = 0.0f;
      int s = 0;
      for (; s + 4 <= ns; s += 4) {
        const float v0 = __ldcg(src + (size_t)s * stride), v1 = __ldcg(src + (size_t)(s + 1) * stride);
        const float v2 = __ldcg(src + (size_t)(s + 2) * stride), v3 = __ldcg(src + (size_t)(s + 3) * stride);
        acc0 = fmaf(wts[r * kMaxSplits + s], v0, acc0);
        acc1 = fmaf(wts[r * kMaxSplits + s + 1], v1, acc1);
        acc2 = fmaf(wts[r * kMaxSplits + s + 2], v2, acc2);
        acc3 = fmaf(wts[r * kMaxSplits + s + 3], v3, acc3);
      }
      for (; s < ns; ++s) acc0 = fmaf(wts[r * kMaxSplits + s], __ldcg(src + (size_t)s * stride), acc0);
      const float acc = (acc0 + acc1) + (acc2 + acc3);
      qs[r * D + c] = (Lr[r] > 0.0f) ? acc / Lr[r] : 0.0f;
    }
    if (tid == 0) p.ws_count[(size_t)n * p.Hkv + h] = 0;  // leave the workspace zeroed
  }
  __syncthreads();

  // ---- out = R o_rot ---------------------------------------------------------
  if constexpr (BLK > 0) smem_fwht_rows<D, BLK>(qs, G);
  for (int idx = tid; idx < G * D; idx += kAttnThreads) {
    const int r = idx / D, c = idx % D;
    const float val = (BLK > 0) ? qs[idx] * p.cb : qs[idx];
    const size_t o_idx = ((size_t)n * p.Hq + (size_t)h * G + r) * D + c;
    if (p.out_bf16)
      reinterpret_cast<__nv_bfloat16*>(p.out)[o_idx] = __float2bfloat16_rn(val);
    else
      reinterpret_cast<float*>(p.out)[o_idx] = val;
  }
}

}  // namespace kvq
