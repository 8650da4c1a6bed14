// kvq_decode.cuh - split-K paged decode attention over the rotated INT4 cache.
//
// SAW-INT4 (Abstract): "fused attention execution" over the quantized paged
// cache. The rotation R is orthogonal and its own inverse, so the kernel
// rotates q once, runs attention in the rotated space directly on the codes,
// and rotates the output back: out = R sum_t p_t v^_t.
//
// Grid (split, kv head, sequence), 4 warps per CTA; the splits of one
// (sequence, kv head) form thread-block clusters of up to 8 CTAs.
//  - Each warp walks its tasks (a task = two consecutive pages of the CTA's
//    page range) through a private ring of 1-D bulk copies (TMA engine)
//    completing on mbarriers: 16*D code bytes (K block, V block) + 64 B
//    scales + 64 B zeros per page. The first copies are issued before q is
//    rotated, so the rotation overlaps them.
//  - Per task, on the tensor cores (mma.m16n8k16, f16 in, f32 accumulate):
//      QK: S[16 rows x 32 tokens] = Qhl[16 x D] * codes^T   (4 n-tiles)
//      PV: O[16 rows x D]        += Phl[16 x 32 tokens] * codes (2 k-steps)
//    A rows 0..7 carry the fp16 "hi" part of up to 8 query heads and rows
//    8..15 the "lo" remainder (x = hi + lo keeps ~22 bits), so one MMA does
//    both halves and a GQA group of up to 8 shares one K/V stream.
//    The 4-bit codes enter as exact normal fp16 values c (or 16c for a nibble
//    at bits 4..7, compensated by 1/16 on the other operand or in the
//    epilogue). Subnormal fp16 operands are avoided on purpose: small
//    products built from them lost precision in the tensor-core accumulation
//    (a systematic bias of ~2^-13 relative, measured on B200).
//    Dequantization is folded into per-token scalars:
//      logit_t = s_t * (q~ . code_t) + z_t * sum(q~)
//      o_rot   = (sum_t p_t s_t code_t + sum_t p_t z_t) / sum_t p_t
//    Online softmax in base 2 (log2 e folded into q~), rescaling only when
//    the running maximum grows.
//  - Warps merge in shared memory; the CTAs of a cluster merge through
//    distributed shared memory into the cluster's first CTA; when a
//    (sequence, kv head) has several clusters, their partial results meet in
//    the workspace and the last cluster to arrive (atomic ticket) combines
//    them. The final CTA applies the inverse rotation and stores.
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
  float* ws_part;             // [B][Hkv][n_parts][G][D + 2]
  int* ws_count;              // [B][Hkv]
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
constexpr int kStages = 3;       // ring depth per warp, in tasks of two pages
constexpr int kMaxSplits = 256;
constexpr int kMaxParts = 64;    // partial results per (sequence, kv head) in the workspace
constexpr int kMaxCluster = 8;

template <int D>
struct AttnSmem {
  static constexpr int kCodeBytes = 16 * D;               // K block + V block of one page-head
  static constexpr int kPageBytes = kCodeBytes + 128;     // + 32 scales + 32 zeros (fp16)
  static constexpr int kStageBytes = 2 * kPageBytes;      // one task = two pages
  static constexpr int kRingBytes = kAttnWarps * kStages * kStageBytes;
  // per-warp merge area (overlays the ring after the page loop)
  static constexpr int kMergeFloatsPerWarp = 8 * D + 3 * 8;
  static constexpr int kMergeBytes = kAttnWarps * kMergeFloatsPerWarp * 4;
  static constexpr int kUnionBytes = kRingBytes > kMergeBytes ? kRingBytes : kMergeBytes;
  static constexpr int kQBytes = 8 * D * 4;               // q rows, then the CTA's merged O
  static constexpr int kMLBytes = 8 * 2 * 4;              // the CTA's merged (M, L) per head
  static constexpr int kWeightBytes = (2 * 8 * kMaxParts + 8) * 4;
  static constexpr int kBarBytes = kAttnWarps * kStages * 8;
  static constexpr int kFlagBytes = kAttnWarps * kStages * 4 + 16;
  static constexpr int kOffQ = kUnionBytes;
  static constexpr int kOffML = kOffQ + kQBytes;
  static constexpr int kOffW = kOffML + kMLBytes;
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

// hi/lo fp16 pair of two floats, packed as the A fragment wants them.
__device__ __forceinline__ void split_pair(float x0, float x1, uint32_t& hi, uint32_t& lo) {
  const __half2 h = __floats2half2_rn(x0, x1);
  const float2 hf = __half22float2(h);
  const __half2 l = __floats2half2_rn(__fsub_rn(x0, hf.x), __fsub_rn(x1, hf.y));
  hi = *reinterpret_cast<const uint32_t*>(&h);
  lo = *reinterpret_cast<const uint32_t*>(&l);
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
  float* cml = reinterpret_cast<float*>(smem + S::kOffML);
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
  const int n_tasks = (p_end > p_begin) ? (p_end - p_begin + 1) / 2 : 0;
  const int n_my = (n_tasks > warp) ? (n_tasks - warp + kAttnWarps - 1) / kAttnWarps : 0;

  uint8_t* ring = smem + warp * kStages * S::kStageBytes;
  const uint32_t ring_s = smem_addr(ring);
  const uint32_t bar0 = smem_addr(&bars[warp * kStages]);
  int* wflags = flags + warp * kStages;
  const int32_t* pt_row = p.page_table + (size_t)n * p.max_pages;

  if (lane == 0) {
    for (int s = 0; s < kStages; ++s) mbar_init(bar0 + 8 * s, 1);
    mbar_init_fence();
  }
  __syncwarp();

  // ---- page ids of this warp's tasks, 32 tasks at a time ---------------------
  // task i of this warp covers pages p_begin + 2*(warp + 4 i) and the next one;
  // INT_MIN marks "no page" (past the split's range).
  int pid_base = 0, pid_a = INT_MIN, pid_b = INT_MIN;
  auto load_ids = [&](int base) {
    const int i = base + lane;
    const int pa = p_begin + 2 * (warp + kAttnWarps * i);
    pid_a = (i < n_my && pa < p_end) ? pt_row[pa] : INT_MIN;
    pid_b = (i < n_my && pa + 1 < p_end) ? pt_row[pa + 1] : INT_MIN;
  };
  load_ids(0);

  // Issue the copies of task i into its ring stage (all lanes call; i grows by one).
  auto issue = [&](int i) {
    if (i - pid_base >= 32) {
      pid_base += 32;
      load_ids(pid_base);
    }
    const int ia = __shfl_sync(FULL, pid_a, i - pid_base);
    const int ib = __shfl_sync(FULL, pid_b, i - pid_base);
    if (lane == 0) {
      const int st = i % kStages;
      const uint32_t bar = bar0 + 8 * st;
      const uint32_t dst = ring_s + st * S::kStageBytes;
      const bool va = ia >= 0 && ia < p.num_pages;
      const bool vb = ib >= 0 && ib < p.num_pages;
      if ((ia != INT_MIN && !va) || (ib != INT_MIN && !vb)) record_error(KVQ_ERR_OUT_OF_RANGE);
      wflags[st] = (va ? 1 : 0) | (vb ? 2 : 0);
      const uint32_t bytes = (va ? S::kPageBytes : 0) + (vb ? S::kPageBytes : 0);
      if (bytes == 0) {
        mbar_arrive(bar);
      } else {
        mbar_arrive_expect_tx(bar, bytes);
        if (va) {
          const size_t ph = (size_t)ia * p.Hkv + h;
          bulk_g2s(dst, p.cache + ph * S::kCodeBytes, S::kCodeBytes, bar);
          bulk_g2s(dst + S::kCodeBytes, p.scales + ph * 32, 64, bar);
          bulk_g2s(dst + S::kCodeBytes + 64, p.zeros + ph * 32, 64, bar);
        }
        if (vb) {
          const size_t ph = (size_t)ib * p.Hkv + h;
          const uint32_t d1 = dst + S::kPageBytes;
          bulk_g2s(d1, p.cache + ph * S::kCodeBytes, S::kCodeBytes, bar);
          bulk_g2s(d1 + S::kCodeBytes, p.scales + ph * 32, 64, bar);
          bulk_g2s(d1 + S::kCodeBytes + 64, p.zeros + ph * 32, 64, bar);
        }
      }
    }
  };

  const int pre = min(n_my, kStages);
  for (int i = 0; i < pre; ++i) issue(i);
  int issued = pre;

  // ---- q~ = R q * (softmax_scale * log2 e), rows >= G are zero --------------
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
      split_pair(qv[8 * u + t] * f, qv[8 * u + t + 4] * f, aq[2 * u + t][0], aq[2 * u + t][1]);
      split_pair(qv[8 * u + t + 2] * f, qv[8 * u + t + 6] * f, aq[2 * u + t][2], aq[2 * u + t][3]);
    }
  }

  // ---- page stream -------------------------------------------------------------
  float o[NT][4];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) o[nt][0] = o[nt][1] = o[nt][2] = o[nt][3] = 0.0f;
  float m_run = -INFINITY, l_run = 0.0f, zs_run = 0.0f;
  bool ok = true;
  int consumed = 0;

  for (int i = 0; i < n_my; ++i) {
    const int st = i % kStages;
    const bool waited = mbar_wait_bounded(bar0 + 8 * st, (i / kStages) & 1);
    if (!__all_sync(FULL, waited)) { ok = false; break; }
    consumed = i + 1;
    const uint8_t* stg = ring + st * S::kStageBytes;
    const int fl = wflags[st];
    const int tok0 = (p_begin + 2 * (warp + kAttnWarps * i)) * 16;  // first token of the task

    // QK on the codes: n-tile nt = token rows 8(nt&1) + g of page nt>>1
    float acc[4][4];
#pragma unroll
    for (int nt = 0; nt < 4; ++nt) {
      acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.0f;
      if ((fl >> (nt >> 1)) & 1) {
        const uint8_t* row = stg + (nt >> 1) * S::kPageBytes + (8 * (nt & 1) + g) * (D / 2) + tig * (4 * W);
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
    }

    // logits (base 2) of this thread's 8 tokens: 8nt + 2tig + {0, 1}
    float lg[8];
#pragma unroll
    for (int nt = 0; nt < 4; ++nt) {
      const uint8_t* sz = stg + (nt >> 1) * S::kPageBytes + S::kCodeBytes;
      const int i2 = 4 * (nt & 1) + tig;  // half2 index of tokens 8(nt&1) + 2tig, +1
      const float2 sk = __half22float2(reinterpret_cast<const __half2*>(sz)[i2]);
      const float2 zk = __half22float2(reinterpret_cast<const __half2*>(sz + 64)[i2]);
      lg[2 * nt] = fmaf((acc[nt][0] + acc[nt][2]) * acc_to_true, sk.x, zk.x * qsum);
      lg[2 * nt + 1] = fmaf((acc[nt][1] + acc[nt][3]) * acc_to_true, sk.y, zk.y * qsum);
      const int t = tok0 + 8 * nt + 2 * tig;
      const bool vp = (fl >> (nt >> 1)) & 1;
      if (!vp || t >= ctx) lg[2 * nt] = -INFINITY;
      if (!vp || t + 1 >= ctx) lg[2 * nt + 1] = -INFINITY;
    }

    // online softmax, rescaling only when the running maximum grows
    float pm = fmaxf(fmaxf(fmaxf(lg[0], lg[1]), fmaxf(lg[2], lg[3])),
                     fmaxf(fmaxf(lg[4], lg[5]), fmaxf(lg[6], lg[7])));
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
    float pv[8];
#pragma unroll
    for (int nt = 0; nt < 4; ++nt) {
      const uint8_t* sz = stg + (nt >> 1) * S::kPageBytes + S::kCodeBytes;
      const int i2 = 4 * (nt & 1) + tig;
      const float2 sv = __half22float2(reinterpret_cast<const __half2*>(sz + 32)[i2]);
      const float2 zv = __half22float2(reinterpret_cast<const __half2*>(sz + 96)[i2]);
      const float p0 = (lg[2 * nt] == -INFINITY) ? 0.0f : fast_exp2(lg[2 * nt] - m_run);
      const float p1 = (lg[2 * nt + 1] == -INFINITY) ? 0.0f : fast_exp2(lg[2 * nt + 1] - m_run);
      l_run += p0 + p1;
      pv[2 * nt] = (p0 > 0.0f) ? p0 * sv.x : 0.0f;
      pv[2 * nt + 1] = (p1 > 0.0f) ? p1 * sv.y : 0.0f;
      zs_run += ((p0 > 0.0f) ? p0 * zv.x : 0.0f) + ((p1 > 0.0f) ? p1 * zv.y : 0.0f);
    }

    // PV on the codes, one k-step per page: A = (p*s_v) hi/lo rows for this
    // thread's tokens, B = code pairs of token rows (2tig, 2tig+1), (2tig+8,
    // 2tig+9); thread group g supplies channels [g*NT, g*NT + NT)
#pragma unroll
    for (int pg = 0; pg < 2; ++pg) {
      if ((fl >> pg) & 1) {
        uint32_t ap[4];
        split_pair(pv[4 * pg], pv[4 * pg + 1], ap[0], ap[1]);
        split_pair(pv[4 * pg + 2], pv[4 * pg + 3], ap[2], ap[3]);
        const uint8_t* vb = stg + pg * S::kPageBytes + 8 * D;
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
    }
    __syncwarp();
    if (issued < n_my) { issue(issued); ++issued; }
  }
  if (!ok) {
    // a copy never completed: give the ones still outstanding a bounded wait
    for (int i = consumed; i < issued; ++i) mbar_wait_bounded(bar0 + 8 * (i % kStages), (i / kStages) & 1);
  }

  // ---- merge the four warps into the CTA's (M, L, O + Z) per head --------------
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
        const float e = fast_exp2(mwr - M);
        O += mw[r * D + c] * e;
        L += mw[8 * D + 8 + r] * e;
        Z += mw[8 * D + 16 + r] * e;
      }
    }
    qs[idx] = O + Z;
    if (c == 0) {
      cml[2 * r] = M;
      cml[2 * r + 1] = L;
    }
  }
  __syncthreads();

  // ---- merge the cluster's CTAs into its first CTA (distributed smem) --------
  const int cs = p.cluster_size;
  if (cs > 1) {
    constexpr int kPer = (8 * D + kAttnThreads - 1) / kAttnThreads;
    float keepO[kPer], keepM[kPer], keepL[kPer];
    cluster_sync_all();  // every CTA's merged result is in its shared memory
    const uint32_t rank = cluster_ctarank();
    if (rank == 0) {
#pragma unroll
      for (int k = 0; k < kPer; ++k) {
        const int idx = tid + k * kAttnThreads;
        keepO[k] = keepM[k] = keepL[k] = 0.0f;
        if (idx < G * D) {
          const int r = idx / D;
          float M = -INFINITY;
          for (int q = 0; q < cs; ++q) M = fmaxf(M, ld_dsmem_f32(&cml[2 * r], q));
          float O = 0.0f, L = 0.0f;
          if (M != -INFINITY) {
            for (int q = 0; q < cs; ++q) {
              const float mq = ld_dsmem_f32(&cml[2 * r], q);
              if (mq == -INFINITY) continue;
              const float e = fast_exp2(mq - M);
              O += e * ld_dsmem_f32(&qs[idx], q);
              L += e * ld_dsmem_f32(&cml[2 * r + 1], q);
            }
          }
          keepO[k] = O;
          keepM[k] = M;
          keepL[k] = L;
        }
      }
    }
    cluster_sync_all();  // the first CTA has read every CTA's shared memory
    if (rank != 0) return;
#pragma unroll
    for (int k = 0; k < kPer; ++k) {
      const int idx = tid + k * kAttnThreads;
      if (idx < G * D) {
        qs[idx] = keepO[k];
        if (idx % D == 0) {
          cml[2 * (idx / D)] = keepM[k];
          cml[2 * (idx / D) + 1] = keepL[k];
        }
      }
    }
    __syncthreads();
  }

  if (p.n_parts == 1) {
    for (int idx = tid; idx < G * D; idx += kAttnThreads) {
      const float L = cml[2 * (idx / D) + 1];
      qs[idx] = (L > 0.0f) ? qs[idx] / L : 0.0f;
    }
  } else {
    // ---- several clusters per (sequence, kv head): meet in the workspace -----
    const int part = split / cs;
    const int np = p.n_parts;
    float* base = p.ws_part + (((size_t)n * p.Hkv + h) * np) * G * (D + 2);
    float* dst = base + (size_t)part * G * (D + 2);
    for (int idx = tid; idx < G * D; idx += kAttnThreads) {
      const int r = idx / D, c = idx % D;
      dst[r * (D + 2) + c] = qs[idx];
      if (c == 0) {
        dst[r * (D + 2) + D] = cml[2 * r];
        dst[r * (D + 2) + D + 1] = cml[2 * r + 1];
      }
    }
    __threadfence();
    __syncthreads();
    int* s_last = flags + kAttnWarps * kStages;
    if (tid == 0) {
      const int prev = atomicAdd(&p.ws_count[(size_t)n * p.Hkv + h], 1);
      *s_last = (prev == np - 1);
    }
    __syncthreads();
    if (!*s_last) return;
    __threadfence();
    float* lsp = wts + 8 * kMaxParts;  // per (head, part) sums
    float* Lr = wts + 16 * kMaxParts;  // per head total
    for (int idx = tid; idx < G * np; idx += kAttnThreads) {
      const int r = idx % G, s = idx / G;
      const float* src = base + ((size_t)s * G + r) * (D + 2) + D;
      wts[r * kMaxParts + s] = __ldcg(src);
      lsp[r * kMaxParts + s] = __ldcg(src + 1);
    }
    __syncthreads();
    for (int r = warp; r < G; r += kAttnWarps) {
      float M = -INFINITY;
      for (int s = lane; s < np; s += 32) M = fmaxf(M, wts[r * kMaxParts + s]);
#pragma unroll
      for (int o2 = 16; o2 > 0; o2 >>= 1) M = fmaxf(M, __shfl_xor_sync(FULL, M, o2));
      float L = 0.0f;
      for (int s = lane; s < np; s += 32) {
        const float ms = wts[r * kMaxParts + s];
        const float e = (ms == -INFINITY) ? 0.0f : fast_exp2(ms - M);
        wts[r * kMaxParts + s] = e;
        L += e * lsp[r * kMaxParts + s];
      }
#pragma unroll
      for (int o2 = 16; o2 > 0; o2 >>= 1) L += __shfl_xor_sync(FULL, L, o2);
      if (lane == 0) Lr[r] = L;
    }
    __syncthreads();
    for (int idx = tid; idx < G * D; idx += kAttnThreads) {
      const int r = idx / D, c = idx % D;
      const float* src = base + (size_t)r * (D + 2) + c;
      const size_t stride = (size_t)G * (D + 2);
      float a0 = 0.0f, a1 = 0.0f, a2 = 0.0f, a3 = 0.0f;
      int s = 0;
      for (; s + 4 <= np; s += 4) {
        const float v0 = __ldcg(src + (size_t)s * stride), v1 = __ldcg(src + (size_t)(s + 1) * stride);
        const float v2 = __ldcg(src + (size_t)(s + 2) * stride), v3 = __ldcg(src + (size_t)(s + 3) * stride);
        a0 = fmaf(wts[r * kMaxParts + s], v0, a0);
        a1 = fmaf(wts[r * kMaxParts + s + 1], v1, a1);
        a2 = fmaf(wts[r * kMaxParts + s + 2], v2, a2);
        a3 = fmaf(wts[r * kMaxParts + s + 3], v3, a3);
      }
      for (; s < np; ++s) a0 = fmaf(wts[r * kMaxParts + s], __ldcg(src + (size_t)s * stride), a0);
      const float acc = (a0 + a1) + (a2 + a3);
      qs[idx] = (Lr[r] > 0.0f) ? acc / Lr[r] : 0.0f;
    }
    if (tid == 0) p.ws_count[(size_t)n * p.Hkv + h] = 0;  // leave the tickets at zero
  }
  __syncthreads();

  // ---- out = R o_rot -------------------------------------------------------------
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
