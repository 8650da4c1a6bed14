// kvq_prefill.cuh - chunked-prefill attention over the rotated INT4 cache on
// the 5th-generation tensor cores.
//
// SAW-INT4 (Abstract): attention is computed directly on the quantized paged
// cache, and the method targets serving many requests at once. A prefill
// chunk brings many queries per sequence, so QK^T and PV become dense
// products and run as tcgen05 MMAs.
//
// Sequence n's chunk is its last qlen context tokens (positions ctx - qlen ..
// ctx - 1), already written to the cache by kv_quant_write; query token i of
// the chunk attends causally to positions 0 .. ctx - qlen + i.
//
// One CTA (8 warps) per (tile of 128 / G chunk tokens x the G query heads of
// one kv head, kv head, sequence): 128 query rows = the MMA's M, row
// r = token (r / G) x head (r % G) = tensor-memory lane r. Two threads share a
// row: warps w and w + 4 (the lane quarter w mod 4 is all that a warp may
// read of tensor memory), each with half of the row's logits and of its
// output columns; they meet once per block to agree on the running maximum.
// The cache is read in blocks of 64 tokens (4 pages), up to the tile's last
// position:
//   - 16-byte cp.async copies of the block's codes, scales and zeros into a
//     double-buffered staging area (the next block loads while this one runs;
//     its page ids were read from the page table a block earlier);
//   - the codes become exact centred integers c - 8 in shared memory: K as
//     fp16, the MMA's B operand [64 tokens][D], and V transposed as bf16,
//     [D][64 tokens], both K-major with the 128-byte swizzle; the 8 moves into
//     the zero point (z + 8 s). Centred, a channel's sum has no fixed sign: the
//     tensor cores' accumulation error then has none either, where with codes
//     0 .. 15 and P' >= 0 it leaned the same way in every channel and R^T's
//     all-ones row added it up (x sqrt(b));
//   - S = Q~ K^T: q~ = R q (softmax scale and log2 e folded in), scaled per
//     row by a power of two that puts its largest element in [2^13, 2^14),
//     enters as fp16 hi + lo (two MMA passes, ~22 significant bits, both parts
//     normal fp16: the tensor cores do not keep subnormal operands exact; fp16
//     alone would move logits on keys with x10 outlier channels), codes are
//     exact, the fp32 accumulator lands in tensor memory:
//     logit = s_t 2^-e (q~ 2^e . (code_t - 8)) + (z_t + 8 s_t) sum(q~);
//   - each thread takes its half of the row's S from tensor memory, masks
//     positions past its own, and runs its share of the online softmax two
//     logits at a time (f32x2; sum p and sum p z_v in registers, the running
//     maximum agreed with the partner thread); rows past the context get scale
//     and offset 0, so that garbage there cannot reach the sums;
//   - P' = p * s_v as bf16 hi + lo (16 significant bits over the fp32 exponent
//     range: small weights never become subnormal) is written to shared memory
//     as the A operand and O_blk = P' V (V codes as exact bf16 integers) goes
//     to a fresh tensor-memory accumulator; the running O, in a second one, is
//     updated on the CUDA cores, O = alpha O + O_blk in fp32. (Accumulating
//     80 blocks into one tensor-memory accumulator with the MMA itself lost
//     precision: 1.3e-2 max-abs at 5000 tokens, against 2.6e-4 at 700.)
// The epilogue divides, rotates back with R^T (warp FWHT) and stores.
#pragma once

#include "kvq_decode.cuh"
#include "kvq_write_tc.cuh"

namespace kvq {

struct PrefillParams {
  const uint16_t* q;          // bf16 [Tq][Hq][D]; sequence n's chunk at rows q_start[n] ..
  const uint8_t* cache;       // [pages][Hkv][2][16][D/2]
  const uint16_t* scales;     // fp16 [pages][Hkv][2][16]
  const uint16_t* zeros;
  const int32_t* page_table;  // [B][max_pages]
  const int32_t* ctx_lens;    // [B]: context lengths including the chunk
  const int32_t* q_start;     // [B + 1]: chunk of sequence n = rows q_start[n] .. q_start[n + 1] - 1
  void* out;                  // [Tq][Hq][D] fp32 or bf16
  int B, Hq, Hkv, G;
  int num_pages, max_pages;
  int out_bf16;
  float qmul;                 // c_b * softmax_scale * log2(e)
  float cb;                   // c_b, 1 for plain INT4
  uint32_t signs[4];          // randomized Hadamard signs, as written
};

constexpr int kPfThreads = 256;  // two threads per query row
constexpr int kPfRows = 128;   // query rows per CTA (MMA M)
constexpr int kPfBlock = 64;   // cache tokens per block (N of S, K of PV)
// tensor-memory columns: S [0, 64), O_blk [64, 64 + D), O [64 + D, 64 + 2D),
// rounded up to a power of two
__host__ __device__ constexpr uint32_t pf_tmem_cols(int d) { return 64 + 2 * d <= 256 ? 256 : 512; }

template <int D>
struct PfSmem {
  static constexpr int kSlot = 16 * D + 128;                 // one page: codes, 32 scales, 32 zeros
  static constexpr int kStageBytes = (kPfBlock / 16) * kSlot;
  static constexpr int kQhi = 0;                             // [128 rows][D] fp16, D/64 swizzle chunks
  static constexpr int kQlo = kQhi + kPfRows * D * 2;
  static constexpr int kK = kQlo + kPfRows * D * 2;          // [64 tokens][D] fp16
  static constexpr int kVt = kK + kPfBlock * D * 2;          // [D][64 tokens] bf16
  static constexpr int kPhi = kVt + D * kPfBlock * 2;        // [128 rows][64 tokens] bf16
  static constexpr int kPlo = kPhi + kPfRows * kPfBlock * 2;
  static constexpr int kStage = kPlo + kPfRows * kPfBlock * 2;
  static constexpr int kSz = kStage + 2 * kStageBytes;       // float [4][64]: s_k, z_k, s_v, z_v
  static constexpr int kPageOk = kSz + 4 * kPfBlock * 4;     // int [4]
  static constexpr int kXch = kPageOk + 16;                  // float [2][128]: the two halves' block maxima
  static constexpr int kQsum = kXch + 2 * kPfRows * 4;       // float [128]
  static constexpr int kQinv = kQsum + kPfRows * 4;          // float [128]: 2^-e of each row
  static constexpr int kBar = kQinv + kPfRows * 4;           // 2 mbarriers
  static constexpr int kTmem = kBar + 16;
  static constexpr int kUsed = kTmem + 16;
  static constexpr int kTotal = kUsed + 1024;                // room to align the base to 1024 B
};

// The pair (x0, x1) as bf16 hi = RN(x) and lo = RN(x - hi), each packed in
// one word (hi + lo keeps 16 significant bits).
__device__ __forceinline__ void hilo_split_bf16(uint64_t x2, uint32_t& hw, uint32_t& lw) {
  float x0, x1;
  f2_unpack(x2, x0, x1);
  const __nv_bfloat162 h = __floats2bfloat162_rn(x0, x1);
  const float2 hf = __bfloat1622float2(h);
  float r0, r1;
  f2_unpack(f2_sub(x2, f2_pack(hf.x, hf.y)), r0, r1);
  const __nv_bfloat162 l = __floats2bfloat162_rn(r0, r1);
  hw = *reinterpret_cast<const uint32_t*>(&h);
  lw = *reinterpret_cast<const uint32_t*>(&l);
}

// Two 4-bit codes of byte k of w -> half2 (low nibble, high nibble) as exact
// centred fp16 integers c - 8 (w4 = w >> 4 puts the high nibble of byte k in
// its low bits; 1024 + c has ulp 1 in fp16 and subtracting 1032 is exact).
__device__ __forceinline__ uint32_t byte_to_half2(uint32_t w, uint32_t w4, uint32_t k) {
  const uint32_t x = prmt(w, w4, k | ((4u + k) << 8));
  const uint32_t biased = (x & 0x000F000Fu) | 0x64006400u;
  uint32_t r;
  asm("sub.rn.f16x2 %0, %1, %2;\n" : "=r"(r) : "r"(biased), "r"(0x64086408u));
  return r;
}

template <int D, int BLK>
__global__ void __launch_bounds__(kPfThreads, 1) kvq_prefill_kernel(const __grid_constant__ PrefillParams p) {
  static_assert(D == 64 || D == 128, "prefill instances exist for D = 64 and 128");
  using S = PfSmem<D>;
  constexpr int E = D / 32;
  constexpr uint32_t kIdescS = (1u << 4) | ((uint32_t)(kPfBlock >> 3) << 17) | ((uint32_t)(kPfRows >> 4) << 24);
  // PV: bf16 A and B (P' hi / lo and V codes)
  constexpr uint32_t kIdescPV = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(D >> 3) << 17) |
                                ((uint32_t)(kPfRows >> 4) << 24);
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024 - (smem_addr(smem_raw) & 1023)) & 1023);
  const uint32_t sb = smem_addr(smem);
  float* sz = reinterpret_cast<float*>(smem + S::kSz);
  int* page_ok = reinterpret_cast<int*>(smem + S::kPageOk);
  float* qsum = reinterpret_cast<float*>(smem + S::kQsum);
  float* qinv = reinterpret_cast<float*>(smem + S::kQinv);
  float* xch = reinterpret_cast<float*>(smem + S::kXch);
  const uint32_t bar_s = sb + S::kBar, bar_pv = bar_s + 8;
  uint32_t* tslot = reinterpret_cast<uint32_t*>(smem + S::kTmem);

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int tile = blockIdx.x, h = blockIdx.y, n = blockIdx.z;
  const int G = p.G, TQ = kPfRows / G;
  const unsigned FULL = 0xffffffffu;

  pdl_wait();  // every input may come from the previous kernel on the stream
  pdl_launch_dependents();
  const int q0 = p.q_start[n], qlen = p.q_start[n + 1] - q0;
  if (qlen <= 0 || tile * TQ >= qlen) return;  // the whole CTA, before any barrier
  int ctx = p.ctx_lens[n];
  // a context shorter than its chunk, past the page table, or a chunk longer
  // than the grid covers (max_q_len too small): the sequence is left unwritten
  if (ctx < qlen || ctx > p.max_pages * 16 || qlen > (int)gridDim.x * TQ) {
    if (tid == 0) record_error(KVQ_ERR_OUT_OF_RANGE);
    return;
  }
  const int pos0 = ctx - qlen + tile * TQ;            // position of the tile's first token
  const int ntok = min(TQ, qlen - tile * TQ);         // tokens of the tile
  const int n_blocks = (pos0 + ntok + kPfBlock - 1) / kPfBlock;

  if (tid == 0) {
    mbar_init(bar_s, 1);
    mbar_init(bar_pv, 1);
    mbar_init_fence();
  }
  if (warp == 0) tmem_alloc(smem_addr(tslot), pf_tmem_cols(D));
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tslot;
  const int quarter = warp & 3, half = warp >> 2;  // tensor-memory lanes; half of the row
  const uint32_t lane_base = (uint32_t)(32 * quarter) << 16;
  // this thread's columns: S [32 half, +32), O_blk and O [D/2 half, +D/2)
  const uint32_t tS = tmem + lane_base + 32 * half;
  const uint32_t tOb = tmem + lane_base + kPfBlock + (D / 2) * half, tO = tOb + D;

  // ---- block fetch: 4 pages of kv head h into staging buffer b & 1 --------
  const int32_t* pt_row = p.page_table + (size_t)n * p.max_pages;
  // The page ids a block needs are read from the page table one block ahead
  // (into registers), so that no fetch waits for that load: pid[k] for this
  // thread's k-th 16-byte chunk of the next fetch, sid for the scales and
  // zeros of token tid (tid < 64).
  constexpr int kChunks = D + 8;  // 16-byte chunks per page: codes, then scales, zeros
  constexpr int kPerThread = (4 * kChunks + kPfThreads - 1) / kPfThreads;
  auto page_id = [&](int lp) { return (lp * 16 < ctx) ? pt_row[lp] : -1; };
  int pid[kPerThread];
  auto load_ids = [&](int b) {
#pragma unroll
    for (int k = 0; k < kPerThread; ++k) {
      const int i = tid + k * kPfThreads;
      pid[k] = (i < 4 * kChunks) ? page_id(4 * b + i / kChunks) : -1;
    }
  };
  auto fetch = [&](int b) {
    uint8_t* st = smem + S::kStage + (b & 1) * S::kStageBytes;
#pragma unroll
    for (int k = 0; k < kPerThread; ++k) {
      const int i = tid + k * kPfThreads;
      const int id = pid[k];
      if (i >= 4 * kChunks || id < 0 || id >= p.num_pages) continue;
      const int pg = i / kChunks, c = i % kChunks;
      const size_t head = (size_t)id * p.Hkv + h;
      const void* src = (c < D) ? static_cast<const void*>(p.cache + head * (16 * D) + 16 * c)
                                : static_cast<const void*>((c < D + 4 ? p.scales : p.zeros) + head * 32 + 8 * ((c - D) & 3));
      cp_async_16(smem_addr(st + pg * S::kSlot + 16 * c), src);
    }
    cp_async_commit();
  };
  load_ids(0);
  fetch(0);
  if (n_blocks > 1) load_ids(1);
  int sid = (tid < kPfBlock) ? page_id(tid >> 4) : -1;  // block 0

  // ---- q~ = R q * (softmax_scale * log2 e) as fp16 hi + lo, sum(q~) per row -
  for (int r = warp; r < kPfRows; r += kPfThreads / 32) {
    const int i = r / G, j = r % G;
    float v[E];
    if (i < ntok) {
      const uint16_t* src = p.q + ((size_t)(q0 + tile * TQ + i) * p.Hq + (size_t)h * G + j) * D + E * lane;
#pragma unroll
      for (int e = 0; e < E; ++e) v[e] = bf16_bits_to_float(src[e]);
      if constexpr (BLK > 0) {
        apply_signs<D>(v, p.signs, lane);
        warp_fwht<D, BLK>(v, lane);
      }
    } else {
#pragma unroll
      for (int e = 0; e < E; ++e) v[e] = 0.0f;
    }
    float sum = 0.0f, amax = 0.0f;
#pragma unroll
    for (int e = 0; e < E; ++e) {
      v[e] *= p.qmul;
      sum += v[e];
      amax = fmaxf(amax, fabsf(v[e]));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      sum += __shfl_xor_sync(FULL, sum, o);
      amax = fmaxf(amax, __shfl_xor_sync(FULL, amax, o));
    }
    // 2^e with amax 2^e in [2^13, 2^14)
    int ex = 0;
    if (amax > 0.0f) {
      (void)frexpf(amax, &ex);  // amax = m 2^ex, m in [0.5, 1)
      ex = 14 - ex;
    }
    const float up = ldexpf(1.0f, ex);
    if (lane == 0) {
      qsum[r] = sum;
      qinv[r] = ldexpf(1.0f, -ex);
    }
    uint32_t hi2[E / 2], lo2[E / 2];
#pragma unroll
    for (int e = 0; e < E; e += 2) {
      hi2[e / 2] = hilo_pair(v[e] * up, v[e + 1] * up, false);
      lo2[e / 2] = hilo_pair(v[e] * up, v[e + 1] * up, true);
    }
    // E = 4 consecutive elements = 8 bytes of one 16-byte swizzle unit
    // E consecutive elements = 2E bytes of one 16-byte swizzle unit
    if constexpr (E == 4) {
      *reinterpret_cast<uint2*>(smem + S::kQhi + sw128_offset(r, E * lane, kPfRows)) = make_uint2(hi2[0], hi2[1]);
      *reinterpret_cast<uint2*>(smem + S::kQlo + sw128_offset(r, E * lane, kPfRows)) = make_uint2(lo2[0], lo2[1]);
    } else {
      *reinterpret_cast<uint32_t*>(smem + S::kQhi + sw128_offset(r, E * lane, kPfRows)) = hi2[0];
      *reinterpret_cast<uint32_t*>(smem + S::kQlo + sw128_offset(r, E * lane, kPfRows)) = lo2[0];
    }
  }

  // this thread's row (= tensor-memory lane)
  const int row = 32 * quarter + lane, ri = row / G;
  const bool row_ok = ri < ntok;
  const int pos_r = pos0 + ri;  // the last position this row attends to
  float m_used = -INFINITY, l_sum = 0.0f, zs = 0.0f;
  float alpha_prev = 1.0f;  // the factor of the block whose O_blk is pending
  // O = alpha O + O_blk, this row, after the block's PV MMA (warp-wide
  // tensor-memory loads and stores; `first`: O := O_blk)
  auto fold = [&](bool first, float alpha) {
#pragma unroll
    for (int c0 = 0; c0 < D / 2; c0 += 32) {
      float ob[32];
      tmem_ld32(tOb + c0, ob);
      if (!first) {
        float o[32];
        tmem_ld32(tO + c0, o);
#pragma unroll
        for (int k = 0; k < 32; ++k) ob[k] = fmaf(alpha, o[k], ob[k]);
      }
      tmem_st32(tO + c0, ob);
    }
  };

  for (int b = 0; b < n_blocks; ++b) {
    if (b + 1 < n_blocks) {
      fetch(b + 1);
      if (b + 2 < n_blocks) load_ids(b + 2);
    }
    else cp_async_commit();
    cp_async_wait<1>();  // block b has landed (this thread's copies)
    // the previous PV MMA read the K, V and P' tiles and wrote O_blk: done
    // first; then fold it into O
    if (b > 0) mbar_wait_bounded(bar_pv, (b - 1) & 1);
    __syncthreads();     // ... and every thread's copies have landed
    tc_fence_after();
    if (b > 0) fold(b == 1, alpha_prev);

    // ---- codes -> exact fp16 operands; scales and zeros per token ----------
    const uint8_t* st = smem + S::kStage + (b & 1) * S::kStageBytes;
    for (int u = tid; u < kPfBlock * (D / 8); u += kPfThreads) {  // K: 8 channels per unit
      const int t = u / (D / 8), c8 = u % (D / 8);
      const uint32_t w = *reinterpret_cast<const uint32_t*>(st + (t >> 4) * S::kSlot + (t & 15) * (D / 2) + 4 * c8);
      const uint32_t w4 = w >> 4;
      *reinterpret_cast<uint4*>(smem + S::kK + sw128_offset(t, 8 * c8, kPfBlock)) =
          make_uint4(byte_to_half2(w, w4, 0), byte_to_half2(w, w4, 1), byte_to_half2(w, w4, 2),
                     byte_to_half2(w, w4, 3));
    }
    for (int u = tid; u < (D / 2) * (kPfBlock / 8); u += kPfThreads) {  // V^T: a channel pair x 8 tokens
      const int cp = u % (D / 2), tg = u / (D / 2);
      uint32_t wa = 0, wb = 0;  // byte cp of tokens 8tg .. 8tg+3, 8tg+4 .. 8tg+7
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const int t0 = 8 * tg + k, t1 = t0 + 4;
        const uint32_t b0 = st[(t0 >> 4) * S::kSlot + 8 * D + (t0 & 15) * (D / 2) + cp];
        const uint32_t b1 = st[(t1 >> 4) * S::kSlot + 8 * D + (t1 & 15) * (D / 2) + cp];
        wa |= b0 << (8 * k);
        wb |= b1 << (8 * k);
      }
      // low nibbles -> channel 2cp, high nibbles -> channel 2cp + 1; pairs of tokens
      const uint32_t wa4 = wa >> 4, wb4 = wb >> 4;
      // tokens k0, k0 + 1 of word x (low nibbles) as exact centred bf16
      // c - 8: 128 + c has ulp 1 in bf16, and subtracting 136 is exact
      auto pair = [](uint32_t x, uint32_t k0) {
        const uint32_t y = prmt(x, 0u, k0 | ((k0 + 1u) << 8));
        const uint32_t biased = (y & 0x000F000Fu) | 0x43004300u;
        uint32_t r;
        asm("sub.rn.bf16x2 %0, %1, %2;\n" : "=r"(r) : "r"(biased), "r"(0x43084308u));
        return r;
      };
      *reinterpret_cast<uint4*>(smem + S::kVt + sw128_offset(2 * cp, 8 * tg, D)) =
          make_uint4(pair(wa, 0), pair(wa, 2), pair(wb, 0), pair(wb, 2));
      *reinterpret_cast<uint4*>(smem + S::kVt + sw128_offset(2 * cp + 1, 8 * tg, D)) =
          make_uint4(pair(wa4 & 0x0F0F0F0Fu, 0), pair(wa4 & 0x0F0F0F0Fu, 2), pair(wb4 & 0x0F0F0F0Fu, 0),
                     pair(wb4 & 0x0F0F0F0Fu, 2));
    }
    if (tid < kPfBlock) {  // token tid of the block
      const int t = tid, pg = t >> 4, lp = 4 * b + pg;
      const int id = sid;
      if (b + 1 < n_blocks) sid = page_id(lp + 4);  // the next block's, read ahead
      const bool ok = id >= 0 && id < p.num_pages;
      if (!ok && lp * 16 < ctx && (t & 15) == 0) record_error(KVQ_ERR_OUT_OF_RANGE);
      const __half* scl = reinterpret_cast<const __half*>(st + pg * S::kSlot + 16 * D);
      const __half* zer = reinterpret_cast<const __half*>(st + pg * S::kSlot + 16 * D + 64);
      // scales, and the zero points of the centred codes: z + 8 s. Rows past
      // the context may hold anything (NaN scales included): they get 0, so
      // that their zero weights cannot turn 0 * garbage into NaN
      const bool live = ok && lp * 16 + (t & 15) < ctx;
      const float s_k = __half2float(scl[t & 15]), s_v = __half2float(scl[16 + (t & 15)]);
      sz[0 * kPfBlock + t] = live ? s_k : 0.0f;
      sz[1 * kPfBlock + t] = live ? fmaf(8.0f, s_k, __half2float(zer[t & 15])) : 0.0f;
      sz[2 * kPfBlock + t] = live ? s_v : 0.0f;
      sz[3 * kPfBlock + t] = live ? fmaf(8.0f, s_v, __half2float(zer[16 + (t & 15)])) : 0.0f;
      if ((t & 15) == 0) page_ok[pg] = ok ? 1 : 0;
    }
    asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");  // operands visible to the MMAs
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    // ---- S = Q~ K^T (hi, then lo) ------------------------------------------
    if (tid == 0) {
#pragma unroll
      for (int half = 0; half < 2; ++half)
#pragma unroll
        for (int s = 0; s < D / 16; ++s) {
          const uint32_t offa = (s >> 2) * (kPfRows * 128) + (s & 3) * 32;
          const uint32_t offb = (s >> 2) * (kPfBlock * 128) + (s & 3) * 32;
          umma_f16_ss(tmem, umma_desc_sw128(sb + (half ? S::kQlo : S::kQhi) + offa),
                      umma_desc_sw128(sb + S::kK + offb), kIdescS, half > 0 || s > 0);
        }
      umma_commit(bar_s);
    }
    mbar_wait_bounded(bar_s, b & 1);
    tc_fence_after();

    // ---- online softmax: this thread's 32 of the row's 64 logits ------------
    constexpr int kH = kPfBlock / 2;
    const int t0 = kH * half;  // first token of this thread's half
    float sv[kH];
    tmem_ld32(tS, sv);
    const float qs = qsum[row], qi = qinv[row];
    // every row sees the whole block, every page is valid: no masks
    const bool open = kPfBlock * b + kPfBlock - 1 <= pos0 &&
                      (page_ok[0] & page_ok[1] & page_ok[2] & page_ok[3]) != 0;
    // logits two at a time (f32x2): fma(S qi, s_k, z_k qs)
    const uint64_t qi2 = f2_pack(qi, qi), qs2 = f2_pack(qs, qs);
#pragma unroll
    for (int t = 0; t < kH; t += 2) {
      const float2 sk = *reinterpret_cast<const float2*>(sz + t0 + t);
      const float2 zk = *reinterpret_cast<const float2*>(sz + kPfBlock + t0 + t);
      f2_unpack(f2_fma(f2_mul(f2_pack(sv[t], sv[t + 1]), qi2), f2_pack(sk.x, sk.y), f2_mul(f2_pack(zk.x, zk.y), qs2)),
                sv[t], sv[t + 1]);
    }
    if (!open) {
#pragma unroll
      for (int t = 0; t < kH; ++t) {
        const int pos = kPfBlock * b + t0 + t;
        const bool live = row_ok && pos <= pos_r && page_ok[(t0 + t) >> 4];
        sv[t] = live ? sv[t] : -INFINITY;
      }
    }
    float mb = -INFINITY;
#pragma unroll
    for (int t = 0; t < kH; t += 2) mb = fmax3(mb, sv[t], sv[t + 1]);
    // the row's block maximum: the two halves meet (warps quarter and
    // quarter + 4, 64 threads, named barrier 1 + quarter)
    xch[half * kPfRows + row] = mb;
    named_bar_sync(1 + quarter, 64);
    mb = fmaxf(mb, xch[(half ^ 1) * kPfRows + row]);
    // online softmax: the running maximum, and the factor for what came before
    // (both halves compute the same values)
    const float m_new = fmaxf(m_used, mb);
    const float alpha = (m_new == -INFINITY || m_used == -INFINITY) ? 0.0f : fast_exp2(m_used - m_new);
    l_sum *= alpha;
    zs *= alpha;
    alpha_prev = alpha;
    m_used = m_new;
    // p and P' = p * s_v as bf16 hi + lo, this half of row `row` of the A
    // operands, two at a time; a masked logit (-inf) gives exp2 = 0, and a
    // row with no visible position yet (m = -inf) subtracts 0 instead
    const float msub = (m_used == -INFINITY) ? 0.0f : m_used;
    const uint64_t m2 = f2_pack(msub, msub);
    uint64_t l2 = f2_pack(0.0f, 0.0f), z2 = l2;
#pragma unroll
    for (int t8 = 0; t8 < kH; t8 += 8) {
      uint32_t hw[4], lw[4];
#pragma unroll
      for (int k = 0; k < 8; k += 2) {
        const int t = t8 + k;
        float d0, d1;
        f2_unpack(f2_sub(f2_pack(sv[t], sv[t + 1]), m2), d0, d1);
        const uint64_t p2 = f2_pack(fast_exp2(d0), fast_exp2(d1));
        const float2 s_v = *reinterpret_cast<const float2*>(sz + 2 * kPfBlock + t0 + t);
        const float2 z_v = *reinterpret_cast<const float2*>(sz + 3 * kPfBlock + t0 + t);
        l2 = f2_add(l2, p2);
        z2 = f2_fma(p2, f2_pack(z_v.x, z_v.y), z2);
        hilo_split_bf16(f2_mul(p2, f2_pack(s_v.x, s_v.y)), hw[k / 2], lw[k / 2]);
      }
      *reinterpret_cast<uint4*>(smem + S::kPhi + sw128_offset(row, t0 + t8, kPfRows)) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
      *reinterpret_cast<uint4*>(smem + S::kPlo + sw128_offset(row, t0 + t8, kPfRows)) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
    }
    {
      float a0, a1, c0, c1;
      f2_unpack(l2, a0, a1);
      f2_unpack(z2, c0, c1);
      l_sum += a0 + a1;
      zs += c0 + c1;
    }
    asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    // ---- O_blk = P' V (hi, then lo) -----------------------------------------
    if (tid == 0) {
#pragma unroll
      for (int half = 0; half < 2; ++half)
#pragma unroll
        for (int s = 0; s < kPfBlock / 16; ++s)
          umma_f16_ss(tmem + kPfBlock, umma_desc_sw128(sb + (half ? S::kPlo : S::kPhi) + 32 * s),
                      umma_desc_sw128(sb + S::kVt + 32 * s), kIdescPV, half > 0 || s > 0);
      umma_commit(bar_pv);
    }
  }
  cp_async_wait<0>();
  mbar_wait_bounded(bar_pv, (n_blocks - 1) & 1);
  tc_fence_after();
  fold(n_blocks == 1, alpha_prev);

  // ---- epilogue: o~ = (O + Z) / L, then R^T per row --------------------------
  // the halves' sums of p and p z: each thread adds its partner's
  xch[half * kPfRows + row] = l_sum;
  named_bar_sync(1 + quarter, 64);
  const float l_all = l_sum + xch[(half ^ 1) * kPfRows + row];
  named_bar_sync(1 + quarter, 64);
  xch[half * kPfRows + row] = zs;
  named_bar_sync(1 + quarter, 64);
  const float z_all = zs + xch[(half ^ 1) * kPfRows + row];
  float* orow = reinterpret_cast<float*>(smem + S::kQhi);  // [128][D] fp32 over the Q tiles
  {
    const float inv = (l_all > 0.0f) ? 1.0f / l_all : 0.0f;
#pragma unroll
    for (int c0 = 0; c0 < D / 2; c0 += 32) {
      float o[32];
      tmem_ld32(tO + c0, o);
      const int cb = (D / 2) * half + c0;  // column of o[0]
#pragma unroll
      for (int k = 0; k < 32; k += 4)
        *reinterpret_cast<float4*>(orow + row * D + ((cb + k + 4 * row) & (D - 1))) =
            make_float4((o[k] + z_all) * inv, (o[k + 1] + z_all) * inv, (o[k + 2] + z_all) * inv,
                        (o[k + 3] + z_all) * inv);
    }
  }
  tc_fence_before();
  __syncthreads();
  for (int r = warp; r < kPfRows; r += kPfThreads / 32) {
    const int i = r / G, j = r % G;
    if (i >= ntok) continue;
    float v[E];
#pragma unroll
    for (int e = 0; e < E; ++e) v[e] = orow[r * D + ((E * lane + e + 4 * r) & (D - 1))];
    if constexpr (BLK > 0) {
      warp_fwht<D, BLK>(v, lane);
      apply_signs<D>(v, p.signs, lane);
    }
    const size_t o_base = ((size_t)(q0 + tile * TQ + i) * p.Hq + (size_t)h * G + j) * D + E * lane;
#pragma unroll
    for (int e = 0; e < E; ++e) {
      const float x = BLK > 0 ? v[e] * p.cb : v[e];
      if (p.out_bf16)
        reinterpret_cast<__nv_bfloat16*>(p.out)[o_base + e] = __float2bfloat16_rn(x);
      else
        reinterpret_cast<float*>(p.out)[o_base + e] = x;
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem, pf_tmem_cols(D));
}

}  // namespace kvq
