// kvq_oscar.cuh - the OScaR variant: INT2 codes after a rotation and a
// per-token scaling, K quantized per channel.
//
// OScaR forum summary, "The OScaR Framework": V^ = Quant(S (R V)) - rotate,
// scale every token so that all tokens suit the quantizer equally, quantize.
// OScaR abstract: the per-channel quantization paradigm for Key tensors,
// Token Norm Imbalance (token norms that differ widely within a group that
// shares quantization parameters) as the error source, INT2.
//
// Readings (the pages give no group size, rule for S or layout):
//  - R: the same block Hadamard as the INT4 path (H_b / sqrt(b), b = 0: none);
//  - S: fp32(1 / n_t) with n_t = ||R k_t||_2 rounded to fp16 (stored), the
//    row multiplied by it, so that K^_t = n_t * dequant(codes); every scaled
//    K row has unit norm up to the fp16 rounding of n_t;
//  - K: per channel c over the 16 tokens of a page, z_c = RD16(min),
//    s_c = smallest fp16 with 3 s_c + z_c >= max, code = rint(fp32(u - z)
//    * fp32(1/s)) in 0..3;
//  - V: token-wise INT2 after R (a per-token S cancels under per-token
//    (s, z), so none is stored);
//  - codes four per byte, the lowest channel in the lowest bits;
//  - a page is quantized whole: a sequence's unfinished last page stays in
//    bf16 (k_tail / v_tail) and the decode reads it exactly.
//
// Layout per (page, kv head), in three pools:
//  cache [pages][Hkv][2][16][D/4]  K codes, then V codes (1024 B at D = 128)
//  kmeta fp16 [pages][Hkv][2][D]   K per-channel s, then z (512 B)
//  tmeta fp16 [pages][Hkv][3][16]  K token norms, V s, V z (96 B)
//
// Decode: split-K over pages, each warp streaming its own pages through a
// cp.async ring. QK on the tensor cores (mma.m16n8k16 f16) by bit planes of
// the codes: A = b0 * s_c, then b1 * (2 s_c), for 16 tokens (each entry s_c
// or 0, exact in fp16), B = q~ as fp16 hi + lo columns (query head, hi/lo),
// built once per CTA; sum_c q~_c z_c comes from one more MMA whose A holds z
// in row 0; logit_t = n_t (dot + sum_c q~_c z_c). PV with the V codes of two
// tokens paired per channel, each 2-bit code moved to its own byte and read
// as e4m3 (exactly code * 2^-9), against p * s_t as hi + lo. The splits'
// partial results go to the workspace; a second kernel (programmatic
// dependent launch) merges them, rotates back and stores.
#pragma once

#include "kvq_decode.cuh"

namespace kvq {

// ----------------------------------------------------------------------------
// write
// ----------------------------------------------------------------------------
struct OscarWriteParams {
  const uint16_t* k;        // bf16 [P * 16][Hkv][D]: token group g = rows 16 g .. 16 g + 15
  const uint16_t* v;
  const int32_t* page_ids;  // [P]
  uint8_t* cache;
  uint16_t* kmeta;
  uint16_t* tmeta;
  int P, Hkv, num_pages;
  float cb;                 // fp32(1/sqrt(b)), 1 for b = 0
};

constexpr int kOscarWriteWarps = 4;

// Shared memory of one write warp: the 16 K and 16 V rows of its (group,
// head) unit as bf16, each row padded by 16 bytes so that the eight row
// addresses of an ldmatrix fall on distinct banks; then per-channel minimum
// and maximum scratch for 64 channels, [8][72] floats each (a row stride of
// 288 bytes keeps the float2 stores of one instruction within two
// wavefronts). 13 KB a warp: four 4-warp CTAs fit on an SM.
struct OscarWriteSmem {
  static constexpr int kRowBytes = 2 * 128 + 16;
  static constexpr int kRows = 32 * kRowBytes;
  static constexpr int kStatStride = 72;
  static constexpr int kStats = 2 * 8 * kStatStride * 4;
  static constexpr int kWarp = kRows + kStats;
  static constexpr int kTotal = kOscarWriteWarps * kWarp;
};

// INT2 (s, z) of a range: z = RD16(mn); s = the smallest fp16 with
// 3 s + z >= mx. need = RU(RU(mx - z) * RU(1/3)) is at least (mx - z) / 3 and
// within a few fp32 ulps of it, so RU16(need) is the answer or one fp16 step
// above it. The step below, pb, is tested exactly in fp32: 3 pb is exact,
// and 3 pb >= mx - z holds exactly when 3 pb >= RU(mx - z) (no fp32 value
// lies strictly between the rounded-down and rounded-up difference).
__device__ __forceinline__ void int2_scale_zero(float mn, float mx, unsigned short& sb, unsigned short& zb,
                                                float& sf, float& zf) {
  const __half zh = __float2half_rd(mn);
  zf = __half2float(zh);
  const float d = __fsub_ru(mx, zf);
  const float need = __fmul_ru(d, 0.333333343f);  // RU(1/3)
  unsigned short s = __half_as_ushort(__float2half_ru(need));
  if (s != 0 && s < 0x7C00) {
    const unsigned short pb = (unsigned short)(s - 1);
    if (__fmul_rn(3.0f, __half2float(__ushort_as_half(pb))) >= d) s = pb;
  }
  sb = s;
  zb = __half_as_ushort(zh);
  sf = __half2float(__ushort_as_half(s));
}

// Bytes 0 of four words, in order, as one word.
__device__ __forceinline__ uint32_t gather_low_bytes(uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  return prmt(prmt(a, b, 0x0040u), prmt(c, d, 0x0040u), 0x5410u);
}

// Two codes rint(fp32(u - z) * fp32(1/s)) (ties to even) as a nibble in
// bits 0-3 of the result (the first code in bits 0-1; the bits above are not
// cleared). Adding 2^23 inside one fma rounds the exact product to an
// integer c in the low mantissa bits of 2^23 + c. No clamp is needed: z <= u
// gives c >= 0, and u - z <= 3 s exactly, so fp32(u - z) * fp32(1/s) <=
// 3 (1 + 2^-24) gives c <= 3 (s = 0 has 1/s read as 0, c = 0).
__device__ __forceinline__ uint32_t int2_code_pair(uint64_t u2, uint64_t z2, uint64_t inv2) {
  const uint64_t r = f2_fma(f2_sub(u2, z2), inv2, f2_pack(8388608.0f, 8388608.0f));
  float r0, r1;
  f2_unpack(r, r0, r1);
  return (__float_as_uint(r1) << 2) + __float_as_uint(r0);
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}

// D = A * B, bf16 operands, fp32 accumulator starting at zero.
__device__ __forceinline__ void mma_bf16_16816_z(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  const float z = 0.0f;
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%10,%10,%10,%10};\n"
      : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1), "f"(z));
}

// Rotate the 16 staged rows at `rows` (bf16, kRowBytes apart) of one warp:
// R x = H_b x / sqrt(b) as H_b = H_{b/16} (x) H_16 (Sylvester order, channel
// 16 G + j). The tensor cores apply H_16 to every 16-channel group (exact
// products, fp32 sums); a butterfly over the groups applies H_{b/16}; b = 0
// multiplies by the identity. Result y[G][nt][t]: channels 16 G + 8 nt +
// 2 tig + {0, 1} (an f32x2 pair) of token g (t = 0) or g + 8 (t = 1).
template <int BLK>
__device__ __forceinline__ void oscar_rotate_rows(uint32_t rows, const uint32_t (&hb)[2][2], float cb,
                                                  uint64_t (&y)[8][2][2]) {
  const int lane = threadIdx.x & 31;
  const uint32_t a_row = rows + ((lane & 7) + ((lane >> 3) & 1) * 8) * OscarWriteSmem::kRowBytes +
                         (lane >> 4) * 16;
#pragma unroll
  for (int G = 0; G < 8; ++G) {
    uint32_t a[4];
    ldsm_x4(a_row + G * 32, a);
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
      float d[4];
      mma_bf16_16816_z(d, a, hb[nt][0], hb[nt][1]);
      y[G][nt][0] = f2_pack(d[0], d[1]);
      y[G][nt][1] = f2_pack(d[2], d[3]);
    }
  }
  if constexpr (BLK >= 32) {
#pragma unroll
    for (int st = 1; st < BLK / 16; st <<= 1)
#pragma unroll
      for (int G = 0; G < 8; ++G)
        if (!(G & st))
#pragma unroll
          for (int nt = 0; nt < 2; ++nt)
#pragma unroll
            for (int t = 0; t < 2; ++t) {
              const uint64_t a = y[G][nt][t], b = y[G + st][nt][t];
              y[G][nt][t] = f2_add(a, b);
              y[G + st][nt][t] = f2_sub(a, b);
            }
    const uint64_t c2 = f2_pack(cb, cb);
#pragma unroll
    for (int G = 0; G < 8; ++G)
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) {
        y[G][nt][0] = f2_mul(y[G][nt][0], c2);
        y[G][nt][1] = f2_mul(y[G][nt][1], c2);
      }
  }
}

// Pack the nibbles of a warp's 16 x 128 codes and store the page's 512
// bytes, one 16-byte store per lane. nib[t][q] byte i holds the nibble of
// (token g or g + 8, k = 4 q + i) where k = 2 G + nt: channels 8 k + 2 tig,
// + 1. Code byte m of a row covers channels 4 m .. 4 m + 3, so byte
// m = 2 k + (tig >> 1) pairs the nibbles of lanes tig = 2 (tig >> 1) (low)
// and + 1 (high).
__device__ __forceinline__ void oscar_store_codes(const uint32_t (&nib)[2][4], uint8_t* dst, bool ok) {
  const int lane = threadIdx.x & 31, g = lane >> 2, tig = lane & 3;
  const bool odd = tig & 1, hi = tig & 2;
  uint32_t b[4];
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    // even lanes assemble token g, odd lanes token g + 8
    const uint32_t r = __shfl_xor_sync(0xffffffffu, odd ? nib[0][q] : nib[1][q], 1);
    const uint32_t mine = odd ? nib[1][q] : nib[0][q];
    b[q] = odd ? (r | (mine << 4)) : (mine | (r << 4));
  }
  // b[q] byte i = byte 8 q + 2 i + (tig >> 1) of the row; lanes tig and
  // tig ^ 2 hold the even and odd bytes: the first stores bytes 0..15, the
  // second 16..31
  const uint32_t r0 = __shfl_xor_sync(0xffffffffu, hi ? b[0] : b[2], 2);
  const uint32_t r1 = __shfl_xor_sync(0xffffffffu, hi ? b[1] : b[3], 2);
  const uint32_t e0 = hi ? r0 : b[0], e1 = hi ? r1 : b[1];
  const uint32_t o0 = hi ? b[2] : r0, o1 = hi ? b[3] : r1;
  const uint4 w = make_uint4(prmt(e0, o0, 0x5140), prmt(e0, o0, 0x7362), prmt(e1, o1, 0x5140),
                             prmt(e1, o1, 0x7362));
  const int row = g + (odd ? 8 : 0);
  if (ok) *reinterpret_cast<uint4*>(dst + row * 32 + (hi ? 16 : 0)) = w;
}

// Persistent: each warp takes (group, head) units unit0, unit0 + stride, ...
// The next unit's K rows are fetched while this unit's K is quantized, its V
// rows while this unit's V is.
template <int D, int BLK>
__global__ void __launch_bounds__(kOscarWriteWarps * 32, 4) kvq_oscar_write_kernel(const OscarWriteParams p) {
  static_assert(D == 128, "the OScaR path is built for head_dim 128");
  using SM = OscarWriteSmem;
  extern __shared__ __align__(128) uint8_t smem[];
  pdl_wait();  // the previous kernel may still read the pools or write K, V
  pdl_launch_dependents();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int g = lane >> 2, tig = lane & 3;
  const unsigned FULL = 0xffffffffu;
  uint8_t* ws = smem + warp * SM::kWarp;
  const uint32_t rows_s = smem_addr(ws);
  float* smin = reinterpret_cast<float*>(ws + SM::kRows);
  float* smax = smin + 8 * SM::kStatStride;
  const int units = p.P * p.Hkv;
  const int stride = gridDim.x * kOscarWriteWarps;
  const size_t row_stride = (size_t)p.Hkv * D;

  // (group, head) of a unit, and of the unit one grid stride later, without
  // a division per unit: unit = grp * Hkv + h
  const int sg = stride / p.Hkv, sh = stride - sg * p.Hkv;
  auto advance = [&](int& grp, int& h) {
    grp += sg;
    h += sh;
    if (h >= p.Hkv) {
      h -= p.Hkv;
      ++grp;
    }
  };
  // one matrix (0: K, 1: V) of a unit: 16 rows of 256 bytes, 8 chunks a lane
  auto stage = [&](int unit, int grp, int h, int which) {
    if (unit < units) {
      const uint16_t* src = (which ? p.v : p.k) + ((size_t)grp * 16 * p.Hkv + h) * D;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int c = lane + 32 * j, r = c >> 4, ch = c & 15;
        cp_async_16(rows_s + (which * 16 + r) * SM::kRowBytes + 16 * ch, src + r * row_stride + 8 * ch);
      }
    }
    cp_async_commit();
  };

  // H_16 (or the identity) as B fragments: k rows 2 tig, + 1 (b0) and
  // 2 tig + 8, + 9 (b1) of column n = 8 nt + g
  uint32_t hb[2][2];
  {
    auto h = [](int k, int n) -> uint32_t {
      if (BLK == 0) return k == n ? 0x3F80u : 0u;
      return (__popc(k & n) & 1) ? 0xBF80u : 0x3F80u;
    };
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
      const int n = 8 * nt + g;
      hb[nt][0] = h(2 * tig, n) | (h(2 * tig + 1, n) << 16);
      hb[nt][1] = h(2 * tig + 8, n) | (h(2 * tig + 9, n) << 16);
    }
  }

  int unit = blockIdx.x * kOscarWriteWarps + warp;
  int grp = unit / p.Hkv, h = unit - grp * p.Hkv;
  stage(unit, grp, h, 0);
  stage(unit, grp, h, 1);
  for (; unit < units; unit += stride, advance(grp, h)) {
    int ngrp = grp, nh = h;  // the next unit's
    advance(ngrp, nh);
    const int page = p.page_ids[grp];
    const bool ok = page >= 0 && page < p.num_pages;
    if (!ok && lane == 0) record_error(KVQ_ERR_OUT_OF_RANGE);
    const size_t ph = (size_t)(ok ? page : 0) * p.Hkv + h;
    uint8_t* kc = p.cache + (ph * 2 + 0) * 16 * (D / 4);
    uint8_t* vc = p.cache + (ph * 2 + 1) * 16 * (D / 4);
    uint16_t* kmeta = p.kmeta + ph * 2 * D;
    uint16_t* tm = p.tmeta + ph * 3 * 16;

    // ---- K: rotate, scale each token by S = fp32(1/n), per-channel INT2 ----
    cp_async_wait<1>();
    __syncwarp();
    uint64_t y[8][2][2];
    oscar_rotate_rows<BLK>(rows_s, hb, p.cb, y);
    __syncwarp();
    stage(unit + stride, ngrp, nh, 0);
    // token norms: an fp32 sum of the squares (no path through its tree has
    // more than 9 roundings, so ||y||^2 is within 2^-20.8 relative and n
    // within 2^-21.5); when n (1 -+ 2^-19) round to different fp16 values
    // for any token of the warp, the warp sums again in fp64, where the
    // squares of fp32 values are exact
    unsigned short nb[2];
    {
      float sq[2];
#pragma unroll
      for (int t = 0; t < 2; ++t) {
        uint64_t acc[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
        for (int G = 0; G < 8; ++G)
#pragma unroll
          for (int nt = 0; nt < 2; ++nt) acc[(2 * G + nt) & 3] = f2_fma(y[G][nt][t], y[G][nt][t], acc[(2 * G + nt) & 3]);
        const uint64_t a2 = f2_add(f2_add(acc[0], acc[1]), f2_add(acc[2], acc[3]));
        float lo, hi;
        f2_unpack(a2, lo, hi);
        sq[t] = lo + hi;
        sq[t] += __shfl_xor_sync(FULL, sq[t], 1);
        sq[t] += __shfl_xor_sync(FULL, sq[t], 2);
      }
      bool unsure = false;
#pragma unroll
      for (int t = 0; t < 2; ++t) {
        const float n32 = __fsqrt_rn(sq[t]);
        nb[t] = __half_as_ushort(__float2half_rn(n32));
        unsure |= __half_as_ushort(__float2half_rn(n32 * (1.0f - 0x1p-19f))) !=
                  __half_as_ushort(__float2half_rn(n32 * (1.0f + 0x1p-19f)));
      }
      if (__any_sync(FULL, unsure)) {
#pragma unroll
        for (int t = 0; t < 2; ++t) {
          double ss = 0.0;
#pragma unroll
          for (int G = 0; G < 8; ++G)
#pragma unroll
            for (int nt = 0; nt < 2; ++nt) {
              float a, b;
              f2_unpack(y[G][nt][t], a, b);
              ss = fma((double)a, (double)a, fma((double)b, (double)b, ss));
            }
          ss += __shfl_xor_sync(FULL, ss, 1);
          ss += __shfl_xor_sync(FULL, ss, 2);
          nb[t] = __half_as_ushort(__double2half(sqrt(ss)));
        }
      }
    }
#pragma unroll
    for (int t = 0; t < 2; ++t) {
      if ((nb[t] & 0x7FFF) >= 0x7C00) nb[t] = 0x7BFF;  // saturate at the largest finite fp16
      const float nf = __half2float(__ushort_as_half(nb[t]));
      const float S = nf > 0.0f ? __frcp_rn(nf) : 0.0f;
      const uint64_t s2 = f2_pack(S, S);
#pragma unroll
      for (int G = 0; G < 8; ++G)
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) y[G][nt][t] = f2_mul(y[G][nt][t], s2);
    }
    if (ok && tig == 0) {
      tm[g] = nb[0];
      tm[g + 8] = nb[1];
    }
    // per-channel min / max over the 16 tokens: tokens g, g + 8 here, then
    // the 8 lanes of each tig through shared memory, 64 channels (groups
    // 4 hc .. 4 hc + 3) at a time
    uint32_t nib[2][4] = {{0u, 0u, 0u, 0u}, {0u, 0u, 0u, 0u}};
#pragma unroll
    for (int hc = 0; hc < 2; ++hc) {
#pragma unroll
      for (int G = 4 * hc; G < 4 * hc + 4; ++G)
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
          float a0, a1, c0, c1;
          f2_unpack(y[G][nt][0], a0, a1);
          f2_unpack(y[G][nt][1], c0, c1);
          const int ch = 16 * (G - 4 * hc) + 8 * nt + 2 * tig;
          *reinterpret_cast<float2*>(smin + g * SM::kStatStride + ch) = make_float2(fminf(a0, c0), fminf(a1, c1));
          *reinterpret_cast<float2*>(smax + g * SM::kStatStride + ch) = make_float2(fmaxf(a0, c0), fmaxf(a1, c1));
        }
      __syncwarp();
      {
        float2 mn = *reinterpret_cast<const float2*>(smin + 2 * lane);
        float2 mx = *reinterpret_cast<const float2*>(smax + 2 * lane);
#pragma unroll
        for (int r = 1; r < 8; ++r) {
          const float2 a = *reinterpret_cast<const float2*>(smin + r * SM::kStatStride + 2 * lane);
          const float2 b = *reinterpret_cast<const float2*>(smax + r * SM::kStatStride + 2 * lane);
          mn = make_float2(fminf(mn.x, a.x), fminf(mn.y, a.y));
          mx = make_float2(fmaxf(mx.x, b.x), fmaxf(mx.y, b.y));
        }
        unsigned short sb0, zb0, sb1, zb1;
        float sf0, sf1, zf0, zf1;
        int2_scale_zero(mn.x, mx.x, sb0, zb0, sf0, zf0);
        int2_scale_zero(mn.y, mx.y, sb1, zb1, sf1, zf1);
        if (ok) {
          *reinterpret_cast<uint32_t*>(kmeta + 64 * hc + 2 * lane) = sb0 | ((uint32_t)sb1 << 16);
          *reinterpret_cast<uint32_t*>(kmeta + D + 64 * hc + 2 * lane) = zb0 | ((uint32_t)zb1 << 16);
        }
        // this lane's columns of row 0 now hold z and 1/s
        *reinterpret_cast<float2*>(smin + 2 * lane) = make_float2(zf0, zf1);
        *reinterpret_cast<float2*>(smax + 2 * lane) =
            make_float2(sf0 > 0.0f ? __frcp_rn(sf0) : 0.0f, sf1 > 0.0f ? __frcp_rn(sf1) : 0.0f);
      }
      __syncwarp();
      uint32_t pk[2][8];  // [token][k - 8 hc]: a nibble in bits 0-3
#pragma unroll
      for (int G = 4 * hc; G < 4 * hc + 4; ++G)
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
          const int ch = 16 * (G - 4 * hc) + 8 * nt + 2 * tig, k = 2 * (G - 4 * hc) + nt;
          const float2 z = *reinterpret_cast<const float2*>(smin + ch);
          const float2 iv = *reinterpret_cast<const float2*>(smax + ch);
          const uint64_t z2 = f2_pack(z.x, z.y), i2 = f2_pack(iv.x, iv.y);
#pragma unroll
          for (int t = 0; t < 2; ++t) pk[t][k] = int2_code_pair(y[G][nt][t], z2, i2);
        }
#pragma unroll
      for (int t = 0; t < 2; ++t)
#pragma unroll
        for (int q = 0; q < 2; ++q)
          nib[t][2 * hc + q] =
              gather_low_bytes(pk[t][4 * q], pk[t][4 * q + 1], pk[t][4 * q + 2], pk[t][4 * q + 3]) & 0x0F0F0F0Fu;
      __syncwarp();  // row 0 of the scratch is read before it is rewritten
    }
    oscar_store_codes(nib, kc, ok);

    // ---- V: rotate, token-wise INT2 ------------------------------------------
    cp_async_wait<1>();
    __syncwarp();
    oscar_rotate_rows<BLK>(rows_s + 16 * SM::kRowBytes, hb, p.cb, y);
    __syncwarp();
    stage(unit + stride, ngrp, nh, 1);
    {
      float mn[2], mx[2];
#pragma unroll
      for (int t = 0; t < 2; ++t) {
        float a, b;
        f2_unpack(y[0][0][t], a, b);
        mn[t] = fminf(a, b);
        mx[t] = fmaxf(a, b);
#pragma unroll
        for (int G = 0; G < 8; ++G)
#pragma unroll
          for (int nt = 0; nt < 2; ++nt) {
            f2_unpack(y[G][nt][t], a, b);
            mn[t] = fmin3(mn[t], a, b);
            mx[t] = fmax3(mx[t], a, b);
          }
        mn[t] = fminf(mn[t], __shfl_xor_sync(FULL, mn[t], 1));
        mx[t] = fmaxf(mx[t], __shfl_xor_sync(FULL, mx[t], 1));
        mn[t] = fminf(mn[t], __shfl_xor_sync(FULL, mn[t], 2));
        mx[t] = fmaxf(mx[t], __shfl_xor_sync(FULL, mx[t], 2));
      }
      uint32_t nib[2][4] = {{0u, 0u, 0u, 0u}, {0u, 0u, 0u, 0u}};
#pragma unroll
      for (int t = 0; t < 2; ++t) {
        unsigned short sb, zb;
        float sf, zf;
        int2_scale_zero(mn[t], mx[t], sb, zb, sf, zf);
        const float iv = (sf > 0.0f) ? __frcp_rn(sf) : 0.0f;
        if (ok && tig == 0) {
          tm[16 + g + 8 * t] = sb;
          tm[32 + g + 8 * t] = zb;
        }
        const uint64_t z2 = f2_pack(zf, zf), i2 = f2_pack(iv, iv);
        uint32_t pk[16];  // [k = 2 G + nt]: a nibble in bits 0-3
#pragma unroll
        for (int G = 0; G < 8; ++G)
#pragma unroll
          for (int nt = 0; nt < 2; ++nt) pk[2 * G + nt] = int2_code_pair(y[G][nt][t], z2, i2);
#pragma unroll
        for (int q = 0; q < 4; ++q)
          nib[t][q] = gather_low_bytes(pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]) & 0x0F0F0F0Fu;
      }
      oscar_store_codes(nib, vc, ok);
    }
  }
  cp_async_wait<0>();
}

// ----------------------------------------------------------------------------
// decode
// ----------------------------------------------------------------------------
struct OscarAttnParams {
  const uint16_t* q;          // bf16 [B][Hq][D]
  const uint8_t* cache;
  const uint16_t* kmeta;
  const uint16_t* tmeta;
  const int32_t* page_table;  // [B][max_pages]: the full pages of each sequence
  const int32_t* ctx_lens;    // [B]
  const uint16_t* k_tail;     // bf16 [B][Hkv][16][D]: the unfinished page, rows 0 .. ctx % 16 - 1
  const uint16_t* v_tail;
  float* ws;                  // [B][Hkv][n_splits][G][D + 2]: O + Z, M, L of each split
  void* out;                  // [B][Hq][D] fp32 or bf16
  int B, Hq, Hkv, G;
  int num_pages, max_pages;
  int n_splits, pages_per_split;
  int out_bf16;
  float qmul;                 // c_b * softmax_scale * log2(e)
  float qraw;                 // softmax_scale * log2(e)
  float cb;
};

constexpr int kOscarWarps = 4;
constexpr int kOscarRing = 4;

template <int D>
struct OscarSmem {
  static constexpr int kCodes = 2 * 16 * (D / 4);               // K then V codes
  static constexpr int kSlot = kCodes + 2 * D * 2 + 3 * 16 * 2; // + kmeta + tmeta
  static constexpr int kRing = kOscarWarps * kOscarRing * kSlot;
  // q~ rows: row r, channels 32 j .. 32 j + 31 at float r * kQRow + j * kQSeg;
  // the padding puts the 16 (row, j) float4 reads of one k-step (when the
  // B fragments are built, once per CTA) in 8 distinct 16-byte bank groups
  static constexpr int kQSeg = 36;
  static constexpr int kQRow = 4 * kQSeg;
  static constexpr int kOffQ = kRing;
  static constexpr int kRes = 4 * (D + 4);                      // floats per state: [4 rows][D + 4]
  static constexpr int kOffRes = kOffQ + 4 * kQRow * 4;         // states: the warps', then the tail's
  static constexpr int kTotal = kOffRes + (kOscarWarps + 1) * kRes * 4;
};

// Four bytes read as e4m3 -> two f16x2 registers (bytes 0, 1 and 2, 3). A
// byte holding a 2-bit code c (bits 0-1, the rest zero) is the e4m3
// subnormal c * 2^-9, which fp16 holds exactly.
__device__ __forceinline__ void e4m3x2_to_f16x2(uint32_t x, uint32_t& lo, uint32_t& hi) {
  asm("{\n .reg .b16 a, b;\n mov.b32 {a, b}, %2;\n cvt.rn.f16x2.e4m3x2 %0, a;\n"
      " cvt.rn.f16x2.e4m3x2 %1, b;\n}\n"
      : "=r"(lo), "=r"(hi)
      : "r"(x));
}

template <int D, int BLK>
__global__ void __launch_bounds__(kOscarWarps * 32) kvq_oscar_decode_kernel(const __grid_constant__ OscarAttnParams p) {
  static_assert(D == 128, "the OScaR path is built for head_dim 128");
  using S = OscarSmem<D>;
  constexpr int R = kOscarRing;
  constexpr int SLOT = S::kSlot;
  constexpr int NJ = D / 16;   // QK k-steps and PV m-tiles
  constexpr int E = D / 32;
  extern __shared__ __align__(128) uint8_t smem[];
  float* qs = reinterpret_cast<float*>(smem + S::kOffQ);
  float* res = reinterpret_cast<float*>(smem + S::kOffRes);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2, tig = lane & 3;
  const int split = blockIdx.x, h = blockIdx.y, n = blockIdx.z;
  const int G = p.G;
  const unsigned FULL = 0xffffffffu;

  pdl_wait();  // the pools may be what the previous kernel wrote
  pdl_launch_dependents();

  int ctx = p.ctx_lens[n];
  const int cap = p.max_pages * 16 + 15;
  if (ctx < 0 || ctx > cap) {
    if (tid == 0) record_error(KVQ_ERR_OUT_OF_RANGE);
    ctx = ctx < 0 ? 0 : cap;
  }
  const int n_full = ctx >> 4, tail = ctx & 15;
  const int p0 = split * p.pages_per_split;
  const int p1 = min(p0 + p.pages_per_split, n_full);
  // a split past the sequence's pages (and not holding its unfinished page)
  // has nothing to add; the merge kernel does not read its workspace rows
  if (p0 >= n_full && !(split == 0 && tail > 0)) return;

  // q~ = R q * qmul for the G query heads of kv head h (rows >= G zero)
  for (int r = warp; r < 4; r += kOscarWarps) {
    float v[E] = {0.0f, 0.0f, 0.0f, 0.0f};
    if (r < G) {
      const uint2 w = *reinterpret_cast<const uint2*>(p.q + ((size_t)n * p.Hq + (size_t)h * G + r) * D + E * lane);
      v[0] = __uint_as_float(w.x << 16);
      v[1] = __uint_as_float(w.x & 0xffff0000u);
      v[2] = __uint_as_float(w.y << 16);
      v[3] = __uint_as_float(w.y & 0xffff0000u);
      if constexpr (BLK > 0) warp_fwht<D, BLK>(v, lane);
#pragma unroll
      for (int e = 0; e < E; ++e) v[e] *= p.qmul;
    }
    *reinterpret_cast<float4*>(qs + r * S::kQRow + (lane >> 3) * S::kQSeg + E * (lane & 7)) =
        make_float4(v[0], v[1], v[2], v[3]);
  }
  __syncthreads();

  // ---- this warp's pages p0 + warp, p0 + warp + 4, ... ----------------------
  uint8_t* ring = smem + warp * (R * SLOT);
  const uint32_t ring_s = smem_addr(ring);
  uint32_t valid = 0;
  int ids = -1;  // page ids of this warp's pages 32 c .. 32 c + 31 (lane i: page 32 c + i)
  auto fetch = [&](int k) {
    if ((k & 31) == 0) {
      const int pl = p0 + warp + (k + lane) * kOscarWarps;
      ids = pl < p1 ? p.page_table[(size_t)n * p.max_pages + pl] : -1;
    }
    const int id = __shfl_sync(FULL, ids, k & 31);
    const int pg = p0 + warp + k * kOscarWarps;
    const int slot = k % R;
    bool ok = false;
    if (pg < p1) {
      ok = id >= 0 && id < p.num_pages;
      if (ok) {
        const size_t ph = (size_t)id * p.Hkv + h;
        const uint8_t* cs = p.cache + ph * S::kCodes;
        const uint8_t* ms = reinterpret_cast<const uint8_t*>(p.kmeta + ph * 2 * D);
        const uint8_t* ts = reinterpret_cast<const uint8_t*>(p.tmeta + ph * 3 * 16);
        const uint32_t dst = ring_s + slot * SLOT;
        cp_async_16(dst + 16 * lane, cs + 16 * lane);
        cp_async_16(dst + 512 + 16 * lane, cs + 512 + 16 * lane);
        cp_async_16(dst + S::kCodes + 16 * lane, ms + 16 * lane);
        cp_async_16_if(dst + S::kCodes + 4 * D + 16 * (lane < 6 ? lane : 0), ts + 16 * (lane < 6 ? lane : 0),
                       lane < 6);
      } else if (lane == 0) {
        record_error(KVQ_ERR_OUT_OF_RANGE);
      }
    }
    valid = ok ? (valid | (1u << slot)) : (valid & ~(1u << slot));
    cp_async_commit();
  };

  float o[NJ][4];
#pragma unroll
  for (int i = 0; i < NJ; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.0f;
  const bool hv = tig < G;                 // this thread's logits belong to query head tig
  float m_run = hv ? -INFINITY : 0.0f, l_run = 0.0f, zs_run = 0.0f;
  const int hd = g >> 1, part = g & 1;     // this thread's B column: head hd, hi (0) or lo (1)
  const int la = 8 * tig + (g >> 1), lb = la + 4;
  // B = q~ of head hd as fp16 hi or lo, the same for every page: k-step j
  // covers channels 32 tig + 4 j .. + 3 (rows 2 tig, + 1 -> channels + 0,
  // + 1; rows 2 tig + 8, + 9 -> + 2, + 3)
  uint32_t bq0[NJ], bq1[NJ];
  {
    const float* qrow = qs + hd * S::kQRow + tig * S::kQSeg;
#pragma unroll
    for (int j = 0; j < NJ; ++j) {
      const float4 qv = *reinterpret_cast<const float4*>(qrow + 4 * j);
      bq0[j] = hilo_pair(qv.x, qv.y, part);
      bq1[j] = hilo_pair(qv.z, qv.w, part);
    }
  }

#pragma unroll
  for (int k = 0; k < R - 1; ++k) fetch(k);
  for (int k = 0; p0 + warp + k * kOscarWarps < p1; ++k) {
    fetch(k + R - 1);
    cp_async_wait<R - 1>();
    __syncwarp();
    if ((valid >> (k % R)) & 1u) {
      const uint8_t* pg = ring + (k % R) * SLOT;
      const uint8_t* kcode = pg;
      const uint8_t* vcode = pg + 16 * (D / 4);
      const __half* ksc = reinterpret_cast<const __half*>(pg + S::kCodes);
      const __half* kze = ksc + D;
      const __half* kno = reinterpret_cast<const __half*>(pg + S::kCodes + 4 * D);
      const __half* vsc = kno + 16;
      const __half* vze = kno + 32;

      // QK by bit planes, code = b0 + 2 b1: A = b0 s_c, then b1 (2 s_c), both
      // exact in fp16 (a select of s_c or 0). The bits of tokens g and g + 8
      // come from K code bytes 8 tig .. 8 tig + 7 (byte 8 tig + j: k-step j,
      // channels 32 tig + 4 j + c' at bits 2 c', 2 c' + 1); each shifted copy
      // of a code word brings one bit position of every byte to bit 7, which
      // prmt (in its sign mode) replicates across a half. sum_c q~_c z_c: an
      // extra MMA whose A holds z in row 0 only.
      const uint2 ra = *reinterpret_cast<const uint2*>(kcode + g * (D / 4) + 8 * tig);
      const uint2 rc = *reinterpret_cast<const uint2*>(kcode + (g + 8) * (D / 4) + 8 * tig);
      float acc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
      float zacc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        const uint32_t xa = half ? ra.y : ra.x, xc = half ? rc.y : rc.x;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int j = 4 * half + i;
          // output bytes 0, 1 <- bit 7 of byte i of the first word, 2, 3 <- of the second
          const uint32_t sel = (8u + i) | ((8u + i) << 4) | ((12u + i) << 8) | ((12u + i) << 12);
          const uint2 sw = *reinterpret_cast<const uint2*>(ksc + 32 * tig + 4 * j);
          const uint2 zw = *reinterpret_cast<const uint2*>(kze + 32 * tig + 4 * j);
          uint32_t s2x, s2y;
          asm("add.rn.f16x2 %0, %1, %1;\n" : "=r"(s2x) : "r"(sw.x));
          asm("add.rn.f16x2 %0, %1, %1;\n" : "=r"(s2y) : "r"(sw.y));
          const uint32_t a0[4] = {prmt(xa << 7, xa << 5, sel) & sw.x, prmt(xc << 7, xc << 5, sel) & sw.x,
                                  prmt(xa << 3, xa << 1, sel) & sw.y, prmt(xc << 3, xc << 1, sel) & sw.y};
          mma_f16_16816(acc, a0, bq0[j], bq1[j]);
          const uint32_t a1[4] = {prmt(xa << 6, xa << 4, sel) & s2x, prmt(xc << 6, xc << 4, sel) & s2x,
                                  prmt(xa << 2, xa, sel) & s2y, prmt(xc << 2, xc, sel) & s2y};
          mma_f16_16816(acc, a1, bq0[j], bq1[j]);
          const uint32_t az[4] = {g == 0 ? zw.x : 0u, 0u, g == 0 ? zw.y : 0u, 0u};
          mma_f16_16816(zacc, az, bq0[j], bq1[j]);
        }
      }
      const float zsum = __shfl_sync(FULL, zacc[0] + zacc[1], tig);  // row 0 = lane tig: head tig

      // logits (base 2) of tokens g and g + 8 for query head tig
      const float n0 = __half2float(kno[g]), n1 = __half2float(kno[g + 8]);
      float lg0 = n0 * (acc[0] + acc[1] + zsum);
      float lg1 = n1 * (acc[2] + acc[3] + zsum);
      if (!hv) lg0 = lg1 = -INFINITY;
      const float sv0 = __half2float(vsc[g]), sv1 = __half2float(vsc[g + 8]);
      const float zv0 = __half2float(vze[g]), zv1 = __half2float(vze[g + 8]);
      // lazy online softmax (as in the INT4 decode)
      const bool sv_big = fmaxf(sv0, sv1) > kBigScale;
      const bool need = (lg0 > m_run + kHead) || (lg1 > m_run + kHead) || sv_big;
      if (__any_sync(FULL, need)) {
        float pm = fmaxf(lg0, lg1);
        pm = fmaxf(pm, __shfl_xor_sync(FULL, pm, 4));
        pm = fmaxf(pm, __shfl_xor_sync(FULL, pm, 8));
        pm = fmaxf(pm, __shfl_xor_sync(FULL, pm, 16));
        const bool big = __any_sync(FULL, sv_big);
        const float mn = (pm > m_run + kHead || (big && pm > m_run)) ? pm : m_run;
        const float alpha = fast_exp2(m_run - mn);
#pragma unroll
        for (int i = 0; i < NJ; ++i) {
          o[i][0] *= alpha; o[i][1] *= alpha; o[i][2] *= alpha; o[i][3] *= alpha;
        }
        l_run *= alpha;
        zs_run *= alpha;
        m_run = mn;
      }
      const float pr0 = fast_exp2(lg0 - m_run), pr1 = fast_exp2(lg1 - m_run);
      l_run += pr0 + pr1;
      zs_run = fmaf(pr0, zv0, fmaf(pr1, zv1, zs_run));
      const float P0 = pr0 * sv0, P1 = pr1 * sv1;
      const float q0 = __shfl_sync(FULL, P0, la), q1 = __shfl_sync(FULL, P0, lb);
      const float q2 = __shfl_sync(FULL, P1, la), q3 = __shfl_sync(FULL, P1, lb);
      const uint32_t bp0 = hilo_pair(q0, q1, part), bp1 = hilo_pair(q2, q3, part);

      // PV: A = V codes^T. Rows g / g + 8 of m-tile i are channels
      // 16 g + 2 i / 16 g + 2 i + 1, k-slots the tokens 2 tig, 2 tig + 1,
      // 2 tig + 8, 2 tig + 9; each token's word holds bytes 4 g .. 4 g + 3
      const uint32_t va = *reinterpret_cast<const uint32_t*>(vcode + (2 * tig) * (D / 4) + 4 * g);
      const uint32_t vb = *reinterpret_cast<const uint32_t*>(vcode + (2 * tig + 1) * (D / 4) + 4 * g);
      const uint32_t vcw = *reinterpret_cast<const uint32_t*>(vcode + (2 * tig + 8) * (D / 4) + 4 * g);
      const uint32_t vd = *reinterpret_cast<const uint32_t*>(vcode + (2 * tig + 9) * (D / 4) + 4 * g);
#pragma unroll
      for (int hb = 0; hb < 2; ++hb) {
        // bytes 2 hb, 2 hb + 1 of the four tokens: channels 16 g + 8 hb .. + 7
        const uint32_t x = prmt(va, vb, hb ? 0x7362 : 0x5140);
        const uint32_t y = prmt(vcw, vd, hb ? 0x7362 : 0x5140);
        uint32_t xl[4], xh[4], yl[4], yh[4];  // [code k]: low half = byte 2 hb, high = byte 2 hb + 1
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          e4m3x2_to_f16x2((x >> (2 * c)) & 0x03030303u, xl[c], xh[c]);
          e4m3x2_to_f16x2((y >> (2 * c)) & 0x03030303u, yl[c], yh[c]);
        }
        // m-tile i = 4 hb + 2 q + r2 covers channels 16 g + 8 hb + 4 q + 2 r2 + {0, 1}:
        // byte q (0 low half, 1 high half), codes 2 r2 and 2 r2 + 1
#pragma unroll
        for (int qb = 0; qb < 2; ++qb)
#pragma unroll
          for (int r2 = 0; r2 < 2; ++r2) {
            const int i = 4 * hb + 2 * qb + r2;
            const uint32_t a[4] = {qb ? xh[2 * r2] : xl[2 * r2], qb ? xh[2 * r2 + 1] : xl[2 * r2 + 1],
                                   qb ? yh[2 * r2] : yl[2 * r2], qb ? yh[2 * r2 + 1] : yl[2 * r2 + 1]};
            mma_f16_16816(o[i], a, bp0, bp1);
          }
      }
    }
    __syncwarp();  // the slot is read out before a later fetch refills it
  }
  cp_async_wait<0>();

  // ---- per-warp state: O[head][channel], then (m, l, zs) ----------------------
#pragma unroll
  for (int o2 = 4; o2 < 32; o2 <<= 1) {
    l_run += __shfl_xor_sync(FULL, l_run, o2);
    zs_run += __shfl_xor_sync(FULL, zs_run, o2);
  }
  {
    float* mine = res + warp * S::kRes + tig * (D + 4);
#pragma unroll
    for (int i = 0; i < NJ; ++i) {
      mine[16 * g + 2 * i] = (o[i][0] + o[i][1]) * 512.0f;
      mine[16 * g + 2 * i + 1] = (o[i][2] + o[i][3]) * 512.0f;
    }
    if (g == 0) {
      mine[D] = m_run;
      mine[D + 1] = l_run;
      mine[D + 2] = zs_run;
    }
  }
  // ---- the unfinished page (split 0, warp 0): bf16 rows as they are -------
  // q . k = (R q) . (R k), so the logits take the unrotated q and k; the
  // weighted sum of the unrotated v is rotated once at the end.
  const bool has_tail = split == 0 && tail > 0;
  if (has_tail && warp == 0) {
    float mt[4], lt[4], ot[4][E], qr[4][E];
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      mt[r] = -INFINITY;
      lt[r] = 0.0f;
      const int rr = r < G ? r : 0;
      const uint2 w = *reinterpret_cast<const uint2*>(p.q + ((size_t)n * p.Hq + (size_t)h * G + rr) * D + E * lane);
      qr[r][0] = __uint_as_float(w.x << 16) * p.qraw;
      qr[r][1] = __uint_as_float(w.x & 0xffff0000u) * p.qraw;
      qr[r][2] = __uint_as_float(w.y << 16) * p.qraw;
      qr[r][3] = __uint_as_float(w.y & 0xffff0000u) * p.qraw;
#pragma unroll
      for (int e = 0; e < E; ++e) ot[r][e] = 0.0f;
    }
    const size_t base = ((size_t)n * p.Hkv + h) * 16 * D + E * lane;
    for (int t = 0; t < tail; ++t) {
      float kr[E], vr[E];
      const uint2 kw = *reinterpret_cast<const uint2*>(p.k_tail + base + (size_t)t * D);
      const uint2 vw = *reinterpret_cast<const uint2*>(p.v_tail + base + (size_t)t * D);
      kr[0] = __uint_as_float(kw.x << 16); kr[1] = __uint_as_float(kw.x & 0xffff0000u);
      kr[2] = __uint_as_float(kw.y << 16); kr[3] = __uint_as_float(kw.y & 0xffff0000u);
      vr[0] = __uint_as_float(vw.x << 16); vr[1] = __uint_as_float(vw.x & 0xffff0000u);
      vr[2] = __uint_as_float(vw.y << 16); vr[3] = __uint_as_float(vw.y & 0xffff0000u);
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        float d = 0.0f;
#pragma unroll
        for (int e = 0; e < E; ++e) d = fmaf(qr[r][e], kr[e], d);
#pragma unroll
        for (int o2 = 16; o2 > 0; o2 >>= 1) d += __shfl_xor_sync(FULL, d, o2);
        const float mn = fmaxf(mt[r], d);
        const float a = fast_exp2(mt[r] - mn), pw = fast_exp2(d - mn);
        lt[r] = fmaf(lt[r], a, pw);
#pragma unroll
        for (int e = 0; e < E; ++e) ot[r][e] = fmaf(ot[r][e], a, pw * vr[e]);
        mt[r] = mn;
      }
    }
    if constexpr (BLK > 0) {
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        warp_fwht<D, BLK>(ot[r], lane);
#pragma unroll
        for (int e = 0; e < E; ++e) ot[r][e] *= p.cb;
      }
    }
    float* st = res + kOscarWarps * S::kRes;
#pragma unroll
    for (int r = 0; r < 4; ++r) {
#pragma unroll
      for (int e = 0; e < E; ++e) st[r * (D + 4) + E * lane + e] = ot[r][e];
      if (lane == 0) {
        st[r * (D + 4) + D] = mt[r];
        st[r * (D + 4) + D + 1] = lt[r];
        st[r * (D + 4) + D + 2] = 0.0f;
      }
    }
  }
  __syncthreads();

  // ---- merge the warps (and the unfinished page) into the split's result -----
  const int nstates = kOscarWarps + (has_tail ? 1 : 0);
  for (int e = tid; e < G * (D / 4); e += kOscarWarps * 32) {
    const int r = e / (D / 4), c4 = 4 * (e % (D / 4));
    float M = -INFINITY;
    for (int s2 = 0; s2 < nstates; ++s2) M = fmaxf(M, res[s2 * S::kRes + r * (D + 4) + D]);
    float4 O = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
    float L = 0.0f, Z = 0.0f;
    if (M != -INFINITY) {
      for (int s2 = 0; s2 < nstates; ++s2) {
        const float* sl = res + s2 * S::kRes + r * (D + 4);
        const float ms = sl[D];
        const float wgt = (ms == -INFINITY) ? 0.0f : fast_exp2(ms - M);
        const float4 v = *reinterpret_cast<const float4*>(sl + c4);
        O.x = fmaf(wgt, v.x, O.x);
        O.y = fmaf(wgt, v.y, O.y);
        O.z = fmaf(wgt, v.z, O.z);
        O.w = fmaf(wgt, v.w, O.w);
        L = fmaf(wgt, sl[D + 1], L);
        Z = fmaf(wgt, sl[D + 2], Z);
      }
    }
    float* dst = p.ws + ((((size_t)n * p.Hkv + h) * p.n_splits + split) * G + r) * (D + 2);
    *reinterpret_cast<float2*>(dst + c4) = make_float2(O.x + Z, O.y + Z);
    *reinterpret_cast<float2*>(dst + c4 + 2) = make_float2(O.z + Z, O.w + Z);
    if (c4 == 0) {
      dst[D] = M;
      dst[D + 1] = L;
    }
  }
}

// Merge the splits of each (sequence, query head), rotate back, store: one
// CTA per query row, warp w taking splits 32 w .. 32 w + 31 (lane i: split
// 32 w + i), so that every load of a row is in flight at once but for the
// channel sums, sixteen splits deep.
template <int D, int BLK>
__global__ void __launch_bounds__(128) kvq_oscar_combine_kernel(const __grid_constant__ OscarAttnParams p) {
  constexpr int E = D / 32;
  static_assert(kMaxSplits <= 128, "four warps of 32 splits");
  __shared__ __align__(16) float part[4][D + 4];
  __shared__ float wmax[4];
  pdl_wait();  // the decode kernel's partial results
  pdl_launch_dependents();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const unsigned FULL = 0xffffffffu;
  const int row = blockIdx.x;  // n * Hq + hq
  const int n = row / p.Hq, hq = row % p.Hq, h = hq / p.G, r = hq % p.G;
  const size_t sstride = (size_t)p.G * (D + 2);
  const float* base = p.ws + (((size_t)n * p.Hkv + h) * p.n_splits * p.G + r) * (D + 2);
  // splits that hold a part of this sequence (the decode kernel returns
  // early from the others and leaves their rows unwritten)
  int ctx = p.ctx_lens[n];
  const int cap = p.max_pages * 16 + 15;
  ctx = ctx < 0 ? 0 : (ctx > cap ? cap : ctx);
  const int ns = ctx == 0 ? 0 : max(1, ((ctx >> 4) + p.pages_per_split - 1) / p.pages_per_split);
  const int s = 32 * warp + lane;
  float ms = -INFINITY, ls = 0.0f;
  if (s < ns) {
    ms = base[s * sstride + D];
    ls = base[s * sstride + D + 1];
  }
  float m = ms;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(FULL, m, o));
  if (lane == 0) wmax[warp] = m;
  __syncthreads();
  const float M = fmaxf(fmaxf(wmax[0], wmax[1]), fmaxf(wmax[2], wmax[3]));
  const float w = (ms == -INFINITY) ? 0.0f : fast_exp2(ms - M);
  float L = w * ls;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) L += __shfl_xor_sync(FULL, L, o);
  float v[E] = {0.0f, 0.0f, 0.0f, 0.0f};
  const int cnt = max(0, min(32, ns - 32 * warp));
  const float* sb = base + (size_t)(32 * warp) * sstride + E * lane;
#pragma unroll 16
  for (int i = 0; i < cnt; ++i) {
    const float wi = __shfl_sync(FULL, w, i);
    const float2 a = *reinterpret_cast<const float2*>(sb + i * sstride);
    const float2 b = *reinterpret_cast<const float2*>(sb + i * sstride + 2);
    v[0] = fmaf(wi, a.x, v[0]);
    v[1] = fmaf(wi, a.y, v[1]);
    v[2] = fmaf(wi, b.x, v[2]);
    v[3] = fmaf(wi, b.y, v[3]);
  }
  *reinterpret_cast<float4*>(&part[warp][E * lane]) = make_float4(v[0], v[1], v[2], v[3]);
  if (lane == 0) part[warp][D] = L;
  __syncthreads();
  if (warp != 0) return;
  float Lt = 0.0f;
#pragma unroll
  for (int e = 0; e < E; ++e) v[e] = 0.0f;
#pragma unroll
  for (int w2 = 0; w2 < 4; ++w2) {
    const float4 a = *reinterpret_cast<const float4*>(&part[w2][E * lane]);
    v[0] += a.x;
    v[1] += a.y;
    v[2] += a.z;
    v[3] += a.w;
    Lt += part[w2][D];
  }
  const float inv = (Lt > 0.0f) ? 1.0f / Lt : 0.0f;
#pragma unroll
  for (int e = 0; e < E; ++e) v[e] *= inv;
  if constexpr (BLK > 0) {
    warp_fwht<D, BLK>(v, lane);
#pragma unroll
    for (int e = 0; e < E; ++e) v[e] *= p.cb;
  }
  const size_t o = (size_t)row * D + E * lane;
  if (p.out_bf16) {
    const uint32_t w0 = (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(v[0])) |
                        ((uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(v[1])) << 16);
    const uint32_t w1 = (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(v[2])) |
                        ((uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(v[3])) << 16);
    *reinterpret_cast<uint2*>(reinterpret_cast<uint16_t*>(p.out) + o) = make_uint2(w0, w1);
  } else {
    *reinterpret_cast<float4*>(reinterpret_cast<float*>(p.out) + o) = make_float4(v[0], v[1], v[2], v[3]);
  }
}

}  // namespace kvq
