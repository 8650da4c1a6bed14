// kvq_write.cuh - fused rotation + token-wise INT4 quantization + paged store.
//
// SAW-INT4 (Abstract): "a fused rotation-quantization kernel that integrates
// directly into paged KV-cache layouts"; OScaR (forum summary, "The OScaR
// Framework"): rotate, then quantize.
//
// Work unit: a warp tile = 32 consecutive tokens of one (kv head, K|V). One
// thread owns one row (token, head, K|V) of D values, so the whole Hadamard
// block, the row min/max and the packing stay in the thread's registers - no
// shuffles. Input rows arrive through cp.async into a per-warp shared buffer
// with an XOR swizzle on 16-byte chunks (conflict-free row reads); the copy of
// tile i+1 is issued before tile i is computed. Packed rows (D/2 bytes) and
// the fp16 s, z go straight to their slot.
#pragma once

#include "kvq_device.cuh"

namespace kvq {

struct WriteParams {
  const uint16_t* k;        // bf16 [T][Hkv][D]
  const uint16_t* v;
  const int64_t* slots;     // [T]
  uint8_t* cache;           // [pages][Hkv][2][16][D/2]
  uint16_t* scales;         // fp16 [pages][Hkv][2][16]
  uint16_t* zeros;
  int T;
  int Hkv;
  long long num_slots;      // num_pages * 16
  int num_tiles;            // ceil(T/32) * Hkv * 2
  float cb;                 // fp32(1/sqrt(b)), 1 for b = 0
};

constexpr int kWriteWarps = 4;

template <int D>
__host__ __device__ constexpr int write_smem_bytes() {
  return kWriteWarps * 32 * D * 2;
}

// In-register fast Walsh-Hadamard transform of each contiguous BLK block
// (Sylvester natural order: y_i = sum_j (-1)^popcount(i&j) x_j).
template <int D, int BLK>
__device__ __forceinline__ void fwht_blocks(float (&x)[D]) {
#pragma unroll
  for (int base = 0; base < D; base += BLK) {
#pragma unroll
    for (int len = 1; len < BLK; len <<= 1) {
#pragma unroll
      for (int i = 0; i < BLK; ++i) {
        if ((i & len) == 0) {
          const float a = x[base + i], b = x[base + i + len];
          x[base + i] = __fadd_rn(a, b);
          x[base + i + len] = __fsub_rn(a, b);
        }
      }
    }
  }
}

template <int D, int BLK>
__global__ void __launch_bounds__(kWriteWarps * 32, 3) kvq_write_kernel(const WriteParams p) {
  constexpr int ROWB = D * 2;       // bytes per bf16 input row
  constexpr int CPR = ROWB / 16;    // 16-byte chunks per row (8 or 16)
  extern __shared__ __align__(128) uint8_t smem[];
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  uint8_t* wbuf = smem + warp * 32 * ROWB;
  const uint32_t wbuf_s = smem_addr(wbuf);
  const int nw = gridDim.x * kWriteWarps;
  int tile = blockIdx.x * kWriteWarps + warp;

  auto issue = [&](int tl) {
    const int kv = tl & 1;
    const int h = (tl >> 1) % p.Hkv;
    const int tb = (tl >> 1) / p.Hkv;
    const uint16_t* src = kv ? p.v : p.k;
#pragma unroll
    for (int j = 0; j < CPR; ++j) {
      const int idx = j * 32 + lane;
      const int r = idx / CPR, c = idx % CPR;
      const int t = tb * 32 + r;
      if (t < p.T) {
        const uint16_t* g = src + ((size_t)t * p.Hkv + h) * D + c * 8;
        cp_async_16(wbuf_s + r * ROWB + ((c ^ (r & (CPR - 1))) * 16), g);
      }
    }
    cp_async_commit();
  };

  if (tile < p.num_tiles) issue(tile);
  for (; tile < p.num_tiles; tile += nw) {
    const int kv = tile & 1;
    const int h = (tile >> 1) % p.Hkv;
    const int tb = (tile >> 1) / p.Hkv;
    const int t = tb * 32 + lane;
    const long long slot = (t < p.T) ? p.slots[t] : -1;

    cp_async_wait_all();
    __syncwarp();
    float x[D];
#pragma unroll
    for (int c = 0; c < CPR; ++c) {
      const uint4 u = *reinterpret_cast<const uint4*>(wbuf + lane * ROWB + ((c ^ (lane & (CPR - 1))) * 16));
      const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        x[c * 8 + 2 * e] = __uint_as_float(w[e] << 16);
        x[c * 8 + 2 * e + 1] = __uint_as_float(w[e] & 0xffff0000u);
      }
    }
    __syncwarp();
    if (tile + nw < p.num_tiles) issue(tile + nw);

    // 1. rotation y = (H_b x) * fp32(1/sqrt(b))
    if constexpr (BLK > 0) {
      fwht_blocks<D, BLK>(x);
#pragma unroll
      for (int c = 0; c < D; ++c) x[c] = __fmul_rn(x[c], p.cb);
    }
    // 2. row min / max
    float mn = x[0], mx = x[0];
#pragma unroll
    for (int c = 1; c < D; ++c) {
      mn = fminf(mn, x[c]);
      mx = fmaxf(mx, x[c]);
    }
    // 3. z = largest fp16 <= mn; s = smallest fp16 with 15 s + z >= mx.
    //    Directed roundings give a candidate at most one fp16 step above the
    //    smallest; the exact test (fp64: 15 s + z is exact there) settles it.
    const __half zh = __float2half_rd(mn);
    const float zf = __half2float(zh);
    const float need = __fdiv_ru(__fsub_ru(mx, zf), 15.0f);
    unsigned short sb = __half_as_ushort(__float2half_ru(need));
    if (sb != 0 && sb < 0x7C00) {
      const unsigned short pb = (unsigned short)(sb - 1);
      const float sp = __half2float(__ushort_as_half(pb));
      if (fma(15.0, (double)sp, (double)zf) >= (double)mx) sb = pb;
    }
    const float sf = __half2float(__ushort_as_half(sb));
    const float inv = (sf > 0.0f) ? __frcp_rn(sf) : 0.0f;
    // 4. code = rint(fp32(y - z) * fp32(1/s)): adding 2^23 inside one fma
    //    rounds the exact product to an integer (ties to even); the code is
    //    then the low bits of the result.
    uint32_t packed[D / 8];
#pragma unroll
    for (int wd = 0; wd < D / 8; ++wd) {
      uint32_t acc = 0;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float tq = __fmaf_rn(__fsub_rn(x[wd * 8 + i], zf), inv, 8388608.0f);
        acc |= (__float_as_uint(tq) & 0xFu) << (4 * i);
      }
      packed[wd] = acc;
    }
    // 5. paged store
    if (slot >= 0 && slot < p.num_slots) {
      const long long page = slot >> 4;
      const int off = (int)(slot & 15);
      const size_t row = (((size_t)page * p.Hkv + h) * 2 + kv) * 16 + off;
      uint4* dst = reinterpret_cast<uint4*>(p.cache + row * (D / 2));
#pragma unroll
      for (int q = 0; q < D / 32; ++q)
        dst[q] = make_uint4(packed[4 * q], packed[4 * q + 1], packed[4 * q + 2], packed[4 * q + 3]);
      p.scales[row] = sb;
      p.zeros[row] = __half_as_ushort(zh);
    } else if (t < p.T && slot != -1) {
      record_error(KVQ_ERR_OUT_OF_RANGE);
    }
  }
  cp_async_wait_all();
}

}  // namespace kvq
