// kvq_write.cuh - token-wise INT4 quantization + paged store without a
// rotation: kv_quant_write with hadamard_block = 0 (plain INT4, the
// comparator of the rotated path). The rotated write (b = 32/64/128) is the
// tensor-core kernel in kvq_write_tc.cuh.
//
// SAW-INT4 (Abstract): one scale per token, codes stored straight into the
// paged cache by the kernel that quantizes them.
//
// Work unit: a warp tile = 32 consecutive tokens of one (kv head, K|V). One
// thread owns one row (token, head, K|V) of D values, so the row min/max and
// the packing stay in the thread's registers - no shuffles. Input rows arrive
// through cp.async into a per-warp shared buffer with an XOR swizzle on
// 16-byte chunks (conflict-free row reads); the copy of tile i+1 is issued
// before tile i is computed. The arithmetic runs on packed fp32 pairs (sm_100
// f32x2: one issue slot per two lanes) where it can: y - z and the rounding
// fma. Packed rows (D/2 bytes) and the fp16 s, z go straight to their slot.
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
  uint32_t signs[4];        // randomized Hadamard: bit c negates channel c before the transform
};

constexpr int kWriteWarps = 4;

template <int D>
__host__ __device__ constexpr int write_smem_bytes() {
  return kWriteWarps * 32 * D * 2;
}

template <int D>
__global__ void __launch_bounds__(kWriteWarps * 32, 3) kvq_write_kernel(const WriteParams p) {
  constexpr int ROWB = D * 2;       // bytes per bf16 input row
  constexpr int CPR = ROWB / 16;    // 16-byte chunks per row (8 or 16)
  constexpr int RPI = 32 / CPR;     // rows covered by one warp-wide copy instruction
  extern __shared__ __align__(128) uint8_t smem[];
  pdl_wait();  // the previous kernel on the stream may still read the cache or write K, V
  pdl_launch_dependents();
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  uint8_t* wbuf = smem + warp * 32 * ROWB;
  const uint32_t wbuf_s = smem_addr(wbuf);
  const int nw = gridDim.x * kWriteWarps;
  int tile = blockIdx.x * kWriteWarps + warp;
  const size_t row_stride = (size_t)p.Hkv * D;  // elements between consecutive tokens
  const int lrow = lane / CPR, lchunk = lane % CPR;

  auto issue = [&](int tl) {
    const int kv = tl & 1;
    const int h = (tl >> 1) % p.Hkv;
    const int tb = (tl >> 1) / p.Hkv;
    const uint16_t* src = (kv ? p.v : p.k) + ((size_t)(tb * 32 + lrow) * p.Hkv + h) * D + lchunk * 8;
#pragma unroll
    for (int j = 0; j < CPR; ++j) {
      const int r = j * RPI + lrow;
      if (tb * 32 + r < p.T)
        cp_async_16(wbuf_s + r * ROWB + ((lchunk ^ (r & (CPR - 1))) * 16), src + (size_t)j * RPI * row_stride);
    }
    cp_async_commit();
  };

  const uint64_t magic2 = f2_pack(8388608.0f, 8388608.0f);

  if (tile < p.num_tiles) issue(tile);
  for (; tile < p.num_tiles; tile += nw) {
    const int kv = tile & 1;
    const int h = (tile >> 1) % p.Hkv;
    const int tb = (tile >> 1) / p.Hkv;
    const int t = tb * 32 + lane;
    const long long slot = (t < p.T) ? p.slots[t] : -1;

    cp_async_wait_all();
    __syncwarp();
    uint64_t xp[D / 2];
#pragma unroll
    for (int c = 0; c < CPR; ++c) {
      const uint4 u = *reinterpret_cast<const uint4*>(wbuf + lane * ROWB + ((c ^ (lane & (CPR - 1))) * 16));
      const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
      for (int e = 0; e < 4; ++e)
        xp[c * 4 + e] = f2_pack(__uint_as_float(w[e] << 16), __uint_as_float(w[e] & 0xffff0000u));
    }
    __syncwarp();
    if (tile + nw < p.num_tiles) issue(tile + nw);

    // 1. row min / max (y = x: no rotation) (four independent 3-input chains each)
    float mn4[4], mx4[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      float a, b;
      f2_unpack(xp[q * (D / 8)], a, b);
      mn4[q] = fminf(a, b);
      mx4[q] = fmaxf(a, b);
#pragma unroll
      for (int i = q * (D / 8) + 1; i < (q + 1) * (D / 8); ++i) {
        f2_unpack(xp[i], a, b);
        mn4[q] = fmin3(mn4[q], a, b);
        mx4[q] = fmax3(mx4[q], a, b);
      }
    }
    const float mn = fminf(fminf(mn4[0], mn4[1]), fminf(mn4[2], mn4[3]));
    const float mx = fmaxf(fmaxf(mx4[0], mx4[1]), fmaxf(mx4[2], mx4[3]));
    // 2. z = largest fp16 <= mn; s = smallest fp16 with 15 s + z >= mx.
    //    Directed roundings give a candidate at most one fp16 step high; the
    //    step below is tested exactly in fp32 (15 s is exact, and
    //    15 s >= mx - z holds exactly when 15 s >= RU(mx - z)).
    const __half zh = __float2half_rd(mn);
    const float zf = __half2float(zh);
    const float dz = __fsub_ru(mx, zf);
    const float need = __fmul_ru(dz, 0.0666666701f);  // RU(1/15)
    unsigned short sb = __half_as_ushort(__float2half_ru(need));
    if (sb != 0 && sb < 0x7C00) {
      const unsigned short pb = (unsigned short)(sb - 1);
      if (__fmul_rn(15.0f, __half2float(__ushort_as_half(pb))) >= dz) sb = pb;
    }
    const float sf = __half2float(__ushort_as_half(sb));
    const float inv = (sf > 0.0f) ? __frcp_rn(sf) : 0.0f;
    // 3. code = rint(fp32(y - z) * fp32(1/s)): adding 2^23 inside one fma
    //    rounds the exact product to an integer (ties to even), leaving the
    //    code in the low 4 bits of the result (above them: the constant
    //    exponent of 2^23). Eight such words shifted by 4i and summed give the
    //    packed word plus a known constant, removed by starting the sum at its
    //    negation.
    const uint64_t z2 = f2_pack(zf, zf);
    const uint64_t inv2 = f2_pack(inv, inv);
    uint32_t packed[D / 8];
#pragma unroll
    for (int wd = 0; wd < D / 8; ++wd) {
      uint32_t acc = 0x05000000u;  // -(0x4B000000 + (0x4B000000 << 4)) mod 2^32
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const uint64_t f = f2_fma(f2_sub(xp[wd * 4 + i], z2), inv2, magic2);
        float lo, hi;
        f2_unpack(f, lo, hi);
        acc += __float_as_uint(lo) << (8 * i);
        acc += __float_as_uint(hi) << (8 * i + 4);
      }
      packed[wd] = acc;
    }
    // 4. paged store
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
