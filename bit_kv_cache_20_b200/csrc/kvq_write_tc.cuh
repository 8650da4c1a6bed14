// kvq_write_tc.cuh - fused rotation + token-wise INT4 quantization + paged
// store, with the rotation on the 5th-generation tensor cores.
//
// SAW-INT4 (Abstract): a single kernel rotates, quantizes and stores each
// row straight into the paged cache; OScaR (forum summary, "The OScaR
// Framework"): rotate first, then quantize.
//
// The block-diagonal Hadamard rotation of a tile of 128 rows (128 consecutive
// tokens of one kv head, K or V) is one dense product Y = X H with X [128 x D]
// bf16 and H [D x D] = diag(H_b) (entries +-1, exact in bf16): D/16
// tcgen05.mma (kind::f16, bf16 x bf16 -> fp32) accumulating in tensor memory.
// The products are exact and the fp32 accumulation stays well inside the
// error bound of a fp32 butterfly (measured on B200: at most 0.11 of it for
// b = 32, 64, 128). The 1/sqrt(b) normalization, the row min/max, the scale
// and zero-point, the codes and the nibble packing run on the CUDA cores in
// the epilogue, one thread per row.
//
// Persistent grid, one CTA per SM, 2 + 4 kTcBufs warps:
//   warp 0       TMA producer: 2-D tiled loads (128-byte swizzle) of X tiles
//                into a ring of kTcStages stages;
//   warp 1       owns the tensor memory and issues the MMAs (one thread) into
//                one of kTcBufs accumulator buffers;
//   warps 2..    kTcBufs epilogue groups of 4 warps (one per tensor-memory
//                lane quarter); group e takes every kTcBufs-th tile of the
//                CTA, so the groups' epilogues overlap one another and the
//                MMAs. (Measured on B200: the DRAM traffic, not the epilogue,
//                bounds the kernel; more groups or stages did not help.)
// mbarriers hand each stage and each accumulator buffer from one role to the
// next; every wait is bounded (a lost wait records KVQ_ERR_TIMEOUT and the
// roles stop), and the CTA waits for its own copies and MMAs before it frees
// the tensor memory and exits.
#pragma once

#include <cuda.h>

#include "kvq_device.cuh"
#include "kvq_write.cuh"

namespace kvq {

constexpr int kTcStages = 4;
constexpr int kTcBufs = 2;  // tensor-memory accumulators = epilogue groups
constexpr int kTcWarps = 2 + 4 * kTcBufs;
constexpr int kTcThreads = kTcWarps * 32;
constexpr int kTcRows = 128;  // rows (tokens) per tile = UMMA M

template <int D>
struct TcSmem {
  static constexpr int kChunkBytes = kTcRows * 128;            // 128 rows x 64 bf16 (one swizzle span)
  static constexpr int kTileBytes = kTcRows * D * 2;           // D / 64 chunks
  static constexpr int kOffH = 0;                              // H as the K-major B operand: D/64 chunks of D x 128 B
  static constexpr int kOffX = D * D * 2;                      // ring of X tiles
  static constexpr int kOffBar = kOffX + kTcStages * kTileBytes;
  // mbarriers: full[kTcStages], empty[kTcStages], tfull[kTcBufs], tempty[kTcBufs], done
  static constexpr int kBars = 2 * kTcStages + 2 * kTcBufs + 1;
  static constexpr int kOffTmem = kOffBar + kBars * 8;
  static constexpr int kUsed = kOffTmem + 16;
  static constexpr int kTotal = kUsed + 1024;                  // room to align the base to 1024 B
};

// Byte offset of element (row, k) in a K-major operand stored as 64-wide
// chunks of `rows` rows x 128 B with the 128-byte swizzle (16-byte unit c of
// a row stored at c ^ (row % 8)).
__host__ __device__ constexpr int sw128_offset(int row, int k, int rows) {
  return (k >> 6) * (rows * 128) + row * 128 + ((((k & 63) >> 3) ^ (row & 7)) << 4) + (k & 7) * 2;
}

// Four bytes of packed codes from eight fp32 words whose low byte holds a
// code (c0 .. c7 in order): byte j = c[2j] | c[2j+1] << 4.
__device__ __forceinline__ uint32_t pack8_codes(const uint32_t (&f)[8]) {
  const uint32_t e = prmt(prmt(f[0], f[2], 0x0040u), prmt(f[4], f[6], 0x0040u), 0x5410u);
  const uint32_t o = prmt(prmt(f[1], f[3], 0x0040u), prmt(f[5], f[7], 0x0040u), 0x5410u);
  return o * 16u + e;
}

template <int D, int BLK>
__global__ void __launch_bounds__(kTcThreads, 1)
    kvq_write_tc_kernel(const __grid_constant__ CUtensorMap tmap_k, const __grid_constant__ CUtensorMap tmap_v,
                        const WriteParams p, const int n_tiles) {
  using S = TcSmem<D>;
  constexpr int KC = D / 64;  // 64-wide K chunks
  constexpr int KS = D / 16;  // MMA k-steps
  // instruction descriptor: fp32 accumulator, bf16 A and B, both K-major,
  // N = D, M = 128
  constexpr uint32_t kIdesc = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(D >> 3) << 17) | ((uint32_t)(kTcRows >> 4) << 24);
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024 - (smem_addr(smem_raw) & 1023)) & 1023);
  const uint32_t sb = smem_addr(smem);
  const uint32_t bar0 = sb + S::kOffBar;
  auto full = [&](int st) { return bar0 + 8 * st; };
  auto empty = [&](int st) { return bar0 + 8 * (kTcStages + st); };
  auto tfull = [&](int j) { return bar0 + 8 * (2 * kTcStages + j); };
  auto tempty = [&](int j) { return bar0 + 8 * (2 * kTcStages + kTcBufs + j); };
  const uint32_t done_bar = bar0 + 8 * (2 * kTcStages + 2 * kTcBufs);
  uint32_t* tslot = reinterpret_cast<uint32_t*>(smem + S::kOffTmem);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  if (tid == 0) {
    for (int st = 0; st < kTcStages; ++st) {
      mbar_init(full(st), 1);
      mbar_init(empty(st), 1);
    }
    for (int j = 0; j < kTcBufs; ++j) {
      mbar_init(tfull(j), 1);
      mbar_init(tempty(j), 4 * 32);
    }
    mbar_init(done_bar, 1);
    mbar_init_fence();
  }
  if (warp == 1) tmem_alloc(smem_addr(tslot), kTcBufs * D);
  tc_fence_before();
  __syncthreads();  // barriers and the tensor-memory address are in place
  tc_fence_after();
  // While warp 0 starts the first copies, the other warps build the B
  // operand [n][k] = H[n][k] sigma_k (H = diag(H_b), unnormalized Sylvester
  // order, symmetric; sigma the randomized signs, all +1 by default), so that
  // Y = X B^T = (R X^T)^T sqrt(b), 16 bytes at a time, then meet on named
  // barrier 1 before the first MMA.
  if (warp != 0) {
    for (int i = tid - 32; i < D * (D / 8); i += kTcThreads - 32) {
      const int n = i / (D / 8), k0 = 8 * (i % (D / 8));
      // sign word of channels k0 .. k0 + 7 (constant indices: no local copy of p)
      const uint32_t sw = k0 < 32 ? p.signs[0] : k0 < 64 ? p.signs[1] : k0 < 96 ? p.signs[2] : p.signs[3];
      uint32_t w[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        uint32_t pair = 0;
#pragma unroll
        for (int hlf = 0; hlf < 2; ++hlf) {
          const int k = k0 + 2 * e + hlf;
          uint32_t bits = 0;  // bf16 0
          if (n / BLK == k / BLK) {
            bits = (__popc((n % BLK) & (k % BLK)) & 1) ? 0xBF80u : 0x3F80u;  // -1, +1
            bits ^= ((sw >> (k & 31)) & 1u) << 15;  // times sigma_k
          }
          pair |= bits << (16 * hlf);
        }
        w[e] = pair;
      }
      *reinterpret_cast<uint4*>(smem + S::kOffH + sw128_offset(n, k0, D)) = make_uint4(w[0], w[1], w[2], w[3]);
    }
    asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");  // H visible to the tensor cores
    named_bar_sync(1, kTcThreads - 32);
  }
  const uint32_t tmem = *tslot;
  const int first = blockIdx.x, stride = gridDim.x;
  // Everything above touched only this CTA's shared and tensor memory, so it
  // overlaps the previous kernel's last CTAs; global memory waits for it.
  pdl_wait();
  pdl_launch_dependents();

  if (warp == 0) {
    // ---- TMA producer --------------------------------------------------------
    if (lane == 0) {
      int i = 0;
      for (int tile = first; tile < n_tiles; tile += stride, ++i) {
        const int st = i % kTcStages;
        if (i >= kTcStages && !mbar_wait_bounded(empty(st), ((i / kTcStages) - 1) & 1)) break;
        const int kv = tile & 1, h = (tile >> 1) % p.Hkv, tb = (tile >> 1) / p.Hkv;
        mbar_arrive_expect_tx(full(st), S::kTileBytes);
        const void* tm = kv ? static_cast<const void*>(&tmap_v) : static_cast<const void*>(&tmap_k);
#pragma unroll
        for (int c = 0; c < KC; ++c)
          tma_load_2d(sb + S::kOffX + st * S::kTileBytes + c * S::kChunkBytes, tm, h * D + 64 * c, tb * kTcRows,
                      full(st));
      }
      // every copy issued has landed before the CTA may exit
      for (int k = max(i - kTcStages, 0); k < i; ++k) mbar_wait_bounded(full(k % kTcStages), (k / kTcStages) & 1);
    }
  } else if (warp == 1) {
    // ---- MMA issuer ----------------------------------------------------------
    if (lane == 0) {
      int i = 0;
      for (int tile = first; tile < n_tiles; tile += stride, ++i) {
        const int st = i % kTcStages, j = i % kTcBufs;
        if (!mbar_wait_bounded(full(st), (i / kTcStages) & 1)) break;
        if (i >= kTcBufs && !mbar_wait_bounded(tempty(j), ((i / kTcBufs) - 1) & 1)) break;
        tc_fence_after();
        const uint32_t xs = sb + S::kOffX + st * S::kTileBytes;
#pragma unroll
        for (int s = 0; s < KS; ++s) {
          const uint32_t off = (s >> 2) * S::kChunkBytes + (s & 3) * 32;
          const uint32_t offb = (s >> 2) * (D * 128) + (s & 3) * 32;
          umma_f16_ss(tmem + j * D, umma_desc_sw128(xs + off), umma_desc_sw128(sb + S::kOffH + offb), kIdesc,
                      s > 0);
        }
        umma_commit(empty(st));  // the stage may be refilled once these MMAs are done
        umma_commit(tfull(j));   // the accumulator is ready for the epilogue
      }
      // every MMA issued has completed before the tensor memory is freed
      umma_commit(done_bar);
      mbar_wait_bounded(done_bar, 0);
    }
  } else {
    // ---- epilogue: one thread per row of the tile ---------------------------
    const int eg = (warp - 2) >> 2;  // epilogue group: takes every kTcBufs-th tile
    const int q = warp & 3;          // tensor-memory lane quarter this warp may read
    const int r = 32 * q + lane;     // row of the tile
    const uint64_t cb2 = f2_pack(p.cb, p.cb);
    const uint64_t magic2 = f2_pack(8388608.0f, 8388608.0f);
    int i = eg;
    for (int tile = first + eg * stride; tile < n_tiles; tile += kTcBufs * stride, i += kTcBufs) {
      const int j = eg;
      const int kv = tile & 1, h = (tile >> 1) % p.Hkv, tb = (tile >> 1) / p.Hkv;
      const int t = tb * kTcRows + r;
      const long long slot = (t < p.T) ? p.slots[t] : -1;  // in flight during the wait
      if (!__all_sync(0xffffffffu, mbar_wait_bounded(tfull(j), (i / kTcBufs) & 1))) break;
      tc_fence_after();
      const uint32_t ta = tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)(j * D);

      // 1. min / max of the unnormalized rotation H x; y = fp32(Hx) * c_b is
      //    monotone in Hx, so min y and max y are the scaled extremes
      float mn4[4] = {INFINITY, INFINITY, INFINITY, INFINITY};
      float mx4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        float v[32];
        tmem_ld32(ta + 32 * c, v);
#pragma unroll
        for (int k = 0; k < 16; ++k) {  // four independent chains
          mn4[k & 3] = fmin3(mn4[k & 3], v[2 * k], v[2 * k + 1]);
          mx4[k & 3] = fmax3(mx4[k & 3], v[2 * k], v[2 * k + 1]);
        }
      }
      const float mn = __fmul_rn(fminf(fminf(mn4[0], mn4[1]), fminf(mn4[2], mn4[3])), p.cb);
      const float mx = __fmul_rn(fmaxf(fmaxf(mx4[0], mx4[1]), fmaxf(mx4[2], mx4[3])), p.cb);
      // 2. z = largest fp16 <= min y; s = smallest fp16 with 15 s + z >= max y
      //    (directed roundings give a candidate at most one fp16 step high;
      //    the step below is tested exactly in fp32: 15 s is exact, and
      //    15 s >= max y - z holds exactly when 15 s >= RU(max y - z))
      const __half zh = __float2half_rd(mn);
      const float zf = __half2float(zh);
      const float dz = __fsub_ru(mx, zf);
      const float need = __fmul_ru(dz, 0.0666666701f);  // RU(1/15)
      unsigned short sbits = __half_as_ushort(__float2half_ru(need));
      if (sbits != 0 && sbits < 0x7C00) {
        const unsigned short pb = (unsigned short)(sbits - 1);
        if (__fmul_rn(15.0f, __half2float(__ushort_as_half(pb))) >= dz) sbits = pb;
      }
      const float sf = __half2float(__ushort_as_half(sbits));
      const float inv = (sf > 0.0f) ? __frcp_rn(sf) : 0.0f;
      const uint64_t z2 = f2_pack(zf, zf), inv2 = f2_pack(inv, inv);
      const bool store = slot >= 0 && slot < p.num_slots;
      if (!store && t < p.T && slot != -1) record_error(KVQ_ERR_OUT_OF_RANGE);
      const size_t row = store ? ((((size_t)(slot >> 4) * p.Hkv + h) * 2 + kv) * 16 + (slot & 15)) : 0;
      uint4* dst = reinterpret_cast<uint4*>(p.cache + row * (D / 2));

      // 3. code = rint(fp32(y - z) * fp32(1/s)) via one fma with 2^23 (the
      //    code lands in the low byte of the result); 32 codes -> 16 bytes
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        float v[32];
        tmem_ld32(ta + 32 * c, v);
        uint32_t words[4];
#pragma unroll
        for (int w = 0; w < 4; ++w) {
          uint32_t f[8];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const uint64_t y2 = f2_mul(f2_pack(v[8 * w + 2 * e], v[8 * w + 2 * e + 1]), cb2);
            const uint64_t q2 = f2_fma(f2_sub(y2, z2), inv2, magic2);
            float lo, hi;
            f2_unpack(q2, lo, hi);
            f[2 * e] = __float_as_uint(lo);
            f[2 * e + 1] = __float_as_uint(hi);
          }
          words[w] = pack8_codes(f);
        }
        if (store) dst[c] = make_uint4(words[0], words[1], words[2], words[3]);
      }
      if (store) {
        p.scales[row] = sbits;
        p.zeros[row] = __half_as_ushort(zh);
      }
      tc_fence_before();
      mbar_arrive(tempty(j));  // the accumulator buffer may be overwritten
    }
  }

  // ---- teardown: every role is done; free the tensor memory --------------
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, kTcBufs * D);
}

}  // namespace kvq
