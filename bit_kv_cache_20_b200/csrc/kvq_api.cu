// kvq_api.cu - the C ABI declared in include/kvq.h: argument checks, device
// selection, grid sizing and kernel dispatch. One translation unit holds every
// kernel, so the device error word is a single symbol per device.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <mutex>
#include <utility>
#include <vector>
#include <climits>
#include <cmath>
#include <cstdint>

#include "../../include/kvq.h"
#include "kvq_decode.cuh"
#include "kvq_write.cuh"
#include "kvq_write_tc.cuh"
#include "kvq_prefill.cuh"
#include "kvq_oscar.cuh"
#include "kvq_selftest.cuh"

namespace {

// Launch with programmatic stream serialization (see KVQ_ATTN_INPUTS_READY in
// kvq.h): the kernel's CTAs may start while the previous kernel on the stream
// drains; every kernel here waits for it (griddepcontrol.wait) before
// touching memory that kernel may have written.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, int smem, cudaStream_t s,
                       Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = (size_t)smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}


constexpr int kMaxDevices = 64;

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

bool valid_block(int D, int b) {
  if (b == 0) return true;
  if (b != 32 && b != 64 && b != 128) return false;
  return b <= D && (D % b) == 0;
}

// Make the device that owns `ptr` current for this runtime. The owner is read
// with the driver's pointer query, which needs no current context, so a
// process that drives several GPUs never touches a device it does not use.
typedef CUresult (*PtrAttrFn)(void*, CUpointer_attribute, CUdeviceptr);

PtrAttrFn pointer_query() {
  static std::atomic<PtrAttrFn> fn{nullptr};
  PtrAttrFn f = fn.load(std::memory_order_acquire);
  if (f) return f;
  void* raw = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPoint("cuPointerGetAttribute", &raw, cudaEnableDefault, &q) != cudaSuccess ||
      q != cudaDriverEntryPointSuccess || !raw) {
    cudaGetLastError();
    return nullptr;
  }
  f = reinterpret_cast<PtrAttrFn>(raw);
  fn.store(f, std::memory_order_release);
  return f;
}

kvq_status select_device_of(const void* ptr, int* dev_out) {
  PtrAttrFn query = pointer_query();
  if (!query) return KVQ_ERR_CUDA;
  unsigned int mtype = 0;
  int ordinal = -1;
  const CUdeviceptr dp = reinterpret_cast<CUdeviceptr>(ptr);
  if (query(&mtype, CU_POINTER_ATTRIBUTE_MEMORY_TYPE, dp) != CUDA_SUCCESS) return KVQ_ERR_INVALID_ARG;
  if (mtype != CU_MEMORYTYPE_DEVICE) return KVQ_ERR_INVALID_ARG;
  if (query(&ordinal, CU_POINTER_ATTRIBUTE_DEVICE_ORDINAL, dp) != CUDA_SUCCESS) return KVQ_ERR_CUDA;
  int cur = -1;
  if (cudaGetDevice(&cur) != cudaSuccess) return KVQ_ERR_CUDA;
  if (cur != ordinal && cudaSetDevice(ordinal) != cudaSuccess) return KVQ_ERR_CUDA;
  *dev_out = ordinal;
  return KVQ_OK;
}

int sm_count(int dev) {
  static std::atomic<int> cache[kMaxDevices];
  if (dev < 0 || dev >= kMaxDevices) return -1;
  int v = cache[dev].load(std::memory_order_relaxed);
  if (v > 0) return v;
  if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
    cudaGetLastError();
    return -1;
  }
  cache[dev].store(v, std::memory_order_relaxed);
  return v;
}

// Resident CTAs per SM of a kernel instance; `cache` is that instance's own
// per-device table.
template <typename K>
int resident_ctas(K kernel, std::atomic<int>* cache, int dev, int threads, int smem) {
  if (dev < 0 || dev >= kMaxDevices) return 1;
  int v = cache[dev].load(std::memory_order_relaxed);
  if (v > 0) return v;
  if (smem > 48 * 1024)
    cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&v, kernel, threads, smem) != cudaSuccess || v < 1) {
    cudaGetLastError();
    v = 1;
  }
  cache[dev].store(v, std::memory_order_relaxed);
  return v;
}

// ---------------------------------------------------------------------------
// kv_quant_write
// ---------------------------------------------------------------------------
template <int D>
kvq_status launch_write(const kvq::WriteParams& p, int dev, cudaStream_t s) {
  auto kern = kvq::kvq_write_kernel<D>;
  constexpr int smem = kvq::write_smem_bytes<D>();
  const int threads = kvq::kWriteWarps * 32;
  static std::atomic<int> occ[kMaxDevices];
  const int per_sm = resident_ctas(kern, occ, dev, threads, smem);
  const long long need = (p.num_tiles + kvq::kWriteWarps - 1) / kvq::kWriteWarps;
  const long long cap = (long long)per_sm * sm_count(dev);
  const int blocks = (int)(need < cap ? need : cap);
  if (launch_pdl(kern, dim3(blocks), dim3(threads), smem, s, p) != cudaSuccess) {
    cudaGetLastError();
    return KVQ_ERR_CUDA;
  }
  return KVQ_OK;
}

// Tiled tensor maps of K and V ([T][Hkv*D] bf16, boxes of 128 rows x 64
// elements, 128-byte swizzle) through the driver's encoder, looked up once.
typedef CUresult (*TmapEncodeFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                 const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                 CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

TmapEncodeFn tmap_encoder() {
  static std::atomic<TmapEncodeFn> fn{nullptr};
  TmapEncodeFn f = fn.load(std::memory_order_acquire);
  if (f) return f;
  void* raw = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &raw, cudaEnableDefault, &q) != cudaSuccess ||
      q != cudaDriverEntryPointSuccess || !raw) {
    cudaGetLastError();
    return nullptr;
  }
  f = reinterpret_cast<TmapEncodeFn>(raw);
  fn.store(f, std::memory_order_release);
  return f;
}

bool make_row_tmap(CUtensorMap* m, const void* base, int T, int Hkv, int D) {
  TmapEncodeFn enc = tmap_encoder();
  if (!enc) return false;
  const cuuint64_t dims[2] = {(cuuint64_t)Hkv * D, (cuuint64_t)T};
  const cuuint64_t strides[1] = {(cuuint64_t)Hkv * D * 2};
  const cuuint32_t box[2] = {64, (cuuint32_t)kvq::kTcRows};
  const cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Rotated write on the tensor cores: persistent grid, one CTA per SM.
template <int D, int BLK>
kvq_status launch_write_tc(const kvq::WriteParams& p, int dev, cudaStream_t s) {
  if (dev < 0 || dev >= kMaxDevices) return KVQ_ERR_UNSUPPORTED;
  CUtensorMap tk, tv;
  if (!make_row_tmap(&tk, p.k, p.T, p.Hkv, D) || !make_row_tmap(&tv, p.v, p.T, p.Hkv, D)) return KVQ_ERR_CUDA;
  const long long tiles = ((long long)p.T + kvq::kTcRows - 1) / kvq::kTcRows * p.Hkv * 2;
  if (tiles > INT_MAX) return KVQ_ERR_INVALID_ARG;
  auto kern = kvq::kvq_write_tc_kernel<D, BLK>;
  constexpr int smem = kvq::TcSmem<D>::kTotal;
  static std::atomic<int> ready[kMaxDevices];
  if (!ready[dev].load(std::memory_order_relaxed)) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess) {
      cudaGetLastError();
      return KVQ_ERR_CUDA;
    }
    ready[dev].store(1, std::memory_order_relaxed);
  }
  const int sms = sm_count(dev);
  if (sms < 1) return KVQ_ERR_CUDA;
  const int grid = (int)(tiles < sms ? tiles : sms);
  if (launch_pdl(kern, dim3(grid), dim3(kvq::kTcThreads), smem, s, tk, tv, p, (int)tiles) != cudaSuccess) {
    cudaGetLastError();
    return KVQ_ERR_CUDA;
  }
  return KVQ_OK;
}

template <int D>
kvq_status dispatch_write(const kvq::WriteParams& p, int b, int dev, cudaStream_t s) {
  switch (b) {
    case 0: return launch_write<D>(p, dev, s);
    case 32: return launch_write_tc<D, 32>(p, dev, s);
    case 64: return launch_write_tc<D, 64>(p, dev, s);
    case 128:
      if constexpr (D >= 128) return launch_write_tc<D, 128>(p, dev, s);
      return KVQ_ERR_UNSUPPORTED;
    default: return KVQ_ERR_UNSUPPORTED;
  }
}

// ---------------------------------------------------------------------------
// paged_decode_attn_int4
// ---------------------------------------------------------------------------
struct SplitPlan {
  int n_splits;         // uniform plan: CTAs per (sequence, kv-head group)
  int pages_per_split;
  int hg;               // kv heads per CTA
  int nc;               // column tiles of 4 query heads
  int n_items;          // per-sequence plan: entries of AttnParams::items (0 = uniform plan)
  int part_slots;       // per-sequence plan: partial-result slots it writes
};

int cols_for(int G) { return G > 4 ? 2 : 1; }

int inst_slot(int D, int b, int hg, int nc, int app) {
  const int bi = (b == 0) ? 0 : (b == 32) ? 1 : (b == 64) ? 2 : 3;
  const int hi = (hg == 4) ? 2 : (hg == 2) ? 1 : 0;
  return ((((D == 64) ? 0 : 1) * 4 + bi) * 6 + hi * 2 + (nc - 1)) * 2 + (app ? 1 : 0);
}
constexpr int kInstSlots = 96;

// Instances exist for HG * NC <= 4 (the plan never asks for more).
template <int D, int BLK, int NC, bool APP>
const void* decode_kernel_ptr(int hg) {
  if constexpr (NC == 1) {
    if (hg == 4) return reinterpret_cast<const void*>(kvq::kvq_decode_kernel<D, BLK, 4, NC, APP>);
  }
  if (hg == 2) return reinterpret_cast<const void*>(kvq::kvq_decode_kernel<D, BLK, 2, NC, APP>);
  if (hg == 1) return reinterpret_cast<const void*>(kvq::kvq_decode_kernel<D, BLK, 1, NC, APP>);
  return nullptr;
}

template <int D, int BLK>
const void* decode_kernel_ptr(int hg, int nc, int app) {
  if (app) return nc == 2 ? decode_kernel_ptr<D, BLK, 2, true>(hg) : decode_kernel_ptr<D, BLK, 1, true>(hg);
  return nc == 2 ? decode_kernel_ptr<D, BLK, 2, false>(hg) : decode_kernel_ptr<D, BLK, 1, false>(hg);
}

const void* decode_kernel_for(int D, int b, int hg, int nc, int app) {
  if (D == 64) {
    if (b == 0) return decode_kernel_ptr<64, 0>(hg, nc, app);
    if (b == 32) return decode_kernel_ptr<64, 32>(hg, nc, app);
    if (b == 64) return decode_kernel_ptr<64, 64>(hg, nc, app);
    return nullptr;
  }
  if (b == 0) return decode_kernel_ptr<128, 0>(hg, nc, app);
  if (b == 32) return decode_kernel_ptr<128, 32>(hg, nc, app);
  if (b == 64) return decode_kernel_ptr<128, 64>(hg, nc, app);
  if (b == 128) return decode_kernel_ptr<128, 128>(hg, nc, app);
  return nullptr;
}

template <int D, int NC>
int decode_smem_bytes_t(int hg) {
  if constexpr (NC == 1) {
    if (hg == 4) return kvq::AttnSmem<D, 4, NC>::kTotal;
  }
  if (hg == 2) return kvq::AttnSmem<D, 2, NC>::kTotal;
  return kvq::AttnSmem<D, 1, NC>::kTotal;
}

int decode_smem_bytes(int D, int hg, int nc) {
  if (D == 64) return nc == 2 ? decode_smem_bytes_t<64, 2>(hg) : decode_smem_bytes_t<64, 1>(hg);
  return nc == 2 ? decode_smem_bytes_t<128, 2>(hg) : decode_smem_bytes_t<128, 1>(hg);
}

// Opt the decode kernel instance into its dynamic shared memory and return
// how many of its CTAs one SM holds (once per device and instance; 0 on error).
int decode_ctas_per_sm(int dev, int D, int b, int hg, int nc, int app) {
  static std::atomic<int> cache[kMaxDevices][kInstSlots];
  if (dev < 0 || dev >= kMaxDevices) return 0;
  const int slot = inst_slot(D, b, hg, nc, app);
  int v = cache[dev][slot].load(std::memory_order_relaxed);
  if (v > 0) return v;
  const void* k = decode_kernel_for(D, b, hg, nc, app);
  const int smem = decode_smem_bytes(D, hg, nc);
  if (!k || cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess ||
      cudaOccupancyMaxActiveBlocksPerMultiprocessor(&v, k, 32 * kvq::attn_warps(nc), smem) != cudaSuccess ||
      v < 1) {
    cudaGetLastError();
    return 0;
  }
  cache[dev][slot].store(v, std::memory_order_relaxed);
  return v;
}

// Choose the kv heads per CTA (HG) and the split of each (sequence, head
// group) into CTAs. For each HG that divides Hkv (with HG * NC <= 4), the
// split count fills the device's resident CTA slots once (as the occupancy
// API reports for that instance) with at least 4 pages per split; the plan
// with the least work per CTA times waves (plus a fixed cost of 8 head-pages
// per CTA) wins, ties going to the smaller HG (fewer partial results).
SplitPlan plan_splits(const kvq_attn_desc* d, int dev, int app) {
  const int nc = cols_for(d->num_q_heads / d->num_kv_heads);
  const int sms = sm_count(dev);
  SplitPlan best = {1, d->max_pages_per_seq, 1, nc, 0, 0};
  long long best_cost = LLONG_MAX;
  for (int hg = 1; hg <= 4; hg <<= 1) {
    if (d->num_kv_heads % hg != 0 || hg * nc > 4) continue;
    const int per_sm = decode_ctas_per_sm(dev, d->head_dim, d->hadamard_block, hg, nc, app);
    if (per_sm < 1 || sms < 1) continue;
    const long long slots = (long long)per_sm * sms;
    const long long units = (long long)d->batch * (d->num_kv_heads / hg);
    long long ns = units > 0 ? slots / units : 1;
    long long ns_cap = d->max_pages_per_seq / 4;
    if (ns_cap > kvq::kMaxSplits) ns_cap = kvq::kMaxSplits;
    if (ns > ns_cap) ns = ns_cap;
    if (ns < 1) ns = 1;
    const long long pps = (d->max_pages_per_seq + ns - 1) / ns;
    ns = (d->max_pages_per_seq + pps - 1) / pps;  // drop splits that would be empty
    const long long waves = (units * ns + slots - 1) / slots;
    const long long cost = (waves < 1 ? 1 : waves) * (pps * hg + 8);
    if (cost < best_cost) {
      best_cost = cost;
      best = {(int)ns, (int)pps, hg, nc, 0, 0};
    }
  }
  return best;
}

// Per-sequence plan from a host copy of the context lengths. Sequence n
// (np_n pages) gets ns_n splits so that no CTA holds much more than T
// head-pages, T the smallest value (not below the average per resident CTA)
// for which the CTAs of split sequences fit in one wave: those CTAs wait for
// one another in the split merge, the others never wait, so the launch may
// take several waves and cannot deadlock. Items (one per (sequence, split),
// each launched for every kv-head group) are ordered longest first, so that
// the block scheduler's waves balance (longest-processing-time order). Cost
// of a plan: max(total work / resident CTAs, the largest CTA) in head-pages
// plus a fixed 8 per CTA; the cheapest kv-head group size wins. Returns false
// when the plan does not fit the parameter block (then the uniform plan runs).
bool plan_lengths(const kvq_attn_desc* d, int dev, int app, SplitPlan* out, uint2* items) {
  const int B = d->batch;
  const int32_t* lens = d->context_lens_host;
  if (!lens || B < 1 || B > kvq::kMaxPlanItems) return false;
  const int nc = cols_for(d->num_q_heads / d->num_kv_heads);
  const int sms = sm_count(dev);
  if (sms < 1) return false;
  static thread_local std::vector<int> np, ns;
  static thread_local std::vector<std::pair<long long, int>> order;
  np.assign(B, 0);
  ns.assign(B, 1);
  long long max_np = 0;
  for (int n = 0; n < B; ++n) {
    long long c = lens[n];
    if (c < 0) c = 0;
    if (c > (long long)d->max_pages_per_seq * KVQ_PAGE_SIZE) c = (long long)d->max_pages_per_seq * KVQ_PAGE_SIZE;
    np[n] = (int)((c + KVQ_PAGE_SIZE - 1) / KVQ_PAGE_SIZE);
    if (np[n] > max_np) max_np = np[n];
  }
  long long best_cost = LLONG_MAX;
  int best_hg = 0;
  long long best_T = 0;
  for (int hg = 1; hg <= 4; hg <<= 1) {
    if (d->num_kv_heads % hg != 0 || hg * nc > 4) continue;
    const int per_sm = decode_ctas_per_sm(dev, d->head_dim, d->hadamard_block, hg, nc, app);
    if (per_sm < 1) continue;
    const long long slots = (long long)per_sm * sms;
    const long long groups = d->num_kv_heads / hg;
    long long total = 0;
    for (int n = 0; n < B; ++n) total += groups * ((long long)np[n] * hg + 8);
    // splits of sequence n at threshold T; the merge waits need their CTAs in one wave
    auto splits = [&](int n, long long T) {
      const long long w = (long long)np[n] * hg;
      long long k = (w + T - 1) / T;
      long long cap = np[n] / 4;  // at least 4 pages per split
      if (cap > kvq::kMaxSplits) cap = kvq::kMaxSplits;
      if (k > cap) k = cap;
      return k < 1 ? 1LL : k;
    };
    auto fits = [&](long long T) {
      long long in_merges = 0, n_items = 0;
      for (int n = 0; n < B; ++n) {
        const long long k = splits(n, T);
        n_items += k;
        if (k > 1) in_merges += k;
      }
      return groups * in_merges <= slots && n_items <= kvq::kMaxPlanItems;
    };
    long long lo = total / slots, hi = max_np * hg + 1;
    if (lo < 1) lo = 1;
    if (lo > hi) lo = hi;
    if (!fits(hi)) continue;
    while (lo < hi) {
      const long long mid = lo + (hi - lo) / 2;
      if (fits(mid)) hi = mid;
      else lo = mid + 1;
    }
    long long largest = 0;
    for (int n = 0; n < B; ++n) {
      const long long k = splits(n, lo);
      const long long w = ((long long)np[n] + k - 1) / k * hg + 8;
      if (w > largest) largest = w;
    }
    const long long cost = std::max((total + slots - 1) / slots, largest);
    if (cost < best_cost) {
      best_cost = cost;
      best_hg = hg;
      best_T = lo;
    }
  }
  if (best_hg == 0) return false;
  const int hg = best_hg;
  order.clear();
  int part_slots = 0;
  for (int n = 0; n < B; ++n) {
    const long long w = (long long)np[n] * hg;
    long long k = (w + best_T - 1) / best_T;
    long long cap = np[n] / 4;
    if (cap > kvq::kMaxSplits) cap = kvq::kMaxSplits;
    if (k > cap) k = cap;
    ns[n] = (int)(k < 1 ? 1 : k);
    const int pps = np[n] > 0 ? (np[n] + ns[n] - 1) / ns[n] : 1;
    if (pps > 0xFFFF) return false;
    for (int sp = 0; sp < ns[n]; ++sp) {
      const long long pages = std::min<long long>(pps, std::max<long long>(np[n] - (long long)sp * pps, 0));
      order.push_back({pages, (n << 8) | sp});
    }
  }
  if ((int)order.size() > kvq::kMaxPlanItems) return false;
  std::stable_sort(order.begin(), order.end(),
                   [](const std::pair<long long, int>& a, const std::pair<long long, int>& b) { return a.first > b.first; });
  // partial-result slots: the splits of one sequence take consecutive slots
  static thread_local std::vector<int> base;
  base.assign(B, 0);
  for (int n = 0; n < B; ++n)
    if (ns[n] > 1) {
      base[n] = part_slots;
      part_slots += ns[n];
    }
  if (part_slots > 0xFFFF) return false;
  for (size_t i = 0; i < order.size(); ++i) {
    const int n = order[i].second >> 8, sp = order[i].second & 0xFF;
    const int pps = np[n] > 0 ? (np[n] + ns[n] - 1) / ns[n] : 1;
    items[i] = make_uint2((uint32_t)n | ((uint32_t)sp << 16) | ((uint32_t)ns[n] << 24),
                          (uint32_t)base[n] | ((uint32_t)pps << 16));
  }
  *out = {0, 0, hg, nc, (int)order.size(), part_slots};
  return true;
}

// Workspace of a per-sequence plan: its partial slots, each holding every
// query head's row.
size_t planned_workspace_bytes(const kvq_attn_desc* d, const SplitPlan& plan) {
  return (size_t)plan.part_slots * d->num_q_heads * (d->head_dim + 4) * sizeof(uint32_t);
}

// Bound on planned_workspace_bytes over every context-length vector: the
// CTAs of split sequences fit in one wave, so at most resident/groups slots.
size_t planned_workspace_bound(const kvq_attn_desc* d, int dev, int app) {
  const int nc = cols_for(d->num_q_heads / d->num_kv_heads);
  const int sms = sm_count(dev);
  size_t best = 0;
  for (int hg = 1; hg <= 4; hg <<= 1) {
    if (d->num_kv_heads % hg != 0 || hg * nc > 4) continue;
    const int per_sm = decode_ctas_per_sm(dev, d->head_dim, d->hadamard_block, hg, nc, app);
    if (per_sm < 1 || sms < 1) continue;
    const size_t slots = (size_t)per_sm * sms * hg / d->num_kv_heads;
    best = std::max(best, slots * d->num_q_heads * (d->head_dim + 4) * sizeof(uint32_t));
  }
  return best;
}

// A randomized-Hadamard sign mask: zero without a rotation, no bit at or
// above D.
bool valid_signs(const uint32_t (&sg)[4], int D, int b) {
  for (int w = 0; w < 4; ++w) {
    const uint32_t allowed = (b == 0) ? 0u : (D >= 32 * (w + 1)) ? 0xFFFFFFFFu : (D <= 32 * w) ? 0u
                                                                  : ((1u << (D - 32 * w)) - 1u);
    if (sg[w] & ~allowed) return false;
  }
  return true;
}

kvq_status check_attn_desc(const kvq_attn_desc* d) {
  if (!d) return KVQ_ERR_INVALID_ARG;
  if (d->batch < 0 || d->num_q_heads < 1 || d->num_kv_heads < 1 || d->num_pages < 1 ||
      d->max_pages_per_seq < 1 || d->page_size != KVQ_PAGE_SIZE)
    return KVQ_ERR_INVALID_ARG;
  if (d->batch > 65535 || d->num_kv_heads > 65535) return KVQ_ERR_INVALID_ARG;
  if (d->num_q_heads % d->num_kv_heads != 0) return KVQ_ERR_INVALID_ARG;
  if (d->max_pages_per_seq > INT_MAX / KVQ_PAGE_SIZE) return KVQ_ERR_INVALID_ARG;
  if (!(d->softmax_scale >= 0.0f) || !std::isfinite(d->softmax_scale)) return KVQ_ERR_INVALID_ARG;
  if (d->out_dtype != 0 && d->out_dtype != 1) return KVQ_ERR_INVALID_ARG;
  if ((d->flags & ~KVQ_ATTN_INPUTS_READY) != 0) return KVQ_ERR_INVALID_ARG;
  const int G = d->num_q_heads / d->num_kv_heads;
  if (d->head_dim != 64 && d->head_dim != 128) return KVQ_ERR_UNSUPPORTED;
  if (G != 1 && G != 2 && G != 4 && G != 8) return KVQ_ERR_UNSUPPORTED;
  if (!valid_block(d->head_dim, d->hadamard_block)) return KVQ_ERR_UNSUPPORTED;
  if (!valid_signs(d->hadamard_signs, d->head_dim, d->hadamard_block)) return KVQ_ERR_INVALID_ARG;
  return KVQ_OK;
}

// Workspace: the splits' partial results, slot-major ([slot][Hq] rows of
// D + 4 words: O + Z, M, L, padding; the uniform plan's slot of split j of
// sequence n is n * n_splits + j), each word stored as ~bits so that zero
// means "not written".
size_t workspace_bytes_for(const kvq_attn_desc* d, const SplitPlan& plan) {
  if (plan.n_items > 0) return planned_workspace_bytes(d, plan);
  if (plan.n_splits <= 1 || d->batch == 0) return 0;
  const size_t G = (size_t)(d->num_q_heads / d->num_kv_heads);
  return (size_t)d->batch * d->num_kv_heads * plan.n_splits * G * (d->head_dim + 4) * sizeof(uint32_t);
}

template <int D, int BLK, int NC, bool APP>
cudaError_t launch_decode_instance(const kvq::AttnParams& p, int hg, int smem, cudaStream_t s) {
  const dim3 grid = p.n_items > 0 ? dim3(p.Hkv / hg, p.n_items, 1) : dim3(p.n_splits, p.Hkv / hg, p.B);
  const dim3 block(32 * kvq::attn_warps(NC));
  cudaError_t e = cudaErrorInvalidValue;
  if constexpr (NC == 1) {
    if (hg == 4) e = launch_pdl(kvq::kvq_decode_kernel<D, BLK, 4, NC, APP>, grid, block, smem, s, p);
  }
  if (hg == 2) e = launch_pdl(kvq::kvq_decode_kernel<D, BLK, 2, NC, APP>, grid, block, smem, s, p);
  else if (hg == 1) e = launch_pdl(kvq::kvq_decode_kernel<D, BLK, 1, NC, APP>, grid, block, smem, s, p);
  if (e != cudaSuccess) cudaGetLastError();
  return e;
}

template <int D, int BLK>
kvq_status launch_attn(const kvq::AttnParams& p, const SplitPlan& plan, int dev, cudaStream_t s) {
  const int app = p.slots_new != nullptr;
  if (decode_ctas_per_sm(dev, D, BLK, plan.hg, plan.nc, app) < 1) return KVQ_ERR_CUDA;
  const int smem = decode_smem_bytes(D, plan.hg, plan.nc);
  cudaError_t e;
  if (app)
    e = plan.nc == 2 ? launch_decode_instance<D, BLK, 2, true>(p, plan.hg, smem, s)
                     : launch_decode_instance<D, BLK, 1, true>(p, plan.hg, smem, s);
  else
    e = plan.nc == 2 ? launch_decode_instance<D, BLK, 2, false>(p, plan.hg, smem, s)
                     : launch_decode_instance<D, BLK, 1, false>(p, plan.hg, smem, s);
  return e == cudaSuccess ? KVQ_OK : KVQ_ERR_CUDA;
}

template <int D>
kvq_status dispatch_attn(const kvq::AttnParams& p, int b, const SplitPlan& plan, int dev, cudaStream_t s) {
  switch (b) {
    case 0: return launch_attn<D, 0>(p, plan, dev, s);
    case 32: return launch_attn<D, 32>(p, plan, dev, s);
    case 64: return launch_attn<D, 64>(p, plan, dev, s);
    case 128:
      if constexpr (D >= 128) return launch_attn<D, 128>(p, plan, dev, s);
      return KVQ_ERR_UNSUPPORTED;
    default: return KVQ_ERR_UNSUPPORTED;
  }
}
// Chunked prefill on the tensor cores (D = 64, 128).
template <int D, int BLK>
kvq_status launch_prefill(const kvq::PrefillParams& p, int max_q_len, int dev, cudaStream_t s) {
  if (dev < 0 || dev >= kMaxDevices) return KVQ_ERR_UNSUPPORTED;
  auto kern = kvq::kvq_prefill_kernel<D, BLK>;
  constexpr int smem = kvq::PfSmem<D>::kTotal;
  static std::atomic<int> ready[kMaxDevices];
  if (!ready[dev].load(std::memory_order_relaxed)) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess) {
      cudaGetLastError();
      return KVQ_ERR_CUDA;
    }
    ready[dev].store(1, std::memory_order_relaxed);
  }
  const int tq = kvq::kPfRows / p.G;
  const dim3 grid((unsigned)(((long long)max_q_len + tq - 1) / tq), p.Hkv, p.B);
  if (launch_pdl(kern, grid, dim3(kvq::kPfThreads), smem, s, p) != cudaSuccess) {
    cudaGetLastError();
    return KVQ_ERR_CUDA;
  }
  return KVQ_OK;
}

}  // namespace

extern "C" {

kvq_status kv_quant_write(const void* k, const void* v, const int64_t* slot_mapping,
                          const int32_t* page_table, uint8_t* cache, void* scales, void* zeros,
                          int32_t hadamard_block, const kvq_write_desc* desc, void* stream) {
  (void)page_table;  // placement is decided by slot_mapping alone
  if (!desc) return KVQ_ERR_INVALID_ARG;
  const kvq_write_desc& d = *desc;
  if (d.num_tokens < 0 || d.num_kv_heads < 1 || d.page_size != KVQ_PAGE_SIZE || d.num_pages < 1)
    return KVQ_ERR_INVALID_ARG;
  if (d.head_dim != 64 && d.head_dim != 128) return KVQ_ERR_UNSUPPORTED;
  if (!valid_block(d.head_dim, hadamard_block)) return KVQ_ERR_UNSUPPORTED;
  if (!valid_signs(d.hadamard_signs, d.head_dim, hadamard_block)) return KVQ_ERR_INVALID_ARG;
  if (d.num_tokens == 0) return KVQ_OK;  // nothing to do; pointers may be NULL
  if (!k || !v || !slot_mapping || !cache || !scales || !zeros) return KVQ_ERR_INVALID_ARG;
  if (!aligned(k, 16) || !aligned(v, 16) || !aligned(cache, 16) || !aligned(scales, 16) ||
      !aligned(zeros, 16) || !aligned(slot_mapping, 8))
    return KVQ_ERR_INVALID_ARG;
  const long long tiles = ((long long)d.num_tokens + 31) / 32 * d.num_kv_heads * 2;
  if (tiles > INT_MAX) return KVQ_ERR_INVALID_ARG;
  int dev = 0;
  kvq_status st = select_device_of(cache, &dev);
  if (st != KVQ_OK) return st;
  kvq::WriteParams p;
  p.k = static_cast<const uint16_t*>(k);
  p.v = static_cast<const uint16_t*>(v);
  p.slots = slot_mapping;
  p.cache = cache;
  p.scales = static_cast<uint16_t*>(scales);
  p.zeros = static_cast<uint16_t*>(zeros);
  p.T = d.num_tokens;
  p.Hkv = d.num_kv_heads;
  p.num_slots = (long long)d.num_pages * KVQ_PAGE_SIZE;
  p.num_tiles = (int)tiles;
  p.cb = hadamard_block > 0 ? (float)(1.0 / std::sqrt((double)hadamard_block)) : 1.0f;
  for (int w = 0; w < 4; ++w) p.signs[w] = d.hadamard_signs[w];
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  return d.head_dim == 64 ? dispatch_write<64>(p, hadamard_block, dev, s)
                          : dispatch_write<128>(p, hadamard_block, dev, s);
}

size_t kvq_attn_workspace_size(const kvq_attn_desc* desc) {
  if (check_attn_desc(desc) != KVQ_OK) return SIZE_MAX;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return SIZE_MAX;
  }
  if (dev < 0 || dev >= kMaxDevices) return SIZE_MAX;
  // the same workspace serves paged_decode_attn_int4 and the decode-append
  // entry point (their kernels may hold different numbers of CTAs per SM)
  size_t need = 0;
  for (int app = 0; app < 2; ++app) {
    need = std::max(need, workspace_bytes_for(desc, plan_splits(desc, dev, app)));
    if (desc->context_lens_host) need = std::max(need, planned_workspace_bound(desc, dev, app));
  }
  return need;
}

namespace {

// The new tokens of a decode-append call (all null for a plain decode).
struct AppendArgs {
  const void* k_new;
  const void* v_new;
  const int64_t* slot_mapping;
};

kvq_status decode_impl(const void* q, const uint8_t* cache, const void* scales, const void* zeros,
                       const int32_t* page_table, const int32_t* context_lens, void* out, void* workspace,
                       size_t workspace_bytes, const kvq_attn_desc* desc, void* stream, const AppendArgs& app) {
  kvq_status st = check_attn_desc(desc);
  if (st != KVQ_OK) return st;
  const kvq_attn_desc& d = *desc;
  if (d.batch == 0) return KVQ_OK;  // nothing to do; pointers may be NULL
  if (!q || !cache || !scales || !zeros || !page_table || !context_lens || !out)
    return KVQ_ERR_INVALID_ARG;
  if (!aligned(cache, 16) || !aligned(scales, 16) || !aligned(zeros, 16) || !aligned(q, 16) ||
      !aligned(page_table, 4) || !aligned(context_lens, 4) || !aligned(out, d.out_dtype ? 2 : 4))
    return KVQ_ERR_INVALID_ARG;
  int dev = 0;
  st = select_device_of(cache, &dev);
  if (st != KVQ_OK) return st;
  if (dev < 0 || dev >= kMaxDevices) return KVQ_ERR_UNSUPPORTED;
  // kernel parameters (with the per-sequence plan's items) live in static
  // storage per thread rather than on the stack: the item table is 8 KB
  static thread_local kvq::AttnParams p;
  SplitPlan plan;
  SplitPlan lp;
  const int app_mode = app.slot_mapping != nullptr;
  if (d.context_lens_host && plan_lengths(&d, dev, app_mode, &lp, p.items) &&
      (lp.part_slots == 0 || (workspace && aligned(workspace, 16) &&
                              workspace_bytes >= planned_workspace_bytes(&d, lp)))) {
    plan = lp;
  } else {
    plan = plan_splits(&d, dev, app_mode);
  }
  const size_t need = workspace_bytes_for(&d, plan);
  if (need > 0 && (!workspace || workspace_bytes < need || !aligned(workspace, 16)))
    return KVQ_ERR_WORKSPACE;
  p.n_items = plan.n_items;
  p.q = static_cast<const uint16_t*>(q);
  p.cache = cache;
  p.scales = static_cast<const uint16_t*>(scales);
  p.zeros = static_cast<const uint16_t*>(zeros);
  p.page_table = page_table;
  p.ctx_lens = context_lens;
  p.out = out;
  p.B = d.batch;
  p.Hq = d.num_q_heads;
  p.Hkv = d.num_kv_heads;
  p.G = d.num_q_heads / d.num_kv_heads;
  p.num_pages = d.num_pages;
  p.max_pages = d.max_pages_per_seq;
  p.n_splits = plan.n_splits;
  p.pages_per_split = plan.pages_per_split;
  p.ws_part = need > 0 ? static_cast<uint32_t*>(workspace) : nullptr;
  p.out_bf16 = d.out_dtype;
  p.inputs_ready = (d.flags & KVQ_ATTN_INPUTS_READY) ? 1 : 0;
  p.k_new = static_cast<const uint16_t*>(app.k_new);
  p.v_new = static_cast<const uint16_t*>(app.v_new);
  p.slots_new = app.slot_mapping;
  p.cache_w = const_cast<uint8_t*>(cache);
  p.scales_w = static_cast<uint16_t*>(const_cast<void*>(scales));
  p.zeros_w = static_cast<uint16_t*>(const_cast<void*>(zeros));
  const double cb = d.hadamard_block > 0 ? 1.0 / std::sqrt((double)d.hadamard_block) : 1.0;
  const double scale = d.softmax_scale > 0.0f ? (double)d.softmax_scale : 1.0 / std::sqrt((double)d.head_dim);
  p.qmul = (float)(cb * scale * 1.4426950408889634);  // log2(e)
  p.cb = (float)cb;
  for (int w = 0; w < 4; ++w) p.signs[w] = d.hadamard_signs[w];
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  return d.head_dim == 64 ? dispatch_attn<64>(p, d.hadamard_block, plan, dev, s)
                          : dispatch_attn<128>(p, d.hadamard_block, plan, dev, s);
}

}  // namespace

kvq_status paged_decode_attn_int4(const void* q, const uint8_t* cache, const void* scales,
                                  const void* zeros, const int32_t* page_table,
                                  const int32_t* context_lens, void* out, void* workspace,
                                  size_t workspace_bytes, const kvq_attn_desc* desc, void* stream) {
  return decode_impl(q, cache, scales, zeros, page_table, context_lens, out, workspace, workspace_bytes,
                     desc, stream, AppendArgs{nullptr, nullptr, nullptr});
}

kvq_status paged_decode_append_attn_int4(const void* q, const void* k_new, const void* v_new,
                                         const int64_t* slot_mapping, uint8_t* cache, void* scales,
                                         void* zeros, const int32_t* page_table,
                                         const int32_t* context_lens, void* out, void* workspace,
                                         size_t workspace_bytes, const kvq_attn_desc* desc, void* stream) {
  if (desc && desc->batch > 0 &&
      (!k_new || !v_new || !slot_mapping || !aligned(k_new, 16) || !aligned(v_new, 16) || !aligned(slot_mapping, 8)))
    return KVQ_ERR_INVALID_ARG;
  return decode_impl(q, cache, scales, zeros, page_table, context_lens, out, workspace, workspace_bytes,
                     desc, stream, AppendArgs{k_new, v_new, slot_mapping});
}

kvq_status paged_prefill_attn_int4(const void* q, const uint8_t* cache, const void* scales,
                                   const void* zeros, const int32_t* page_table,
                                   const int32_t* context_lens, const int32_t* q_start, int32_t max_q_len,
                                   void* out, const kvq_attn_desc* desc, void* stream) {
  kvq_status st = check_attn_desc(desc);
  if (st != KVQ_OK) return st;
  const kvq_attn_desc& d = *desc;
  if (max_q_len < 0) return KVQ_ERR_INVALID_ARG;
  if (d.batch == 0 || max_q_len == 0) return KVQ_OK;
  if (!q || !cache || !scales || !zeros || !page_table || !context_lens || !q_start || !out)
    return KVQ_ERR_INVALID_ARG;
  if (!aligned(cache, 16) || !aligned(scales, 16) || !aligned(zeros, 16) || !aligned(q, 16) ||
      !aligned(page_table, 4) || !aligned(context_lens, 4) || !aligned(q_start, 4) ||
      !aligned(out, d.out_dtype ? 2 : 4))
    return KVQ_ERR_INVALID_ARG;
  int dev = 0;
  st = select_device_of(cache, &dev);
  if (st != KVQ_OK) return st;
  kvq::PrefillParams p;
  p.q = static_cast<const uint16_t*>(q);
  p.cache = cache;
  p.scales = static_cast<const uint16_t*>(scales);
  p.zeros = static_cast<const uint16_t*>(zeros);
  p.page_table = page_table;
  p.ctx_lens = context_lens;
  p.q_start = q_start;
  p.out = out;
  p.B = d.batch;
  p.Hq = d.num_q_heads;
  p.Hkv = d.num_kv_heads;
  p.G = d.num_q_heads / d.num_kv_heads;
  p.num_pages = d.num_pages;
  p.max_pages = d.max_pages_per_seq;
  p.out_bf16 = d.out_dtype;
  const double cb = d.hadamard_block > 0 ? 1.0 / std::sqrt((double)d.hadamard_block) : 1.0;
  const double scale = d.softmax_scale > 0.0f ? (double)d.softmax_scale : 1.0 / std::sqrt((double)d.head_dim);
  p.qmul = (float)(cb * scale * 1.4426950408889634);  // log2(e)
  p.cb = (float)cb;
  for (int w = 0; w < 4; ++w) p.signs[w] = d.hadamard_signs[w];
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  switch (d.hadamard_block) {
    case 0: return d.head_dim == 64 ? launch_prefill<64, 0>(p, max_q_len, dev, s)
                                    : launch_prefill<128, 0>(p, max_q_len, dev, s);
    case 32: return d.head_dim == 64 ? launch_prefill<64, 32>(p, max_q_len, dev, s)
                                     : launch_prefill<128, 32>(p, max_q_len, dev, s);
    case 64: return d.head_dim == 64 ? launch_prefill<64, 64>(p, max_q_len, dev, s)
                                     : launch_prefill<128, 64>(p, max_q_len, dev, s);
    case 128: return launch_prefill<128, 128>(p, max_q_len, dev, s);
    default: return KVQ_ERR_UNSUPPORTED;
  }
}

// ---------------------------------------------------------------------------
// OScaR variant
// ---------------------------------------------------------------------------
}  // extern "C"

namespace {

// Persistent write grid: at most one wave of resident CTAs.
template <int BLK>
kvq_status launch_oscar_write(const kvq::OscarWriteParams& p, int dev, cudaStream_t s) {
  static std::atomic<int> occ[kMaxDevices];
  constexpr int smem = kvq::OscarWriteSmem::kTotal;
  auto kern = kvq::kvq_oscar_write_kernel<128, BLK>;
  const int per_sm = resident_ctas(kern, occ, dev, kvq::kOscarWriteWarps * 32, smem);
  const long long units = (long long)p.P * p.Hkv;
  const long long need = (units + kvq::kOscarWriteWarps - 1) / kvq::kOscarWriteWarps;
  const long long wave = (long long)per_sm * std::max(sm_count(dev), 1);
  const dim3 grid((unsigned)std::min(need, wave));
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess ||
      launch_pdl(kern, grid, dim3(kvq::kOscarWriteWarps * 32), smem, s, p) != cudaSuccess) {
    cudaGetLastError();
    return KVQ_ERR_CUDA;
  }
  return KVQ_OK;
}

kvq_status check_oscar_desc(const kvq_oscar_attn_desc* d) {
  if (!d) return KVQ_ERR_INVALID_ARG;
  if (d->batch < 0 || d->batch > 65535 || d->num_q_heads < 1 || d->num_kv_heads < 1 ||
      d->num_kv_heads > 65535 || d->num_pages < 1 || d->max_pages_per_seq < 1 ||
      d->max_pages_per_seq > INT_MAX / KVQ_PAGE_SIZE - 1)
    return KVQ_ERR_INVALID_ARG;
  if (d->num_q_heads % d->num_kv_heads != 0) return KVQ_ERR_INVALID_ARG;
  if ((long long)d->batch * d->num_q_heads > INT_MAX) return KVQ_ERR_INVALID_ARG;  // one merge CTA per row
  if (!(d->softmax_scale >= 0.0f) || !std::isfinite(d->softmax_scale)) return KVQ_ERR_INVALID_ARG;
  if (d->out_dtype != 0 && d->out_dtype != 1) return KVQ_ERR_INVALID_ARG;
  const int G = d->num_q_heads / d->num_kv_heads;
  if (d->head_dim != 128 || (G != 1 && G != 2 && G != 4)) return KVQ_ERR_UNSUPPORTED;
  if (!valid_block(d->head_dim, d->hadamard_block)) return KVQ_ERR_UNSUPPORTED;
  return KVQ_OK;
}

// Splits per (sequence, kv head): enough to fill the device's resident decode
// CTAs once, and at most 64 pages per split (short CTAs balance sequences of
// different lengths over several waves); at least two pages per split.
void oscar_plan(const kvq_oscar_attn_desc* d, int dev, int* ns, int* pps) {
  static std::atomic<int> occ[kMaxDevices];
  int per_sm = 1;
  if (dev >= 0 && dev < kMaxDevices)
    per_sm = resident_ctas(kvq::kvq_oscar_decode_kernel<128, 128>, occ, dev, kvq::kOscarWarps * 32,
                           kvq::OscarSmem<128>::kTotal);
  const long long slots = (long long)per_sm * std::max(sm_count(dev), 1);
  const long long units = std::max<long long>((long long)d->batch * d->num_kv_heads, 1);
  long long n = std::max<long long>(slots / units, (d->max_pages_per_seq + 63) / 64);
  const long long cap = std::max<long long>(d->max_pages_per_seq / 2, 1);
  if (n > cap) n = cap;
  if (n > kvq::kMaxSplits) n = kvq::kMaxSplits;
  if (n < 1) n = 1;
  const long long p = (d->max_pages_per_seq + n - 1) / n;
  *ns = (int)((d->max_pages_per_seq + p - 1) / p);
  *pps = (int)p;
}

size_t oscar_ws_bytes(const kvq_oscar_attn_desc* d, int ns) {
  const size_t G = (size_t)(d->num_q_heads / d->num_kv_heads);
  return (size_t)d->batch * d->num_kv_heads * ns * G * (d->head_dim + 2) * sizeof(float);
}

template <int BLK>
kvq_status launch_oscar_decode(const kvq::OscarAttnParams& p, cudaStream_t s) {
  constexpr int smem = kvq::OscarSmem<128>::kTotal;
  auto kern = kvq::kvq_oscar_decode_kernel<128, BLK>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess ||
      launch_pdl(kern, dim3(p.n_splits, p.Hkv, p.B), dim3(kvq::kOscarWarps * 32), smem, s, p) != cudaSuccess ||
      launch_pdl(kvq::kvq_oscar_combine_kernel<128, BLK>, dim3((unsigned)((long long)p.B * p.Hq)), dim3(128), 0,
                 s, p) != cudaSuccess) {
    cudaGetLastError();
    return KVQ_ERR_CUDA;
  }
  return KVQ_OK;
}

}  // namespace

extern "C" {

kvq_status kv_quant_write_oscar(const void* k, const void* v, const int32_t* page_ids, uint8_t* cache,
                                void* kmeta, void* tmeta, int32_t hadamard_block,
                                const kvq_oscar_write_desc* desc, void* stream) {
  if (!desc) return KVQ_ERR_INVALID_ARG;
  const kvq_oscar_write_desc& d = *desc;
  if (d.num_groups < 0 || d.num_kv_heads < 1 || d.num_pages < 1) return KVQ_ERR_INVALID_ARG;
  // units (group, head) and unit + grid stride must stay in int
  if ((long long)d.num_groups * d.num_kv_heads > INT_MAX / 2) return KVQ_ERR_INVALID_ARG;
  if (d.head_dim != 128 || !valid_block(d.head_dim, hadamard_block)) return KVQ_ERR_UNSUPPORTED;
  if (d.num_groups == 0) return KVQ_OK;
  if (!k || !v || !page_ids || !cache || !kmeta || !tmeta) return KVQ_ERR_INVALID_ARG;
  if (!aligned(k, 16) || !aligned(v, 16) || !aligned(cache, 16) || !aligned(kmeta, 16) || !aligned(tmeta, 16) ||
      !aligned(page_ids, 4))
    return KVQ_ERR_INVALID_ARG;
  int dev = 0;
  kvq_status st = select_device_of(cache, &dev);
  if (st != KVQ_OK) return st;
  kvq::OscarWriteParams p;
  p.k = static_cast<const uint16_t*>(k);
  p.v = static_cast<const uint16_t*>(v);
  p.page_ids = page_ids;
  p.cache = cache;
  p.kmeta = static_cast<uint16_t*>(kmeta);
  p.tmeta = static_cast<uint16_t*>(tmeta);
  p.P = d.num_groups;
  p.Hkv = d.num_kv_heads;
  p.num_pages = d.num_pages;
  p.cb = hadamard_block > 0 ? (float)(1.0 / std::sqrt((double)hadamard_block)) : 1.0f;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  switch (hadamard_block) {
    case 0: return launch_oscar_write<0>(p, dev, s);
    case 32: return launch_oscar_write<32>(p, dev, s);
    case 64: return launch_oscar_write<64>(p, dev, s);
    default: return launch_oscar_write<128>(p, dev, s);
  }
}

size_t kvq_oscar_workspace_size(const kvq_oscar_attn_desc* desc) {
  if (check_oscar_desc(desc) != KVQ_OK) return SIZE_MAX;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return SIZE_MAX;
  }
  int ns = 1, pps = 1;
  oscar_plan(desc, dev, &ns, &pps);
  return oscar_ws_bytes(desc, ns);
}

kvq_status paged_decode_attn_oscar(const void* q, const uint8_t* cache, const void* kmeta, const void* tmeta,
                                   const int32_t* page_table, const int32_t* context_lens, const void* k_tail,
                                   const void* v_tail, void* out, void* workspace, size_t workspace_bytes,
                                   const kvq_oscar_attn_desc* desc, void* stream) {
  kvq_status st = check_oscar_desc(desc);
  if (st != KVQ_OK) return st;
  const kvq_oscar_attn_desc& d = *desc;
  if (d.batch == 0) return KVQ_OK;
  if (!q || !cache || !kmeta || !tmeta || !page_table || !context_lens || !k_tail || !v_tail || !out)
    return KVQ_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(cache, 16) || !aligned(kmeta, 16) || !aligned(tmeta, 16) ||
      !aligned(k_tail, 16) || !aligned(v_tail, 16) || !aligned(page_table, 4) || !aligned(context_lens, 4) ||
      !aligned(out, d.out_dtype ? 8 : 16))
    return KVQ_ERR_INVALID_ARG;
  int dev = 0;
  st = select_device_of(cache, &dev);
  if (st != KVQ_OK) return st;
  int ns = 1, pps = 1;
  oscar_plan(&d, dev, &ns, &pps);
  if (!workspace || !aligned(workspace, 16) || workspace_bytes < oscar_ws_bytes(&d, ns)) return KVQ_ERR_WORKSPACE;
  kvq::OscarAttnParams p;
  p.q = static_cast<const uint16_t*>(q);
  p.cache = cache;
  p.kmeta = static_cast<const uint16_t*>(kmeta);
  p.tmeta = static_cast<const uint16_t*>(tmeta);
  p.page_table = page_table;
  p.ctx_lens = context_lens;
  p.k_tail = static_cast<const uint16_t*>(k_tail);
  p.v_tail = static_cast<const uint16_t*>(v_tail);
  p.ws = static_cast<float*>(workspace);
  p.out = out;
  p.B = d.batch;
  p.Hq = d.num_q_heads;
  p.Hkv = d.num_kv_heads;
  p.G = d.num_q_heads / d.num_kv_heads;
  p.num_pages = d.num_pages;
  p.max_pages = d.max_pages_per_seq;
  p.n_splits = ns;
  p.pages_per_split = pps;
  p.out_bf16 = d.out_dtype;
  const double cb = d.hadamard_block > 0 ? 1.0 / std::sqrt((double)d.hadamard_block) : 1.0;
  const double scale = d.softmax_scale > 0.0f ? (double)d.softmax_scale : 1.0 / std::sqrt((double)d.head_dim);
  p.qmul = (float)(cb * scale * 1.4426950408889634);
  p.qraw = (float)(scale * 1.4426950408889634);
  p.cb = (float)cb;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  switch (d.hadamard_block) {
    case 0: return launch_oscar_decode<0>(p, s);
    case 32: return launch_oscar_decode<32>(p, s);
    case 64: return launch_oscar_decode<64>(p, s);
    default: return launch_oscar_decode<128>(p, s);
  }
}

kvq_status kvq_selftest_bounded_wait(int32_t which, void* stream) {
  if (which != 0 && which != 1) return KVQ_ERR_INVALID_ARG;
  kvq::kvq_selftest_wait_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(which);
  if (cudaGetLastError() != cudaSuccess) return KVQ_ERR_CUDA;
  return KVQ_OK;
}

kvq_status kvq_selftest_occupy(int32_t ctas, int32_t microseconds, void* stream) {
  if (ctas < 1 || ctas > 65535 || microseconds < 0 || microseconds > 1000000) return KVQ_ERR_INVALID_ARG;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return KVQ_ERR_CUDA;
  }
  int smem_max = 0;
  if (cudaDeviceGetAttribute(&smem_max, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess) {
    cudaGetLastError();
    return KVQ_ERR_CUDA;
  }
  const int smem = smem_max - 8 * 1024;  // most of an SM's shared memory
  if (cudaFuncSetAttribute(kvq::kvq_selftest_occupy_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) !=
      cudaSuccess) {
    cudaGetLastError();
    return KVQ_ERR_CUDA;
  }
  kvq::kvq_selftest_occupy_kernel<<<ctas, 32, smem, static_cast<cudaStream_t>(stream)>>>(
      1000ull * (unsigned long long)microseconds);
  if (cudaGetLastError() != cudaSuccess) return KVQ_ERR_CUDA;
  return KVQ_OK;
}

kvq_status kvq_set_device(int32_t device) {
  if (device < 0) return KVQ_ERR_INVALID_ARG;
  if (cudaSetDevice(device) != cudaSuccess) {
    cudaGetLastError();
    return KVQ_ERR_CUDA;
  }
  return KVQ_OK;
}

const char* kvq_status_string(int32_t status) {
  switch (status) {
    case KVQ_OK: return "KVQ_OK";
    case KVQ_ERR_INVALID_ARG: return "KVQ_ERR_INVALID_ARG";
    case KVQ_ERR_UNSUPPORTED: return "KVQ_ERR_UNSUPPORTED";
    case KVQ_ERR_OUT_OF_RANGE: return "KVQ_ERR_OUT_OF_RANGE";
    case KVQ_ERR_WORKSPACE: return "KVQ_ERR_WORKSPACE";
    case KVQ_ERR_TIMEOUT: return "KVQ_ERR_TIMEOUT";
    case KVQ_ERR_CUDA: return "KVQ_ERR_CUDA";
    default: return "KVQ_ERR_UNKNOWN";
  }
}

int32_t kvq_abi_version(void) { return KVQ_ABI_VERSION; }

}  // extern "C"

// ---------------------------------------------------------------------------
// paged_decode_attn_int4_static_ws: the decode step without a caller-provided
// workspace, for callers that cannot allocate device memory. The split-K
// scratch is this file-scope array (one per device that loads the library).
// ---------------------------------------------------------------------------
static __device__ __align__(256) unsigned char g_static_workspace[KVQ_STATIC_WORKSPACE_BYTES];

namespace {

std::mutex g_static_ws_mutex;
void* g_static_ws_ptr[kMaxDevices] = {};
CUcontext g_static_ws_ctx[kMaxDevices] = {};

typedef CUresult (*CtxGetFn)(CUcontext*);

CtxGetFn ctx_query() {
  static std::atomic<CtxGetFn> fn{nullptr};
  CtxGetFn f = fn.load(std::memory_order_acquire);
  if (f) return f;
  void* raw = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &raw, cudaEnableDefault, &q) != cudaSuccess ||
      q != cudaDriverEntryPointSuccess || !raw) {
    cudaGetLastError();
    return nullptr;
  }
  f = reinterpret_cast<CtxGetFn>(raw);
  fn.store(f, std::memory_order_release);
  return f;
}

// Device address of g_static_workspace on `dev` (which must be current). In
// host code the array's name is only a host-side stand-in, so the address is
// looked up with cudaGetSymbolAddress once per device - again whenever the
// device's current context is another one than at the last lookup (after a
// cudaDeviceReset the module, and the array, may be loaded elsewhere).
kvq_status static_workspace_on(int dev, void** out) {
  std::lock_guard<std::mutex> lock(g_static_ws_mutex);
  CtxGetFn get = ctx_query();
  CUcontext ctx = nullptr;
  if (get && get(&ctx) != CUDA_SUCCESS) ctx = nullptr;
  if (!g_static_ws_ptr[dev] || ctx != g_static_ws_ctx[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_static_workspace) != cudaSuccess || p == nullptr) {
      cudaGetLastError();
      return KVQ_ERR_CUDA;
    }
    g_static_ws_ptr[dev] = p;
    g_static_ws_ctx[dev] = ctx;
  }
  *out = g_static_ws_ptr[dev];
  return KVQ_OK;
}

}  // namespace

extern "C" kvq_status paged_decode_attn_int4_static_ws(const void* q, const uint8_t* cache,
                                                       const void* scales, const void* zeros,
                                                       const int32_t* page_table,
                                                       const int32_t* context_lens, void* out,
                                                       const kvq_attn_desc* desc, void* stream) {
  kvq_status st = check_attn_desc(desc);
  if (st != KVQ_OK) return st;
  if (desc->batch == 0) return KVQ_OK;
  if (!cache || !aligned(cache, 16)) return KVQ_ERR_INVALID_ARG;
  int dev = 0;
  st = select_device_of(cache, &dev);  // makes the cache's device current
  if (st != KVQ_OK) return st;
  if (dev < 0 || dev >= kMaxDevices) return KVQ_ERR_UNSUPPORTED;
  const size_t need = workspace_bytes_for(desc, plan_splits(desc, dev, 0));
  if (need > KVQ_STATIC_WORKSPACE_BYTES) return KVQ_ERR_WORKSPACE;
  void* ws = nullptr;
  st = static_workspace_on(dev, &ws);
  if (st != KVQ_OK) return st;
  // a per-sequence plan (host lengths given) runs when its partials fit too
  return paged_decode_attn_int4(q, cache, scales, zeros, page_table, context_lens, out, ws,
                                (size_t)KVQ_STATIC_WORKSPACE_BYTES, desc, stream);
}

extern "C" kvq_status kvq_get_device_error(void* stream) {
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(st) != cudaSuccess) {
    cudaGetLastError();
    return KVQ_ERR_CUDA;
  }
  int v = 0, zero = 0;
  if (cudaMemcpyFromSymbol(&v, kvq::g_device_error, sizeof(int)) != cudaSuccess ||
      cudaMemcpyToSymbol(kvq::g_device_error, &zero, sizeof(int)) != cudaSuccess) {
    cudaGetLastError();
    return KVQ_ERR_CUDA;
  }
  if (v == KVQ_ERR_TIMEOUT) {
    // words that arrived after a merge gave up may remain in the static
    // split-K array, which no caller can reach: clear it
    int dev = 0;
    void* ws = nullptr;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices ||
        static_workspace_on(dev, &ws) != KVQ_OK ||
        cudaMemsetAsync(ws, 0, KVQ_STATIC_WORKSPACE_BYTES, st) != cudaSuccess ||
        cudaStreamSynchronize(st) != cudaSuccess) {
      cudaGetLastError();
      return KVQ_ERR_CUDA;
    }
  }
  return static_cast<kvq_status>(v);
}

extern "C" size_t kvq_static_workspace_nonzero(void) {
  static unsigned char host[KVQ_STATIC_WORKSPACE_BYTES];
  static std::mutex m;
  std::lock_guard<std::mutex> lock(m);
  if (cudaMemcpyFromSymbol(host, g_static_workspace, KVQ_STATIC_WORKSPACE_BYTES) != cudaSuccess) {
    cudaGetLastError();
    return SIZE_MAX;
  }
  size_t n = 0;
  for (size_t i = 0; i < KVQ_STATIC_WORKSPACE_BYTES; ++i) n += host[i] != 0;
  return n;
}
