// kvq_api.cu - the C ABI declared in include/kvq.h: argument checks, device
// selection, grid sizing and kernel dispatch. One translation unit holds every
// kernel, so the device error word is a single symbol per device.
#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>
#include <mutex>
#include <climits>
#include <cmath>
#include <cstdint>

#include "../../include/kvq.h"
#include "kvq_decode.cuh"
#include "kvq_write.cuh"

namespace {

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
template <int D, int BLK>
kvq_status launch_write(const kvq::WriteParams& p, int dev, cudaStream_t s) {
  auto kern = kvq::kvq_write_kernel<D, BLK>;
  constexpr int smem = kvq::write_smem_bytes<D>();
  const int threads = kvq::kWriteWarps * 32;
  static std::atomic<int> occ[kMaxDevices];
  const int per_sm = resident_ctas(kern, occ, dev, threads, smem);
  const long long need = (p.num_tiles + kvq::kWriteWarps - 1) / kvq::kWriteWarps;
  const long long cap = (long long)per_sm * sm_count(dev);
  const int blocks = (int)(need < cap ? need : cap);
  kern<<<blocks, threads, smem, s>>>(p);
  return cudaGetLastError() == cudaSuccess ? KVQ_OK : KVQ_ERR_CUDA;
}

template <int D>
kvq_status dispatch_write(const kvq::WriteParams& p, int b, int dev, cudaStream_t s) {
  switch (b) {
    case 0: return launch_write<D, 0>(p, dev, s);
    case 32: return launch_write<D, 32>(p, dev, s);
    case 64: return launch_write<D, 64>(p, dev, s);
    case 128:
      if constexpr (D >= 128) return launch_write<D, 128>(p, dev, s);
      return KVQ_ERR_UNSUPPORTED;
    default: return KVQ_ERR_UNSUPPORTED;
  }
}

// ---------------------------------------------------------------------------
// paged_decode_attn_int4
// ---------------------------------------------------------------------------
struct SplitPlan {
  int n_splits;         // CTAs per (sequence, kv-head group)
  int pages_per_split;
  int cluster;          // CTAs per thread-block cluster (divides n_splits)
  int n_parts;          // clusters per (sequence, kv-head group) = partials in the workspace
  int hg;               // kv heads per CTA
};

// kv heads served by one CTA: 4, 2 or 1, whichever largest divides Hkv.
int heads_per_cta(int Hkv) { return (Hkv % 4 == 0) ? 4 : (Hkv % 2 == 0) ? 2 : 1; }

int inst_slot(int D, int b, int hg) {
  const int bi = (b == 0) ? 0 : (b == 32) ? 1 : (b == 64) ? 2 : 3;
  const int hi = (hg == 4) ? 2 : (hg == 2) ? 1 : 0;
  return ((D == 64) ? 0 : 12) + bi * 3 + hi;
}
constexpr int kInstSlots = 24;

template <int D, int BLK>
const void* decode_kernel_ptr(int hg) {
  if (hg == 4) return reinterpret_cast<const void*>(kvq::kvq_decode_kernel<D, BLK, 4>);
  if (hg == 2) return reinterpret_cast<const void*>(kvq::kvq_decode_kernel<D, BLK, 2>);
  return reinterpret_cast<const void*>(kvq::kvq_decode_kernel<D, BLK, 1>);
}

const void* decode_kernel_for(int D, int b, int hg) {
  if (D == 64) {
    if (b == 0) return decode_kernel_ptr<64, 0>(hg);
    if (b == 32) return decode_kernel_ptr<64, 32>(hg);
    if (b == 64) return decode_kernel_ptr<64, 64>(hg);
    return nullptr;
  }
  if (b == 0) return decode_kernel_ptr<128, 0>(hg);
  if (b == 32) return decode_kernel_ptr<128, 32>(hg);
  if (b == 64) return decode_kernel_ptr<128, 64>(hg);
  if (b == 128) return decode_kernel_ptr<128, 128>(hg);
  return nullptr;
}

int decode_smem_bytes(int D) {
  return D == 64 ? kvq::AttnSmem<64>::kTotal : kvq::AttnSmem<128>::kTotal;
}

// Opt the decode kernel instance into its dynamic shared memory (once per
// device and instance).
bool prepare_decode_kernel(int dev, int D, int b, int hg) {
  static std::atomic<int> done[kMaxDevices][kInstSlots];
  const int slot = inst_slot(D, b, hg);
  if (done[dev][slot].load(std::memory_order_relaxed)) return true;
  const void* k = decode_kernel_for(D, b, hg);
  if (!k || cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, decode_smem_bytes(D)) !=
                cudaSuccess) {
    cudaGetLastError();
    return false;
  }
  done[dev][slot].store(1, std::memory_order_relaxed);
  return true;
}

// Clusters of `cs` decode CTAs that can be resident at once on the device.
int max_active_clusters(int dev, int D, int b, int hg, int cs) {
  static std::atomic<int> cache[kMaxDevices][kInstSlots][kvq::kMaxCluster + 1];
  const int slot = inst_slot(D, b, hg);
  int v = cache[dev][slot][cs].load(std::memory_order_relaxed);
  if (v > 0) return v;
  if (!prepare_decode_kernel(dev, D, b, hg)) return 0;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(cs, 1, 1);
  cfg.blockDim = dim3(kvq::kAttnThreads, 1, 1);
  cfg.dynamicSmemBytes = decode_smem_bytes(D);
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = cs;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, decode_kernel_for(D, b, hg), &cfg) != cudaSuccess || n < 1) {
    cudaGetLastError();
    return 0;
  }
  cache[dev][slot][cs].store(n, std::memory_order_relaxed);
  return n;
}

// Split each (sequence, kv-head group) into CTAs grouped in thread-block
// clusters (which merge on chip), choosing the cluster size and the split
// count so that every CTA of the launch is resident at once (one wave, as the
// occupancy API reports for clusters of that size) and each split keeps at
// least 8 pages. Larger clusters are preferred (fewer partial results); a
// smaller one must buy more than 10 % more splits. Only with more than one
// cluster per (sequence, head group) do partial results go through the
// workspace and a combine kernel.
SplitPlan plan_splits(const kvq_attn_desc* d, int dev) {
  const int hg = heads_per_cta(d->num_kv_heads);
  const long long units = (long long)d->batch * (d->num_kv_heads / hg);
  long long cap = d->max_pages_per_seq / 8;
  if (cap < 1) cap = 1;
  if (cap > kvq::kMaxSplits) cap = kvq::kMaxSplits;
  SplitPlan best = {1, d->max_pages_per_seq, 1, 1, hg};
  if (units <= 0 || cap == 1) return best;
  for (int cs = kvq::kMaxCluster; cs >= 1; --cs) {
    const int mac = max_active_clusters(dev, d->head_dim, d->hadamard_block, hg, cs);
    const long long per_unit = mac / units;  // clusters per (sequence, head group) in one wave
    if (per_unit < 1) continue;
    long long parts = per_unit;
    if (parts > cap / cs) parts = cap / cs;
    if (parts > kvq::kMaxParts) parts = kvq::kMaxParts;
    if (parts < 1) continue;
    const long long ns = parts * cs;
    if (ns * 10 > best.n_splits * 11LL) best = {(int)ns, 0, cs, (int)parts, hg};
  }
  best.pages_per_split = (d->max_pages_per_seq + best.n_splits - 1) / best.n_splits;
  return best;
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
  const int G = d->num_q_heads / d->num_kv_heads;
  if (d->head_dim != 64 && d->head_dim != 128) return KVQ_ERR_UNSUPPORTED;
  if (G != 1 && G != 2 && G != 4 && G != 8) return KVQ_ERR_UNSUPPORTED;
  if (!valid_block(d->head_dim, d->hadamard_block)) return KVQ_ERR_UNSUPPORTED;
  return KVQ_OK;
}

size_t workspace_bytes_for(const kvq_attn_desc* d, const SplitPlan& plan) {
  if (plan.n_parts <= 1 || d->batch == 0) return 0;
  const size_t G = (size_t)(d->num_q_heads / d->num_kv_heads);
  return (size_t)d->batch * d->num_kv_heads * plan.n_parts * G * (d->head_dim + 2) * sizeof(float);
}

template <int D, int BLK>
kvq_status launch_attn(const kvq::AttnParams& p, int hg, int dev, cudaStream_t s) {
  if (dev < 0 || dev >= kMaxDevices) return KVQ_ERR_UNSUPPORTED;
  if (!prepare_decode_kernel(dev, D, BLK, hg)) return KVQ_ERR_CUDA;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(p.n_splits, p.Hkv / hg, p.B);
  cfg.blockDim = dim3(kvq::kAttnThreads, 1, 1);
  cfg.dynamicSmemBytes = kvq::AttnSmem<D>::kTotal;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = p.cluster_size;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e;
  if (hg == 4) e = cudaLaunchKernelEx(&cfg, kvq::kvq_decode_kernel<D, BLK, 4>, p);
  else if (hg == 2) e = cudaLaunchKernelEx(&cfg, kvq::kvq_decode_kernel<D, BLK, 2>, p);
  else e = cudaLaunchKernelEx(&cfg, kvq::kvq_decode_kernel<D, BLK, 1>, p);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return KVQ_ERR_CUDA;
  }
  if (p.n_parts > 1) {
    // merge the clusters' partial results; launched as a programmatic
    // dependent so its CTAs are scheduled while the main grid drains
    cudaLaunchConfig_t c2 = {};
    c2.gridDim = dim3(p.G, p.Hkv, p.B);
    c2.blockDim = dim3(D, 1, 1);
    c2.dynamicSmemBytes = 0;
    c2.stream = s;
    cudaLaunchAttribute a2[1];
    a2[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    a2[0].val.programmaticStreamSerializationAllowed = 1;
    c2.attrs = a2;
    c2.numAttrs = 1;
    if (cudaLaunchKernelEx(&c2, kvq::kvq_decode_combine_kernel<D, BLK>, p) != cudaSuccess) {
      cudaGetLastError();
      return KVQ_ERR_CUDA;
    }
  }
  return cudaGetLastError() == cudaSuccess ? KVQ_OK : KVQ_ERR_CUDA;
}

template <int D>
kvq_status dispatch_attn(const kvq::AttnParams& p, int b, int hg, int dev, cudaStream_t s) {
  switch (b) {
    case 0: return launch_attn<D, 0>(p, hg, dev, s);
    case 32: return launch_attn<D, 32>(p, hg, dev, s);
    case 64: return launch_attn<D, 64>(p, hg, dev, s);
    case 128:
      if constexpr (D >= 128) return launch_attn<D, 128>(p, hg, dev, s);
      return KVQ_ERR_UNSUPPORTED;
    default: return KVQ_ERR_UNSUPPORTED;
  }
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
  return workspace_bytes_for(desc, plan_splits(desc, dev));
}

kvq_status paged_decode_attn_int4(const void* q, const uint8_t* cache, const void* scales,
                                  const void* zeros, const int32_t* page_table,
                                  const int32_t* context_lens, void* out, void* workspace,
                                  size_t workspace_bytes, const kvq_attn_desc* desc, void* stream) {
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
  const SplitPlan plan = plan_splits(&d, dev);
  const size_t need = workspace_bytes_for(&d, plan);
  if (need > 0 && (!workspace || workspace_bytes < need || !aligned(workspace, 16)))
    return KVQ_ERR_WORKSPACE;
  kvq::AttnParams p;
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
  p.cluster_size = plan.cluster;
  p.n_parts = plan.n_parts;
  p.ws_part = need > 0 ? static_cast<float*>(workspace) : nullptr;
  p.out_bf16 = d.out_dtype;
  const double cb = d.hadamard_block > 0 ? 1.0 / std::sqrt((double)d.hadamard_block) : 1.0;
  const double scale = d.softmax_scale > 0.0f ? (double)d.softmax_scale : 1.0 / std::sqrt((double)d.head_dim);
  p.qmul = (float)(cb * scale * 1.4426950408889634);  // log2(e)
  p.cb = (float)cb;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  return d.head_dim == 64 ? dispatch_attn<64>(p, d.hadamard_block, plan.hg, dev, s)
                          : dispatch_attn<128>(p, d.hadamard_block, plan.hg, dev, s);
}

kvq_status kvq_get_device_error(void* stream) {
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) {
    cudaGetLastError();
    return KVQ_ERR_CUDA;
  }
  int v = 0, zero = 0;
  if (cudaMemcpyFromSymbol(&v, kvq::g_device_error, sizeof(int)) != cudaSuccess ||
      cudaMemcpyToSymbol(kvq::g_device_error, &zero, sizeof(int)) != cudaSuccess) {
    cudaGetLastError();
    return KVQ_ERR_CUDA;
  }
  return static_cast<kvq_status>(v);
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

// Device address of g_static_workspace on `dev` (which must be current). In
// host code the array's name is only a host-side stand-in, so the address is
// looked up once per device and cached.
kvq_status static_workspace_on(int dev, void** out) {
  std::lock_guard<std::mutex> lock(g_static_ws_mutex);
  if (!g_static_ws_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_static_workspace) != cudaSuccess || p == nullptr) {
      cudaGetLastError();
      return KVQ_ERR_CUDA;
    }
    g_static_ws_ptr[dev] = p;
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
  const size_t need = workspace_bytes_for(desc, plan_splits(desc, dev));
  if (need > KVQ_STATIC_WORKSPACE_BYTES) return KVQ_ERR_WORKSPACE;
  void* ws = nullptr;
  if (need > 0) {
    st = static_workspace_on(dev, &ws);
    if (st != KVQ_OK) return st;
  }
  return paged_decode_attn_int4(q, cache, scales, zeros, page_table, context_lens, out, ws,
                                need > 0 ? (size_t)KVQ_STATIC_WORKSPACE_BYTES : 0, desc, stream);
}
