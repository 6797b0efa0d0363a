// C-ABI entry points of libmla (declared in include/mla.h): descriptor
// validation, buffer sizing, TMA descriptor encoding and kernel launches.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>
#include <math.h>
#include <mutex>

#include "common.cuh"
#include "mla.h"

namespace mla {

cudaError_t launch_plan(const PlanArgs& args, cudaStream_t stream);
cudaError_t launch_combine(const CombineArgs& args, int tasks, cudaStream_t stream);
cudaError_t launch_merge(const MergeArgs& args, cudaStream_t stream);
const void* decode_kernel_ptr(bool fp8);
int decode_smem_bytes(bool fp8);
int decode_threads(bool fp8);
cudaError_t launch_decode(const CacheMaps& maps, const DecodeArgs& args, int workers, bool fp8,
                          cudaStream_t stream);

namespace {

constexpr int kMaxDevices = 64;

struct DeviceInfo {
  bool ready = false;
  int sms = 0;
  int max_clusters = 0;  // co-resident 2-CTA clusters of the decode kernel
};

std::mutex g_mu;
DeviceInfo g_dev[kMaxDevices];
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

// Per-device set-up: opt in to the decode kernel's shared memory and find how
// many of its clusters fit at once.
bool device_info(DeviceInfo* out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return false;
  std::lock_guard<std::mutex> lock(g_mu);
  DeviceInfo& d = g_dev[dev];
  if (!d.ready) {
    int sms = 0, optin = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return false;
    if (cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess) return false;
    // both cache formats' kernels: the worker count is the smaller of their co-resident clusters
    int clusters = sms / 2;
    for (int f = 0; f < 2; ++f) {
      const bool fp8 = f == 1;
      if (optin < decode_smem_bytes(fp8)) return false;
      if (cudaFuncSetAttribute(decode_kernel_ptr(fp8), cudaFuncAttributeMaxDynamicSharedMemorySize,
                               decode_smem_bytes(fp8)) != cudaSuccess)
        return false;
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3(2 * (sms / 2), 1, 1);
      cfg.blockDim = dim3(decode_threads(fp8), 1, 1);
      cfg.dynamicSmemBytes = decode_smem_bytes(fp8);
      int c = 0;
      if (cudaOccupancyMaxActiveClusters(&c, decode_kernel_ptr(fp8), &cfg) != cudaSuccess) {
        cudaGetLastError();
        c = sms / 2;
      }
      if (c < clusters) clusters = c;
    }
    d.sms = sms;
    d.max_clusters = clusters;
    d.ready = true;
  }
  *out = d;
  return true;
}

PFN_cuTensorMapEncodeTiled_v12000 encoder() {
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_encode) {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  }
  return g_encode;
}

mla_status_t check_desc(const mla_decode_desc_t* d) {
  if (!d) return MLA_ERR_INVALID_ARG;
  if (d->batch < 0 || d->q_len < 1 || d->num_heads < 1 || d->num_pages < 1 || d->max_pages_per_seq < 1 ||
      d->topk < 0 || (d->causal != 0 && d->causal != 1) || d->num_sms < 0)
    return MLA_ERR_INVALID_ARG;
  if (!(d->softmax_scale > 0.f) || !isfinite(d->softmax_scale)) return MLA_ERR_INVALID_ARG;
  if (d->topk > 0 && d->causal) return MLA_ERR_INVALID_ARG;  // a sparse row's tokens are the listed ones
  if (d->d_latent != kDLatent || d->d_rope != kDRope || d->page_size != kPage) return MLA_ERR_UNSUPPORTED;
  if (d->num_heads > kMaxHeads) return MLA_ERR_UNSUPPORTED;
  const long long tasks = (long long)d->batch * d->q_len;
  const long long rows = (long long)d->num_pages * kPage;
  if (tasks > (1 << 24) || rows > 0x7fffffffLL || (long long)d->max_pages_per_seq * kPage > 0x7fffffffLL)
    return MLA_ERR_UNSUPPORTED;
  // The plan kernel lays every task's pages end to end in 32-bit prefix sums:
  // the largest total a descriptor allows must stay below 2^31.
  const long long pages_per_task =
      d->topk > 0 ? ((long long)d->topk + kPage - 1) / kPage : (long long)d->max_pages_per_seq;
  if (tasks * pages_per_task > 0x7fffffffLL) return MLA_ERR_UNSUPPORTED;
  return MLA_OK;
}

int workers_for(const mla_decode_desc_t* d, const DeviceInfo& info) {
  int sms = info.sms;
  if (d->num_sms > 0 && d->num_sms < sms) sms = d->num_sms;
  int w = sms / 2;
  if (w > info.max_clusters) w = info.max_clusters;
  return w < 1 ? 1 : w;
}

size_t plan_bytes_for(const mla_decode_desc_t* d) {
  const int tasks = d->batch * d->q_len;
  return ((size_t)plan_words(tasks) * sizeof(int32_t) + 15) & ~(size_t)15;
}

size_t workspace_bytes_for(const mla_decode_desc_t* d, int workers) {
  const int slots = workers + d->batch * d->q_len;
  return part_o_bytes(slots, d->num_heads) + part_lse_bytes(slots, d->num_heads);
}

bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

}  // namespace

// The driver's tensor-map encoder, shared with the other entry points.
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() { return encoder(); }

}  // namespace mla

using namespace mla;

extern "C" {

size_t mla_plan_bytes(const mla_decode_desc_t* desc) {
  if (check_desc(desc) != MLA_OK) return 0;
  return plan_bytes_for(desc);
}

int32_t mla_num_workers(const mla_decode_desc_t* desc) {
  if (check_desc(desc) != MLA_OK) return 0;
  DeviceInfo info;
  if (!device_info(&info)) return 0;
  return workers_for(desc, info);
}

size_t mla_workspace_bytes(const mla_decode_desc_t* desc) {
  if (check_desc(desc) != MLA_OK) return 0;
  DeviceInfo info;
  if (!device_info(&info)) return 0;
  return workspace_bytes_for(desc, workers_for(desc, info));
}

mla_status_t mla_decode_plan(const mla_decode_desc_t* desc, const int32_t* seq_lens, void* plan, size_t plan_bytes,
                             mla_stream_t stream) {
  mla_status_t st = check_desc(desc);
  if (st != MLA_OK) return st;
  if (!plan || (!seq_lens && desc->batch > 0) || !aligned16(plan)) return MLA_ERR_INVALID_ARG;
  if (plan_bytes < plan_bytes_for(desc)) return MLA_ERR_WORKSPACE_TOO_SMALL;
  DeviceInfo info;
  if (!device_info(&info)) return MLA_ERR_CUDA;
  PlanArgs a;
  a.seq_lens = seq_lens;
  a.plan = reinterpret_cast<int32_t*>(plan);
  a.batch = desc->batch;
  a.q_len = desc->q_len;
  a.heads = desc->num_heads;
  a.max_pages_per_seq = desc->max_pages_per_seq;
  a.topk = desc->topk;
  a.causal = desc->causal;
  a.workers = workers_for(desc, info);
  return launch_plan(a, (cudaStream_t)stream) == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
}

}  // extern "C"

namespace mla {
namespace {

mla_status_t decode_impl(const mla_decode_desc_t* desc, void* plan, const void* q, const void* kv_cache,
                         const int32_t* block_table, const int32_t* seq_lens, const int32_t* topk_indices, void* out,
                         float* lse, void* workspace, size_t workspace_bytes, bool fp8, mla_stream_t stream) {
  mla_status_t st = check_desc(desc);
  if (st != MLA_OK) return st;
  if (desc->batch == 0) return MLA_OK;  // nothing to read or write; empty tensors may be NULL
  if (!plan || !q || !kv_cache || !block_table || !seq_lens || !out || !lse || !workspace)
    return MLA_ERR_INVALID_ARG;
  if (desc->topk > 0 && !topk_indices) return MLA_ERR_INVALID_ARG;
  if (!aligned16(plan) || !aligned16(q) || !aligned16(kv_cache) || !aligned16(out) || !aligned16(workspace) ||
      ((uintptr_t)lse & 3u) || ((uintptr_t)block_table & 3u) || ((uintptr_t)seq_lens & 3u) ||
      ((uintptr_t)topk_indices & 3u))
    return MLA_ERR_INVALID_ARG;
  DeviceInfo info;
  if (!device_info(&info)) return MLA_ERR_CUDA;
  const int workers = workers_for(desc, info);
  if (workspace_bytes < workspace_bytes_for(desc, workers)) return MLA_ERR_WORKSPACE_TOO_SMALL;

  PFN_cuTensorMapEncodeTiled_v12000 enc = encoder();
  if (!enc) return MLA_ERR_CUDA;
  // bf16 cache: a 2-D tensor [num_pages * 64 rows, 576 columns] of bf16:
  // 64-column boxes with 128-byte swizzle (latent columns) and 32-column
  // boxes with 64-byte swizzle (rope columns), 64 rows (page) or 1 row
  // (gather). fp8 cache: [num_pages * 64 rows, 656 bytes] of uint8: boxes of
  // 128 code bytes (no swizzle), 64 rope bytes (64-byte swizzle) and the
  // 16 bytes holding the scale.
  CacheMaps maps;
  const bool f8 = fp8;
  cuuint64_t dims[2] = {(cuuint64_t)(f8 ? kF8RowBytes : kDQK), (cuuint64_t)desc->num_pages * kPage};
  cuuint64_t strides[1] = {(cuuint64_t)(f8 ? kF8RowBytes : kDQK * 2)};
  cuuint32_t elem[2] = {1, 1};
  auto encode = [&](CUtensorMap* m, cuuint32_t cols, cuuint32_t rows, CUtensorMapSwizzle sw) {
    cuuint32_t box[2] = {cols, rows};
    return enc(m, f8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
               const_cast<void*>(kv_cache), dims, strides, box, elem, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
  };
  if (!f8) {
    if (!encode(&maps.tile, 64, kPage, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !encode(&maps.row, 64, 1, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !encode(&maps.rope_tile, 32, kPage, CU_TENSOR_MAP_SWIZZLE_64B) ||
        !encode(&maps.rope_row, 32, 1, CU_TENSOR_MAP_SWIZZLE_64B))
      return MLA_ERR_CUDA;
    maps.scale_tile = maps.tile;
    maps.scale_row = maps.row;
  } else if (!encode(&maps.tile, 128, kPage, CU_TENSOR_MAP_SWIZZLE_NONE) ||
             !encode(&maps.row, 128, 1, CU_TENSOR_MAP_SWIZZLE_NONE) ||
             !encode(&maps.rope_tile, 64, kPage, CU_TENSOR_MAP_SWIZZLE_64B) ||
             !encode(&maps.rope_row, 64, 1, CU_TENSOR_MAP_SWIZZLE_64B) ||
             !encode(&maps.scale_tile, 16, kPage, CU_TENSOR_MAP_SWIZZLE_NONE) ||
             !encode(&maps.scale_row, 16, 1, CU_TENSOR_MAP_SWIZZLE_NONE)) {
    return MLA_ERR_CUDA;
  }

  const int slots = workers + desc->batch * desc->q_len;
  DecodeArgs a;
  a.q = reinterpret_cast<const __nv_bfloat16*>(q);
  a.block_table = block_table;
  a.seq_lens = seq_lens;
  a.indices = topk_indices;
  a.cache = static_cast<const uint8_t*>(kv_cache);
  a.out = reinterpret_cast<__nv_bfloat16*>(out);
  a.lse = lse;
  a.part_o = reinterpret_cast<float*>(workspace);
  a.part_lse = reinterpret_cast<float*>(reinterpret_cast<char*>(workspace) + part_o_bytes(slots, desc->num_heads));
  a.plan = reinterpret_cast<int32_t*>(plan);
  a.batch = desc->batch;
  a.q_len = desc->q_len;
  a.heads = desc->num_heads;
  a.num_pages = desc->num_pages;
  a.max_pages_per_seq = desc->max_pages_per_seq;
  a.topk = desc->topk;
  a.scale_log2 = desc->softmax_scale * 1.4426950408889634f;
  return launch_decode(maps, a, workers, fp8, (cudaStream_t)stream) == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
}

}  // namespace
}  // namespace mla

extern "C" {

mla_status_t mla_decode(const mla_decode_desc_t* desc, void* plan, const void* q, const void* kv_cache,
                        const int32_t* block_table, const int32_t* seq_lens, const int32_t* topk_indices, void* out,
                        float* lse, void* workspace, size_t workspace_bytes, mla_stream_t stream) {
  return decode_impl(desc, plan, q, kv_cache, block_table, seq_lens, topk_indices, out, lse, workspace,
                     workspace_bytes, false, stream);
}

mla_status_t mla_decode_fp8(const mla_decode_desc_t* desc, void* plan, const void* q, const void* kv_cache_fp8,
                            const int32_t* block_table, const int32_t* seq_lens, const int32_t* topk_indices,
                            void* out, float* lse, void* workspace, size_t workspace_bytes, mla_stream_t stream) {
  return decode_impl(desc, plan, q, kv_cache_fp8, block_table, seq_lens, topk_indices, out, lse, workspace,
                     workspace_bytes, true, stream);
}

mla_status_t mla_combine(const mla_decode_desc_t* desc, void* plan, const void* workspace, size_t workspace_bytes,
                         void* out, float* lse, mla_stream_t stream) {
  mla_status_t st = check_desc(desc);
  if (st != MLA_OK) return st;
  if (desc->batch == 0) return MLA_OK;
  if (!plan || !workspace || !out || !lse) return MLA_ERR_INVALID_ARG;
  if (!aligned16(plan) || !aligned16(workspace) || !aligned16(out) || ((uintptr_t)lse & 3u))
    return MLA_ERR_INVALID_ARG;
  DeviceInfo info;
  if (!device_info(&info)) return MLA_ERR_CUDA;
  const int workers = workers_for(desc, info);
  if (workspace_bytes < workspace_bytes_for(desc, workers)) return MLA_ERR_WORKSPACE_TOO_SMALL;
  const int tasks = desc->batch * desc->q_len;
  if (tasks == 0) return MLA_OK;
  const int slots = workers + tasks;
  CombineArgs a;
  a.part_o = reinterpret_cast<const float*>(workspace);
  a.part_lse =
      reinterpret_cast<const float*>(reinterpret_cast<const char*>(workspace) + part_o_bytes(slots, desc->num_heads));
  a.plan = reinterpret_cast<const int32_t*>(plan);
  a.out = reinterpret_cast<__nv_bfloat16*>(out);
  a.lse = lse;
  a.q_len = desc->q_len;
  a.heads = desc->num_heads;
  return launch_combine(a, tasks, (cudaStream_t)stream) == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
}

mla_status_t mla_get_error(const void* plan, uint32_t* error_bits, mla_stream_t stream) {
  if (!plan) return MLA_ERR_INVALID_ARG;
  if (cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess) return MLA_ERR_CUDA;
  uint32_t bits = 0;
  if (cudaMemcpy(&bits, plan, sizeof(bits), cudaMemcpyDeviceToHost) != cudaSuccess) return MLA_ERR_CUDA;
  if (error_bits) *error_bits = bits;
  if (bits & kErrTimeout) return MLA_ERR_DEVICE_TIMEOUT;
  if (bits) return MLA_ERR_DEVICE_BOUNDS;
  return MLA_OK;
}

mla_status_t mla_merge(const mla_merge_desc_t* desc, const void* part_out, const float* part_lse, void* out, float* lse,
                       mla_stream_t stream) {
  if (!desc) return MLA_ERR_INVALID_ARG;
  if (desc->parts < 1 || desc->rows < 0) return MLA_ERR_INVALID_ARG;
  if (desc->d_latent != kDLatent) return MLA_ERR_UNSUPPORTED;
  if (desc->rows == 0) return MLA_OK;
  if ((desc->rows + 7) / 8 > 0x7fffffffLL || desc->rows * desc->parts > (1LL << 40)) return MLA_ERR_UNSUPPORTED;
  if (!part_out || !part_lse || !out || !lse) return MLA_ERR_INVALID_ARG;
  if (!aligned16(part_out) || !aligned16(out) || ((uintptr_t)part_lse & 3u) || ((uintptr_t)lse & 3u))
    return MLA_ERR_INVALID_ARG;
  MergeArgs a;
  a.part_out = reinterpret_cast<const __nv_bfloat16*>(part_out);
  a.part_lse = part_lse;
  a.out = reinterpret_cast<__nv_bfloat16*>(out);
  a.lse = lse;
  a.parts = desc->parts;
  a.rows = desc->rows;
  return launch_merge(a, (cudaStream_t)stream) == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
}

const char* mla_status_string(mla_status_t s) {
  switch (s) {
    case MLA_OK: return "ok";
    case MLA_ERR_INVALID_ARG: return "invalid argument";
    case MLA_ERR_UNSUPPORTED: return "unsupported configuration";
    case MLA_ERR_WORKSPACE_TOO_SMALL: return "plan or workspace buffer too small";
    case MLA_ERR_CUDA: return "CUDA error";
    case MLA_ERR_DEVICE_BOUNDS: return "out-of-range length, page id or index seen on device";
    case MLA_ERR_DEVICE_TIMEOUT: return "device pipeline wait timed out";
  }
  return "unknown status";
}

}  // extern "C"

// ---------------------------------------------------------------------------
// mla_decode_noalloc: the full decode step (plan + decode + combine) with its
// scratch (plan buffer and split partials) in a fixed array of device memory
// that this library defines, for callers that cannot allocate device memory.

namespace mla {
namespace {

constexpr size_t kNoAllocScratchBytes = 32u << 20;  // 32 MiB, held by every device that loads the library

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

void* g_noalloc_ptr[kMaxDevices] = {};

// Device address of the scratch array for the current device. In host code
// the array's name is only a stand-in, so the address is looked up once per
// device (the first call on a device does it, with that device current).
bool noalloc_scratch(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return false;
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_noalloc_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) {
      cudaGetLastError();
      return false;
    }
    g_noalloc_ptr[dev] = p;
  }
  *out = g_noalloc_ptr[dev];
  return true;
}

size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

// Scratch layout: [plan | partial outputs | partial LSEs]. The split partials
// need one slot per (worker, task) overlap, worst case workers + tasks. The
// call fits when the plan plus tasks + 1 slots (one worker) fit; then up to
// *max_workers workers do. Every quantity is compared before it is
// subtracted, so no size can wrap.
bool noalloc_fit(const mla_decode_desc_t* desc, long long* max_workers) {
  const size_t plan = align256(plan_bytes_for(desc));
  const size_t per_slot = part_o_bytes(1, desc->num_heads) + part_lse_bytes(1, desc->num_heads);
  const long long tasks = (long long)desc->batch * desc->q_len;
  if (plan >= kNoAllocScratchBytes) return false;
  const long long slots = (long long)((kNoAllocScratchBytes - plan) / per_slot);
  if (slots < tasks + 1) return false;
  *max_workers = slots - tasks;
  return true;
}

}  // namespace
}  // namespace mla

extern "C" mla_status_t mla_decode_noalloc(const mla_decode_desc_t* desc, const int32_t* seq_lens, const void* q,
                                           const void* kv_cache, const int32_t* block_table,
                                           const int32_t* topk_indices, void* out, float* lse,
                                           mla_stream_t stream) {
  mla_status_t st = check_desc(desc);
  if (st != MLA_OK) return st;
  if (desc->batch == 0) return MLA_OK;
  if (!seq_lens || !q || !kv_cache || !block_table || !out || !lse) return MLA_ERR_INVALID_ARG;
  if (desc->topk > 0 && !topk_indices) return MLA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(kv_cache) || !aligned16(out) || ((uintptr_t)lse & 3u) ||
      ((uintptr_t)block_table & 3u) || ((uintptr_t)seq_lens & 3u) || ((uintptr_t)topk_indices & 3u))
    return MLA_ERR_INVALID_ARG;  // checked here so that nothing is launched for a bad call
  // Sizing first, on the host alone: nothing touches the device for a call
  // whose plan and partials cannot fit.
  long long max_workers = 0;
  if (!noalloc_fit(desc, &max_workers)) return MLA_ERR_WORKSPACE_TOO_SMALL;
  DeviceInfo info;
  if (!device_info(&info)) return MLA_ERR_CUDA;
  void* scratch = nullptr;
  if (!noalloc_scratch(&scratch)) return MLA_ERR_CUDA;

  const size_t plan_bytes = plan_bytes_for(desc);
  long long workers = workers_for(desc, info);
  if (workers > max_workers) workers = max_workers;

  mla_decode_desc_t d = *desc;
  d.num_sms = (int32_t)(2 * workers);
  void* plan = scratch;
  void* ws = static_cast<char*>(scratch) + align256(plan_bytes);
  const size_t ws_bytes = workspace_bytes_for(&d, (int)workers);
  st = mla_decode_plan(&d, seq_lens, plan, plan_bytes, stream);
  if (st != MLA_OK) return st;
  st = mla_decode(&d, plan, q, kv_cache, block_table, seq_lens, topk_indices, out, lse, ws, ws_bytes, stream);
  if (st != MLA_OK) return st;
  return mla_combine(&d, plan, ws, ws_bytes, out, lse, stream);
}
