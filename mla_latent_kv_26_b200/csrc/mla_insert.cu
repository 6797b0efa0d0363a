// Latent-cache insert: kv_norm (RMSNorm) of each new token's 512-wide latent,
// the rotary embedding of its 64-wide rope key, and the write of both into the
// token's row of the paged cache, in one pass.
//
// "深度解读DeepSeek：源码解读 DeepSeek-V3", section "MLA": the down projection's
// output splits into the latent (512) and k_pe (64); k_pe is rotated and the
// absorbed branch caches kv_norm(latent) and the rotated k_pe at the token's
// position. "DeepSeek-V2-Lite 模型结构详解", section "四、RMSNorm": a row is
// divided by sqrt(mean(x^2) + eps) in float32, cast back to the input dtype,
// then multiplied by the weight. Rotation: consecutive pairs (x[2i], x[2i+1])
// turned by the caller's (cos, sin) for the token's position and pair i,
// in float32, rounded to bf16.
//
// Layout of the work: one warp per token, 40 warps per SM (5 blocks of 8,
// which caps a thread at 48 registers). Measured on B200 for a 64 x 1024-token
// prefill insert: more resident warps beat more tokens in flight per warp
// (1 token x 40 warps: 27.4 us; 2 x 24: 29.0 us; 4 x 16: 30.7 us). Lane
// l holds latent elements [8l, 8l+8) and [256+8l, 256+8l+8) (each warp-wide
// 16-byte load covers 512 contiguous bytes) and rope pair l. The kernel is
// HBM-bound: per token it reads the 1152-byte input row, 256 bytes of cos/sin,
// the sequence id, the position and one block-table entry, and writes the
// 1152-byte cache row; the weight (1 KB) stays in L1/L2.
#include <cuda_runtime.h>
#include <math.h>

#include "common.cuh"
#include "mla.h"
#include "sm100.cuh"

namespace mla {

struct InsertArgs {
  const __nv_bfloat16* kv;      // [N, 576]
  const __nv_bfloat16* weight;  // [512]
  const float* cos;             // [max_positions, 32]
  const float* sin;             // [max_positions, 32]
  const int32_t* seq_ids;       // [N]
  const int32_t* positions;     // [N]
  const int32_t* block_table;   // [batch, max_pages_per_seq]
  __nv_bfloat16* cache;         // [num_pages, 64, 576]
  uint32_t* error;              // device word or nullptr
  int num_tokens, batch, max_pages_per_seq, num_pages, max_positions;
  float eps;
};

namespace {

// Device error bit of a token whose sequence id or position is out of range
// (MLA_DEVERR_POSITION; the other bits are shared with decode).
constexpr uint32_t kErrInsertPos = 0x10u;

#ifndef MLA_INSERT_UNROLL
#define MLA_INSERT_UNROLL 1
#endif
#ifndef MLA_INSERT_BLOCKS
#define MLA_INSERT_BLOCKS 5
#endif
constexpr int kInsertWarps = 8;                        // warps per block
constexpr int kInsertUnroll = MLA_INSERT_UNROLL;       // tokens in flight per warp
constexpr int kInsertBlocksPerSM = MLA_INSERT_BLOCKS;  // resident blocks per SM (sets the register cap)

MLA_DEV float bf_lo(uint32_t v) { return __uint_as_float(v << 16); }
MLA_DEV float bf_hi(uint32_t v) { return __uint_as_float(v & 0xffff0000u); }


// x (8 bf16 in a uint4) scaled by inv, rounded to bf16, times w (8 bf16),
// rounded to bf16: the page's order. The product of two bf16 values is exact
// in float32, so the second rounding is the correctly rounded bf16 product.
MLA_DEV uint32_t norm2(uint32_t x, uint32_t w, float inv) {
  const uint32_t y = ptx::pack_bf16x2(bf_lo(x) * inv, bf_hi(x) * inv);
  return ptx::pack_bf16x2(bf_lo(y) * bf_lo(w), bf_hi(y) * bf_hi(w));
}
MLA_DEV uint4 norm8(uint4 x, uint4 w, float inv) {
  return make_uint4(norm2(x.x, w.x, inv), norm2(x.y, w.y, inv), norm2(x.z, w.z, inv), norm2(x.w, w.w, inv));
}
MLA_DEV float sumsq2(uint32_t x) { return bf_lo(x) * bf_lo(x) + bf_hi(x) * bf_hi(x); }
MLA_DEV float sumsq8(uint4 x) { return sumsq2(x.x) + sumsq2(x.y) + sumsq2(x.z) + sumsq2(x.w); }

// Two floats -> two e4m3 codes (round to nearest even, saturating at +-448),
// `lo` in the low byte.
MLA_DEV uint32_t e4m3x2(float lo, float hi) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}
// Eight bf16 values (a uint4) divided by s (IEEE quotients) -> eight e4m3 codes.
MLA_DEV uint2 codes8(uint4 v, float s) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  uint32_t c[4];
#pragma unroll
  for (int u = 0; u < 4; ++u) c[u] = e4m3x2(__fdiv_rn(bf_lo(w[u]), s), __fdiv_rn(bf_hi(w[u]), s));
  return make_uint2(c[0] | (c[1] << 16), c[2] | (c[3] << 16));
}
MLA_DEV float absmax2(uint32_t v) { return fmaxf(fabsf(bf_lo(v)), fabsf(bf_hi(v))); }
MLA_DEV float absmax8(uint4 v) { return fmaxf(fmaxf(absmax2(v.x), absmax2(v.y)), fmaxf(absmax2(v.z), absmax2(v.w))); }

// kF8: the row is written in the fp8 cache format (656 bytes: 512 e4m3 codes
// of the latent divided by its per-token scale amax / 448, the rope as bf16,
// the float32 scale, 12 zero bytes), from the same bf16 latent values the
// bf16 format stores.
template <bool kF8>
__global__ void __launch_bounds__(kInsertWarps * 32, kInsertBlocksPerSM) mla_insert_kernel(const InsertArgs a) {
  const int lane = threadIdx.x & 31;
  const int warp = blockIdx.x * kInsertWarps + (threadIdx.x >> 5);
  const int stride = gridDim.x * kInsertWarps * kInsertUnroll;
  const uint4* w4 = reinterpret_cast<const uint4*>(a.weight);
  const int max_pos = min(a.max_pages_per_seq * kPage, a.max_positions);
  uint32_t err = 0;

  for (int n0 = warp * kInsertUnroll; n0 < a.num_tokens; n0 += stride) {
    uint4 xa[kInsertUnroll], xb[kInsertUnroll];
    uint32_t xr[kInsertUnroll];
    float c[kInsertUnroll], s[kInsertUnroll];
    long long row[kInsertUnroll];  // destination row of the cache, -1 = skip
    int bs[kInsertUnroll], ps[kInsertUnroll];
    // the index chain first (sequence, position -> block table), so that its
    // two round trips overlap the row loads
#pragma unroll
    for (int u = 0; u < kInsertUnroll; ++u) {
      const int n = min(n0 + u, a.num_tokens - 1);
      bs[u] = __ldg(a.seq_ids + n);
      ps[u] = __ldg(a.positions + n);
    }
#pragma unroll
    for (int u = 0; u < kInsertUnroll; ++u) {
      const int n = min(n0 + u, a.num_tokens - 1);
      const uint4* src = reinterpret_cast<const uint4*>(a.kv + (size_t)n * kDQK);
      xa[u] = __ldcs(src + lane);  // read once: evict-first
      xb[u] = __ldcs(src + 32 + lane);
      xr[u] = __ldcs(reinterpret_cast<const unsigned int*>(src + 64) + lane);
    }
#pragma unroll
    for (int u = 0; u < kInsertUnroll; ++u) {
      const int n = n0 + u;
      row[u] = -1;
      if (n >= a.num_tokens) continue;
      const int b = bs[u], p = ps[u];
      if (b < 0 || b >= a.batch || p < 0 || p >= max_pos) {
        err |= kErrInsertPos;
        continue;
      }
      const int page = __ldg(a.block_table + (size_t)b * a.max_pages_per_seq + p / kPage);
      c[u] = __ldg(a.cos + (size_t)p * (kDRope / 2) + lane);
      s[u] = __ldg(a.sin + (size_t)p * (kDRope / 2) + lane);
      if (page < 0 || page >= a.num_pages) {
        err |= kErrPageId;
        continue;
      }
      row[u] = (long long)page * kPage + p % kPage;
    }
#pragma unroll
    for (int u = 0; u < kInsertUnroll; ++u) {
      if (row[u] < 0) continue;  // uniform across the warp
      float ss = sumsq8(xa[u]) + sumsq8(xb[u]);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
      const float inv = 1.0f / sqrtf(ss * (1.0f / kDLatent) + a.eps);
      const float x0 = bf_lo(xr[u]), x1 = bf_hi(xr[u]);
      const uint4 ya = norm8(xa[u], __ldg(w4 + lane), inv);  // the weight stays in L1
      const uint4 yb = norm8(xb[u], __ldg(w4 + 32 + lane), inv);
      const uint32_t rope = ptx::pack_bf16x2(x0 * c[u] - x1 * s[u], x0 * s[u] + x1 * c[u]);
      if constexpr (!kF8) {
        uint4* dst = reinterpret_cast<uint4*>(a.cache + (size_t)row[u] * kDQK);
        dst[lane] = ya;
        dst[32 + lane] = yb;
        reinterpret_cast<uint32_t*>(dst + 64)[lane] = rope;
      } else {
        float amax = fmaxf(absmax8(ya), absmax8(yb));
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
        const float scale = amax > 0.f ? __fdiv_rn(amax, 448.0f) : 1.0f;
        uint8_t* dst = reinterpret_cast<uint8_t*>(a.cache) + (size_t)row[u] * kF8RowBytes;
        *reinterpret_cast<uint2*>(dst + 8 * lane) = codes8(ya, scale);
        *reinterpret_cast<uint2*>(dst + 256 + 8 * lane) = codes8(yb, scale);
        *reinterpret_cast<uint32_t*>(dst + kF8RopeOff + 4 * lane) = rope;
        if (lane == 0) *reinterpret_cast<uint4*>(dst + kF8ScaleOff) = make_uint4(__float_as_uint(scale), 0u, 0u, 0u);
      }
    }
  }
  if (err && lane == 0 && a.error) atomicOr(a.error, err);
}

bool aligned(const void* p, uintptr_t a) { return ((uintptr_t)p & (a - 1)) == 0; }

}  // namespace

cudaError_t launch_insert(const InsertArgs& a, bool fp8, cudaStream_t stream) {
  if (a.num_tokens == 0) return cudaSuccess;
  int dev = 0, sms = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  const int per_block = kInsertWarps * kInsertUnroll;
  const int need = (a.num_tokens + per_block - 1) / per_block;
  const int grid = need < sms * kInsertBlocksPerSM ? need : sms * kInsertBlocksPerSM;
  if (fp8) mla_insert_kernel<true><<<grid, kInsertWarps * 32, 0, stream>>>(a);
  else mla_insert_kernel<false><<<grid, kInsertWarps * 32, 0, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace mla

namespace {
mla_status_t cache_insert(const mla_insert_desc_t* desc, const void* kv, const void* weight, const float* cos_table,
                          const float* sin_table, const int32_t* seq_ids, const int32_t* positions,
                          const int32_t* block_table, void* kv_cache, uint32_t* error_word, bool fp8,
                          mla_stream_t stream) {
  using namespace mla;
  if (!desc) return MLA_ERR_INVALID_ARG;
  if (desc->num_tokens < 0 || desc->batch < 0 || desc->max_pages_per_seq < 1 || desc->num_pages < 1 ||
      desc->max_positions < 1 || !(desc->eps >= 0.0f) || !isfinite(desc->eps))
    return MLA_ERR_INVALID_ARG;
  if (desc->d_latent != kDLatent || desc->d_rope != kDRope || desc->page_size != kPage) return MLA_ERR_UNSUPPORTED;
  // positions and cache rows are 32-bit in the kernel
  if ((long long)desc->max_pages_per_seq * kPage > 0x7fffffffLL || (long long)desc->num_pages * kPage > 0x7fffffffLL)
    return MLA_ERR_UNSUPPORTED;
  if (desc->num_tokens == 0) return MLA_OK;
  if (!kv || !weight || !cos_table || !sin_table || !seq_ids || !positions || !block_table || !kv_cache)
    return MLA_ERR_INVALID_ARG;
  if (!aligned(kv, 16) || !aligned(weight, 16) || !aligned(kv_cache, 16) || !aligned(cos_table, 4) ||
      !aligned(sin_table, 4) || !aligned(error_word, 4))
    return MLA_ERR_INVALID_ARG;
  InsertArgs a;
  a.kv = static_cast<const __nv_bfloat16*>(kv);
  a.weight = static_cast<const __nv_bfloat16*>(weight);
  a.cos = cos_table;
  a.sin = sin_table;
  a.seq_ids = seq_ids;
  a.positions = positions;
  a.block_table = block_table;
  a.cache = static_cast<__nv_bfloat16*>(kv_cache);
  a.error = error_word;
  a.num_tokens = desc->num_tokens;
  a.batch = desc->batch;
  a.max_pages_per_seq = desc->max_pages_per_seq;
  a.num_pages = desc->num_pages;
  a.max_positions = desc->max_positions;
  a.eps = desc->eps;
  return launch_insert(a, fp8, (cudaStream_t)stream) == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
}
}  // namespace

extern "C" MLA_API mla_status_t mla_cache_insert(const mla_insert_desc_t* desc, const void* kv, const void* weight,
                                                 const float* cos_table, const float* sin_table,
                                                 const int32_t* seq_ids, const int32_t* positions,
                                                 const int32_t* block_table, void* kv_cache, uint32_t* error_word,
                                                 mla_stream_t stream) {
  return cache_insert(desc, kv, weight, cos_table, sin_table, seq_ids, positions, block_table, kv_cache, error_word,
                      false, stream);
}

extern "C" MLA_API mla_status_t mla_cache_insert_fp8(const mla_insert_desc_t* desc, const void* kv,
                                                     const void* weight, const float* cos_table,
                                                     const float* sin_table, const int32_t* seq_ids,
                                                     const int32_t* positions, const int32_t* block_table,
                                                     void* kv_cache_fp8, uint32_t* error_word, mla_stream_t stream) {
  return cache_insert(desc, kv, weight, cos_table, sin_table, seq_ids, positions, block_table, kv_cache_fp8,
                      error_word, true, stream);
}
