// Definitions shared by the libmla kernels and the host entry points.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <stdint.h>

namespace mla {

constexpr int kPage = 64;        // tokens per cache page
constexpr int kDLatent = 512;    // c_kv width
constexpr int kDRope = 64;       // k_pe width
constexpr int kDQK = 576;        // cached values per token
// fp8 cache row: e4m3 latent codes [0, 512), bf16 rope [512, 640), f32 scale
// [640, 644), zero [644, 656).
constexpr int kF8RowBytes = 656;
constexpr int kF8RopeOff = 512;
constexpr int kF8ScaleOff = 640;
constexpr int kRowsPerTask = 128;  // heads handled by one worker (one TMEM lane each)
constexpr int kMaxHeads = 128;

// Plan buffer (int32 words):
//   [0] device error word   [1] number of tasks T   [2] pages per worker (quota)
//   [3] total pages         [4] workers             [5] heads     [6..7] reserved
//   [8 .. 8+T]      prefix[t]: first global page of task t (prefix[T] = total)
//   [9+T .. 9+2T)   ntok[t]: tokens (or index slots) of task t after validation
constexpr int kPlanHeader = 8;
constexpr int kPlanErr = 0, kPlanTasks = 1, kPlanQuota = 2, kPlanTotal = 3, kPlanWorkers = 4, kPlanHeads = 5;

__host__ __device__ inline int plan_prefix_off() { return kPlanHeader; }
__host__ __device__ inline int plan_ntok_off(int tasks) { return kPlanHeader + tasks + 1; }
__host__ __device__ inline int plan_words(int tasks) { return kPlanHeader + 2 * tasks + 1; }

constexpr uint32_t kErrSeqLen = 0x1u, kErrPageId = 0x2u, kErrIndex = 0x4u, kErrTimeout = 0x8u;

struct PlanArgs {
  const int32_t* seq_lens;
  int32_t* plan;
  int batch, q_len, heads, max_pages_per_seq, topk, causal, workers;
};

struct DecodeArgs {
  const __nv_bfloat16* q;       // [B, Sq, H, 576]
  const int32_t* block_table;   // [B, max_pages_per_seq]
  const int32_t* seq_lens;      // [B]
  const int32_t* indices;       // [B, Sq, topk] or nullptr
  __nv_bfloat16* out;           // [B, Sq, H, 512]
  float* lse;                   // [B, Sq, H]
  float* part_o;                // [slots, H, 512]
  float* part_lse;              // [slots, 2, H]
  int32_t* plan;
  int batch, q_len, heads, num_pages, max_pages_per_seq, topk;
  float scale_log2;             // softmax_scale * log2(e)
};

// Tensor maps of the cache viewed as a 2-D tensor [num_pages * 64 rows, 576
// columns] of bf16: boxes of 64 columns (128-byte swizzle) and of 32 columns
// (64-byte swizzle), each 64 rows high for page tiles and 1 row high for
// gathers.
//
// fp8 cache [num_pages * 64 rows, 656 bytes]: `tile` / `row` are boxes of 128
// code bytes (no swizzle), the rope boxes 64 bytes wide (64-byte swizzle),
// and `scale_tile` / `scale_row` 16-byte boxes at the scale's offset.
struct CacheMaps {
  CUtensorMap tile;
  CUtensorMap row;
  CUtensorMap rope_tile;
  CUtensorMap rope_row;
  CUtensorMap scale_tile;
  CUtensorMap scale_row;
};

struct CombineArgs {
  const float* part_o;
  const float* part_lse;  // [slots, 2, H]
  const int32_t* plan;
  __nv_bfloat16* out;
  float* lse;
  int q_len, heads;
};

struct MergeArgs {
  const __nv_bfloat16* part_out;  // [parts, rows, 512]
  const float* part_lse;          // [parts, rows]
  __nv_bfloat16* out;             // [rows, 512]
  float* lse;                     // [rows]
  int parts;
  long long rows;
};

// Workspace layout: part_o then part_lse.
__host__ __device__ inline size_t part_o_bytes(int slots, int heads) {
  return (size_t)slots * heads * kDLatent * sizeof(float);
}
// one LSE per (slot, CTA half, head): each half of a split row has its own normaliser
__host__ __device__ inline size_t part_lse_bytes(int slots, int heads) {
  return (size_t)slots * 2 * heads * sizeof(float);
}

}  // namespace mla
