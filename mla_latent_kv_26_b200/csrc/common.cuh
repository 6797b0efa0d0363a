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
//   [0] device error word   [1] number of tasks T   [2] quota of group 0
//   [3] total pages         [4] workers             [5] heads
//   [6] worker groups G     [7] workers per group Wg
//   [8 .. 8+T]      prefix[u]: first global page of plan position u (prefix[T] = total)
//   [9+T .. 9+2T)   ntok[u]: tokens (or index slots) of position u after validation
constexpr int kPlanHeader = 8;
constexpr int kPlanErr = 0, kPlanTasks = 1, kPlanQuota = 2, kPlanTotal = 3, kPlanWorkers = 4, kPlanHeads = 5;
constexpr int kPlanGroups = 6, kPlanGroupWorkers = 7;

__host__ __device__ inline int plan_prefix_off() { return kPlanHeader; }
__host__ __device__ inline int plan_ntok_off(int tasks) { return kPlanHeader + tasks + 1; }
__host__ __device__ inline int plan_words(int tasks) { return kPlanHeader + 2 * tasks + 1; }

// Worker groups: with several dense query tokens per sequence (2..8, no
// top-k) and at least 4 workers per token, the workers form G = Sq equal
// groups and group g takes token g of every sequence. The tokens of one
// sequence read the same pages, and the groups walk them in step, so a page
// fetched for one token is still in L2 for the others. Otherwise G = 1.
__host__ __device__ inline int plan_groups(int q_len, int topk, int workers) {
  return (q_len >= 2 && q_len <= 8 && topk == 0 && workers / q_len >= 4) ? q_len : 1;
}

// Plan order: with G > 1 groups, position u holds query token u / B of
// sequence u % B (token-major, so a group's positions are contiguous); with
// G = 1 it is query row u = b * Sq + i.
struct TaskMap {
  int groups, batch, q_len;
  __host__ __device__ int seq(int u) const { return groups > 1 ? u % batch : u / q_len; }
  __host__ __device__ int tok(int u) const { return groups > 1 ? u / batch : u % q_len; }
  __host__ __device__ int row(int u) const { return groups > 1 ? (u % batch) * q_len + u / batch : u; }
};

// Group g of a plan: positions [t0, t1), global pages [base, end), split
// over workers [w0, w0 + Wg) in runs of `quota` pages.
struct PlanGroup {
  int t0, t1, base, end, quota, w0;
};
__device__ inline PlanGroup plan_group(const int32_t* plan, int g) {
  const int T = plan[kPlanTasks], G = plan[kPlanGroups], Wg = plan[kPlanGroupWorkers];
  const int32_t* prefix = plan + plan_prefix_off();
  PlanGroup r;
  r.t0 = g * (T / G);
  r.t1 = r.t0 + T / G;
  r.base = prefix[r.t0];
  r.end = prefix[r.t1];
  r.quota = max(1, (r.end - r.base + Wg - 1) / Wg);
  r.w0 = g * Wg;
  return r;
}

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
  const uint8_t* cache;         // the cache's first byte (row copies of gathered tokens)
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
