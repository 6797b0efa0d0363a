// Steps a1 (split schedule) and a8 (LSE merge of split partials).
#include <math.h>

#include "common.cuh"
#include "sm100.cuh"

namespace mla {

// One block of 1024 threads. Plan position u (query token TaskMap::tok(u)
// of sequence TaskMap::seq(u)) gets ntok[u] tokens (index slots when sparse)
// and ceil(ntok/64) pages; prefix[] lays the positions' pages end to end;
// worker j of group g owns the group's pages [j*quota_g, (j+1)*quota_g).
__global__ void __launch_bounds__(1024) mla_plan_kernel(PlanArgs a) {
  __shared__ int s_scan[32];
  __shared__ int s_carry;
  __shared__ unsigned s_err;
  const int tid = threadIdx.x;
  const int T = a.batch * a.q_len;
  int32_t* prefix = a.plan + plan_prefix_off();
  int32_t* ntok = a.plan + plan_ntok_off(T);
  if (tid == 0) {
    s_carry = 0;
    s_err = 0u;
  }
  __syncthreads();
  const long long cap = (long long)a.max_pages_per_seq * kPage;
  const int G = plan_groups(a.q_len, a.topk, a.workers);
  const TaskMap map{G, a.batch, a.q_len};
  for (int base = 0; base < T; base += 1024) {
    const int t = base + tid;
    int pages = 0;
    if (t < T) {
      const int b = map.seq(t), i = map.tok(t);
      const int L = a.seq_lens[b];
      const bool ok = L >= 0 && (long long)L <= cap;
      int n = 0;
      if (ok) n = a.topk > 0 ? a.topk : (a.causal ? max(L - a.q_len + i + 1, 0) : L);
      else atomicOr(&s_err, kErrSeqLen);
      ntok[t] = n;
      pages = (n + kPage - 1) / kPage;
    }
    // inclusive scan: within each warp by shuffles, then over the 32 warp totals
    const int lane = tid & 31, warp = tid >> 5;
    int v = pages;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int n = __shfl_up_sync(~0u, v, off);
      if (lane >= off) v += n;
    }
    if (lane == 31) s_scan[warp] = v;
    __syncthreads();
    if (warp == 0) {
      int w = s_scan[lane];
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const int n = __shfl_up_sync(~0u, w, off);
        if (lane >= off) w += n;
      }
      s_scan[lane] = w;
    }
    __syncthreads();
    if (t < T) prefix[t] = s_carry + (warp > 0 ? s_scan[warp - 1] : 0) + v - pages;
    __syncthreads();
    if (tid == 1023) s_carry += s_scan[31];
    __syncthreads();
  }
  if (tid == 0) {
    const int total = s_carry;
    prefix[T] = total;
    const int Wg = a.workers / G;
    const int pages0 = prefix[T / G];  // pages of group 0 (prefix[0] = 0)
    a.plan[kPlanErr] = (int32_t)s_err;
    a.plan[kPlanTasks] = T;
    a.plan[kPlanQuota] = max(1, (pages0 + Wg - 1) / Wg);
    a.plan[kPlanTotal] = total;
    a.plan[kPlanWorkers] = a.workers;
    a.plan[kPlanHeads] = a.heads;
    a.plan[kPlanGroups] = G;
    a.plan[kPlanGroupWorkers] = Wg;
  }
}

// grid (T, ceil(H/8)), 256 threads: one warp per (task, head) row.
// Unsplit tasks were finished by the decode kernel; empty tasks get out = 0,
// lse = -inf; split tasks merge their partials (slot = worker + task). Each
// half of the 512 output columns was normalised on its own (one per CTA of
// the worker), so each half merges with its own LSEs:
// lse = M + ln sum_w exp(lse_w - M), out = sum_w exp(lse_w - lse) * o_w.
__global__ void __launch_bounds__(256) mla_combine_kernel(CombineArgs a) {
  ptx::grid_dependency_wait();  // the decode's partials (programmatic launch)
  const int T = a.plan[kPlanTasks];
  const int t = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int h = blockIdx.y * 8 + warp;
  if (t >= T || h >= a.heads) return;
  const int G = a.plan[kPlanGroups];
  const PlanGroup grp = plan_group(a.plan, t / (T / G));
  const int32_t* prefix = a.plan + plan_prefix_off();
  const int p0 = prefix[t], p1 = prefix[t + 1];
  const TaskMap map{G, T / G, G};  // with G > 1, q_len = G; with G = 1, row(t) = t
  const size_t row = (size_t)map.row(t) * a.heads + h;
  __nv_bfloat16* orow = a.out + row * kDLatent;
  const int w0 = grp.w0 + (p0 - grp.base) / grp.quota;
  const int w1 = p1 > p0 ? grp.w0 + (p1 - 1 - grp.base) / grp.quota : w0;
  if (p1 > p0 && w0 == w1) return;

  float m[2] = {-INFINITY, -INFINITY};
  if (p1 > p0) {
    for (int w = w0; w <= w1; ++w) {
#pragma unroll
      for (int g = 0; g < 2; ++g) m[g] = fmaxf(m[g], a.part_lse[((size_t)(w + t) * 2 + g) * a.heads + h]);
    }
  }
  if (m[0] == -INFINITY) {
    const __nv_bfloat162 z = __floats2bfloat162_rn(0.f, 0.f);
    for (int j = 0; j < 4; ++j) {
      __nv_bfloat162* dst = reinterpret_cast<__nv_bfloat162*>(orow + lane * 4 + 128 * j);
      dst[0] = z;
      dst[1] = z;
    }
    if (lane == 0) a.lse[row] = -INFINITY;
    return;
  }
  float acc[16];
#pragma unroll
  for (int j = 0; j < 16; ++j) acc[j] = 0.f;
  float sum[2] = {0.f, 0.f};
  for (int w = w0; w <= w1; ++w) {
    const size_t srow = (size_t)(w + t) * a.heads + h;
    float e[2];
#pragma unroll
    for (int g = 0; g < 2; ++g) {
      const float l = a.part_lse[((size_t)(w + t) * 2 + g) * a.heads + h];
      e[g] = (l == -INFINITY) ? 0.f : expf(l - m[g]);
      sum[g] += e[g];
    }
    const float4* src = reinterpret_cast<const float4*>(a.part_o + srow * kDLatent);
#pragma unroll
    for (int j = 0; j < 4; ++j) {  // columns lane*4 + 128 j: j < 2 in the first half
      const float ej = e[j >> 1];
      const float4 v = src[lane + 32 * j];
      acc[4 * j + 0] += ej * v.x;
      acc[4 * j + 1] += ej * v.y;
      acc[4 * j + 2] += ej * v.z;
      acc[4 * j + 3] += ej * v.w;
    }
  }
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const float inv = 1.f / sum[j >> 1];
    __nv_bfloat162* dst = reinterpret_cast<__nv_bfloat162*>(orow + lane * 4 + 128 * j);
    dst[0] = __floats2bfloat162_rn(acc[4 * j + 0] * inv, acc[4 * j + 1] * inv);
    dst[1] = __floats2bfloat162_rn(acc[4 * j + 2] * inv, acc[4 * j + 3] * inv);
  }
  if (lane == 0) a.lse[row] = m[0] + logf(sum[0]);
}

// Merge of `parts` results of the same rows computed over disjoint token
// sets (one per context-parallel shard): one warp per row, lane l holding
// columns [8l, 8l + 8) and [256 + 8l, 256 + 8l + 8).
// lse = M + ln sum_i exp(lse_i - M), out = sum_i exp(lse_i - lse) * out_i;
// parts with lse_i = -inf weigh nothing; all empty: out = 0, lse = -inf.
__global__ void __launch_bounds__(256) mla_merge_kernel(MergeArgs a) {
  const long long row = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= a.rows) return;
  float m = -INFINITY;
  for (int i = 0; i < a.parts; ++i) m = fmaxf(m, a.part_lse[(size_t)i * a.rows + row]);
  float acc[16];
#pragma unroll
  for (int j = 0; j < 16; ++j) acc[j] = 0.f;
  float sum = 0.f;
  if (m != -INFINITY) {
    for (int i = 0; i < a.parts; ++i) {
      const float l = a.part_lse[(size_t)i * a.rows + row];
      if (l == -INFINITY) continue;
      const float e = expf(l - m);
      sum += e;
      const uint4* src = reinterpret_cast<const uint4*>(a.part_out + ((size_t)i * a.rows + row) * kDLatent);
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const uint4 v = src[lane + 32 * h];
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[u]));
          acc[8 * h + 2 * u] += e * f.x;
          acc[8 * h + 2 * u + 1] += e * f.y;
        }
      }
    }
  }
  const float inv = sum > 0.f ? 1.f / sum : 0.f;
  uint4* dst = reinterpret_cast<uint4*>(a.out + (size_t)row * kDLatent);
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    uint32_t w[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      __nv_bfloat162 b = __floats2bfloat162_rn(acc[8 * h + 2 * u] * inv, acc[8 * h + 2 * u + 1] * inv);
      w[u] = *reinterpret_cast<uint32_t*>(&b);
    }
    dst[lane + 32 * h] = make_uint4(w[0], w[1], w[2], w[3]);
  }
  if (lane == 0) a.lse[row] = sum > 0.f ? m + logf(sum) : -INFINITY;
}

cudaError_t launch_merge(const MergeArgs& args, cudaStream_t stream) {
  const long long blocks = (args.rows + 7) / 8;
  mla_merge_kernel<<<(unsigned)blocks, 256, 0, stream>>>(args);
  return cudaGetLastError();
}

cudaError_t launch_plan(const PlanArgs& args, cudaStream_t stream) {
  mla_plan_kernel<<<1, 1024, 0, stream>>>(args);
  return cudaGetLastError();
}

// Launched with programmatic stream serialization behind the decode: its
// blocks take SMs as decode CTAs finish and wait for the whole decode.
cudaError_t launch_combine(const CombineArgs& args, int tasks, cudaStream_t stream) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(tasks, (args.heads + 7) / 8, 1);
  cfg.blockDim = dim3(256, 1, 1);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, mla_combine_kernel, args);
}

}  // namespace mla
