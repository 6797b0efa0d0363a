// Sparse-attention indexer: fp8 index scores and their top-k positions.
//
// "DeepSeek-V3.2-Exp unboxing", the Indexer section: for every query token
// the indexer scores all cached keys of its sequence and keeps the highest
// scoring positions for the sparse attention that follows. The scoring call
// is fp8_index(q [b, m, h, d] fp8, q_s [b, m, h] fp32, k [b, n, d] fp8,
// k_s [b, n] fp32) -> o [b, m, n] fp32, with the model's per-head weights
// passed as q_s and the fp8 key cache's per-token scales as k_s. The kernel
// body is not printed; this file computes (the reading stated in the header)
//
//   o[b, i, t] = k_s[b, t] * sum_h q_s[b, i, h] * max(0, q[b, i, h, :] . k[b, t, :])
//
// mla_index_kernel: one CTA per SM, persistent over work items (sequence,
// group of G query tokens, tile of 128 keys), items of one CTA contiguous so
// that a query group stays in shared memory while its key tiles stream by.
//   warp 0      TMA producer: key tiles [128 keys x 128 B] into a 6-stage
//               ring, the query group [G*h rows x 128 B] into one of two
//               buffers when the group changes (128-byte swizzle, K-major)
//   warp 1      tcgen05 issuer: D[128 keys, G*h] = K_tile . Q_group^T, four
//               kind::f8f6f4 MMAs (K = 32 each) into one of two TMEM buffers
//   warps 2-9   epilogue, two groups of four warps taking alternate tiles
//               (group g reads TMEM buffer g), one TMEM lane (key) per
//               thread: ReLU, head weights, key scale, one fp32 score per
//               (query, key), coalesced stores. With one group the epilogue
//               set the pace (the kernel took 92.6 us against 55.8 us with
//               the epilogue's arithmetic left out).
//
// mla_topk_kernel: one cluster of C CTAs (C = 1..8) per row; CTA c owns the
// positions [c * chunk, (c + 1) * chunk) of the row, kept in shared memory
// as order-preserving 32-bit keys. Four 8-bit radix passes (histograms
// merged across the cluster through distributed shared memory) find the
// k-th largest key exactly; the selected positions are then written in
// increasing order (prefix sums over threads and over the cluster's CTAs),
// ties at the threshold going to the smaller positions.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>
#include <math.h>

#include <mutex>

#include "common.cuh"
#include "mla.h"
#include "sm100.cuh"

namespace mla {

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder();

namespace idx {

using namespace ptx;

// Instruction descriptor, kind::f8f6f4: e4m3 A and B (format code 0), fp32
// accumulator, both K-major.
__host__ __device__ constexpr uint32_t idesc_e4m3_f32(int M, int N) {
  return (1u << 4) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

// D[tmem] (+)= A[smem] * B[smem] with 8-bit floating-point operands (K = 32
// per instruction); issued by one thread.
MLA_DEV void mma_ss_f8(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.u32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// 32x32b shape, 16 columns: thread i of the warp reads TMEM lane (base lane + i).
MLA_DEV void tmem_ld_32x32b_16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
        "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}

MLA_DEV uint32_t cluster_nctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_nctarank;" : "=r"(r));
  return r;
}

// 4-byte load from a shared-memory address of any CTA of the cluster (an
// address made by map_to_rank).
MLA_DEV uint32_t ld_shared_cluster_u32(uint32_t cluster_addr) {
  uint32_t v;
  asm volatile("ld.shared::cluster.u32 %0, [%1];" : "=r"(v) : "r"(cluster_addr) : "memory");
  return v;
}

constexpr int kThreads = 320;   // producer, MMA issuer, 2 x 4 epilogue warps
constexpr int kStages = 6;
constexpr int kKeys = 128;                 // keys per tile: the MMA's M
constexpr int kDim = 128;                  // index head width d: 128 fp8 = one 128-byte swizzle row
constexpr int kTileBytes = kKeys * kDim;   // 16 KB
constexpr int kMaxN = 256;                 // MMA N: query group x heads
constexpr int kQBytes = kMaxN * kDim;      // 32 KB
constexpr int kSmem = 1024 + kStages * kTileBytes + 2 * kQBytes;
constexpr uint32_t kTmemCols = 2 * kMaxN;
// A pipeline wait gives up after MLA_WAIT_LIMIT_NS (2 s: only a broken
// device gets there; a test build sets a few hundred nanoseconds to make the
// waits run out). The waits that let copies and MMAs in flight finish before
// the CTA exits keep the 2 s limit in every build.
#ifndef MLA_WAIT_LIMIT_NS
#define MLA_WAIT_LIMIT_NS 2000000000ull
#endif
constexpr uint64_t kTimeoutNs = MLA_WAIT_LIMIT_NS;
constexpr uint64_t kDrainNs = 2000000000ull;
constexpr uint32_t kErrTimeoutBit = 0x8u;

struct Args {
  const float* q_s;  // [b, m, h]
  const float* k_s;  // [b, n]
  float* o;          // [b, m, n]
  uint32_t* err;     // device word or nullptr
  int b, m, h, n;
  int G, N;          // queries per group, MMA N = G * h
  int groups, tiles; // per sequence: ceil(m / G) query groups, ceil(n / 128) key tiles
  long long items, per_cta;
};

struct Maps {
  CUtensorMap k;  // [b * n rows, 128 columns] e4m3
  CUtensorMap q;  // [b * m * h rows, 128 columns] e4m3, boxes of N rows
};

struct Bars {
  uint64_t full[kStages], empty[kStages];
  uint64_t q_full[2], q_empty[2];
  uint64_t t_full[2], t_empty[2];
  uint64_t done;
  uint32_t tmem;
  uint32_t abort_flag;
};

struct Waiter {
  Bars* bars;
  uint32_t* err;
  MLA_DEV bool aborted() const { return *reinterpret_cast<volatile uint32_t*>(&bars->abort_flag) != 0; }
  MLA_DEV void fail() {
    *reinterpret_cast<volatile uint32_t*>(&bars->abort_flag) = 1u;
    if (err) atomicOr(err, kErrTimeoutBit);
  }
  // Bounded wait; gives up at once after another thread gave up unless `drain`.
  MLA_DEV bool wait(uint64_t* bar, uint32_t parity, bool drain = false) {
    const uint32_t a = smem_addr(bar);
    if (mbar_try_wait(a, parity)) return true;
    const uint64_t t0 = global_timer_ns();
    const uint64_t limit = drain ? kDrainNs : kTimeoutNs;
    while (true) {
      if (mbar_try_wait(a, parity)) return true;
      if (!drain && aborted()) return false;
      if (global_timer_ns() - t0 > limit) {
        fail();
        return false;
      }
    }
  }
  MLA_DEV bool wait_warp(uint64_t* bar, uint32_t parity) { return __all_sync(~0u, wait(bar, parity)); }
};

// Position (sequence, query group, key tile) of work item `it`, advanced one
// item at a time without divisions.
struct ItemCursor {
  int bb, g, j, groups, tiles;
  MLA_DEV void init(long long it, const Args& a) {
    groups = a.groups;
    tiles = a.tiles;
    j = (int)(it % tiles);
    const long long bg = it / tiles;
    g = (int)(bg % groups);
    bb = (int)(bg / groups);
  }
  MLA_DEV void next() {
    if (++j == tiles) {
      j = 0;
      if (++g == groups) {
        g = 0;
        ++bb;
      }
    }
  }
};

__global__ void __launch_bounds__(kThreads, 1) mla_index_kernel(const __grid_constant__ Maps maps, const Args a) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ Bars bars;
  const uint32_t base = (smem_addr(smem_raw) + 1023u) & ~1023u;
  const uint32_t ring = base;                          // kStages key tiles
  const uint32_t qbuf = base + kStages * kTileBytes;   // two query-group buffers
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  Waiter W{&bars, a.err};

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(smem_addr(&bars.full[s]), 1);
      mbar_init(smem_addr(&bars.empty[s]), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(smem_addr(&bars.q_full[i]), 1);
      mbar_init(smem_addr(&bars.q_empty[i]), 1);
      mbar_init(smem_addr(&bars.t_full[i]), 1);
      mbar_init(smem_addr(&bars.t_empty[i]), 4);  // the four epilogue warps of group i
    }
    mbar_init(smem_addr(&bars.done), 1);
    bars.abort_flag = 0u;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&maps.k);
    prefetch_tmap(&maps.q);
  }
  if (warp == 1) {
    tmem_alloc(smem_addr(&bars.tmem), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars.tmem;

  const long long i0 = (long long)blockIdx.x * a.per_cta;
  const long long i1 = min(i0 + a.per_cta, a.items);
  ItemCursor cur;
  cur.init(i0, a);

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    int k = 0, nq = 0;  // key tiles and query groups whose loads were issued
    if (lane == 0) {
      for (long long it = i0; it < i1; ++it, cur.next()) {
        if (it == i0 || cur.j == 0) {  // a new query group
          const int qb = nq & 1;
          if (!W.wait(&bars.q_empty[qb], ((nq >> 1) & 1) ^ 1)) break;
          mbar_arrive_expect_tx(smem_addr(&bars.q_full[qb]), (uint32_t)(a.N * kDim));
          tma_load_2d(qbuf + qb * kQBytes, &maps.q, 0, (cur.bb * a.m + cur.g * a.G) * a.h,
                      smem_addr(&bars.q_full[qb]));
          ++nq;
        }
        const int s = k % kStages;
        if (!W.wait(&bars.empty[s], ((k / kStages) & 1) ^ 1)) break;
        mbar_arrive_expect_tx(smem_addr(&bars.full[s]), kTileBytes);
        tma_load_2d(ring + s * kTileBytes, &maps.k, 0, cur.bb * a.n + cur.j * kKeys, smem_addr(&bars.full[s]));
        ++k;
      }
      // every issued copy lands before the CTA can exit
      for (int d = max(0, k - kStages); d < k; ++d) W.wait(&bars.full[d % kStages], (d / kStages) & 1, true);
      for (int d = max(0, nq - 2); d < nq; ++d) W.wait(&bars.q_full[d & 1], (d >> 1) & 1, true);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc = idesc_e4m3_f32(kKeys, a.N);
      int k = 0, qi = -1;
      for (long long it = i0; it < i1; ++it, cur.next()) {
        if (it == i0 || cur.j == 0) {  // a new query group
          if (qi >= 0) mma_commit(smem_addr(&bars.q_empty[qi & 1]));  // the old group's MMAs are issued
          ++qi;
          if (!W.wait(&bars.q_full[qi & 1], (qi >> 1) & 1)) break;
        }
        const int s = k % kStages, tb = k & 1;
        if (!W.wait(&bars.full[s], (k / kStages) & 1)) break;
        if (!W.wait(&bars.t_empty[tb], ((k >> 1) & 1) ^ 1)) break;
        tc_fence_after();
        const uint32_t sa = ring + s * kTileBytes, sb = qbuf + (qi & 1) * kQBytes;
        // K-step u: both operands advance 32 bytes along their swizzled rows
#pragma unroll
        for (int u = 0; u < kDim / 32; ++u)
          mma_ss_f8(tmem + (uint32_t)(tb * kMaxN), smem_desc_sw128(sa + 32 * u, 16, 1024),
                    smem_desc_sw128(sb + 32 * u, 16, 1024), idesc, u > 0 ? 1u : 0u);
        mma_commit(smem_addr(&bars.empty[s]));
        mma_commit(smem_addr(&bars.t_full[tb]));
        ++k;
      }
      mma_commit(smem_addr(&bars.done));
      W.wait(&bars.done, 0, true);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue
    const int quad = warp & 3;
    const int grp = (warp - 2) >> 2;   // tiles k with k % 2 == grp, TMEM buffer grp
    const int row = quad * 32 + lane;  // key within the tile = TMEM lane
    const uint32_t lanes = tmem + ((uint32_t)(quad * 32) << 16);
    int k = grp;
    // the key scale of this group's next item is loaded while this one is computed
    auto key_scale = [&](const ItemCursor& c) -> float {
      const int t = c.j * kKeys + row;
      return t < a.n ? __ldg(a.k_s + (size_t)c.bb * a.n + t) : 0.f;
    };
    if (grp) cur.next();
    float ks_next = i0 + grp < i1 ? key_scale(cur) : 0.f;
    for (long long it = i0 + grp; it < i1; it += 2, k += 2) {
      const int tb = grp;
      const ItemCursor c = cur;
      const float ks = ks_next;
      cur.next();
      cur.next();
      if (it + 2 < i1) ks_next = key_scale(cur);
      if (!W.wait_warp(&bars.t_full[tb], (k >> 1) & 1)) break;
      tc_fence_after();
      const int bb = c.bb, g = c.g;
      const int t = c.j * kKeys + row;
      const bool valid = t < a.n;
      const int nq = min(a.G, a.m - g * a.G);
      for (int qj = 0; qj < nq; ++qj) {
        const int mq = g * a.G + qj;
        const float4* w4 = reinterpret_cast<const float4*>(a.q_s + ((size_t)bb * a.m + mq) * a.h);
        float acc4[4] = {0.f, 0.f, 0.f, 0.f};  // four independent chains over the heads
        for (int c0 = 0; c0 < a.h; c0 += 64) {
          const int nc = min(4, (a.h - c0) >> 4);  // 16-column loads in this round (h is a multiple of 16)
          uint32_t v[4][16];
#pragma unroll
          for (int c = 0; c < 4; ++c)
            if (c < nc) tmem_ld_32x32b_16(lanes + (uint32_t)(tb * kMaxN + qj * a.h + c0 + 16 * c), v[c]);
          tmem_wait_ld();
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            if (c < nc) {
#pragma unroll
              for (int e = 0; e < 16; e += 4) {
                const float4 w = __ldg(w4 + ((c0 + 16 * c + e) >> 2));
                acc4[0] = fmaf(w.x, fmaxf(__uint_as_float(v[c][e + 0]), 0.f), acc4[0]);
                acc4[1] = fmaf(w.y, fmaxf(__uint_as_float(v[c][e + 1]), 0.f), acc4[1]);
                acc4[2] = fmaf(w.z, fmaxf(__uint_as_float(v[c][e + 2]), 0.f), acc4[2]);
                acc4[3] = fmaf(w.w, fmaxf(__uint_as_float(v[c][e + 3]), 0.f), acc4[3]);
              }
            }
          }
        }
        if (valid) a.o[((size_t)bb * a.m + mq) * a.n + t] = ((acc4[0] + acc4[1]) + (acc4[2] + acc4[3])) * ks;
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_addr(&bars.t_empty[tb]));
    }
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// ---------------------------------------------------------------------------- top-k

constexpr int kTopkThreads = 1024;
constexpr int kTopkTarget = 16384;  // positions per CTA the cluster size aims at
constexpr int kTopkMaxCached = 49152;  // positions per CTA kept in shared memory (192 KB)

struct TopkArgs {
  const float* scores;   // [rows, n]
  const int32_t* lens;   // [rows] or nullptr
  int32_t* out;          // [rows, k]
  int rows, n, k, chunk, cached;
};

// Order-preserving key of a float: larger float <=> larger key; -0 is +0.
MLA_DEV uint32_t order_key(float x) {
  uint32_t u = __float_as_uint(x);
  if (u == 0x80000000u) u = 0u;
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Exclusive prefix sum over the block's 1024 threads; *total gets the sum.
MLA_DEV uint32_t block_exclusive_scan(uint32_t v, uint32_t* warp_tot, uint32_t* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(~0u, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) warp_tot[warp] = x;
  __syncthreads();
  if (warp == 0) {
    uint32_t w = warp_tot[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(~0u, w, o);
      if (lane >= o) w += y;
    }
    warp_tot[lane] = w;  // inclusive over warps
  }
  __syncthreads();
  const uint32_t before = (warp > 0 ? warp_tot[warp - 1] : 0u) + x - v;
  *total = warp_tot[31];
  __syncthreads();  // warp_tot is reused by the next scan
  return before;
}

// Four 8-bit radix digits, most significant first. Each warp counts into its
// own 256-bin histogram (the first digits of real scores fall in few bins,
// and one shared histogram would serialise the whole block on them); the
// warps' histograms are summed per CTA, then across the cluster.
__global__ void __launch_bounds__(kTopkThreads, 1) mla_topk_kernel(const TopkArgs a) {
  extern __shared__ __align__(16) uint32_t keys[];
  __shared__ uint32_t whist[32][256];  // per-warp histograms
  __shared__ uint32_t hist[2][256];    // this CTA's sums, read by the cluster (double-buffered by pass)
  __shared__ uint32_t warp_tot[32];
  __shared__ uint32_t counts[2];  // this CTA's keys above the threshold, keys equal to it
  __shared__ uint32_t pick[2];    // radix pass result: bin, keys in higher bins
  __shared__ uint32_t wsum[2][32];  // per warp: keys above, keys equal (selection)
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int C = (int)cluster_nctarank(), c = (int)cluster_ctarank();
  const int row = (int)cluster_id_x();
  const int L = a.lens ? min(max(__ldg(a.lens + row), 0), a.n) : a.n;
  const int lo = c * a.chunk;
  const int cnt = max(0, min(lo + a.chunk, L) - lo);
  const float* src = a.scores + (size_t)row * a.n + lo;
  if (a.cached)
    for (int i = tid; i < cnt; i += kTopkThreads) keys[i] = order_key(__ldg(src + i));
  __syncthreads();
  auto key_at = [&](int i) -> uint32_t { return a.cached ? keys[i] : order_key(__ldg(src + i)); };

  const int K = min(a.k, L);
  const bool take_all = K == L;  // uniform over the cluster: every CTA sees the same row
  uint32_t prefix = 0u, mask = 0u, krem = (uint32_t)K;
  if (!take_all) {
#pragma unroll 1
    for (int p = 0; p < 4; ++p) {
      const int shift = 24 - 8 * p;
      for (int b = lane; b < 256; b += 32) whist[warp][b] = 0u;
      __syncwarp();
      for (int i = tid; i < cnt; i += kTopkThreads) {
        const uint32_t key = key_at(i);
        if ((key & mask) == prefix) atomicAdd(&whist[warp][(key >> shift) & 255u], 1u);
      }
      __syncthreads();
      uint32_t* h = hist[p & 1];
      if (tid < 256) {
        uint32_t v = 0u;
#pragma unroll 8
        for (int w = 0; w < 32; ++w) v += whist[w][tid];
        h[tid] = v;
      }
      cluster_sync();  // every CTA's histogram of this pass is complete
      // bin b = 255 - tid: an inclusive scan over tid counts the keys in bins >= b
      uint32_t tot = 0u;
      if (tid < 256) {
        const uint32_t a_local = smem_addr(&h[255 - tid]);
        for (int r = 0; r < C; ++r) tot += ld_shared_cluster_u32(map_to_rank(a_local, (uint32_t)r));
      }
      uint32_t sum;
      const uint32_t above = block_exclusive_scan(tot, warp_tot, &sum);  // keys in bins > b
      if (tid < 256 && above < krem && krem <= above + tot) {
        pick[0] = (uint32_t)(255 - tid);
        pick[1] = above;
      }
      __syncthreads();
      krem -= pick[1];
      prefix |= pick[0] << shift;
      mask |= 0xFFu << shift;
      __syncthreads();  // pick and the warp histograms are rewritten by the next pass
    }
  }
  // prefix is now the k-th largest key T; krem keys equal to T are taken, the
  // ones at the smallest positions (take_all: every position below L).
  // Selection: warp w walks positions [w * per, (w + 1) * per) in rounds of
  // 32 consecutive positions (lane order = position order), so prefix counts
  // come from ballots.
  const uint32_t T = prefix;
  const int per = ((cnt + 32 * 32 - 1) / (32 * 32)) * 32;  // positions per warp, a multiple of 32
  const int w0 = warp * per, w1 = min(w0 + per, cnt);
  uint32_t gt = 0u, eq = 0u;
  for (int base = w0; base < w1; base += 32) {
    const int i = base + lane;
    const uint32_t key = i < w1 ? key_at(i) : 0u;
    gt += __popc(__ballot_sync(~0u, i < w1 && (take_all || key > T)));
    eq += __popc(__ballot_sync(~0u, i < w1 && !take_all && key == T));
  }
  if (lane == 0) {
    wsum[0][warp] = gt;
    wsum[1][warp] = eq;
  }
  __syncthreads();
  // this warp's offsets among the CTA's warps (a short serial sum per lane 0)
  uint32_t g_pre = 0u, e_pre = 0u, g_cta = 0u, e_cta = 0u;
  for (int w = 0; w < 32; ++w) {
    const uint32_t gw = wsum[0][w], ew = wsum[1][w];
    if (w < warp) {
      g_pre += gw;
      e_pre += ew;
    }
    g_cta += gw;
    e_cta += ew;
  }
  if (tid == 0) {
    counts[0] = g_cta;
    counts[1] = e_cta;
  }
  cluster_sync();  // every CTA's counts are visible
  // where this CTA's selections start: the CTAs before it in rank order
  uint32_t e_before = 0u, out_base = 0u;
  for (int r = 0; r < c; ++r) {
    const uint32_t g_r = ld_shared_cluster_u32(map_to_rank(smem_addr(&counts[0]), (uint32_t)r));
    const uint32_t e_r = ld_shared_cluster_u32(map_to_rank(smem_addr(&counts[1]), (uint32_t)r));
    const uint32_t take_r = min(e_r, krem > e_before ? krem - e_before : 0u);
    out_base += g_r + take_r;
    e_before += e_r;
  }
  const uint32_t take_cta = min(e_cta, krem > e_before ? krem - e_before : 0u);
  // ties this warp takes: those of the CTA's first take_cta ties that fall in it
  uint32_t ties_seen = e_pre;                       // CTA ties at positions before this round
  uint32_t taken_before = min(e_pre, take_cta);     // ties taken by earlier warps
  uint32_t w = out_base + g_pre + taken_before;     // output slot of this warp's next selection
  int32_t* orow = a.out + (size_t)row * a.k;
  const uint32_t below = (1u << lane) - 1u;
  for (int base = w0; base < w1; base += 32) {
    const int i = base + lane;
    const uint32_t key = i < w1 ? key_at(i) : 0u;
    const bool is_gt = i < w1 && (take_all || key > T);
    const bool is_eq = i < w1 && !take_all && key == T;
    const uint32_t eqm = __ballot_sync(~0u, is_eq);
    const bool take_eq = is_eq && ties_seen + __popc(eqm & below) < take_cta;
    const uint32_t selm = __ballot_sync(~0u, is_gt || take_eq);
    if (is_gt || take_eq) orow[w + __popc(selm & below)] = lo + i;
    w += __popc(selm);
    ties_seen += __popc(eqm);
  }
  if (c == C - 1)
    for (int i = K + tid; i < a.k; i += kTopkThreads) orow[i] = -1;
  cluster_sync();  // no CTA leaves while another may still read its counters
}

// ---------------------------------------------------------------------------- host side

std::mutex g_mu;
bool g_ready[64] = {};

bool aligned(const void* p, uintptr_t n) { return ((uintptr_t)p & (n - 1)) == 0; }

bool setup_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return false;
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_ready[dev]) {
    if (cudaFuncSetAttribute((const void*)mla_index_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem) !=
            cudaSuccess ||
        cudaFuncSetAttribute((const void*)mla_topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             kTopkMaxCached * 4) != cudaSuccess)
      return false;
    g_ready[dev] = true;
  }
  return true;
}

mla_status_t check_index(const mla_index_desc_t* d) {
  if (!d) return MLA_ERR_INVALID_ARG;
  if (d->batch < 0 || d->q_len < 1 || d->num_heads < 1 || d->num_keys < 0) return MLA_ERR_INVALID_ARG;
  if (d->head_dim != kDim || d->num_heads % 16 != 0 || d->num_heads > kMaxN) return MLA_ERR_UNSUPPORTED;
  if ((long long)d->batch * d->q_len * d->num_heads > 0x7fffffffLL || (long long)d->batch * d->num_keys > 0x7fffffffLL)
    return MLA_ERR_UNSUPPORTED;
  return MLA_OK;
}

}  // namespace idx
}  // namespace mla

using namespace mla;

extern "C" MLA_API mla_status_t mla_index_scores(const mla_index_desc_t* desc, const void* q, const float* q_s,
                                                 const void* k, const float* k_s, float* scores,
                                                 uint32_t* error_word, mla_stream_t stream) {
  mla_status_t st = idx::check_index(desc);
  if (st != MLA_OK) return st;
  if (desc->batch == 0 || desc->num_keys == 0) return MLA_OK;
  if (!q || !q_s || !k || !k_s || !scores) return MLA_ERR_INVALID_ARG;
  if (!idx::aligned(q, 16) || !idx::aligned(k, 16) || !idx::aligned(q_s, 16) || !idx::aligned(k_s, 4) ||
      !idx::aligned(scores, 4) || !idx::aligned(error_word, 4))
    return MLA_ERR_INVALID_ARG;
  if (!idx::setup_device()) return MLA_ERR_CUDA;
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return MLA_ERR_CUDA;
  PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
  if (!enc) return MLA_ERR_CUDA;

  idx::Args a;
  a.q_s = q_s;
  a.k_s = k_s;
  a.o = scores;
  a.err = error_word;
  a.b = desc->batch;
  a.m = desc->q_len;
  a.h = desc->num_heads;
  a.n = desc->num_keys;
  a.G = idx::kMaxN / a.h < a.m ? idx::kMaxN / a.h : a.m;
  a.N = a.G * a.h;
  a.groups = (a.m + a.G - 1) / a.G;
  a.tiles = (a.n + idx::kKeys - 1) / idx::kKeys;
  a.items = (long long)a.b * a.groups * a.tiles;
  const long long grid = a.items < sms ? a.items : sms;
  a.per_cta = (a.items + grid - 1) / grid;

  idx::Maps maps;
  cuuint32_t elem[2] = {1, 1};
  cuuint64_t kdims[2] = {(cuuint64_t)idx::kDim, (cuuint64_t)a.b * a.n};
  cuuint64_t qdims[2] = {(cuuint64_t)idx::kDim, (cuuint64_t)a.b * a.m * a.h};
  cuuint64_t stride[1] = {(cuuint64_t)idx::kDim};
  cuuint32_t kbox[2] = {(cuuint32_t)idx::kDim, (cuuint32_t)idx::kKeys};
  cuuint32_t qbox[2] = {(cuuint32_t)idx::kDim, (cuuint32_t)a.N};
  if (enc(&maps.k, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(k), kdims, stride, kbox, elem,
          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS ||
      enc(&maps.q, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(q), qdims, stride, qbox, elem,
          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return MLA_ERR_CUDA;
  idx::mla_index_kernel<<<(unsigned)grid, idx::kThreads, idx::kSmem, (cudaStream_t)stream>>>(maps, a);
  return cudaGetLastError() == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
}

extern "C" MLA_API mla_status_t mla_topk(const mla_topk_desc_t* desc, const float* scores, const int32_t* valid_lens,
                                         int32_t* indices, mla_stream_t stream) {
  if (!desc) return MLA_ERR_INVALID_ARG;
  if (desc->rows < 0 || desc->num_keys < 0 || desc->k < 1) return MLA_ERR_INVALID_ARG;
  if (desc->rows == 0) return MLA_OK;
  if ((desc->num_keys > 0 && !scores) || !indices) return MLA_ERR_INVALID_ARG;
  if (!idx::aligned(scores, 4) || !idx::aligned(valid_lens, 4) || !idx::aligned(indices, 4))
    return MLA_ERR_INVALID_ARG;
  if ((long long)desc->rows * 8 > 0x7fffffffLL) return MLA_ERR_UNSUPPORTED;
  if (!idx::setup_device()) return MLA_ERR_CUDA;
  const int n = desc->num_keys;
  int C = 1;
  while (C < 8 && (n + C - 1) / C > idx::kTopkTarget) C *= 2;
  idx::TopkArgs a;
  a.scores = scores;
  a.lens = valid_lens;
  a.out = indices;
  a.rows = desc->rows;
  a.n = n;
  a.k = desc->k;
  a.chunk = ((n + C - 1) / C + 3) & ~3;
  a.cached = a.chunk <= idx::kTopkMaxCached ? 1 : 0;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(desc->rows * C), 1, 1);
  cfg.blockDim = dim3(idx::kTopkThreads, 1, 1);
  cfg.dynamicSmemBytes = a.cached ? (size_t)a.chunk * 4 : 0;
  cfg.stream = (cudaStream_t)stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = (unsigned)C;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, idx::mla_topk_kernel, a) == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
}
