// Steps a2-a7: split-KV MLA decode over the paged latent cache on sm_100a.
//
// One worker = a cluster of two CTAs on two SMs. A task (one query token of
// one sequence, up to 128 heads) is processed by both CTAs together, each
// owning half of the 512 latent output columns:
//
//   CTA rank 0: loads cache columns [0, 320); scores over columns [0, 288);
//               output columns [0, 256)
//   CTA rank 1: loads cache columns [256, 576); scores over [288, 576);
//               output columns [256, 512)
//
// The full fp32 output accumulator of 128 heads x 512 columns is exactly one
// SM's tensor memory, so it is split across the pair; the score contraction
// is split the same way. Each CTA sends its partial score tile to the peer
// through distributed shared memory (st.async) as 24-bit floats (fp32 rounded
// to its top three bytes: relative error <= 2^-16), which cuts the cross-SM
// traffic by a quarter (the SM-to-SM path sustains ~15 B/clk per direction),
// and adds the peer's partial to its own fp32 partial. Each CTA then runs its
// own online softmax over its half of the output columns: the halves need not
// agree bit for bit; each is a consistent softmax average.
//
// Per CTA (448 threads):
//   warp 0      TMA producer: 64-token pages (block table) or 64 gathered rows
//               (top-k indices, tile::gather4) into a 4-stage ring, 5 boxes of
//               64 rows x 128 B (128-byte swizzle) per stage
//   warp 1      tcgen05 issuer: S = Q_slice * K_slice^T (M=128 heads, N=64
//               tokens, K=288, A = Q in TMEM), two tiles ahead of
//               O += P * V (M=128, N=256, K=64, A = P in TMEM, B = the same
//               stage read MN-major)
//   warps 2-9   softmax: two threads per head row, 32 tokens each; own
//               partial scores prefetched from TMEM a tile ahead (so S runs
//               two tiles ahead), plus the peer's 24-bit partial; online
//               softmax in base 2 with lazy rescaling, P into TMEM; epilogue
//   warps 10-13 sender: read each partial S tile from TMEM as soon as it is
//               computed, round it to 24-bit floats and push it into the peer's receive
//               slot, so remote-store backpressure never stalls the softmax
//               warps; also relays "receive slot read" to the peer
//
// TMEM columns: O [0,256) | Q [256,400) | S [400,464) | P [464,496).
#include <cuda.h>
#include <math.h>

#include "common.cuh"
#include "sm100.cuh"

namespace mla {
namespace dec {

using namespace ptx;

constexpr int kThreads = 448;
constexpr int kStages = 4;
constexpr int kXSlots = 2;
constexpr int kBoxBytes = kPage * 128;  // 64 rows x 64 bf16 (one 128-B swizzle row each)
constexpr int kBoxesPerStage = 5;       // 320 columns per CTA
constexpr int kStageBytes = kBoxesPerStage * kBoxBytes;
constexpr int kXBytes = kRowsPerTask * 64 * 3;  // one 24-bit partial score tile (per slot)
constexpr int kSSteps = 18;                     // 288 columns / 16 per MMA
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kTmemO = 0, kTmemQ = 256, kTmemS = 400, kTmemP = 464;
constexpr float kRescaleThreshold = 8.0f;  // log2 units: tolerate p up to 2^8 before rescaling O
constexpr uint64_t kTimeoutNs = 2000000000ull;
// Shared memory: [misc | stage ring | receive slots]; the stage ring must be
// 1024-byte aligned (128-byte swizzle atoms), which holds when the dynamic
// shared memory base is (checked at run time).
constexpr int kMiscBytes = 3072;
constexpr int kSmemBytes = kMiscBytes + kStages * kStageBytes + kXSlots * kXBytes;

struct Misc {
  uint64_t full[kStages];
  uint64_t empty[kStages];
  uint64_t s_full, s_free, p_full, p_free, o_full, o_empty, q_full, mma_done;
  uint64_t x_full[kXSlots], x_empty[kXSlots], x_read[kXSlots];
  uint64_t pair_bar[4];
  uint64_t stage_mask[kStages];
  uint32_t tmem_base;
  uint32_t abort_flag;
  uint32_t xdummy;  // target of the peer's 4-byte "slot read" stores
  float red_max[2][2][kRowsPerTask];
};
static_assert(sizeof(Misc) <= kMiscBytes, "misc region too small");

// Bounded waits: a wait that runs out sets the CTA's abort flag and the
// device error word, and every later wait returns at once.
struct Waiter {
  Misc* misc;
  uint32_t* err;

  MLA_DEV bool aborted() const { return *reinterpret_cast<volatile uint32_t*>(&misc->abort_flag) != 0; }
  MLA_DEV void fail() {
    *reinterpret_cast<volatile uint32_t*>(&misc->abort_flag) = 1u;
    atomicOr(err, kErrTimeout);
  }
  template <bool kCluster>
  MLA_DEV bool wait_impl(uint64_t* bar, uint32_t parity, bool honour_abort) {
    const uint32_t a = smem_addr(bar);
    if (kCluster ? mbar_try_wait_cluster(a, parity) : mbar_try_wait(a, parity)) return true;
    const uint64_t t0 = global_timer_ns();
    while (true) {
      if (kCluster ? mbar_try_wait_cluster(a, parity) : mbar_try_wait(a, parity)) return true;
      if (honour_abort && aborted()) return false;
      if (global_timer_ns() - t0 > kTimeoutNs) {
        fail();
        return false;
      }
    }
  }
  MLA_DEV bool wait(uint64_t* bar, uint32_t parity) { return wait_impl<false>(bar, parity, true); }
  MLA_DEV bool wait_cluster(uint64_t* bar, uint32_t parity) { return wait_impl<true>(bar, parity, true); }
  MLA_DEV bool drain(uint64_t* bar, uint32_t parity) { return wait_impl<false>(bar, parity, false); }
  // Every lane waits (each gets the acquire); the outcome is made warp-uniform
  // so that no lane leaves a loop its warp-mates stay in.
  MLA_DEV bool wait_warp(uint64_t* bar, uint32_t parity) { return __all_sync(~0u, wait(bar, parity)); }
  MLA_DEV bool wait_cluster_warp(uint64_t* bar, uint32_t parity) {
    return __all_sync(~0u, wait_cluster(bar, parity));
  }
};

// The worker's contiguous range of global pages, walked task by task.
struct Cursor {
  const int32_t* prefix;
  int T, lo, hi, t;

  MLA_DEV void init(const int32_t* plan, int worker) {
    T = plan[kPlanTasks];
    const int quota = plan[kPlanQuota];
    const int total = plan[kPlanTotal];
    prefix = plan + plan_prefix_off();
    lo = worker * quota;
    hi = min(lo + quota, total);
    if (lo >= total || T <= 0) {
      t = T;
      return;
    }
    int a = 0, b = T - 1;  // largest t with prefix[t] <= lo
    while (a < b) {
      const int mid = (a + b + 1) >> 1;
      if (prefix[mid] <= lo) a = mid;
      else b = mid - 1;
    }
    t = a;
  }
  MLA_DEV bool next(int& task, int& pg0, int& pg1, bool& split) {
    while (t < T && prefix[t] < hi) {
      const int cur = t++;
      const int p0 = prefix[cur], p1 = prefix[cur + 1];
      const int a = max(lo, p0), b = min(hi, p1);
      if (a < b) {
        task = cur;
        pg0 = a - p0;
        pg1 = b - p0;
        split = !(pg0 == 0 && pg1 == p1 - p0);
        return true;
      }
    }
    return false;
  }
};

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    mla_decode_kernel(const __grid_constant__ CUtensorMap tm_tile, const __grid_constant__ CUtensorMap tm_row,
                      const DecodeArgs a) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  Misc* misc = reinterpret_cast<Misc*>(smem_raw);
  const uint32_t raw_base = smem_addr(smem_raw);
  const uint32_t stage_base = raw_base + kMiscBytes;
  const uint32_t xbuf = stage_base + kStages * kStageBytes;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t crank = cluster_ctarank();
  const uint32_t peer = crank ^ 1u;
  const int worker = (int)cluster_id_x();
  Waiter W{misc, reinterpret_cast<uint32_t*>(a.plan + kPlanErr)};

  if (stage_base & 1023u) {  // cannot place the swizzled ring: refuse instead of corrupting
    if (threadIdx.x == 0) atomicOr(W.err, kErrTimeout);
    return;
  }
  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(smem_addr(&misc->full[s]), 1);
      mbar_init(smem_addr(&misc->empty[s]), 1);
    }
    mbar_init(smem_addr(&misc->s_full), 1);
    mbar_init(smem_addr(&misc->s_free), 12);  // 8 softmax + 4 sender warps
    mbar_init(smem_addr(&misc->p_full), 8);
    mbar_init(smem_addr(&misc->p_free), 1);
    mbar_init(smem_addr(&misc->o_full), 1);
    mbar_init(smem_addr(&misc->o_empty), 8);
    mbar_init(smem_addr(&misc->q_full), 8);
    mbar_init(smem_addr(&misc->mma_done), 1);
    for (int xs = 0; xs < kXSlots; ++xs) {
      mbar_init(smem_addr(&misc->x_full[xs]), 1);
      mbar_init(smem_addr(&misc->x_empty[xs]), 1);
      mbar_init(smem_addr(&misc->x_read[xs]), 8);
    }
    for (int qd = 0; qd < 4; ++qd) mbar_init(smem_addr(&misc->pair_bar[qd]), 2);
    misc->abort_flag = 0u;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tm_tile);
    prefetch_tmap(&tm_row);
  }
  if (warp == 1) {
    tmem_alloc(smem_addr(&misc->tmem_base), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  cluster_sync();
  tc_fence_after();
  const uint32_t tmem = misc->tmem_base;
  const int col0 = crank ? 256 : 0;  // first cache column loaded by this CTA

  Cursor cur;
  cur.init(a.plan, worker);
  const int T = cur.T;
  const int32_t* ntok_arr = a.plan + plan_ntok_off(T);
  int task = 0, pg0 = 0, pg1 = 0;
  bool split = false;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    int k = 0;
    while (cur.next(task, pg0, pg1, split)) {
      const int b = task / a.q_len, qi = task % a.q_len;
      const int ntok = ntok_arr[task];
      const int32_t* bt_row = a.block_table + (size_t)b * a.max_pages_per_seq;
      if (a.topk == 0) {
        for (int i0 = pg0; i0 < pg1; i0 += 32) {
          const int i = i0 + lane;
          int pid = 0;
          bool pok = false;
          if (i < pg1) {
            pid = bt_row[i];
            pok = (unsigned)pid < (unsigned)a.num_pages;
            if (!pok) atomicOr(W.err, kErrPageId);
          }
          const int cnt = min(32, pg1 - i0);
          for (int jj = 0; jj < cnt; ++jj, ++k) {
            const int page = __shfl_sync(~0u, pid, jj);
            const int ok = __shfl_sync(~0u, pok ? 1 : 0, jj);
            const int tile = i0 + jj;
            const int nvalid = min(kPage, ntok - tile * kPage);
            const uint64_t mask = !ok ? 0ull : (nvalid >= kPage ? ~0ull : ((1ull << nvalid) - 1ull));
            const int s = k % kStages;
            if (!W.wait_warp(&misc->empty[s], ((k / kStages) & 1) ^ 1)) goto producer_done;
            if (lane == 0) {
              misc->stage_mask[s] = mask;
              const uint32_t fb = smem_addr(&misc->full[s]);
              mbar_arrive_expect_tx(fb, kStageBytes);
              const int row = (ok ? page : 0) * kPage;
              const uint32_t dst = stage_base + s * kStageBytes;
#pragma unroll
              for (int bx = 0; bx < kBoxesPerStage; ++bx)
                tma_load_2d(dst + bx * kBoxBytes, &tm_tile, col0 + 64 * bx, row, fb);
            }
            __syncwarp();
          }
        }
      } else {
        const int32_t* idx_row = a.indices + (size_t)(b * a.q_len + qi) * a.topk;
        const int L = a.seq_lens[b];
        for (int tile = pg0; tile < pg1; ++tile, ++k) {
          int rows[2];
          bool valid[2];
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const int slot = tile * kPage + lane + 32 * h;
            const int idx = slot < ntok ? idx_row[slot] : -1;
            const bool in_range = idx >= 0 && idx < L;
            if (slot < ntok && !in_range && idx != -1) atomicOr(W.err, kErrIndex);
            int pid = 0;
            bool pok = false;
            if (in_range) {
              pid = bt_row[idx / kPage];
              pok = (unsigned)pid < (unsigned)a.num_pages;
              if (!pok) atomicOr(W.err, kErrPageId);
            }
            rows[h] = pok ? pid * kPage + (idx % kPage) : 0;
            valid[h] = pok;
          }
          const uint64_t mask =
              (uint64_t)__ballot_sync(~0u, valid[0]) | ((uint64_t)__ballot_sync(~0u, valid[1]) << 32);
          int r[4];
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const int src = (4 * lane + u) & 31;
            const int r0 = __shfl_sync(~0u, rows[0], src);
            const int r1 = __shfl_sync(~0u, rows[1], src);
            r[u] = lane < 8 ? r0 : r1;
          }
          const int s = k % kStages;
          if (!W.wait_warp(&misc->empty[s], ((k / kStages) & 1) ^ 1)) goto producer_done;
          const uint32_t fb = smem_addr(&misc->full[s]);
          if (lane == 0) {
            misc->stage_mask[s] = mask;
            mbar_arrive_expect_tx(fb, kStageBytes);
          }
          __syncwarp();
          if (lane < 16) {
            const uint32_t dst = stage_base + s * kStageBytes + lane * 4 * 128;
#pragma unroll
            for (int bx = 0; bx < kBoxesPerStage; ++bx)
              tma_gather4(dst + bx * kBoxBytes, &tm_row, col0 + 64 * bx, r[0], r[1], r[2], r[3], fb);
          }
          __syncwarp();
        }
      }
    }
  producer_done:
    // Let every issued copy land before the CTA can exit.
    for (int d = max(0, k - kStages); d < k; ++d) W.drain(&misc->full[d % kStages], (d / kStages) & 1);
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idS = idesc_bf16_f32(128, 64, 0, 0);
      constexpr uint32_t idO = idesc_bf16_f32(128, 256, 0, 1);
      int k = 0, j = 0;
      // S for tile kk into the (single) S buffer, once the stage landed and the
      // softmax warps have read the previous S.
      auto issue_s = [&](int kk) -> bool {
        const int s = kk % kStages;
        if (!W.wait(&misc->full[s], (kk / kStages) & 1)) return false;
        if (kk > 0 && !W.wait(&misc->s_free, (kk - 1) & 1)) return false;
        tc_fence_after();
        const uint32_t sb = stage_base + s * kStageBytes;
#pragma unroll
        for (int ks = 0; ks < kSSteps; ++ks) {
          const int c = (crank ? 32 : 0) + 16 * ks;  // column relative to col0
          const uint32_t baddr = sb + (c >> 6) * kBoxBytes + (c & 63) * 2;
          mma_tmem_a(tmem + kTmemS, tmem + kTmemQ + 8 * ks, smem_desc_sw128(baddr, 16, 1024), idS, ks > 0 ? 1u : 0u);
        }
        mma_commit(smem_addr(&misc->s_full));
        return true;
      };
      // O (+)= P V for tile kk; releases the P buffer and the stage.
      auto issue_pv = [&](int kk, bool first, int item) -> bool {
        if (!W.wait(&misc->p_full, kk & 1)) return false;
        if (first && item > 0 && !W.wait(&misc->o_empty, (item - 1) & 1)) return false;
        tc_fence_after();
        const int s = kk % kStages;
        const uint32_t vb = stage_base + s * kStageBytes;
#pragma unroll
        for (int u = 0; u < 4; ++u)
          mma_tmem_a(tmem + kTmemO, tmem + kTmemP + 8 * u, smem_desc_sw128(vb + u * 2048, kBoxBytes, 1024), idO,
                     (first && u == 0) ? 0u : 1u);
        mma_commit(smem_addr(&misc->p_free));
        mma_commit(smem_addr(&misc->empty[s]));
        return true;
      };
      while (cur.next(task, pg0, pg1, split)) {
        if (!W.wait(&misc->q_full, j & 1)) break;
        const int n = pg1 - pg0;
        // S runs two tiles ahead of PV: the softmax warps read S(k+i+1) into
        // registers when they start tile k+i, which frees the buffer for
        // S(k+i+2) before PV(k+i) can be issued.
        bool ok = issue_s(k);
        if (ok && n > 1) ok = issue_s(k + 1);
        for (int i = 0; ok && i < n; ++i) {
          if (i + 2 < n) ok = issue_s(k + i + 2);
          if (ok) ok = issue_pv(k + i, i == 0, j);
        }
        if (!ok) break;
        k += n;
        mma_commit(smem_addr(&misc->o_full));
        ++j;
      }
      mma_commit(smem_addr(&misc->mma_done));
      W.drain(&misc->mma_done, 0);
    }
    __syncwarp();
  } else if (warp >= 2 && warp <= 9) {
    // ------------------------------------------------------------ softmax
    const int sw = warp - 2;
    const int quad = warp & 3;  // TMEM lane quadrant this warp may access
    const int hh = sw >> 2;     // token half of the tile / column half of O
    const int row = quad * 32 + lane;
    const uint32_t lane_base = (uint32_t)(quad * 32) << 16;
    const bool row_valid = row < a.heads;
    // active sender warps x 32 lanes x 12 chunks x 16 B arrive per slot use
    const uint32_t xbytes = (uint32_t)((a.heads + 31) / 32) * 6144u;
    const bool expect_thread = (warp == 4 && lane == 0);
    const int tid_sm = threadIdx.x - 64;
    // This warp's chunks of a receive slot: quadrant block [12 chunks][32 lanes]
    // x 16 B; the lane's row is 64 packed 24-bit values (48 words), chunks
    // 6*hh .. 6*hh+5 hold this thread's 32 tokens.
    const uint32_t xoff = (uint32_t)quad * 6144u + (uint32_t)(6 * hh) * 512u + (uint32_t)lane * 16u;
    int k = 0, j = 0, pair_n = 0;

    auto pair_sync = [&]() -> bool {
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_addr(&misc->pair_bar[quad]));
      return W.wait_warp(&misc->pair_bar[quad], (pair_n++) & 1);
    };
    // Own fp32 partial scores of tile kk into registers; frees the S buffer.
    auto fetch = [&](int kk, uint32_t(&dst)[32]) -> bool {
      if (!W.wait_warp(&misc->s_full, kk & 1)) return false;
      tc_fence_after();
      tmem_ld_32(tmem + lane_base + kTmemS + 32 * hh, dst);
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_addr(&misc->s_free));
      return true;
    };

    while (cur.next(task, pg0, pg1, split)) {
      const size_t qrow = (size_t)task * a.heads + row;
      {
        uint32_t qv[72];
        if (row_valid) {
          const uint4* src = reinterpret_cast<const uint4*>(a.q + qrow * kDQK + crank * 288 + hh * 144);
#pragma unroll
          for (int u = 0; u < 18; ++u) {
            const uint4 v = src[u];
            qv[4 * u + 0] = v.x;
            qv[4 * u + 1] = v.y;
            qv[4 * u + 2] = v.z;
            qv[4 * u + 3] = v.w;
          }
        } else {
#pragma unroll
          for (int u = 0; u < 72; ++u) qv[u] = 0u;
        }
        const uint32_t qa = tmem + lane_base + kTmemQ + 72 * hh;
        tmem_st_32(qa, *reinterpret_cast<const uint32_t(*)[32]>(&qv[0]));
        tmem_st_32(qa + 32, *reinterpret_cast<const uint32_t(*)[32]>(&qv[32]));
        tmem_st_8(qa + 64, *reinterpret_cast<const uint32_t(*)[8]>(&qv[64]));
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_addr(&misc->q_full));
      }

      float m_run = -INFINITY, l_run = 0.f;
      const int ntiles = pg1 - pg0;
      uint32_t own[32], nxt[32];
      if (!fetch(k, own)) goto softmax_done;
      for (int i = 0; i < ntiles; ++i, ++k) {
        const int s = k % kStages;
        const int xs = k & 1;
        if (i + 1 < ntiles && !fetch(k + 1, nxt)) goto softmax_done;
        // the peer's partial scores of tile k (sent about a tile earlier)
        if (expect_thread) mbar_arrive_expect_tx(smem_addr(&misc->x_full[xs]), xbytes);
        if (!W.wait_warp(&misc->x_full[xs], (k >> 1) & 1)) goto softmax_done;
        float sc[32];
        {
          uint32_t w[24];
#pragma unroll
          for (int c = 0; c < 6; ++c) {
            const uint4 v = ld_shared_v4(xbuf + xs * kXBytes + xoff + c * 512);
            w[4 * c + 0] = v.x;
            w[4 * c + 1] = v.y;
            w[4 * c + 2] = v.z;
            w[4 * c + 3] = v.w;
          }
#pragma unroll
          for (int g = 0; g < 8; ++g) {
            float f[4];
            unpack24x4(w[3 * g], w[3 * g + 1], w[3 * g + 2], f);
#pragma unroll
            for (int e = 0; e < 4; ++e) sc[4 * g + e] = __uint_as_float(own[4 * g + e]) + f[e];
          }
        }
#pragma unroll
        for (int c = 0; c < 32; ++c) own[c] = nxt[c];
        // slot read (the arrive's release orders the loads before it); the
        // sender warp relays this to the peer
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_addr(&misc->x_read[xs]));

        // mask (written by the producer before the stage's full barrier)
        if (!W.wait_warp(&misc->full[s], (k / kStages) & 1)) goto softmax_done;
        const uint64_t mask64 = misc->stage_mask[s];
        const uint32_t mask = (uint32_t)(mask64 >> (32 * hh));
        if (mask != ~0u) {
#pragma unroll
          for (int c = 0; c < 32; ++c) sc[c] = ((mask >> c) & 1u) ? sc[c] : -INFINITY;
        }
        float mx[16];
#pragma unroll
        for (int c = 0; c < 16; ++c) mx[c] = fmaxf(sc[c], sc[c + 16]);
#pragma unroll
        for (int c = 0; c < 8; ++c) mx[c] = fmaxf(mx[c], mx[c + 8]);
#pragma unroll
        for (int c = 0; c < 4; ++c) mx[c] = fmaxf(mx[c], mx[c + 4]);
        // the scale is positive: scaling after the max is the same as before it
        const float mloc = fmaxf(fmaxf(mx[0], mx[2]), fmaxf(mx[1], mx[3])) * a.scale_log2;
        misc->red_max[k & 1][hh][row] = mloc;
        if (!pair_sync()) goto softmax_done;
        const float mtile = fmaxf(misc->red_max[k & 1][0][row], misc->red_max[k & 1][1][row]);
        const float m_new = fmaxf(m_run, mtile);
        float alpha = 1.f;
        bool corr = false;
        if (m_new > m_run + kRescaleThreshold) {
          alpha = ex2(m_run - m_new);
          l_run *= alpha;
          m_run = m_new;
          corr = i > 0;
        }
        const float m_use = (m_run == -INFINITY) ? 0.f : m_run;
        const float sl2 = a.scale_log2;
        uint32_t pp[16];
        float ps[16];
#pragma unroll
        for (int c = 0; c < 16; ++c) {
          const float p0 = ex2(fmaf(sc[2 * c], sl2, -m_use));
          const float p1 = ex2(fmaf(sc[2 * c + 1], sl2, -m_use));
          pp[c] = pack_bf16x2(p0, p1);
          ps[c] = p0 + p1;
        }
#pragma unroll
        for (int c = 0; c < 8; ++c) ps[c] += ps[c + 8];
#pragma unroll
        for (int c = 0; c < 4; ++c) ps[c] += ps[c + 4];
        l_run += (ps[0] + ps[2]) + (ps[1] + ps[3]);

        // PV of the previous tile must be done before O and P are touched
        if (k > 0 && !W.wait_warp(&misc->p_free, (k - 1) & 1)) goto softmax_done;
        tc_fence_after();
        if (__any_sync(~0u, corr)) {
          const float f = corr ? alpha : 1.f;
#pragma unroll 1
          for (int c = 0; c < 4; ++c) {
            uint32_t o[32];
            const uint32_t oa = tmem + lane_base + kTmemO + 128 * hh + 32 * c;
            tmem_ld_32(oa, o);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * f);
            tmem_st_32(oa, o);
          }
        }
        tmem_st_16(tmem + lane_base + kTmemP + 16 * hh, pp);
        if (mask64 != ~0ull) {
          // masked tokens' V rows may hold anything (even NaN): zero them so 0 * V stays 0
          const uint32_t sb = stage_base + s * kStageBytes;
          for (int e = tid_sm; e < kPage * 32; e += 256) {
            const int r = e >> 5, c = e & 31;
            if (!((mask64 >> r) & 1ull)) st_shared_v4(sb + (c >> 3) * kBoxBytes + r * 128 + (c & 7) * 16, make_uint4(0, 0, 0, 0));
          }
          fence_proxy_async_smem();
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_addr(&misc->p_full));
      }

      // ------------------------------------------------------------ epilogue
      // The two threads of a row combine their fp32 row sums through red_max
      // (slot (k & 1) was last read before the previous pair sync); the extra
      // sync keeps the next tile's max from overwriting it too early.
      misc->red_max[k & 1][hh][row] = l_run;
      if (!pair_sync()) goto softmax_done;
      {
        const float l_tot = misc->red_max[k & 1][0][row] + misc->red_max[k & 1][1][row];
        if (!pair_sync()) goto softmax_done;
        if (!W.wait_warp(&misc->o_full, j & 1)) goto softmax_done;
        tc_fence_after();
        const float inv = l_tot > 0.f ? 1.f / l_tot : 0.f;
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          uint32_t o[32];
          tmem_ld_32(tmem + lane_base + kTmemO + 128 * hh + 32 * c, o);
          tmem_wait_ld();
          if (row_valid) {
            const int col = (int)crank * 256 + 128 * hh + 32 * c;
            if (!split) {
              uint4* dst = reinterpret_cast<uint4*>(a.out + qrow * kDLatent + col);
#pragma unroll
              for (int u = 0; u < 4; ++u) {
                uint4 v;
                v.x = pack_bf16x2(__uint_as_float(o[8 * u + 0]) * inv, __uint_as_float(o[8 * u + 1]) * inv);
                v.y = pack_bf16x2(__uint_as_float(o[8 * u + 2]) * inv, __uint_as_float(o[8 * u + 3]) * inv);
                v.z = pack_bf16x2(__uint_as_float(o[8 * u + 4]) * inv, __uint_as_float(o[8 * u + 5]) * inv);
                v.w = pack_bf16x2(__uint_as_float(o[8 * u + 6]) * inv, __uint_as_float(o[8 * u + 7]) * inv);
                dst[u] = v;
              }
            } else {
              float4* dst = reinterpret_cast<float4*>(
                  a.part_o + ((size_t)(worker + task) * a.heads + row) * kDLatent + col);
#pragma unroll
              for (int u = 0; u < 8; ++u)
                dst[u] = make_float4(__uint_as_float(o[4 * u + 0]) * inv, __uint_as_float(o[4 * u + 1]) * inv,
                                     __uint_as_float(o[4 * u + 2]) * inv, __uint_as_float(o[4 * u + 3]) * inv);
            }
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_addr(&misc->o_empty));
        if (hh == 0 && row_valid) {
          // each CTA's half has its own normaliser; the unsplit LSE comes from rank 0
          const float lse = l_tot > 0.f ? (m_run + log2f(l_tot)) * 0.69314718055994530942f : -INFINITY;
          if (split) a.part_lse[((size_t)(worker + task) * 2 + crank) * a.heads + row] = lse;
          else if (crank == 0) a.lse[qrow] = lse;
        }
      }
      ++j;
    }
  softmax_done:
    __syncwarp();
  } else if (warp >= 10) {
    // ------------------------------------------------------------ sender
    const int quad = warp & 3;
    const uint32_t lane_base = (uint32_t)(quad * 32) << 16;
    const bool warp_active = quad * 32 < a.heads;
    const bool expect_thread = (warp == 10 && lane == 0);
    uint32_t xfull_peer[kXSlots], xbuf_peer[kXSlots], xempty_peer[kXSlots];
#pragma unroll
    for (int xs = 0; xs < kXSlots; ++xs) {
      xfull_peer[xs] = map_to_rank(smem_addr(&misc->x_full[xs]), peer);
      xempty_peer[xs] = map_to_rank(smem_addr(&misc->x_empty[xs]), peer);
      xbuf_peer[xs] = map_to_rank(xbuf + xs * kXBytes, peer) + (uint32_t)quad * 6144u + (uint32_t)lane * 16u;
    }
    const uint32_t xdummy_peer = map_to_rank(smem_addr(&misc->xdummy), peer);
    // Warp 12 tells the peer that this CTA's softmax warps have read receive
    // slot kk % 2. The local wait acquires their (released) reads; the 4-byte
    // remote store that follows completes on the peer's x_empty barrier.
    auto relay_read = [&](int kk) -> bool {
      if (warp != 10) return true;
      if (!W.wait_warp(&misc->x_read[kk & 1], (kk >> 1) & 1)) return false;
      if (lane == 0) st_async_b32(xdummy_peer, (uint32_t)kk, xempty_peer[kk & 1]);
      return true;
    };
    int k = 0;
    bool ok = true;
    while (ok && cur.next(task, pg0, pg1, split)) {
      for (int i = pg0; i < pg1; ++i, ++k) {
        if (!W.wait_warp(&misc->s_full, k & 1)) { ok = false; break; }
        tc_fence_after();
        uint32_t sr[64];
        tmem_ld_32(tmem + lane_base + kTmemS, *reinterpret_cast<uint32_t(*)[32]>(&sr[0]));
        tmem_ld_32(tmem + lane_base + kTmemS + 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[32]));
        tmem_wait_ld();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_addr(&misc->s_free));
        // the peer must have read this slot's previous contents (tile k - 2)
        const int xs = k & 1;
        if (k >= 2 && expect_thread) mbar_arrive_expect_tx(smem_addr(&misc->x_empty[xs]), 4u);
        if (!W.wait_cluster_warp(&misc->x_empty[xs], ((k >> 1) & 1) ^ 1)) { ok = false; break; }
        if (warp_active) {
          uint32_t w[48];
#pragma unroll
          for (int g = 0; g < 16; ++g) pack24x4(&sr[4 * g], &w[3 * g]);
#pragma unroll
          for (int c = 0; c < 12; ++c)
            st_async_v4(xbuf_peer[xs] + c * 512, w[4 * c], w[4 * c + 1], w[4 * c + 2], w[4 * c + 3], xfull_peer[xs]);
        }
        if (k >= 1 && !relay_read(k - 1)) { ok = false; break; }
      }
    }
    if (ok && k >= 1) ok = relay_read(k - 1);
    // Collect the peer's last "slot read" stores so none is in flight at exit.
    if (ok) {
      for (int xs = 0; xs < kXSlots; ++xs) {
        const int uses = (k + 1 - xs) / 2;  // tiles k' < k with k' % 2 == xs
        if (uses > 0) {
          if (expect_thread) mbar_arrive_expect_tx(smem_addr(&misc->x_empty[xs]), 4u);
          W.wait_cluster_warp(&misc->x_empty[xs], (uses - 1) & 1);
        }
      }
    }
    __syncwarp();
  }

  // ------------------------------------------------------------ teardown
  tc_fence_before();
  cluster_sync();  // no remote access to this CTA's shared memory after this point
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace dec

// Host-side handles (used by mla_api.cu).
const void* decode_kernel_ptr() { return reinterpret_cast<const void*>(&dec::mla_decode_kernel); }
int decode_smem_bytes() { return dec::kSmemBytes; }
int decode_threads() { return dec::kThreads; }

cudaError_t launch_decode(const CUtensorMap& tm_tile, const CUtensorMap& tm_row, const DecodeArgs& args, int workers,
                          cudaStream_t stream) {
  dec::mla_decode_kernel<<<2 * workers, dec::kThreads, dec::kSmemBytes, stream>>>(tm_tile, tm_row, args);
  return cudaGetLastError();
}

}  // namespace mla
