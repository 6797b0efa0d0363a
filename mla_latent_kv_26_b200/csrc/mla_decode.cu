// Steps a2-a7: split-KV MLA decode over the paged latent cache on sm_100a.
//
// One worker = a cluster of two CTAs on two SMs. A task (one query token of
// one sequence, up to 128 heads) is processed by both CTAs together:
//
//   CTA rank 0: loads cache columns [0, 320); partial scores over columns
//               [0, 288); output columns [0, 256)
//   CTA rank 1: loads cache columns [256, 576); partial scores over [288, 576);
//               output columns [256, 512)
//
// The fp32 output accumulator of 128 heads x 512 columns is exactly one SM's
// tensor memory, so the pair splits the output columns, and the score
// contraction with them. The softmax of each head row is owned by one CTA:
// in every 32-lane TMEM quadrant, CTA r owns lanes [16r, 16r+16). For each
// 64-token tile, a CTA sends the peer the partial scores of the rows the peer
// owns (24-bit floats, fp32 rounded to its top three bytes, relative error
// <= 2^-16; 12 KB), receives the peer's partials of its own rows, runs the
// online softmax for its 64 rows, and sends back their P (bf16) together with
// the per-row rescale factor, running max and running sum (9 KB). Both CTAs
// then hold the same P for all 128 rows and accumulate their output halves
// with it. (The SM-to-SM path sustains ~15 B/clk per direction, so the
// exchange volume, not the arithmetic, decides this layout.)
//
// Per CTA (320 threads):
//   warp 0      TMA producer: 64-token pages (block table) or 64 gathered rows
//               (top-k indices, tile::gather4) into a 4-stage ring, 5 boxes of
//               64 rows x 128 B (128-byte swizzle) per stage
//   warp 1      tcgen05 issuer: S = Q_slice * K_slice^T (M=128 heads, N=64
//               tokens, K=288, A = Q in TMEM) one tile ahead of
//               O += P * V (M=128, N=256, K=64, A = P in shared memory, B = the
//               same stage read MN-major); it polls both queues and issues
//               whichever is ready
//   warps 2-5   softmax, one per quadrant: 16 owned rows x 64 tokens, two
//               threads per row (16x32bx2 TMEM accesses); P of the owned rows
//               into this CTA's P buffer and, by one bulk copy per quadrant,
//               into the peer's; epilogue of the owned rows
//   warps 6-9   helpers, one per quadrant, for the rows the peer owns: send
//               their partial scores, apply the peer's rescale factors, epilogue
//               of those rows; warp 8 also relays "receive slot read" tokens
//
// P is double-buffered in shared memory (128 heads x 64 tokens bf16, K-major,
// 128-byte swizzle, identical offsets in both CTAs). The PV commit arrives on
// the P-buffer barrier of both CTAs, so a buffer is rewritten only after both
// CTAs' PV of two tiles earlier completed.
//
// TMEM columns: O [0,256) | Q [256,400) | S [400,464).
#include <cuda.h>
#include <math.h>

#include "common.cuh"
#include "sm100.cuh"

namespace mla {
namespace dec {

using namespace ptx;

constexpr int kThreads = 320;
constexpr int kStages = 4;
constexpr int kBoxBytes = kPage * 128;  // 64 rows x 64 bf16 (one 128-B swizzle row each)
constexpr int kBoxesPerStage = 5;       // 320 columns per CTA
constexpr int kStageBytes = kBoxesPerStage * kBoxBytes;
constexpr int kSSteps = 18;             // 288 columns / 16 per MMA
// Partial-score slot: per quadrant, 32 threads x 6 chunks of 16 B (16 rows x 64 tokens x 3 B).
constexpr int kXQuadBytes = 32 * 6 * 16;
constexpr int kXBytes = 4 * kXQuadBytes;
// P buffer: 128 rows of 64 bf16 (one 128-byte swizzle row each).
constexpr int kPSlotBytes = 128 * 128;
constexpr int kPQuadBytes = 16 * 128;    // the 16 rows a CTA owns in one quadrant
// Rescale factor, running max and running sum of the peer's rows: 16 B per row.
constexpr int kStatBytes = 64 * 16;
constexpr int kStatQuadBytes = 16 * 16;
constexpr int kXSlots = 2;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kTmemO = 0, kTmemQ = 256, kTmemS = 400;
constexpr float kRescaleThreshold = 8.0f;  // log2 units: tolerate p up to 2^8 before rescaling O
constexpr uint64_t kTimeoutNs = 2000000000ull;
// Shared memory: [misc | stage ring | P buffers | score slots | stat slots];
// the stage ring and the P buffers must be 1024-byte aligned (128-byte
// swizzle atoms), which holds when the dynamic shared memory base is (checked
// at run time).
constexpr int kMiscBytes = 3072;
constexpr int kSmemBytes = kMiscBytes + kStages * kStageBytes + kXSlots * (kPSlotBytes + kXBytes + kStatBytes);
static_assert(kSmemBytes <= 232448, "shared memory budget");

struct Misc {
  uint64_t full[kStages];
  uint64_t empty[kStages];
  uint64_t s_full, s_free, o_full, o_empty, q_full, mma_done;
  uint64_t p_full[kXSlots], p_free[kXSlots];
  uint64_t x_full[kXSlots], x_empty[kXSlots], x_read[kXSlots];
  uint64_t pm_full[kXSlots];
  uint64_t stage_mask[kStages];
  uint32_t tmem_base;
  uint32_t abort_flag;
  uint32_t xdummy[4];  // targets of the peer's 4-byte "slot read" stores
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
  const uint32_t pbuf = stage_base + kStages * kStageBytes;  // P buffers (1024-aligned)
  const uint32_t xbuf = pbuf + kXSlots * kPSlotBytes;         // score slots
  const uint32_t statbuf = xbuf + kXSlots * kXBytes;          // stat slots

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
    mbar_init(smem_addr(&misc->s_free), 8);   // 4 softmax + 4 helper warps
    mbar_init(smem_addr(&misc->o_full), 1);
    mbar_init(smem_addr(&misc->o_empty), 8);
    mbar_init(smem_addr(&misc->q_full), 8);
    mbar_init(smem_addr(&misc->mma_done), 1);
    for (int xs = 0; xs < kXSlots; ++xs) {
      mbar_init(smem_addr(&misc->x_full[xs]), 1);
      mbar_init(smem_addr(&misc->x_empty[xs]), 1);
      mbar_init(smem_addr(&misc->x_read[xs]), 4);
      mbar_init(smem_addr(&misc->pm_full[xs]), 1);
      mbar_init(smem_addr(&misc->p_full[xs]), 8);   // 4 softmax + 4 helper warps
      mbar_init(smem_addr(&misc->p_free[xs]), 2);   // the PV commits of both CTAs
    }
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

  // Quadrant roles shared by the softmax and helper warps.
  const int quad = warp & 3;
  const bool quad_active = quad * 32 < a.heads;
  const uint32_t n_active = (uint32_t)((a.heads + 31) / 32);
  const int rl = lane & 15;   // row within a 16-lane half
  const int th = lane >> 4;   // token half (scores) / column half (O) of this thread
  const int own_row = quad * 32 + 16 * (int)crank + rl;
  const int peer_row = quad * 32 + 16 * (int)peer + rl;
  const uint32_t own_lanes = tmem + ((uint32_t)(quad * 32 + 16 * (int)crank) << 16);
  const uint32_t peer_lanes = tmem + ((uint32_t)(quad * 32 + 16 * (int)peer) << 16);

  // Q (this CTA's 288 columns) into TMEM: the softmax warp writes columns
  // [0,144) of its quadrant's 32 rows, the helper warp [144,288).
  auto write_q = [&](int half) {
    const int row = quad * 32 + lane;
    const size_t qrow = (size_t)task * a.heads + row;
    uint32_t qv[72];
    if (row < a.heads) {
      const uint4* src = reinterpret_cast<const uint4*>(a.q + qrow * kDQK + crank * 288 + half * 144);
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
    const uint32_t qa = tmem + ((uint32_t)(quad * 32) << 16) + kTmemQ + 72 * half;
    tmem_st_32(qa, *reinterpret_cast<const uint32_t(*)[32]>(&qv[0]));
    tmem_st_32(qa + 32, *reinterpret_cast<const uint32_t(*)[32]>(&qv[32]));
    tmem_st_8(qa + 64, *reinterpret_cast<const uint32_t(*)[8]>(&qv[64]));
    tmem_wait_st();
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(smem_addr(&misc->q_full));
  };
  // Rescale O rows of a 16-lane half by f (per thread: its row's factor).
  auto rescale_o = [&](uint32_t lanes, float f) {
#pragma unroll 1
    for (int c = 0; c < 4; ++c) {
      uint32_t o[32];
      tmem_ld_16x32bx2_32<128>(lanes + kTmemO + 32 * c, o);
      tmem_wait_ld();
#pragma unroll
      for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * f);
      tmem_st_16x32bx2_32<128>(lanes + kTmemO + 32 * c, o);
    }
  };
  // Epilogue for a 16-lane half: out / partials of rows `row` (per thread), columns th*128 + [0,128).
  auto write_rows = [&](uint32_t lanes, int row, float inv, float lse, bool write_lse) {
    const bool valid = row < a.heads;
    const size_t qrow = (size_t)task * a.heads + row;
#pragma unroll 1
    for (int c = 0; c < 4; ++c) {
      uint32_t o[32];
      tmem_ld_16x32bx2_32<128>(lanes + kTmemO + 32 * c, o);
      tmem_wait_ld();
      if (valid) {
        const int col = (int)crank * 256 + th * 128 + 32 * c;
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
          float4* dst =
              reinterpret_cast<float4*>(a.part_o + ((size_t)(worker + task) * a.heads + row) * kDLatent + col);
#pragma unroll
          for (int u = 0; u < 8; ++u)
            dst[u] = make_float4(__uint_as_float(o[4 * u + 0]) * inv, __uint_as_float(o[4 * u + 1]) * inv,
                                 __uint_as_float(o[4 * u + 2]) * inv, __uint_as_float(o[4 * u + 3]) * inv);
        }
      }
    }
    if (valid && th == 0) {
      if (split) a.part_lse[((size_t)(worker + task) * 2 + crank) * a.heads + row] = lse;
      else if (write_lse) a.lse[qrow] = lse;
    }
  };
  // Drain the last phases of a slot barrier fed by 4-byte remote tokens.
  auto drain_tokens = [&](uint64_t* bars, int uses_total, uint32_t bytes, bool expect) {
    for (int xs = 0; xs < kXSlots; ++xs) {
      const int uses = (uses_total + 1 - xs) / 2;
      if (uses > 0) {
        if (expect) mbar_arrive_expect_tx(smem_addr(&bars[xs]), bytes);
        W.wait_cluster_warp(&bars[xs], (uses - 1) & 1);
      }
    }
  };

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
      // S for tile kk into the (single) S buffer.
      auto issue_s = [&](int kk) {
        const uint32_t sb = stage_base + (kk % kStages) * kStageBytes;
#pragma unroll
        for (int ks = 0; ks < kSSteps; ++ks) {
          const int c = (crank ? 32 : 0) + 16 * ks;  // column relative to col0
          const uint32_t baddr = sb + (c >> 6) * kBoxBytes + (c & 63) * 2;
          mma_tmem_a(tmem + kTmemS, tmem + kTmemQ + 8 * ks, smem_desc_sw128(baddr, 16, 1024), idS, ks > 0 ? 1u : 0u);
        }
        mma_commit(smem_addr(&misc->s_full));
      };
      // O (+)= P V for tile kk; releases the P buffer (in both CTAs) and the stage.
      auto issue_pv = [&](int kk, bool first) {
        const int s = kk % kStages;
        const uint32_t vb = stage_base + s * kStageBytes;
        const uint32_t pb = pbuf + (kk & 1) * kPSlotBytes;
#pragma unroll
        for (int u = 0; u < 4; ++u)
          mma_ss(tmem + kTmemO, smem_desc_sw128(pb + 32 * u, 16, 1024), smem_desc_sw128(vb + u * 2048, kBoxBytes, 1024),
                 idO, (first && u == 0) ? 0u : 1u);
        mma_commit_cluster(smem_addr(&misc->p_free[kk & 1]), (uint16_t)0x3);
        mma_commit(smem_addr(&misc->empty[s]));
      };
      int k = 0, j = 0;
      bool ok = true;
      while (ok && cur.next(task, pg0, pg1, split)) {
        if (!W.wait(&misc->q_full, j & 1)) break;
        const int n = pg1 - pg0;
        // Poll both queues: S(kk) needs its stage and the previous S read out;
        // PV(kk) needs both CTAs' P of tile kk (and, for the first tile of a
        // task, the previous task's epilogue done with O).
        int ns = 0, np = 0;
        uint64_t t0 = global_timer_ns();
        while (np < n) {
          bool progress = false;
          if (ns < n) {
            const int kk = k + ns;
            if (mbar_test_wait(smem_addr(&misc->full[kk % kStages]), (kk / kStages) & 1) &&
                (kk == 0 || mbar_test_wait(smem_addr(&misc->s_free), (kk - 1) & 1))) {
              tc_fence_after();
              issue_s(kk);
              ++ns;
              progress = true;
            }
          }
          if (np < ns) {
            const int kk = k + np;
            if (mbar_test_wait(smem_addr(&misc->p_full[kk & 1]), (kk >> 1) & 1) &&
                (np > 0 || j == 0 || mbar_test_wait(smem_addr(&misc->o_empty), (j - 1) & 1))) {
              tc_fence_after();
              issue_pv(kk, np == 0);
              ++np;
              progress = true;
            }
          }
          if (progress) {
            t0 = global_timer_ns();
          } else if (W.aborted()) {
            ok = false;
            break;
          } else if (global_timer_ns() - t0 > kTimeoutNs) {
            W.fail();
            ok = false;
            break;
          }
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
  } else if (warp >= 2 && warp <= 5) {
    // ------------------------------------------------------------ softmax (owned rows)
    const bool expect_thread = (quad == 0 && lane == 0);
    const int tid_sm = (warp - 2) * 32 + lane;  // 0..127
    // This thread's 64 bytes of P: row own_row, tokens 32*th .. +31, as four
    // 16-byte chunks of the 128-byte swizzled row.
    const uint32_t prow = (uint32_t)own_row * 128u;
    uint32_t pchunk[4];
#pragma unroll
    for (int c = 0; c < 4; ++c) pchunk[c] = prow + ((uint32_t)((4 * th + c) ^ (own_row & 7)) << 4);
    const uint32_t pquad = (uint32_t)(quad * 32 + 16 * (int)crank) * 128u;  // first owned row of the quadrant
    // peer addresses of slot 0; slot 1 follows at the same stride as here
    const uint32_t pm_full_peer = map_to_rank(smem_addr(&misc->pm_full[0]), peer);
    const uint32_t pbuf_peer = map_to_rank(pbuf, peer) + pquad;
    const uint32_t stat_peer =
        map_to_rank(statbuf, peer) + (uint32_t)(quad * kStatQuadBytes) + (uint32_t)rl * 16u;
    const uint32_t xoff = (uint32_t)(quad * kXQuadBytes) + (uint32_t)lane * 16u;
    const uint32_t xbytes = n_active * (uint32_t)kXQuadBytes;
    int k = 0, j = 0;

    while (cur.next(task, pg0, pg1, split)) {
      write_q(0);
      float m_run = -INFINITY, l_run = 0.f;
      const int ntiles = pg1 - pg0;
      for (int i = 0; i < ntiles; ++i, ++k) {
        const int s = k % kStages;
        const int xs = k & 1;
        // own partial scores of this tile (this thread: its row, tokens 32*th..+31)
        uint32_t own[32];
        if (!W.wait_warp(&misc->s_full, k & 1)) goto softmax_done;
        tc_fence_after();
        tmem_ld_16x32bx2_32<32>(own_lanes + kTmemS, own);
        tmem_wait_ld();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_addr(&misc->s_free));
        // the peer's partial scores of these rows
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
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_addr(&misc->x_read[xs]));

        // mask (written by the producer before the stage's full barrier)
        if (!W.wait_warp(&misc->full[s], (k / kStages) & 1)) goto softmax_done;
        const uint64_t mask64 = misc->stage_mask[s];
        const uint32_t mask = (uint32_t)(mask64 >> (32 * th));
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
        const float mtile = fmaxf(mloc, __shfl_xor_sync(~0u, mloc, 16));  // the row's other half
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
        const float l_row = l_run + __shfl_xor_sync(~0u, l_run, 16);

        // P buffer xs is free once both CTAs' PV of tile k-2 completed
        if (k >= 2 && !W.wait_cluster_warp(&misc->p_free[xs], ((k >> 1) & 1) ^ 1)) goto softmax_done;
        const uint32_t pb = pbuf + xs * kPSlotBytes;
#pragma unroll
        for (int c = 0; c < 4; ++c)
          st_shared_v4(pb + pchunk[c], make_uint4(pp[4 * c], pp[4 * c + 1], pp[4 * c + 2], pp[4 * c + 3]));
        fence_proxy_async_smem();  // P is read by the bulk copy and the tensor core
        __syncwarp();
        if (quad_active) {
          // the same rows into the peer's P buffer, and the rows' rescale factor and running stats
          if (lane == 0)
            bulk_copy_to_cta(pbuf_peer + xs * kPSlotBytes, pb + pquad, (uint32_t)kPQuadBytes, pm_full_peer + 8u * xs);
          if (th == 0)
            st_async_v4(stat_peer + xs * kStatBytes, __float_as_uint(corr ? alpha : 1.f), __float_as_uint(m_run),
                        __float_as_uint(l_row), 0u, pm_full_peer + 8u * xs);
        }
        if (__any_sync(~0u, corr)) {
          // O of these rows must hold PV of tile k-1 before it is rescaled
          if (!W.wait_cluster_warp(&misc->p_free[xs ^ 1], ((k - 1) >> 1) & 1)) goto softmax_done;
          tc_fence_after();
          rescale_o(own_lanes, corr ? alpha : 1.f);
          tmem_wait_st();
        }
        if (mask64 != ~0ull) {
          // masked tokens' V rows may hold anything (even NaN): zero them so 0 * V stays 0
          const uint32_t sb = stage_base + s * kStageBytes;
          for (int e = tid_sm; e < kPage * 32; e += 128) {
            const int r = e >> 5, c = e & 31;
            if (!((mask64 >> r) & 1ull))
              st_shared_v4(sb + (c >> 3) * kBoxBytes + r * 128 + (c & 7) * 16, make_uint4(0, 0, 0, 0));
          }
          fence_proxy_async_smem();
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_addr(&misc->p_full[xs]));
      }

      // ------------------------------------------------------------ epilogue (owned rows)
      {
        const float l_row = l_run + __shfl_xor_sync(~0u, l_run, 16);
        if (!W.wait_warp(&misc->o_full, j & 1)) goto softmax_done;
        tc_fence_after();
        const float inv = l_row > 0.f ? 1.f / l_row : 0.f;
        const float lse = l_row > 0.f ? (m_run + log2f(l_row)) * 0.69314718055994530942f : -INFINITY;
        write_rows(own_lanes, own_row, inv, lse, true);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_addr(&misc->o_empty));
      }
      ++j;
    }
  softmax_done:
    // Both CTAs' last PV commits arrive here; collect them before exit.
    if (!W.aborted())
      for (int kk = max(0, k - 2); kk < k; ++kk) W.wait_cluster(&misc->p_free[kk & 1], (kk >> 1) & 1);
    __syncwarp();
  } else if (warp >= 6) {
    // ------------------------------------------------------------ helper (rows the peer owns)
    const bool lead = (quad == 0 && lane == 0);  // warp 8, lane 0: expects and relays
    const uint32_t xfull_peer = map_to_rank(smem_addr(&misc->x_full[0]), peer);
    const uint32_t xempty_peer = map_to_rank(smem_addr(&misc->x_empty[0]), peer);
    const uint32_t xbuf_peer = map_to_rank(xbuf, peer) + (uint32_t)(quad * kXQuadBytes) + (uint32_t)lane * 16u;
    const uint32_t xdummy_peer = map_to_rank(smem_addr(&misc->xdummy[quad]), peer);
    const uint32_t pmbytes = n_active * (uint32_t)(kPQuadBytes + kStatQuadBytes);
    int k = 0, j = 0;
    bool ok = true;
    float pm = -INFINITY, pl = 0.f;  // the owner's running max / sum of this thread's row

    // Partial scores of tile kk for the rows the peer owns -> the peer's slot kk % 2.
    auto send_s = [&](int kk) -> bool {
      if (!W.wait_warp(&misc->s_full, kk & 1)) return false;
      tc_fence_after();
      uint32_t sr[32];
      tmem_ld_16x32bx2_32<32>(peer_lanes + kTmemS, sr);
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_addr(&misc->s_free));
      uint32_t w[24];
#pragma unroll
      for (int g = 0; g < 8; ++g) pack24x4(&sr[4 * g], &w[3 * g]);
      const int xs = kk & 1;
      if (kk >= 2 && lead) mbar_arrive_expect_tx(smem_addr(&misc->x_empty[xs]), 4u);
      if (!W.wait_cluster_warp(&misc->x_empty[xs], ((kk >> 1) & 1) ^ 1)) return false;
      if (quad_active) {
#pragma unroll
        for (int c = 0; c < 6; ++c)
          st_async_v4(xbuf_peer + xs * kXBytes + c * 512, w[4 * c], w[4 * c + 1], w[4 * c + 2], w[4 * c + 3],
                      xfull_peer + 8u * xs);
      }
      return true;
    };
    // This CTA's softmax warps have read score slot kk % 2: tell the peer
    // (their arrives released the reads; this wait acquires them).
    auto relay_read = [&](int kk) -> bool {
      if (quad != 0) return true;
      if (!W.wait_warp(&misc->x_read[kk & 1], (kk >> 1) & 1)) return false;
      if (lane == 0) st_async_b32(xdummy_peer, (uint32_t)kk, xempty_peer + 8u * (kk & 1));
      return true;
    };
    // The peer's P of tile kk landed in P buffer kk % 2: rescale the O rows
    // the peer owns by their factor (rare), then release PV(kk).
    auto accept_p = [&](int kk) -> bool {
      const int xs = kk & 1;
      if (lead) mbar_arrive_expect_tx(smem_addr(&misc->pm_full[xs]), pmbytes);
      if (!W.wait_cluster_warp(&misc->pm_full[xs], (kk >> 1) & 1)) return false;
      const uint4 stv = ld_shared_v4(statbuf + xs * kStatBytes + (uint32_t)(quad * kStatQuadBytes) + (uint32_t)rl * 16u);
      const float alpha = __uint_as_float(stv.x);
      pm = __uint_as_float(stv.y);
      pl = __uint_as_float(stv.z);
      const bool corr = alpha != 1.f;
      if (__any_sync(~0u, corr)) {
        if (!W.wait_cluster_warp(&misc->p_free[xs ^ 1], ((kk - 1) >> 1) & 1)) return false;
        tc_fence_after();
        rescale_o(peer_lanes, corr ? alpha : 1.f);
        tmem_wait_st();
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_addr(&misc->p_full[xs]));
      return true;
    };

    while (ok && cur.next(task, pg0, pg1, split)) {
      write_q(1);
      const int n = pg1 - pg0;
      ok = send_s(k);
      for (int i = 0; ok && i < n; ++i) {
        if (i + 1 < n) ok = send_s(k + i + 1);
        if (ok) ok = relay_read(k + i);
        if (ok) ok = accept_p(k + i);
      }
      if (!ok) break;
      k += n;
      // ------------------------------------------------------------ epilogue (rows the peer owns)
      if (!W.wait_warp(&misc->o_full, j & 1)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const float inv = pl > 0.f ? 1.f / pl : 0.f;
      const float lse = pl > 0.f ? (pm + log2f(pl)) * 0.69314718055994530942f : -INFINITY;
      write_rows(peer_lanes, peer_row, inv, lse, false);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_addr(&misc->o_empty));
      ++j;
    }
    // the peer relays "slot read" for every score tile sent; collect the last ones before exit
    if (ok) drain_tokens(misc->x_empty, k, 4u, lead);
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
