// Steps a2-a7: split-KV MLA decode over the paged latent cache on sm_100a.
//
// One worker = a cluster of two CTAs on two SMs. A task (one query token of
// one sequence, up to 128 heads) is processed by both CTAs together; CTA rank
// r loads, for every 64-token tile, cache columns [256r, 256r + 256) (its
// output columns) and [512 + 32r, 512 + 32r + 32) (half of the rope part),
// and contracts its partial scores over those 288 columns.
//
// The fp32 output accumulator of 128 heads x 512 columns is exactly one SM's
// tensor memory, so the pair splits the output columns, and the score
// contraction with them. The softmax of each head row is owned by one CTA:
// in every 32-lane TMEM quadrant, CTA r owns lanes [16r, 16r+16). For each
// tile, a CTA sends the peer the partial scores of the rows the peer owns
// (23-bit block fixed point in 3 bytes, one power-of-two scale per row; 12 KB),
// receives the peer's partials of its own rows, runs the online softmax for
// its 64 rows, and sends back their P (bf16) together with the per-row
// rescale factor, running max and running sum (9 KB). Both CTAs then hold the
// same P for all 128 rows and accumulate their output halves with it.
//
// Per CTA (448 threads):
//   warp 0      producer: 64-token pages (block table, TMA) or 64 gathered
//               rows (top-k indices; tile::gather4 for latent boxes 0-1 and
//               the rope box, 16-byte cp.async for boxes 2-3) into a 4-stage
//               ring; a stage is four boxes of 64 rows x 128 B (128-byte
//               swizzle) and one box of 64 rows x 64 B (64-byte swizzle)
//   warp 1      tcgen05 issuer: S = Q_slice * K_slice^T (M=128 heads, N=64
//               tokens, K=288; A = Q in TMEM, its rope columns from shared
//               memory) into one of two S buffers, and O += P * V (M=128,
//               N=256, K=64, A = P in shared memory, B = the stage read
//               MN-major); it polls both queues, PV first
//   warps 2-5   softmax, one per quadrant: 16 owned rows x 64 tokens, two
//               threads per row (16x32bx2 TMEM accesses); P of the owned rows
//               into this CTA's P buffer and, by one bulk copy per quadrant,
//               into the peer's; epilogue of the owned rows
//   warps 6-9   senders, one per quadrant, for the rows the peer owns: send
//               their partial scores; warp 8 also relays "receive slot read"
//               tokens
//   warps 10-13 acceptors, one per quadrant, for the rows the peer owns: apply
//               the peer's rescale factors, epilogue of those rows
//
// S is double-buffered in TMEM, so the S of tile k + 1 (and its exchange)
// proceeds while the softmax warps work on tile k. P is double-buffered in
// shared memory (128 heads x 64 tokens bf16, K-major, 128-byte swizzle,
// identical offsets in both CTAs). The PV commit arrives on the P-buffer
// barrier of both CTAs, so a buffer is rewritten only after both CTAs' PV of
// two tiles earlier completed.
//
// TMEM columns: O [0,256) | Q [256,384) | S buffers [384,448), [448,512).
#include <cuda.h>
#include <math.h>

#include "common.cuh"
#include "sm100.cuh"

namespace mla {
namespace dec {

using namespace ptx;

constexpr int kThreads = 448;
constexpr int kStages = 4;
constexpr int kBoxBytes = kPage * 128;  // 64 rows x 64 bf16 (one 128-B swizzle row each)
constexpr int kVBoxes = 4;              // this CTA's 256 output columns, 4 boxes of 64
constexpr int kRopeBoxBytes = kPage * 64;  // 64 rows x 32 bf16 (one 64-byte swizzle row each)
constexpr int kRopeOff = kVBoxes * kBoxBytes;
constexpr int kStageBytes = kRopeOff + kRopeBoxBytes;
// fp8 cache: the CTA's 256 latent columns arrive as e4m3 codes in two boxes
// of 64 rows x 128 B (no swizzle) in the upper half of the stage's latent
// region, the rope box as above, and the rows' scales (16 B each) after it;
// two converter warps then write the bf16 latent boxes in place. Every TMA
// destination is 128-byte aligned: a page's scales arrive as one box of
// 64 x 16 B (row r at 16 r), gathered rows four at a time into 128-byte slots
// (row r at 128 (r / 4) + 16 (r % 4)).
constexpr int kThreadsF8 = 512;
constexpr int kF8CodeBoxBytes = kPage * 128;
constexpr int kF8CodeOff = 2 * kBoxBytes;
constexpr int kF8ScaleStageOff = kStageBytes;
constexpr int kF8ScaleBytes = 16 * 128;  // room for the gathered layout
constexpr int kStageBytesF8 = kStageBytes + kF8ScaleBytes;
constexpr int kF8LoadBytes = 2 * kF8CodeBoxBytes + kRopeBoxBytes + kPage * 16;
// Score slot: per quadrant, 32 threads x 6 chunks of 16 B (16 rows x 64
// tokens of 23-bit fixed point in 3 bytes), then per quadrant 16 row
// exponents of 4 B.
// Each quadrant's part (data, then its 16 row exponents) is contiguous, so
// that one bulk copy per quadrant sends it.
constexpr int kXChunks = 6;
constexpr int kXQuadBytes = 32 * kXChunks * 16;
constexpr int kXExpBytes = 16 * 4;
constexpr int kXQuadStride = kXQuadBytes + kXExpBytes;
constexpr int kXBytes = 4 * kXQuadStride;
// One score slot, and one staging buffer from which the sender warps' bulk
// copies read: the partials of tile k are staged only after the peer has read
// tile k - 1 out of its slot, which also means the copy of tile k - 1 has
// finished reading the staging buffer. (A second slot, measured, did not
// shorten the step.)
constexpr int kXSlots = 1;
// P buffer: 128 rows of 64 bf16 (one 128-byte swizzle row each).
constexpr int kPSlotBytes = 128 * 128;
constexpr int kPQuadBytes = 16 * 128;    // the 16 rows a CTA owns in one quadrant
// Rescale factor, running max and running sum of the peer's rows: 16 B per row.
constexpr int kStatBytes = 64 * 16;
constexpr int kStatQuadBytes = 16 * 16;
constexpr int kPSlots = 2;
constexpr uint32_t kTmemCols = 512;
// Q: this CTA's 256 output columns in TMEM (two bf16 per TMEM column), its
// 32 rope columns in shared memory (no-swizzle K-major core matrices of 8
// rows x 16 B). S buffer b (tile k uses b = k % 2) starts at kTmemS + 64 b.
constexpr uint32_t kTmemO = 0, kTmemQ = 256, kTmemS = 384;
constexpr int kQRopeBytes = 128 * 64;  // 128 rows x 32 bf16
constexpr uint32_t kQRopeLbo = 128, kQRopeSbo = 512;
constexpr float kRescaleThreshold = 8.0f;  // log2 units: tolerate p up to 2^8 before rescaling O
constexpr uint64_t kTimeoutNs = 2000000000ull;
// Shared memory: [misc | stage ring | P buffers | score slot | stat slots | Q rope];
// the stage ring and the P buffers must be 1024-byte aligned (128-byte
// swizzle atoms), which holds when the dynamic shared memory base is (checked
// at run time).
constexpr int kMiscBytes = 1024;
template <bool kF8>
constexpr int smem_bytes() {
  return kMiscBytes + kStages * (kF8 ? kStageBytesF8 : kStageBytes) + kPSlots * (kPSlotBytes + kStatBytes) +
         (kXSlots + 1) * kXBytes + kQRopeBytes;
}
static_assert(smem_bytes<false>() <= 232448 && smem_bytes<true>() <= 232448, "shared memory budget");
static_assert(kStageBytesF8 % 1024 == 0, "stages hold 128-byte swizzle atoms");

struct Misc {
  uint64_t full[kStages];
  uint64_t empty[kStages];
  uint64_t s_full[2], s_free[2], o_full, o_empty, q_full, mma_done;
  uint64_t p_full[kPSlots], p_free[kPSlots], pm_full[kPSlots];
  uint64_t x_full[kXSlots], x_empty[kXSlots], x_read[kXSlots];
  uint64_t stage_mask[kStages];
  uint64_t conv_full[kStages];  // fp8 cache: stage converted to bf16
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

// The worker's contiguous range of global pages (inside its group's
// positions), walked task by task in plan order.
struct Cursor {
  const int32_t* prefix;
  int T, lo, hi, t, tend;

  MLA_DEV void init(const int32_t* plan, int worker) {
    T = plan[kPlanTasks];
    prefix = plan + plan_prefix_off();
    const int G = plan[kPlanGroups], Wg = plan[kPlanGroupWorkers];
    const int g = worker / Wg;
    t = tend = T;
    lo = hi = 0;
    if (T <= 0 || g >= G) return;  // no tasks, or one of the workers left over by the grouping
    const PlanGroup grp = plan_group(plan, g);
    lo = grp.base + (worker - grp.w0) * grp.quota;
    hi = min(lo + grp.quota, grp.end);
    tend = grp.t1;
    if (lo >= grp.end) {
      t = tend;
      return;
    }
    // largest t in the group with prefix[t] <= lo: a 32-way search by the
    // whole warp (one round of loads per factor 32 of the range instead of
    // one per halving; every lane of the calling warp takes part)
    const int lane = threadIdx.x & 31;
    int a = grp.t0, b = grp.t1 - 1;
    while (a < b) {
      const int step = (b - a + 31) / 32;
      const int q = min(a + (lane + 1) * step, b);
      const unsigned le = __ballot_sync(~0u, prefix[q] <= lo);  // a prefix of the lanes (prefix is nondecreasing)
      const int m = __popc(le);
      const int qm = __shfl_sync(~0u, q, max(m - 1, 0));  // last probe at or before the answer
      const int qn = __shfl_sync(~0u, q, min(m, 31));     // first probe after it (m < 32)
      if (m == 0) {
        b = qn - 1;
      } else {
        a = qm;                      // m == 32: the last probe is b itself, so a = b
        if (m < 32) b = qn - 1;
      }
    }
    t = a;
  }
  MLA_DEV bool next(int& task, int& pg0, int& pg1, bool& split) {
    while (t < tend && prefix[t] < hi) {
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

template <bool kF8>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kF8 ? kThreadsF8 : kThreads, 1)
    mla_decode_kernel(const __grid_constant__ CacheMaps maps, const DecodeArgs a) {
  constexpr int kSB = kF8 ? kStageBytesF8 : kStageBytes;  // stage stride
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  Misc* misc = reinterpret_cast<Misc*>(smem_raw);
  const uint32_t raw_base = smem_addr(smem_raw);
  const uint32_t stage_base = raw_base + kMiscBytes;
  const uint32_t pbuf = stage_base + kStages * kSB;  // P buffers (1024-aligned)
  const uint32_t xbuf = pbuf + kPSlots * kPSlotBytes;         // score slots
  const uint32_t xstage = xbuf + kXSlots * kXBytes;           // outgoing partial scores
  const uint32_t statbuf = xstage + kXBytes;                  // stat slots
  const uint32_t qrope = statbuf + kPSlots * kStatBytes;      // rope columns of Q

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t crank = cluster_ctarank();
  const uint32_t peer = crank ^ 1u;
  const int worker = (int)cluster_id_x();
  Waiter W{misc, reinterpret_cast<uint32_t*>(a.plan + kPlanErr)};

  if (stage_base & 1023u) {  // cannot place the swizzled ring: refuse instead of corrupting
    grid_dependency_wait();   // the plan kernel writes the error word too
    if (threadIdx.x == 0) atomicOr(W.err, kErrTimeout);
    return;
  }
  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      // bf16 gathers: 32 cp.async arrivals + lane 0's arrive with the TMA bytes
      mbar_init(smem_addr(&misc->full[s]), (!kF8 && a.topk > 0) ? 33 : 1);
      mbar_init(smem_addr(&misc->empty[s]), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(smem_addr(&misc->s_full[b]), 1);
      mbar_init(smem_addr(&misc->s_free[b]), 8);   // 4 softmax + 4 sender warps
    }
    mbar_init(smem_addr(&misc->o_full), 1);
    mbar_init(smem_addr(&misc->o_empty), 8);  // 4 softmax + 4 acceptor warps
    mbar_init(smem_addr(&misc->q_full), 8);   // 4 softmax + 4 sender warps
    mbar_init(smem_addr(&misc->mma_done), 1);
    for (int x = 0; x < kXSlots; ++x) {
      mbar_init(smem_addr(&misc->x_full[x]), 1);
      mbar_init(smem_addr(&misc->x_empty[x]), 1);
      mbar_init(smem_addr(&misc->x_read[x]), 4);
    }
    for (int ps = 0; ps < kPSlots; ++ps) {
      mbar_init(smem_addr(&misc->pm_full[ps]), 1);
      mbar_init(smem_addr(&misc->p_full[ps]), 8);   // 4 softmax + 4 acceptor warps
      mbar_init(smem_addr(&misc->p_free[ps]), 2);   // the PV commits of both CTAs
    }
    for (int s = 0; s < kStages; ++s) mbar_init(smem_addr(&misc->conv_full[s]), 2);  // the two converter warps
    misc->abort_flag = 0u;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&maps.tile);
    prefetch_tmap(&maps.row);
    prefetch_tmap(&maps.rope_tile);
    prefetch_tmap(&maps.rope_row);
  }
  if (warp == 1) {
    tmem_alloc(smem_addr(&misc->tmem_base), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  cluster_sync();
  tc_fence_after();
  const uint32_t tmem = misc->tmem_base;
  // Everything above overlaps the plan kernel (programmatic launch); the
  // plan, q and the cache are read only after it has finished.
  grid_dependency_wait();
  // Cache columns of this CTA: output columns [vcol0, vcol0 + 256) in four
  // 128-byte-swizzled boxes, and rope columns [rcol0, rcol0 + 32) in one
  // 64-byte-swizzled box; the scores are contracted over both (288 columns).
  const int vcol0 = 256 * (int)crank;
  const int rcol0 = kDLatent + 32 * (int)crank;

  Cursor cur;
  cur.init(a.plan, worker);
  const int T = cur.T;
  const TaskMap tmap{a.plan[kPlanGroups], a.batch, a.q_len};
  const int32_t* ntok_arr = a.plan + plan_ntok_off(T);
  int task = 0, pg0 = 0, pg1 = 0;
  bool split = false;

  // Quadrant roles shared by the softmax, sender and acceptor warps.
  const int quad = warp & 3;
  const bool quad_active = quad * 32 < a.heads;
  const uint32_t n_active = (uint32_t)((a.heads + 31) / 32);
  const int rl = lane & 15;   // row within a 16-lane half
  const int th = lane >> 4;   // token half (scores) / column half (O) of this thread
  const int own_row = quad * 32 + 16 * (int)crank + rl;
  const int peer_row = quad * 32 + 16 * (int)peer + rl;
  const uint32_t own_lanes = tmem + ((uint32_t)(quad * 32 + 16 * (int)crank) << 16);
  const uint32_t peer_lanes = tmem + ((uint32_t)(quad * 32 + 16 * (int)peer) << 16);

  // Q (this CTA's 288 score columns): the softmax warp writes
  // Q[vcol0, vcol0 + 128) of its quadrant's 32 rows into TMEM, the sender
  // warp Q[vcol0 + 128, vcol0 + 256) into TMEM and Q[rcol0, rcol0 + 32) into
  // shared memory.
  auto write_q = [&](int half) {
    const int row = quad * 32 + lane;
    const size_t qrow = (size_t)tmap.row(task) * a.heads + row;
    const bool valid = row < a.heads;
    const uint4* src = reinterpret_cast<const uint4*>(a.q + qrow * kDQK + vcol0 + half * 128);
    uint32_t qv[64];
#pragma unroll
    for (int u = 0; u < 16; ++u) {
      const uint4 v = valid ? src[u] : make_uint4(0, 0, 0, 0);
      qv[4 * u + 0] = v.x;
      qv[4 * u + 1] = v.y;
      qv[4 * u + 2] = v.z;
      qv[4 * u + 3] = v.w;
    }
    const uint32_t qa = tmem + ((uint32_t)(quad * 32) << 16) + kTmemQ + 64 * half;
    tmem_st_32(qa, *reinterpret_cast<const uint32_t(*)[32]>(&qv[0]));
    tmem_st_32(qa + 32, *reinterpret_cast<const uint32_t(*)[32]>(&qv[32]));
    if (half == 1) {
      const uint4* rsrc = reinterpret_cast<const uint4*>(a.q + qrow * kDQK + rcol0);
      uint32_t rv[16];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const uint4 v = valid ? rsrc[u] : make_uint4(0, 0, 0, 0);
        rv[4 * u + 0] = v.x;
        rv[4 * u + 1] = v.y;
        rv[4 * u + 2] = v.z;
        rv[4 * u + 3] = v.w;
      }
      // core matrix (row / 8, column / 8) of 8 rows x 16 B
#pragma unroll
      for (int u = 0; u < 4; ++u)
        st_shared_v4(qrope + (uint32_t)(row >> 3) * kQRopeSbo + (uint32_t)u * kQRopeLbo + (uint32_t)(row & 7) * 16u,
                     make_uint4(rv[4 * u], rv[4 * u + 1], rv[4 * u + 2], rv[4 * u + 3]));
      fence_proxy_async_smem();  // read by the tensor core
    }
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
    const size_t qrow = (size_t)tmap.row(task) * a.heads + row;
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
  // The peer's 4-byte "slot read" tokens of the last two tiles sent (the
  // ones no send waited for) are collected before exit.
  auto drain_x_empty = [&](int tiles, bool expect) {
    for (int t = max(0, tiles - kXSlots); t < tiles; ++t) {
      if (expect) mbar_arrive_expect_tx(smem_addr(&misc->x_empty[t % kXSlots]), 4u);
      W.wait_cluster_warp(&misc->x_empty[t % kXSlots], (t / kXSlots) & 1);
    }
  };

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    int k = 0;
    while (cur.next(task, pg0, pg1, split)) {
      const int b = tmap.seq(task), qi = tmap.tok(task);
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
              const int row = (ok ? page : 0) * kPage;
              const uint32_t dst = stage_base + s * kSB;
              if constexpr (kF8) {
                // codes of this CTA's columns (bytes [256 r, 256 r + 256)), rope, scales
                mbar_arrive_expect_tx(fb, kF8LoadBytes);
                tma_load_2d(dst + kF8CodeOff, &maps.tile, vcol0, row, fb);
                tma_load_2d(dst + kF8CodeOff + kF8CodeBoxBytes, &maps.tile, vcol0 + 128, row, fb);
                tma_load_2d(dst + kRopeOff, &maps.rope_tile, kF8RopeOff + 64 * (int)crank, row, fb);
                tma_load_2d(dst + kF8ScaleStageOff, &maps.scale_tile, kF8ScaleOff, row, fb);
              } else {
                mbar_arrive_expect_tx(fb, kStageBytes);
#pragma unroll
                for (int bx = 0; bx < kVBoxes; ++bx)
                  tma_load_2d(dst + bx * kBoxBytes, &maps.tile, vcol0 + 64 * bx, row, fb);
                tma_load_2d(dst + kRopeOff, &maps.rope_tile, rcol0, row, fb);
              }
            }
            __syncwarp();
          }
        }
      } else {
        const int32_t* idx_row = a.indices + (size_t)(b * a.q_len + qi) * a.topk;
        const int L = a.seq_lens[b];
        // Index slots in batches of 4 tiles (8 per lane): the next batch's
        // indices are loaded before this batch's block-table lookups, and the
        // 8 lookups of a batch go out together, so a batch costs about one
        // round trip to memory instead of two per tile.
        int nidx[8];
        auto load_idx = [&](int t0, int (&dst)[8]) {
#pragma unroll
          for (int h = 0; h < 8; ++h) {
            const int slot = t0 * kPage + 32 * h + lane;
            dst[h] = (t0 + (h >> 1) < pg1 && slot < ntok) ? idx_row[slot] : -1;
          }
        };
        load_idx(pg0, nidx);
        for (int t0 = pg0; t0 < pg1; t0 += 4) {
          int idx[8];
#pragma unroll
          for (int h = 0; h < 8; ++h) idx[h] = nidx[h];
          if (t0 + 4 < pg1) load_idx(t0 + 4, nidx);
          int rows8[8];
          bool valid8[8];
#pragma unroll
          for (int h = 0; h < 8; ++h) {
            const int slot = t0 * kPage + 32 * h + lane;
            const bool in_range = idx[h] >= 0 && idx[h] < L;
            if (t0 + (h >> 1) < pg1 && slot < ntok && !in_range && idx[h] != -1) atomicOr(W.err, kErrIndex);
            const int pid = in_range ? bt_row[idx[h] / kPage] : 0;
            const bool pok = in_range && (unsigned)pid < (unsigned)a.num_pages;
            if (in_range && !pok) atomicOr(W.err, kErrPageId);
            rows8[h] = pok ? pid * kPage + (idx[h] % kPage) : 0;
            valid8[h] = pok;
          }
#pragma unroll
          for (int tt = 0; tt < 4; ++tt) {
            if (t0 + tt >= pg1) break;
            const int rows[2] = {rows8[2 * tt], rows8[2 * tt + 1]};
            const uint64_t mask = (uint64_t)__ballot_sync(~0u, valid8[2 * tt]) |
                                  ((uint64_t)__ballot_sync(~0u, valid8[2 * tt + 1]) << 32);
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
            if constexpr (!kF8) {
              // Two engines at once: tile::gather4 (TMA) brings latent boxes 0
              // and 1 and the rope box, 16-byte cp.async copies by the whole
              // warp bring latent boxes 2 and 3 (row t of the tile is rows[h]
              // of lane t % 32, h = t / 32; lane l copies chunk l % 8 of box
              // 2 + (l / 8) % 2 of row 2 i + l / 16, 128-byte swizzle: chunk ^
              // (t % 8)), the layout a TMA load of those boxes writes. Per
              // SM, each path alone moves a gathered tile at about the same
              // rate, one warp issuing. The barrier expects 32 cp.async
              // arrivals and lane 0's arrive with the TMA bytes.
              const uint32_t dst = stage_base + s * kSB;
              if (lane == 0) {
                misc->stage_mask[s] = mask;
                mbar_arrive_expect_tx(fb, 2 * kBoxBytes + kRopeBoxBytes);
              }
              __syncwarp();
              if (lane < 16) {
#pragma unroll
                for (int bx = 0; bx < 2; ++bx)
                  tma_gather4(dst + bx * kBoxBytes + lane * 4 * 128, &maps.row, vcol0 + 64 * bx, r[0], r[1], r[2], r[3],
                              fb);
                tma_gather4(dst + kRopeOff + lane * 4 * 64, &maps.rope_row, rcol0, r[0], r[1], r[2], r[3], fb);
              }
              const uint32_t bx = 2u + (uint32_t)((lane >> 3) & 1);
              const uint32_t cc = (uint32_t)(lane & 7);
              const size_t col_off = (size_t)(vcol0 + 64 * (int)bx + 8 * (int)cc) * 2;
#pragma unroll 4
              for (int i2 = 0; i2 < kPage / 2; ++i2) {
                const int t = 2 * i2 + (lane >> 4);
                const int rid = __shfl_sync(~0u, t < 32 ? rows[0] : rows[1], t & 31);
                cp_async_16(dst + bx * kBoxBytes + (uint32_t)t * 128u + ((cc ^ (uint32_t)(t & 7)) << 4),
                            a.cache + (size_t)rid * (kDQK * 2) + col_off);
              }
              cp_async_arrive_noinc(fb);
              __syncwarp();
              ++k;
              continue;
            }
            if (lane == 0) {
              misc->stage_mask[s] = mask;
              mbar_arrive_expect_tx(fb, kF8 ? kF8LoadBytes : kStageBytes);
            }
            __syncwarp();
            if (lane < 16) {
              // lane l gathers tile rows 4l .. 4l+3
              const uint32_t dst = stage_base + s * kSB;
              if constexpr (kF8) {
                tma_gather4(dst + kF8CodeOff + lane * 4 * 128, &maps.row, vcol0, r[0], r[1], r[2], r[3], fb);
                tma_gather4(dst + kF8CodeOff + kF8CodeBoxBytes + lane * 4 * 128, &maps.row, vcol0 + 128, r[0], r[1],
                            r[2], r[3], fb);
                tma_gather4(dst + kRopeOff + lane * 4 * 64, &maps.rope_row, kF8RopeOff + 64 * (int)crank, r[0], r[1],
                            r[2], r[3], fb);
                tma_gather4(dst + kF8ScaleStageOff + lane * 128, &maps.scale_row, kF8ScaleOff, r[0], r[1], r[2], r[3],
                            fb);
              } else {
#pragma unroll
                for (int bx = 0; bx < kVBoxes; ++bx)
                  tma_gather4(dst + bx * kBoxBytes + lane * 4 * 128, &maps.row, vcol0 + 64 * bx, r[0], r[1], r[2], r[3],
                              fb);
                tma_gather4(dst + kRopeOff + lane * 4 * 64, &maps.rope_row, rcol0, r[0], r[1], r[2], r[3], fb);
              }
            }
            __syncwarp();
            ++k;
          }
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
      // S for tile kk into S buffer kk % 2: K-step ks < 16 contracts columns
      // [16 ks, 16 ks + 16) of the four output-column boxes (A = Q in TMEM),
      // ks = 16, 17 the two halves of the rope box (A = Q rope in shared
      // memory). A descriptor plus (byte offset >> 4) describes the same layout
      // at that offset.
      const uint64_t dq = smem_desc_noswz(qrope, kQRopeLbo, kQRopeSbo);
      auto issue_s = [&](int kk) {
        const uint32_t sb = stage_base + (kk % kStages) * kSB;
        const uint32_t sd = tmem + kTmemS + 64u * (uint32_t)(kk & 1);
        const uint64_t d0 = smem_desc_sw128(sb, 16, 1024);
        const uint64_t dr = smem_desc_sw64(sb + kRopeOff, 512);
#pragma unroll
        for (int ks = 0; ks < 16; ++ks) {
          const uint32_t off = (uint32_t)((ks >> 2) * kBoxBytes + (ks & 3) * 32);
          mma_tmem_a(sd, tmem + kTmemQ + 8 * ks, d0 + (off >> 4), idS, ks > 0 ? 1u : 0u);
        }
        mma_ss(sd, dq, dr, idS, 1u);
        mma_ss(sd, dq + ((2 * kQRopeLbo) >> 4), dr + (32 >> 4), idS, 1u);
        mma_commit(smem_addr(&misc->s_full[kk & 1]));
      };
      // O (+)= P V for tile kk; releases the P buffer (in both CTAs) and the stage.
      auto issue_pv = [&](int kk, bool first) {
        const int s = kk % kStages;
        const uint64_t dv = smem_desc_sw128(stage_base + s * kSB, kBoxBytes, 1024);
        const uint64_t dp = smem_desc_sw128(pbuf + (kk & 1) * kPSlotBytes, 16, 1024);
        // K-step u: P advances 32 B along its swizzled rows, V 16 rows (2048 B)
        mma_ss(tmem + kTmemO, dp, dv, idO, first ? 0u : 1u);
        mma_ss(tmem + kTmemO, dp + (32 >> 4), dv + (2048 >> 4), idO, 1u);
        mma_ss(tmem + kTmemO, dp + (64 >> 4), dv + (4096 >> 4), idO, 1u);
        mma_ss(tmem + kTmemO, dp + (96 >> 4), dv + (6144 >> 4), idO, 1u);
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
        uint64_t t0 = 0;  // start of the current stretch without progress (0: none)
        while (np < n) {
          bool progress = false;
          // PV first: an S issued ahead of a ready PV delays it by a whole S
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
          if (ns < n) {
            const int kk = k + ns;
            // a stage is ready once loaded (and, for the fp8 cache, converted)
            if (mbar_test_wait(smem_addr(kF8 ? &misc->conv_full[kk % kStages] : &misc->full[kk % kStages]),
                               (kk / kStages) & 1) &&
                (kk < 2 || mbar_test_wait(smem_addr(&misc->s_free[kk & 1]), ((kk >> 1) & 1) ^ 1))) {
              // gathered bf16 rows partly written by cp.async (generic proxy):
              // order them before the tensor core's reads
              if (!kF8 && a.topk > 0) fence_proxy_async_smem();
              tc_fence_after();
              // all 18 MMAs back to back: the tensor pipe overlaps dependent MMAs
              // only while they are queued together
              issue_s(kk);
              ++ns;
              progress = true;
            }
          }
          // the clock is read only while nothing is ready (reading it is slow)
          if (progress) {
            t0 = 0;
          } else if (W.aborted()) {
            ok = false;
            break;
          } else {
            const uint64_t now = global_timer_ns();
            if (t0 == 0) {
              t0 = now;
            } else if (now - t0 > kTimeoutNs) {
              W.fail();
              ok = false;
              break;
            }
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
    const uint32_t xoff = (uint32_t)(quad * kXQuadStride) + (uint32_t)lane * 16u;
    const uint32_t xbytes = n_active * (uint32_t)kXQuadStride;
    const uint32_t xexp = xbuf + (uint32_t)(quad * kXQuadStride + kXQuadBytes) + (uint32_t)rl * 4u;
    int k = 0, j = 0;

    while (cur.next(task, pg0, pg1, split)) {
      write_q(0);
      float m_run = -INFINITY, l_run = 0.f;
      const int ntiles = pg1 - pg0;
      // own partial scores of the current tile (this thread: its row, tokens
      // 32*th..+31); the next tile's are loaded at the end of this one when
      // they are already complete, so the TMEM read overlaps the tile's tail
      uint32_t own[32];
      bool own_loading = false;
      for (int i = 0; i < ntiles; ++i, ++k) {
        const int s = k % kStages;
        const int xs = k & 1;
        if (!own_loading) {
          if (!W.wait_warp(&misc->s_full[k & 1], (k >> 1) & 1)) goto softmax_done;
          tc_fence_after();
          tmem_ld_16x32bx2_32<32>(own_lanes + kTmemS + 64u * (uint32_t)(k & 1), own);
        }
        own_loading = false;
        tmem_wait_ld();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_addr(&misc->s_free[k & 1]));
        // the peer's partial scores of these rows, in slot k % 2
        const uint32_t xslot = (uint32_t)(k % kXSlots) * kXBytes;
        if (expect_thread) mbar_arrive_expect_tx(smem_addr(&misc->x_full[k % kXSlots]), xbytes);
        if (!W.wait_warp(&misc->x_full[k % kXSlots], (k / kXSlots) & 1)) goto softmax_done;
        float sc[32];
        {
          uint32_t w[24];
#pragma unroll
          for (int c = 0; c < kXChunks; ++c) {
            const uint4 v = ld_shared_v4(xbuf + xslot + xoff + c * 512);
            w[4 * c + 0] = v.x;
            w[4 * c + 1] = v.y;
            w[4 * c + 2] = v.z;
            w[4 * c + 3] = v.w;
          }
          const float inv = fx23_inv(ld_shared_u32(xexp + xslot));
          const float bias = fx23_bias(inv);
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            float v0, v1, v2, v3;
            fx23_unpack4(w[3 * c], w[3 * c + 1], w[3 * c + 2], inv, bias, v0, v1, v2, v3);
            const float2 s01 = add2_rn(make_float2(__uint_as_float(own[4 * c + 0]), __uint_as_float(own[4 * c + 1])),
                                       make_float2(v0, v1));
            const float2 s23 = add2_rn(make_float2(__uint_as_float(own[4 * c + 2]), __uint_as_float(own[4 * c + 3])),
                                       make_float2(v2, v3));
            sc[4 * c + 0] = s01.x;
            sc[4 * c + 1] = s01.y;
            sc[4 * c + 2] = s23.x;
            sc[4 * c + 3] = s23.y;
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_addr(&misc->x_read[k % kXSlots]));

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
        const float2 sl2 = make_float2(a.scale_log2, a.scale_log2), nm = make_float2(-m_use, -m_use);
        uint32_t pp[16];
        float2 ps[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
        // two scores per packed instruction: the exponent arguments and the
        // row sum (four packed accumulators)
#pragma unroll
        for (int c = 0; c < 16; ++c) {
          const float2 e = fma2_rn(make_float2(sc[2 * c], sc[2 * c + 1]), sl2, nm);
          const float2 p = make_float2(ex2(e.x), ex2(e.y));
          pp[c] = pack_bf16x2(p.x, p.y);
          ps[c & 3] = add2_rn(ps[c & 3], p);
        }
        ps[0] = add2_rn(ps[0], ps[2]);
        ps[1] = add2_rn(ps[1], ps[3]);
        ps[0] = add2_rn(ps[0], ps[1]);
        l_run += ps[0].x + ps[0].y;
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
          const uint32_t sb = stage_base + s * kSB;
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
        if (i + 1 < ntiles &&
            __all_sync(~0u, mbar_test_wait(smem_addr(&misc->s_full[(k + 1) & 1]), ((k + 1) >> 1) & 1))) {
          tc_fence_after();
          tmem_ld_16x32bx2_32<32>(own_lanes + kTmemS + 64u * (uint32_t)((k + 1) & 1), own);
          own_loading = true;
        }
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
  } else if (warp >= 6 && warp <= 9) {
    // ------------------------------------------------------------ sender (rows the peer owns)
    const bool lead = (quad == 0 && lane == 0);  // warp 8, lane 0: expects and relays
    // peer addresses of slot 0; slot 1 follows at the same stride as here
    const uint32_t xfull_peer = map_to_rank(smem_addr(&misc->x_full[0]), peer);
    const uint32_t xempty_peer = map_to_rank(smem_addr(&misc->x_empty[0]), peer);
    const uint32_t xquad_peer = map_to_rank(xbuf, peer) + (uint32_t)(quad * kXQuadStride);
    const uint32_t xquad_stage = xstage + (uint32_t)(quad * kXQuadStride);
    const uint32_t xdummy_peer = map_to_rank(smem_addr(&misc->xdummy[quad]), peer);
    int k = 0;
    bool ok = true;

    // This CTA's softmax warps have read score slot kk % 2 for tile kk: tell
    // the peer (their arrives released the reads; this wait acquires them).
    auto relay_read = [&](int kk) -> bool {
      if (quad != 0) return true;
      if (!W.wait_warp(&misc->x_read[kk % kXSlots], (kk / kXSlots) & 1)) return false;
      if (lane == 0) st_async_b32(xdummy_peer, (uint32_t)kk, xempty_peer + 8u * (uint32_t)(kk % kXSlots));
      return true;
    };
    // Partial scores of tile kk for the rows the peer owns -> the peer's slot.
    // The relay for tile kk - 1 goes out first: it must precede the wait for
    // the peer's relay of the same tile (with one slot per CTA, the reverse
    // order deadlocks), and sending it before the S wait keeps the peer's
    // score send from waiting on this CTA's S.
    auto send_s = [&](int kk) -> bool {
      if (kk >= 1 && !relay_read(kk - 1)) return false;
      if (!W.wait_warp(&misc->s_full[kk & 1], (kk >> 1) & 1)) return false;
      tc_fence_after();
      uint32_t sr[32];
      tmem_ld_16x32bx2_32<32>(peer_lanes + kTmemS + 64u * (uint32_t)(kk & 1), sr);
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_addr(&misc->s_free[kk & 1]));
      // 23-bit fixed point with the row's exponent; masked tokens (any value,
      // even NaN) neither set the scale nor matter after the receiver masks them
      const int s = kk % kStages;
      if (!W.wait_warp(&misc->full[s], (kk / kStages) & 1)) return false;
      const uint32_t msk = (uint32_t)(misc->stage_mask[s] >> (32 * th));
      float amax = 0.f;
      if (msk == ~0u) {  // every token valid (the common case): a max tree, no bit tests
        float t[16];
#pragma unroll
        for (int c = 0; c < 16; ++c) t[c] = fmaxf(fabsf(__uint_as_float(sr[c])), fabsf(__uint_as_float(sr[c + 16])));
#pragma unroll
        for (int c = 0; c < 8; ++c) t[c] = fmaxf(t[c], t[c + 8]);
#pragma unroll
        for (int c = 0; c < 4; ++c) t[c] = fmaxf(t[c], t[c + 4]);
        amax = fmaxf(fmaxf(t[0], t[2]), fmaxf(t[1], t[3]));
      } else {
#pragma unroll
        for (int c = 0; c < 32; ++c)
          if ((msk >> c) & 1u) amax = fmaxf(amax, fabsf(__uint_as_float(sr[c])));
      }
      amax = fmaxf(amax, __shfl_xor_sync(~0u, amax, 16));
      const uint32_t ex = fx23_exponent(fx23_headroom(amax));
      const float mult = fx23_mult(ex);
      uint32_t w[24];
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        uint32_t c0, c1, c2, c3;
        fx23_code2(__uint_as_float(sr[4 * c]), __uint_as_float(sr[4 * c + 1]), mult, c0, c1);
        fx23_code2(__uint_as_float(sr[4 * c + 2]), __uint_as_float(sr[4 * c + 3]), mult, c2, c3);
        fx23_pack4(c0, c1, c2, c3, w[3 * c], w[3 * c + 1], w[3 * c + 2]);
      }
      // the peer's softmax warps have read its slot for tile kk - kXSlots (so
      // that copy has also finished reading this CTA's staging buffer)
      const int xs = kk % kXSlots;
      if (kk >= kXSlots && lead) mbar_arrive_expect_tx(smem_addr(&misc->x_empty[xs]), 4u);
      if (!W.wait_cluster_warp(&misc->x_empty[xs], ((kk / kXSlots) & 1) ^ 1)) return false;
      if (quad_active) {
        // stage this quadrant's part, then one bulk copy into the peer's slot
#pragma unroll
        for (int c = 0; c < kXChunks; ++c)
          st_shared_v4(xquad_stage + (uint32_t)(c * 512) + (uint32_t)lane * 16u,
                       make_uint4(w[4 * c], w[4 * c + 1], w[4 * c + 2], w[4 * c + 3]));
        if (th == 0) st_shared_u32(xquad_stage + (uint32_t)kXQuadBytes + (uint32_t)rl * 4u, ex);
        fence_proxy_async_smem();  // read by the bulk copy
        __syncwarp();
        if (lane == 0)
          bulk_copy_to_cta(xquad_peer + (uint32_t)xs * kXBytes, xquad_stage, (uint32_t)kXQuadStride,
                           xfull_peer + 8u * (uint32_t)xs);
      }
      return true;
    };

    int js = 0;
    while (ok && cur.next(task, pg0, pg1, split)) {
      write_q(1);
      const int n = pg1 - pg0;
      for (int i = 0; ok && i < n; ++i) ok = send_s(k + i);
      if (!ok) break;
      k += n;
      ++js;
    }
    if (ok && k > 0) ok = relay_read(k - 1);
    // the peer relays "slot read" for every score tile sent; collect the last one before exit
    if (ok) drain_x_empty(k, lead);
    __syncwarp();
  } else if (warp >= 10 && warp < 14) {
    // ------------------------------------------------------------ acceptor (rows the peer owns)
    const bool lead = (quad == 0 && lane == 0);  // warp 12, lane 0: expects the P messages
    const uint32_t pmbytes = n_active * (uint32_t)(kPQuadBytes + kStatQuadBytes);
    int k = 0, j = 0;
    bool ok = true;
    float pm = -INFINITY, pl = 0.f;  // the owner's running max / sum of this thread's row

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
      const int n = pg1 - pg0;
      for (int i = 0; ok && i < n; ++i) ok = accept_p(k + i);
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
    __syncwarp();
  }

  if constexpr (kF8) {
    if (warp >= 14) {
      // ---------------------------------------------------------- converters (fp8 cache)
      // Thread r (0..63) expands row r of each tile: its 256 codes (code box
      // 0: columns 0..127, box 1: 128..255, 128 bytes per row) into the four
      // bf16 boxes (128-byte swizzle). Every output row overlaps only the
      // same row's codes (box 2 over code box 0, box 3 over code box 1), so
      // a thread's writes never cover bytes another thread still has to read:
      // columns 0..191 are converted in place chunk by chunk (their outputs
      // land on codes the thread has already read), the last 64 codes are
      // read into registers before box 3 is written. Chunks are taken in an
      // order rotated by the row, which spreads a warp's accesses over the
      // shared-memory banks.
      const int r = (warp - 14) * 32 + lane;
      const uint32_t sw = (uint32_t)(r & 7);
      int k = 0;
      bool ok = true;
      while (ok && cur.next(task, pg0, pg1, split)) {
        for (int i = pg0; i < pg1; ++i, ++k) {
          const int s = k % kStages;
          if (!W.wait_warp(&misc->full[s], (k / kStages) & 1)) {
            ok = false;
            break;
          }
          const uint32_t sb = stage_base + s * kSB;
          const uint32_t soff = a.topk > 0 ? (uint32_t)((r >> 2) * 128 + (r & 3) * 16) : (uint32_t)(r * 16);
          const float sc = __uint_as_float(ld_shared_u32(sb + kF8ScaleStageOff + soff));
          const uint32_t codes = sb + kF8CodeOff + (uint32_t)r * 128u;
          // 16 codes (columns 16 q .. 16 q + 15) -> two 16-byte chunks of bf16 box q / 4
          auto put = [&](int q, uint4 c) {
            const uint32_t box = sb + (uint32_t)((q >> 2) * kBoxBytes) + (uint32_t)r * 128u;
            const uint32_t c0 = (uint32_t)(2 * (q & 3));
            st_shared_v4(box + ((c0 ^ sw) << 4), dequant8_e4m3(c.x, c.y, sc));
            st_shared_v4(box + (((c0 + 1u) ^ sw) << 4), dequant8_e4m3(c.z, c.w, sc));
          };
#pragma unroll 1
          for (int c = 0; c < 8; ++c) {  // columns 0..127 -> boxes 0, 1
            const int q = (c + r) & 7;
            put(q, ld_shared_v4(codes + (uint32_t)q * 16u));
          }
#pragma unroll 1
          for (int c = 0; c < 4; ++c) {  // columns 128..191 -> box 2, over code box 0's row
            const int q = 8 + ((c + r) & 3);
            put(q, ld_shared_v4(codes + kF8CodeBoxBytes + (uint32_t)(q - 8) * 16u));
          }
          uint4 last[4];  // columns 192..255: read all, then box 3 over code box 1's row
#pragma unroll
          for (int c = 0; c < 4; ++c)
            last[c] = ld_shared_v4(codes + kF8CodeBoxBytes + 64u + (uint32_t)((c + r) & 3) * 16u);
#pragma unroll
          for (int c = 0; c < 4; ++c) put(12 + ((c + r) & 3), last[c]);
          fence_proxy_async_smem();  // read by the tensor core
          __syncwarp();
          if (lane == 0) mbar_arrive(smem_addr(&misc->conv_full[s]));
        }
      }
      __syncwarp();
    }
  }

  // ------------------------------------------------------------ teardown
  // The combine may launch once every CTA is here (its blocks then wait for
  // the whole grid); triggering earlier would park them beside running CTAs.
  allow_dependents();
  tc_fence_before();
  cluster_sync();  // no remote access to this CTA's shared memory after this point
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace dec

// Host-side handles (used by mla_api.cu).
const void* decode_kernel_ptr(bool fp8) {
  return fp8 ? reinterpret_cast<const void*>(&dec::mla_decode_kernel<true>)
             : reinterpret_cast<const void*>(&dec::mla_decode_kernel<false>);
}
int decode_smem_bytes(bool fp8) { return fp8 ? dec::smem_bytes<true>() : dec::smem_bytes<false>(); }
int decode_threads(bool fp8) { return fp8 ? dec::kThreadsF8 : dec::kThreads; }

// Launched with programmatic stream serialization: the CTAs start (barriers,
// TMEM, cluster sync) while the plan kernel before them still runs, and wait
// for it before reading anything it or earlier work produced.
cudaError_t launch_decode(const CacheMaps& maps, const DecodeArgs& args, int workers, bool fp8,
                          cudaStream_t stream) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * workers, 1, 1);
  cfg.blockDim = dim3(fp8 ? dec::kThreadsF8 : dec::kThreads, 1, 1);
  cfg.dynamicSmemBytes = fp8 ? dec::smem_bytes<true>() : dec::smem_bytes<false>();
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return fp8 ? cudaLaunchKernelEx(&cfg, dec::mla_decode_kernel<true>, maps, args)
             : cudaLaunchKernelEx(&cfg, dec::mla_decode_kernel<false>, maps, args);
}

}  // namespace mla
