// Thin inline-PTX wrappers for the sm_100a features the decode kernel uses:
// mbarriers, TMA tile and gather4 loads, cluster/DSMEM access (asynchronous
// remote stores, bulk copies), tcgen05 (TMEM allocation, MMA, commit,
// loads/stores, fences), and the 23-bit block fixed-point packing of the
// score exchange. Written from the public PTX ISA.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <stdint.h>

#define MLA_DEV __device__ __forceinline__

namespace mla {
namespace ptx {

MLA_DEV uint32_t smem_addr(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }

MLA_DEV uint64_t global_timer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

MLA_DEV uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
MLA_DEV uint32_t cluster_id_x() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%clusterid.x;" : "=r"(r));
  return r;
}

// Address of the same shared-memory variable in CTA `rank` of the cluster.
MLA_DEV uint32_t map_to_rank(uint32_t addr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
  return r;
}

MLA_DEV void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}


// ---------------------------------------------------------------- mbarrier

MLA_DEV void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
MLA_DEV void fence_mbar_init() { asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory"); }

MLA_DEV void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
MLA_DEV void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}

MLA_DEV bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t done;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(done)
      : "r"(bar), "r"(parity)
      : "memory");
  return done != 0;
}
// Same, with cluster-scope acquire: for phases completed by remote arrivals.
MLA_DEV bool mbar_try_wait_cluster(uint32_t bar, uint32_t parity) {
  uint32_t done;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(done)
      : "r"(bar), "r"(parity)
      : "memory");
  return done != 0;
}

// Non-blocking probe of a phase (never suspends the thread).
MLA_DEV bool mbar_test_wait(uint32_t bar, uint32_t parity) {
  uint32_t done;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(done)
      : "r"(bar), "r"(parity)
      : "memory");
  return done != 0;
}

// ---------------------------------------------------------------- fences

MLA_DEV void fence_proxy_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

// ---------------------------------------------------------------- TMA

MLA_DEV void prefetch_tmap(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(map) : "memory");
}

// 2-D tile load: box at (c0 = column, c1 = row) into shared memory; completes
// bytes on `bar`.
MLA_DEV void tma_load_2d(uint32_t dst, const CUtensorMap* map, int32_t c0, int32_t c1, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
          dst),
      "l"(map), "r"(c0), "r"(c1), "r"(bar)
      : "memory");
}

// Row gather: four rows r0..r3 of a one-row-high box at column c0, written
// to consecutive box rows at dst.
MLA_DEV void tma_gather4(uint32_t dst, const CUtensorMap* map, int32_t c0, int32_t r0, int32_t r1, int32_t r2,
                         int32_t r3, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile::gather4.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, "
      "%4, %5, %6}], [%7];" ::"r"(dst),
      "l"(map), "r"(c0), "r"(r0), "r"(r1), "r"(r2), "r"(r3), "r"(bar)
      : "memory");
}

// 16-byte asynchronous copy global -> shared (L2 only), and the arrive on an
// mbarrier that fires once all of this thread's earlier cp.async copies have
// landed (.noinc: the arrival counts toward the barrier's expected count).
MLA_DEV void cp_async_16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
MLA_DEV void cp_async_arrive_noinc(uint32_t bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(bar) : "memory");
}

// Programmatic dependent launch: a kernel launched with programmatic stream
// serialization may start while the previous kernel in the stream runs;
// grid_dependency_wait() returns once that kernel has completed and its
// writes are visible. allow_dependents() lets the next such kernel launch.
MLA_DEV void grid_dependency_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
MLA_DEV void allow_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// ---------------------------------------------------------------- DSMEM

// 16-byte asynchronous store into another CTA's shared memory; completes 16
// bytes on that CTA's barrier.
MLA_DEV void st_async_v4(uint32_t cluster_addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d,
                         uint32_t cluster_bar) {
  asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.v4.b32 [%0], {%1, %2, %3, %4}, [%5];" ::"r"(
                   cluster_addr),
               "r"(a), "r"(b), "r"(c), "r"(d), "r"(cluster_bar)
               : "memory");
}

// 4-byte asynchronous store into another CTA's shared memory; completes 4
// bytes on that CTA's barrier.
MLA_DEV void st_async_b32(uint32_t cluster_addr, uint32_t v, uint32_t cluster_bar) {
  asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.b32 [%0], %1, [%2];" ::"r"(cluster_addr), "r"(v),
               "r"(cluster_bar)
               : "memory");
}

// Bulk copy of `bytes` (multiple of 16, both addresses 16-byte aligned) from
// this CTA's shared memory to another CTA's; completes the bytes on that
// CTA's barrier. Written through the async proxy.
MLA_DEV void bulk_copy_to_cta(uint32_t dst_cluster, uint32_t src_cta, uint32_t bytes, uint32_t cluster_bar) {
  asm volatile("cp.async.bulk.shared::cluster.shared::cta.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                   dst_cluster),
               "r"(src_cta), "r"(bytes), "r"(cluster_bar)
               : "memory");
}

MLA_DEV uint32_t ld_shared_u32(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared.b32 %0, [%1];" : "=r"(v) : "r"(addr));
  return v;
}
MLA_DEV uint4 ld_shared_v4(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
  return v;
}
MLA_DEV void st_shared_u32(uint32_t addr, uint32_t v) {
  asm volatile("st.shared.b32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}
MLA_DEV void st_shared_v4(uint32_t addr, uint4 v) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
               : "memory");
}

// ---------------------------------------------------------------- tcgen05

MLA_DEV void tmem_alloc(uint32_t dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem), "r"(ncols)
               : "memory");
}
MLA_DEV void tmem_relinquish() { asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;"); }
MLA_DEV void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

MLA_DEV void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
MLA_DEV void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// Shared-memory matrix descriptor, 128-byte swizzle. `lbo` / `sbo` in bytes:
// K-major: sbo = stride between 8-row groups (lbo unused);
// MN-major: lbo = stride between 64-element MN blocks, sbo = stride between
// 8-row K groups.
MLA_DEV uint64_t smem_desc_sw128(uint32_t addr, uint32_t lbo, uint32_t sbo) {
  return (uint64_t)((addr & 0x3FFFFu) >> 4) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
         ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46) | (2ull << 61);
}

// Shared-memory matrix descriptor, 64-byte swizzle, K-major: rows of 64 B,
// `sbo` = stride between 8-row groups.
MLA_DEV uint64_t smem_desc_sw64(uint32_t addr, uint32_t sbo) {
  return (uint64_t)((addr & 0x3FFFFu) >> 4) | (1ull << 16) | ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46) |
         (4ull << 61);
}

// Shared-memory matrix descriptor, no swizzle, K-major: 8x16-byte core
// matrices; `lbo` = bytes between core matrices adjacent in K, `sbo` = bytes
// between 8-row groups.
MLA_DEV uint64_t smem_desc_noswz(uint32_t addr, uint32_t lbo, uint32_t sbo) {
  return (uint64_t)((addr & 0x3FFFFu) >> 4) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
         ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46);
}

// Instruction descriptor, kind::f16: bf16 A and B, fp32 accumulator.
__host__ __device__ constexpr uint32_t idesc_bf16_f32(int M, int N, int a_mn_major, int b_mn_major) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)a_mn_major << 15) | ((uint32_t)b_mn_major << 16) |
         ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}


// D[tmem] (+)= A[tmem] * B[smem]; issued by one thread.
MLA_DEV void mma_tmem_a(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.u32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// D[tmem] (+)= A[smem] * B[smem]; issued by one thread.
MLA_DEV void mma_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.u32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Arrive on the barrier at shared-memory offset `bar` of every CTA in
// `cta_mask` once all previously issued tcgen05 async ops of this thread
// complete (the arrive is multicast; nothing is loaded).
MLA_DEV void mma_commit_cluster(uint32_t bar, uint16_t cta_mask) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
                   bar),
               "h"(cta_mask)
               : "memory");
}

// Arrive on `bar` once all previously issued tcgen05 async ops of this thread complete.
MLA_DEV void mma_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar) : "memory");
}

MLA_DEV void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
MLA_DEV void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

MLA_DEV void tmem_st_32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]),
      "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]),
      "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]),
      "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}


// 16x32bx2 shape: threads 0-15 access lanes base..base+15 at columns [c, c+n),
// threads 16-31 the same lanes at columns [c+split, c+split+n).
template <int kSplit>
MLA_DEV void tmem_ld_16x32bx2_32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.16x32bx2.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32], %33;"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
        "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]),
        "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
        "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr), "n"(kSplit));
}
template <int kSplit>
MLA_DEV void tmem_st_16x32bx2_32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.16x32bx2.x32.b32 [%0], %33, {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]),
      "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]),
      "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]),
      "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31]), "n"(kSplit)
      : "memory");
}

// ---------------------------------------------------------------- math

// Hardware base-2 exponential (MUFU.EX2), ~2 ulp; ex2(-inf) = +0.
MLA_DEV float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// 23-bit block fixed point (one power-of-two scale per row of 64 values):
// with E the biased exponent of the row's largest magnitude (at least 22),
// q = round(x * 2^(148 - E)) lies in [-(2^22 - 1), 2^22 - 1] and
// x = q * 2^(E - 148), so the absolute error is at most
// 2^(E - 149) <= max|x| * 2^-22. Four values travel in three 32-bit words.
MLA_DEV uint32_t fx23_exponent(float amax) { return max((__float_as_uint(amax) >> 23) & 0xFFu, 22u); }
MLA_DEV float fx23_mult(uint32_t e) { return __uint_as_float((275u - e) << 23); }  // 2^(148 - e)
MLA_DEV float fx23_inv(uint32_t e) { return __uint_as_float((e - 21u) << 23); }    // 2^(e - 148)
// Four codes (low three bytes of each) -> three words.
MLA_DEV void fx23_pack4(uint32_t c0, uint32_t c1, uint32_t c2, uint32_t c3, uint32_t& w0, uint32_t& w1, uint32_t& w2) {
  w0 = __byte_perm(c0, c1, 0x4210);
  w1 = __byte_perm(c1, c2, 0x5421);
  w2 = __byte_perm(c2, c3, 0x6542);
}
// q * inv from a 23-bit field u: 2^23 + u is rebuilt as float bits, and
// (2^23 + u) * inv - (2^23 + 2^22) * inv is exact in one FMA.
MLA_DEV float fx23_bias(float inv) { return -12582912.0f * inv; }
// Three words -> four values.
MLA_DEV void fx23_unpack4(uint32_t w0, uint32_t w1, uint32_t w2, float inv, float bias, float& v0, float& v1,
                          float& v2, float& v3);

// Two floats -> bf16x2 (round to nearest even), `lo` in the low half.
MLA_DEV uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// Eight e4m3 codes (two words, lowest byte first) times a float32 scale,
// each product rounded to float32 and then to bf16: eight bf16 in a uint4.
// The hardware widens two codes at a time to f16 (exact: every e4m3 value is
// an f16 normal or zero), f16 -> float32 is exact, the product is one FMUL.
// Both products of a pair come from one packed two-lane multiply
// (mul.rn.f32x2: two IEEE round-to-nearest float32 products).
MLA_DEV float2 mul2_rn(float2 a, float s) {
  float2 d;
  asm("{\n\t.reg .b64 pa, pb, pd;\n\tmov.b64 pa, {%2, %3};\n\tmov.b64 pb, {%4, %4};\n\t"
      "mul.rn.f32x2 pd, pa, pb;\n\tmov.b64 {%0, %1}, pd;\n\t}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(s));
  return d;
}
// a + b and a * b + c on two float32 lanes at once (add.rn.f32x2 /
// fma.rn.f32x2: the same IEEE results as two FADD / FFMA).
MLA_DEV float2 add2_rn(float2 a, float2 b) {
  float2 d;
  asm("{\n\t.reg .b64 pa, pb, pd;\n\tmov.b64 pa, {%2, %3};\n\tmov.b64 pb, {%4, %5};\n\t"
      "add.rn.f32x2 pd, pa, pb;\n\tmov.b64 {%0, %1}, pd;\n\t}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return d;
}
MLA_DEV float2 fma2_rn(float2 a, float2 b, float2 c) {
  float2 d;
  asm("{\n\t.reg .b64 pa, pb, pc, pd;\n\tmov.b64 pa, {%2, %3};\n\tmov.b64 pb, {%4, %5};\n\t"
      "mov.b64 pc, {%6, %7};\n\tfma.rn.f32x2 pd, pa, pb, pc;\n\tmov.b64 {%0, %1}, pd;\n\t}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
  return d;
}
// Three words -> four values, the FMAs two lanes at a time.
MLA_DEV void fx23_unpack4(uint32_t w0, uint32_t w1, uint32_t w2, float inv, float bias, float& v0, float& v1,
                          float& v2, float& v3) {
  const auto f = [](uint32_t bits24) { return __uint_as_float((bits24 & 0x00FFFFFFu) | 0x4B000000u); };
  const float2 ib = make_float2(inv, inv), bb = make_float2(bias, bias);
  const float2 a = fma2_rn(make_float2(f(w0), f(__byte_perm(w0, w1, 0x0543))), ib, bb);
  const float2 b = fma2_rn(make_float2(f(__byte_perm(w1, w2, 0x0432)), f(w2 >> 8)), ib, bb);
  v0 = a.x;
  v1 = a.y;
  v2 = b.x;
  v3 = b.y;
}
// x * mult + 1.5 * 2^23 has unit spacing: its low 23 bits are
// round(x mult) + 2^22 (bit 23, the exponent's lowest bit, is 0 while
// |round(x mult)| < 2^22). Two codes at a time, the FMAs on two lanes and no
// clamp: with the row's exponent taken from fx23_headroom(max|x|), every
// |x| <= max|x| gives |round(x * mult)| <= 2^22 - 1. (Values outside that range - masked
// tokens, which the receiver discards - stay inside their own 3-byte field.)
MLA_DEV void fx23_code2(float x0, float x1, float mult, uint32_t& c0, uint32_t& c1) {
  constexpr float kMagic = 12582912.0f;
  const float2 y = fma2_rn(make_float2(x0, x1), make_float2(mult, mult), make_float2(kMagic, kMagic));
  c0 = __float_as_uint(y.x);
  c1 = __float_as_uint(y.y);
}
// max|x| * (1 + 2^-22): the exponent then leaves half a unit of headroom
// below 2^22 (only rows whose maximum lies in the top 2^-22 of its binade
// move to the next exponent).
MLA_DEV float fx23_headroom(float amax) { return amax * 1.0000002384185791f; }
MLA_DEV uint4 dequant8_e4m3(uint32_t w0, uint32_t w1, float s) {
  const uint32_t w[2] = {w0, w1};
  uint32_t o[4];
#pragma unroll
  for (int h = 0; h < 2; ++h) {
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      const __nv_fp8x2_storage_t pair = (__nv_fp8x2_storage_t)((w[h] >> (16 * q)) & 0xFFFFu);
      const float2 f = mul2_rn(__half22float2(__half2(__nv_cvt_fp8x2_to_halfraw2(pair, __NV_E4M3))), s);
      o[2 * h + q] = pack_bf16x2(f.x, f.y);
    }
  }
  return make_uint4(o[0], o[1], o[2], o[3]);
}

}  // namespace ptx
}  // namespace mla
