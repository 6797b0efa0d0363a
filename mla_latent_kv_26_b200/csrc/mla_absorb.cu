// The two per-head projections around the latent decode ("absorb" and
// "un-absorb"), as tcgen05 GEMMs.
//
// "深度解读DeepSeek：源码解读 DeepSeek-V3", section "MLA", the absorbed branch:
// wkv_b viewed as [H, 256, 512]; its rows [0, 128) of head h are W_UK[h]
// (128 x 512) and rows [128, 256) are W_UV[h]. The query's no-rope part is
// projected into the latent space, q_lat[h] = W_UK[h]^T q_nope[h] (512 wide),
// and attention runs against the latent cache; its latent output is projected
// back per head, o[h] = W_UV[h] o_lat[h] (128 wide). "DeepSeek-V2-Lite 模型结构
// 详解", section "五、MLA：注意力" (the two absorption identities).
//
// absorb:    q_abs[t, h] = ( W_UK[h]^T q[t, h, 0:128]  ||  q[t, h, 128:192] )   -> [T, H, 576]
//            D[t, j] = sum_d Q[t, d] W[d, j]: M = tokens (128 per tile), N = 256
//            (one half of the 512 latent columns per CTA), K = 128. A = Q from
//            shared memory, K-major; B = W_UK, MN-major (its rows are K).
// un-absorb: o[t, h] = W_UV[h] o_lat[t, h]                                       -> [T, H, 128]
//            D[t, v] = sum_j O[t, j] W[v, j]: M = tokens, N = 128, K = 512 in
//            four chunks of 128 through a 3-stage ring. B = W_UV, K-major.
//
// Operands arrive by TMA in 128-row x 64-column boxes with 128-byte swizzle;
// token rows past T read as zeros. The fp32 accumulator lives in TMEM (lane =
// token row) and is rounded to bf16 by the four warps of the CTA. For decode
// batches both GEMMs are bound by reading the weights (2 x 16.8 MB at H = 128).
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include "common.cuh"
#include "mla.h"
#include "sm100.cuh"

namespace mla {

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder();

namespace gemm {

using namespace ptx;

constexpr int kThreads = 128;
constexpr int kBox = 128 * 128;            // bytes of one 128-row x 64-column bf16 box
constexpr int kAbsorbSmem = 6 * kBox;      // Q (2 boxes; q_pe after the MMAs) + one half of W_UK (4 boxes)
constexpr int kUnStages = 3;
constexpr int kUnStageBytes = 4 * kBox;    // O chunk (2 boxes) + W_UV chunk (2 boxes)
constexpr int kUnSmem = kUnStages * kUnStageBytes;
constexpr int kAlignPad = 1024;            // the dynamic buffer is aligned up to 1024 B
constexpr long long kWaitCycles = 4000000000ll;  // ~2 s at 2 GHz: only a broken device gets here
constexpr uint32_t kErrTimeoutBit = 0x8u;

struct Maps {
  CUtensorMap act;  // activations: [T rows, H * width columns] bf16
  CUtensorMap w;    // wkv_b: [H * 256 rows, 512 columns] bf16
  CUtensorMap out;  // result: [T rows, H * out_width columns] bf16 (TMA stores; rows past T are not written)
};

struct Args {
  const __nv_bfloat16* q;  // absorb: [T, H, 192] (for the q_pe copy)
  __nv_bfloat16* out;      // absorb: [T, H, 576]; un-absorb: [T, H, 128]
  uint32_t* error;         // device word or nullptr
  int tokens, heads;
};

struct Bars {
  uint64_t full[kUnStages];
  uint64_t empty[kUnStages];
  uint64_t done;
  uint32_t tmem;
  int fail;
};

// Bounded wait on an mbarrier phase; false if it did not complete in time.
MLA_DEV bool wait_bounded(uint32_t bar, uint32_t parity) {
  if (mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity))
    if (clock64() - t0 > kWaitCycles) return false;
  return true;
}

// 32x32b shape, 32 columns: thread i of the warp reads TMEM lane (base lane + i).
MLA_DEV void tmem_ld_32x32b_32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
        "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]),
        "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
        "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}

// 32 fp32 accumulator columns of this thread's row -> 32 bf16 at dst (64 B).
MLA_DEV void store_row_bf16(__nv_bfloat16* dst, const uint32_t (&r)[32]) {
  uint4* d = reinterpret_cast<uint4*>(dst);
#pragma unroll
  for (int u = 0; u < 4; ++u)
    d[u] = make_uint4(pack_bf16x2(__uint_as_float(r[8 * u + 0]), __uint_as_float(r[8 * u + 1])),
                      pack_bf16x2(__uint_as_float(r[8 * u + 2]), __uint_as_float(r[8 * u + 3])),
                      pack_bf16x2(__uint_as_float(r[8 * u + 4]), __uint_as_float(r[8 * u + 5])),
                      pack_bf16x2(__uint_as_float(r[8 * u + 6]), __uint_as_float(r[8 * u + 7])));
}

// TMA store of a 2-D box from shared memory (completion tracked by the
// issuing thread's bulk async-group).
MLA_DEV void tma_store_2d(const CUtensorMap* map, uint32_t src, int32_t c0, int32_t c1) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.tile.bulk_group [%0, {%1, %2}], [%3];" ::"l"(map), "r"(c0),
               "r"(c1), "r"(src)
               : "memory");
}
MLA_DEV void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
MLA_DEV void bulk_wait_read() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }

// The epilogue's staging: this thread's TMEM lane (token row `row`) holds
// 32 * nchunks fp32 columns; they are rounded to bf16 and written as row
// `row` of 64-column boxes (128 bytes per row, 128-byte swizzle) at `boxes`,
// the layout a TMA store of those boxes reads.
MLA_DEV void stage_rows_bf16(uint32_t taddr, int nchunks, uint32_t boxes, int row) {
#pragma unroll 1
  for (int c = 0; c < nchunks; ++c) {
    uint32_t r[32];
    tmem_ld_32x32b_32(taddr + 32u * c, r);
    tmem_wait_ld();
    const uint32_t rowp = boxes + (uint32_t)((c >> 1) * kBox + row * 128);
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const uint32_t j = (uint32_t)((c & 1) * 4 + u);  // 16-byte chunk of the 128-byte row
      st_shared_v4(rowp + ((j ^ (uint32_t)(row & 7)) << 4),
                   make_uint4(pack_bf16x2(__uint_as_float(r[8 * u + 0]), __uint_as_float(r[8 * u + 1])),
                              pack_bf16x2(__uint_as_float(r[8 * u + 2]), __uint_as_float(r[8 * u + 3])),
                              pack_bf16x2(__uint_as_float(r[8 * u + 4]), __uint_as_float(r[8 * u + 5])),
                              pack_bf16x2(__uint_as_float(r[8 * u + 6]), __uint_as_float(r[8 * u + 7]))));
    }
  }
  fence_proxy_async_smem();  // read by the TMA store
}

MLA_DEV uint32_t aligned_base(uint8_t* raw) { return (smem_addr(raw) + (kAlignPad - 1)) & ~(uint32_t)(kAlignPad - 1); }

// Common prologue: barriers and the TMEM allocation (warp 0).
MLA_DEV void setup(Bars* bars, uint32_t cols) {
  if (threadIdx.x == 0) {
    for (int s = 0; s < kUnStages; ++s) {
      mbar_init(smem_addr(&bars->full[s]), 1);
      mbar_init(smem_addr(&bars->empty[s]), 1);
    }
    mbar_init(smem_addr(&bars->done), 1);
    bars->fail = 0;
    fence_mbar_init();
  }
  if (threadIdx.x < 32) {
    tmem_alloc(smem_addr(&bars->tmem), cols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
}

MLA_DEV void teardown(Bars* bars, uint32_t tmem, uint32_t cols) {
  tc_fence_before();
  __syncthreads();
  if (threadIdx.x < 32) {
    tc_fence_after();
    tmem_dealloc(tmem, cols);
  }
}

MLA_DEV void record_timeout(Bars* bars, uint32_t* error) {
  bars->fail = 1;
  if (error) atomicOr(error, kErrTimeoutBit);
}

__global__ void __launch_bounds__(kThreads, 1) mla_absorb_q_kernel(const __grid_constant__ Maps maps, const Args a) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ Bars bars;
  const uint32_t sa = aligned_base(smem_raw);  // Q: 2 boxes (d 0-63, 64-127)
  const uint32_t sb = sa + 2 * kBox;           // W_UK half: 4 boxes of 64 latent columns
  const int h = blockIdx.x, nh = blockIdx.y, m0 = blockIdx.z * 128;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  setup(&bars, 256);
  const uint32_t tmem = bars.tmem;

  if (threadIdx.x == 0) {
    const uint32_t full = smem_addr(&bars.full[0]), done = smem_addr(&bars.done);
    mbar_arrive_expect_tx(full, 6 * kBox);
#pragma unroll
    for (int b = 0; b < 2; ++b) tma_load_2d(sa + b * kBox, &maps.act, h * 192 + 64 * b, m0, full);
#pragma unroll
    for (int b = 0; b < 4; ++b) tma_load_2d(sb + b * kBox, &maps.w, nh * 256 + 64 * b, h * 256, full);
    bool ok = wait_bounded(full, 0);
    if (ok) {
      tc_fence_after();
      constexpr uint32_t idesc = idesc_bf16_f32(128, 256, 0, 1);
      // K-step ks: A advances 32 B inside a 64-column box (4 steps per box);
      // B (MN-major) advances 16 of its K rows = 2048 B; its 64-column N blocks are kBox apart.
#pragma unroll
      for (int ks = 0; ks < 8; ++ks)
        mma_ss(tmem, smem_desc_sw128(sa + (ks >> 2) * kBox + (ks & 3) * 32, 16, 1024),
               smem_desc_sw128(sb + ks * 2048, kBox, 1024), idesc, ks > 0 ? 1u : 0u);
      mma_commit(done);
      ok = wait_bounded(done, 0);
      // q_pe passes through: into the Q buffer, which the MMAs are done with
      if (ok && nh == 0) {
        mbar_arrive_expect_tx(smem_addr(&bars.full[1]), kBox);
        tma_load_2d(sa, &maps.act, h * 192 + 128, m0, smem_addr(&bars.full[1]));
      }
    } else {
      wait_bounded(full, 0);  // give the copies in flight a last chance to land
    }
    if (!ok) record_timeout(&bars, a.error);
  }
  __syncthreads();
  tc_fence_after();
  // epilogue: the 256 result columns, rounded to bf16, staged over the W_UK
  // boxes (the MMAs are done with them) and written by four TMA stores
  if (!bars.fail) stage_rows_bf16(tmem + ((uint32_t)(32 * warp) << 16), 8, sb, 32 * warp + lane);
  __syncthreads();
  if (threadIdx.x == 0 && !bars.fail) {
    const int col = h * (kDLatent + kDRope) + nh * 256;
#pragma unroll
    for (int b = 0; b < 4; ++b) tma_store_2d(&maps.out, sb + b * kBox, col + 64 * b, m0);
    if (nh == 0) {
      if (wait_bounded(smem_addr(&bars.full[1]), 0)) tma_store_2d(&maps.out, sa, h * (kDLatent + kDRope) + kDLatent, m0);
      else record_timeout(&bars, a.error);
    }
    bulk_commit();
    bulk_wait_read();  // the stores have read shared memory before the CTA can exit
  }
  teardown(&bars, tmem, 256);
}

__global__ void __launch_bounds__(kThreads, 1) mla_unabsorb_o_kernel(const __grid_constant__ Maps maps, const Args a) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ Bars bars;
  const uint32_t base = aligned_base(smem_raw);  // stage s: O chunk (2 boxes) then W_UV chunk (2 boxes)
  const int h = blockIdx.x, m0 = blockIdx.y * 128;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  setup(&bars, 128);
  const uint32_t tmem = bars.tmem;

  if (threadIdx.x == 0) {
    auto load_chunk = [&](int c) {
      const int s = c % kUnStages;
      const uint32_t st = base + s * kUnStageBytes, full = smem_addr(&bars.full[s]);
      mbar_arrive_expect_tx(full, kUnStageBytes);
#pragma unroll
      for (int b = 0; b < 2; ++b) {
        tma_load_2d(st + b * kBox, &maps.act, h * kDLatent + 128 * c + 64 * b, m0, full);
        tma_load_2d(st + (2 + b) * kBox, &maps.w, 128 * c + 64 * b, h * 256 + 128, full);
      }
    };
    for (int c = 0; c < kUnStages; ++c) load_chunk(c);
    constexpr uint32_t idesc = idesc_bf16_f32(128, 128, 0, 0);
    bool ok = true;
    int landed = kUnStages;  // chunks whose loads were issued
    for (int c = 0; c < 4 && ok; ++c) {
      const int s = c % kUnStages;
      const uint32_t st = base + s * kUnStageBytes;
      ok = wait_bounded(smem_addr(&bars.full[s]), (c / kUnStages) & 1);
      if (!ok) break;
      tc_fence_after();
      // 8 K-steps of 16 over the chunk's 128 columns: 4 per 64-column box, 32 B apart
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) {
        const uint32_t off = (uint32_t)((ks >> 2) * kBox + (ks & 3) * 32);
        mma_ss(tmem, smem_desc_sw128(st + off, 16, 1024), smem_desc_sw128(st + 2 * kBox + off, 16, 1024), idesc,
               (c > 0 || ks > 0) ? 1u : 0u);
      }
      mma_commit(smem_addr(&bars.empty[s]));
      if (c + kUnStages < 4) {
        // the stage is rewritten once the MMAs reading it are done
        ok = wait_bounded(smem_addr(&bars.empty[s]), 0);
        if (ok) {
          load_chunk(c + kUnStages);
          ++landed;
        }
      }
    }
    if (ok) {
      mma_commit(smem_addr(&bars.done));
      ok = wait_bounded(smem_addr(&bars.done), 0);
    } else {
      // give every issued copy a last chance to land before the CTA exits
      for (int c = max(0, landed - kUnStages); c < landed; ++c)
        wait_bounded(smem_addr(&bars.full[c % kUnStages]), (c / kUnStages) & 1);
    }
    if (!ok) record_timeout(&bars, a.error);
  }
  __syncthreads();
  tc_fence_after();
  // epilogue: 128 result columns in two boxes staged over stage 0 (the MMAs
  // are done with it), written by two TMA stores
  if (!bars.fail) stage_rows_bf16(tmem + ((uint32_t)(32 * warp) << 16), 4, base, 32 * warp + lane);
  __syncthreads();
  if (threadIdx.x == 0 && !bars.fail) {
#pragma unroll
    for (int b = 0; b < 2; ++b) tma_store_2d(&maps.out, base + b * kBox, h * 128 + 64 * b, m0);
    bulk_commit();
    bulk_wait_read();
  }
  teardown(&bars, tmem, 128);
}

bool aligned(const void* p, uintptr_t n) { return ((uintptr_t)p & (n - 1)) == 0; }

mla_status_t check(const mla_absorb_desc_t* d) {
  if (!d) return MLA_ERR_INVALID_ARG;
  if (d->num_tokens < 0 || d->num_heads < 1) return MLA_ERR_INVALID_ARG;
  if (d->num_tokens > 65535 * 128) return MLA_ERR_UNSUPPORTED;  // token tiles are a grid dimension
  if (d->d_nope != 128 || d->d_rope != kDRope || d->d_latent != kDLatent || d->d_v != 128 ||
      d->num_heads > kMaxHeads)
    return MLA_ERR_UNSUPPORTED;
  return MLA_OK;
}

// act: [T rows, H * width columns]; w: wkv_b as [H * 256 rows, 512 columns];
// out: [T rows, H * out_width columns].
bool encode_maps(Maps* m, const void* act, int tokens, int heads, int width, const void* wkv_b, void* out,
                 int out_width) {
  PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
  if (!enc) return false;
  cuuint32_t box[2] = {64, 128};
  cuuint32_t elem[2] = {1, 1};
  cuuint64_t adims[2] = {(cuuint64_t)heads * width, (cuuint64_t)tokens};
  cuuint64_t astr[1] = {(cuuint64_t)heads * width * 2};
  cuuint64_t wdims[2] = {(cuuint64_t)kDLatent, (cuuint64_t)heads * 256};
  cuuint64_t wstr[1] = {(cuuint64_t)kDLatent * 2};
  cuuint64_t odims[2] = {(cuuint64_t)heads * out_width, (cuuint64_t)tokens};
  cuuint64_t ostr[1] = {(cuuint64_t)heads * out_width * 2};
  return enc(&m->act, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(act), adims, astr, box, elem,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS &&
         enc(&m->w, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(wkv_b), wdims, wstr, box, elem,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS &&
         enc(&m->out, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, out, odims, ostr, box, elem, CU_TENSOR_MAP_INTERLEAVE_NONE,
             CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

cudaError_t set_smem(const void* kernel, int bytes) {
  return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
}

}  // namespace gemm
}  // namespace mla

using namespace mla;

extern "C" MLA_API mla_status_t mla_absorb_query(const mla_absorb_desc_t* desc, const void* q, const void* wkv_b,
                                                 void* q_abs, uint32_t* error_word, mla_stream_t stream) {
  mla_status_t st = gemm::check(desc);
  if (st != MLA_OK) return st;
  if (desc->num_tokens == 0) return MLA_OK;
  if (!q || !wkv_b || !q_abs) return MLA_ERR_INVALID_ARG;
  if (!gemm::aligned(q, 16) || !gemm::aligned(wkv_b, 16) || !gemm::aligned(q_abs, 16) ||
      !gemm::aligned(error_word, 4))
    return MLA_ERR_INVALID_ARG;
  gemm::Maps maps;
  if (!gemm::encode_maps(&maps, q, desc->num_tokens, desc->num_heads, 192, wkv_b, q_abs, kDLatent + kDRope))
    return MLA_ERR_CUDA;
  const int smem = gemm::kAbsorbSmem + gemm::kAlignPad;
  if (gemm::set_smem((const void*)gemm::mla_absorb_q_kernel, smem) != cudaSuccess) return MLA_ERR_CUDA;
  gemm::Args a{static_cast<const __nv_bfloat16*>(q), static_cast<__nv_bfloat16*>(q_abs), error_word,
               desc->num_tokens, desc->num_heads};
  dim3 grid(desc->num_heads, 2, (desc->num_tokens + 127) / 128);
  gemm::mla_absorb_q_kernel<<<grid, gemm::kThreads, smem, (cudaStream_t)stream>>>(maps, a);
  return cudaGetLastError() == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
}

extern "C" MLA_API mla_status_t mla_unabsorb_output(const mla_absorb_desc_t* desc, const void* o_lat,
                                                    const void* wkv_b, void* out, uint32_t* error_word,
                                                    mla_stream_t stream) {
  mla_status_t st = gemm::check(desc);
  if (st != MLA_OK) return st;
  if (desc->num_tokens == 0) return MLA_OK;
  if (!o_lat || !wkv_b || !out) return MLA_ERR_INVALID_ARG;
  if (!gemm::aligned(o_lat, 16) || !gemm::aligned(wkv_b, 16) || !gemm::aligned(out, 16) ||
      !gemm::aligned(error_word, 4))
    return MLA_ERR_INVALID_ARG;
  gemm::Maps maps;
  if (!gemm::encode_maps(&maps, o_lat, desc->num_tokens, desc->num_heads, kDLatent, wkv_b, out, 128))
    return MLA_ERR_CUDA;
  const int smem = gemm::kUnSmem + gemm::kAlignPad;
  if (gemm::set_smem((const void*)gemm::mla_unabsorb_o_kernel, smem) != cudaSuccess) return MLA_ERR_CUDA;
  gemm::Args a{nullptr, static_cast<__nv_bfloat16*>(out), error_word, desc->num_tokens, desc->num_heads};
  dim3 grid(desc->num_heads, (desc->num_tokens + 127) / 128);
  gemm::mla_unabsorb_o_kernel<<<grid, gemm::kThreads, smem, (cudaStream_t)stream>>>(maps, a);
  return cudaGetLastError() == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
}
