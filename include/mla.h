/*
 * libmla — MLA (multi-head latent attention) decode over a paged latent KV
 * cache, for NVIDIA B200 (sm_100a).
 *
 * What one decode step computes (for every sequence b, query token i, head h):
 *
 *   T      = visible cache positions of (b, i): dense t < L_b, or
 *            t <= L_b - Sq + i when causal, or the listed top-k positions
 *   row(t) = kv_cache[block_table[b][t / 64]][t % 64][0:576]  (c_kv[512] || k_pe[64])
 *   s_t    = scale * ( q[b,i,h,0:512] . row(t)[0:512] + q[b,i,h,512:576] . row(t)[512:576] )
 *   lse    = ln sum_t exp(s_t)
 *   out    = sum_t exp(s_t - lse) * row(t)[0:512]
 *
 * This is the absorbed branch of DeepSeek's MLA as printed in
 * "深度解读DeepSeek：源码解读 DeepSeek-V3", section "MLA" (two-term score
 * against kv_cache and pe_cache, float32 softmax, latent PV), with W_UK
 * folded into q and W_UV left to the caller ("DeepSeek-V2-Lite 模型结构详解",
 * section "五、MLA：注意力", the two absorption identities). The scale is
 * 1/sqrt(192): a query/key head is 128 content + 64 RoPE dimensions (same
 * page, "为什么 Q/K 是 192 维而 V 只有 128 维").
 *
 * Calling sequence, all asynchronous on one stream, no host synchronisation
 * (so it can be captured in a CUDA graph):
 *
 *   mla_decode_plan  -> split schedule from device seq_lens
 *   mla_decode       -> attention; unsplit rows final, split rows as partials
 *   mla_combine      -> LSE merge of partials into out / lse
 *
 * Ownership: the caller owns every buffer (plan, workspace, inputs, outputs).
 * The library allocates no device memory and keeps no state between calls
 * beyond per-device launch attributes. Pointers are device pointers unless
 * stated otherwise. q, kv_cache and out must be 16-byte aligned and densely
 * packed row-major with the shapes given below.
 *
 * Errors: argument problems are reported synchronously, before any launch,
 * as MLA_ERR_INVALID_ARG / MLA_ERR_UNSUPPORTED / MLA_ERR_WORKSPACE_TOO_SMALL;
 * launch failures as MLA_ERR_CUDA. Problems only visible on the device
 * (a length beyond the block table, a page id outside the cache, a sparse
 * index outside [0, L_b)) never trap: the offending tokens are skipped
 * (rows attend to the remaining tokens; a row left with none gets out = 0,
 * lse = -inf) and a bit is set in the plan's error word, read by
 * mla_get_error. Every pipeline wait inside the kernels is bounded; a wait
 * that runs out sets MLA_DEVERR_TIMEOUT and the kernel returns.
 */
#ifndef LIBMLA_MLA_H_
#define LIBMLA_MLA_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define MLA_API __attribute__((visibility("default")))
#else
#define MLA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* A cudaStream_t (NULL = legacy default stream). */
typedef struct CUstream_st* mla_stream_t;

typedef enum {
  MLA_OK = 0,
  MLA_ERR_INVALID_ARG = 1,         /* NULL / misaligned pointer, negative size, bad flag */
  MLA_ERR_UNSUPPORTED = 2,         /* valid but not implemented (e.g. H > 128, d_latent != 512, or
                                      B * Sq * max_pages_per_seq (dense) / B * Sq * ceil(topk / 64)
                                      (sparse) pages of work at or above 2^31) */
  MLA_ERR_WORKSPACE_TOO_SMALL = 3, /* plan or workspace buffer smaller than the sizing query says */
  MLA_ERR_CUDA = 4,                /* a CUDA runtime/driver call failed */
  MLA_ERR_DEVICE_BOUNDS = 5,       /* mla_get_error: bad length, page id or index seen on device */
  MLA_ERR_DEVICE_TIMEOUT = 6       /* mla_get_error: a bounded device wait ran out */
} mla_status_t;

/* Bits of the device error word (mla_get_error). */
#define MLA_DEVERR_SEQ_LEN 0x1u /* seq_lens[b] < 0 or > max_pages_per_seq * 64: sequence skipped */
#define MLA_DEVERR_PAGE_ID 0x2u /* block_table entry outside [0, num_pages): that page skipped */
#define MLA_DEVERR_INDEX 0x4u   /* sparse index outside [-1, L_b): that index skipped */
#define MLA_DEVERR_TIMEOUT 0x8u /* a pipeline wait ran out: results are invalid */
#define MLA_DEVERR_POSITION 0x10u /* mla_cache_insert: sequence id or position out of range: token skipped */

typedef struct {
  int32_t batch;             /* B >= 0 */
  int32_t q_len;             /* Sq >= 1: new query tokens per sequence (2 = MTP pair) */
  int32_t num_heads;         /* H: 1..128 */
  int32_t d_latent;          /* must be 512 (kv_lora_rank) */
  int32_t d_rope;            /* must be 64 (qk_rope_head_dim) */
  int32_t page_size;         /* must be 64 tokens */
  int32_t num_pages;         /* physical pages in kv_cache, >= 1 */
  int32_t max_pages_per_seq; /* block_table row stride (entries), >= 1 */
  int32_t topk;              /* 0: dense; > 0: sparse, topk indices per (b, i) */
  int32_t causal;            /* dense only: 1 = query i sees t <= L_b - Sq + i */
  float softmax_scale;       /* > 0; 1/sqrt(192) for DeepSeek V2/V3 */
  int32_t num_sms;           /* SMs to spread the work over; 0 = all SMs of the current device */
} mla_decode_desc_t;

/* Bytes of the plan buffer for this descriptor (0 if the descriptor is invalid).
 * The plan holds a small header, per-task page prefix sums and token counts,
 * and the device error word. */
MLA_API size_t mla_plan_bytes(const mla_decode_desc_t* desc);

/* Bytes of the workspace: fp32 partial outputs and LSEs for the worst-case
 * number of splits (one slot per (worker, task) overlap), so that no host
 * synchronisation is needed to size it (0 if the descriptor is invalid). */
MLA_API size_t mla_workspace_bytes(const mla_decode_desc_t* desc);

/* Number of 2-CTA workers (clusters) the decode kernel runs on the current
 * device for this descriptor (0 if invalid). Plan, decode and combine must
 * see the same value, i.e. the same device and desc->num_sms. */
MLA_API int32_t mla_num_workers(const mla_decode_desc_t* desc);

/* Step a1: split schedule. seq_lens: device int32 [B] (tokens cached per
 * sequence, including the Sq new ones). Writes the plan (device buffer of at
 * least mla_plan_bytes) and clears its error word. One small kernel. */
MLA_API mla_status_t mla_decode_plan(const mla_decode_desc_t* desc, const int32_t* seq_lens, void* plan,
                             size_t plan_bytes, mla_stream_t stream);

/* Steps a2-a7: attention over the latent cache.
 *   q            bf16 [B, Sq, H, 576]  absorbed queries (q_lat[512] || q_pe[64])
 *   kv_cache     bf16 [num_pages, 64, 576]  (c_kv[512] || k_pe[64] per token)
 *   block_table  int32 [B, max_pages_per_seq]  page ids of each sequence, in order
 *   seq_lens     int32 [B]  (the array given to mla_decode_plan)
 *   topk_indices int32 [B, Sq, topk] logical positions in [0, L_b), -1 = skip;
 *                NULL when desc->topk == 0
 *   out          bf16 [B, Sq, H, 512]   lse  fp32 [B, Sq, H] (natural log)
 *   workspace    at least mla_workspace_bytes
 * Rows whose task is not split are final after this call; the others are
 * final after mla_combine. */
MLA_API mla_status_t mla_decode(const mla_decode_desc_t* desc, void* plan, const void* q, const void* kv_cache,
                        const int32_t* block_table, const int32_t* seq_lens, const int32_t* topk_indices,
                        void* out, float* lse, void* workspace, size_t workspace_bytes, mla_stream_t stream);

/* Steps a2-a7 over an fp8 latent cache: the same attention as mla_decode,
 * with the cached latent kept as e4m3 codes and a per-token scale (the
 * deployment format of "DeepSeek-V3.2-Exp unboxing", the Indexer section,
 * whose reference code imitates it by casting the latent to fp8 and back to
 * bf16). kv_cache_fp8 is [num_pages, 64, 656] bytes, one 656-byte row per
 * token: bytes [0, 512) the e4m3 codes of c_kv (column order), [512, 640)
 * k_pe as 64 bf16, [640, 644) the float32 scale s, [644, 656) zero. The
 * decode uses c_kv[j] = bf16(float32(code[j] * s)) and k_pe unchanged; every
 * other argument, the plan, the workspace and mla_combine are those of
 * mla_decode (plan with mla_decode_plan for the same descriptor). The
 * kernel loads 656 bytes per token instead of 1152 and expands the codes to
 * exactly those bf16 values in shared memory before the tensor-core steps.
 * The rows of a page that a sequence does not reach may hold anything (they
 * are masked). */
MLA_API mla_status_t mla_decode_fp8(const mla_decode_desc_t* desc, void* plan, const void* q,
                                    const void* kv_cache_fp8, const int32_t* block_table, const int32_t* seq_lens,
                                    const int32_t* topk_indices, void* out, float* lse, void* workspace,
                                    size_t workspace_bytes, mla_stream_t stream);

/* Step a8: merge split partials by LSE (lse = ln sum_i exp(lse_i),
 * out = sum_i exp(lse_i - lse) out_i) and write empty rows as out = 0,
 * lse = -inf. Must follow mla_decode on the same stream. */
MLA_API mla_status_t mla_combine(const mla_decode_desc_t* desc, void* plan, const void* workspace, size_t workspace_bytes,
                         void* out, float* lse, mla_stream_t stream);

/* Synchronises the stream, reads the plan's device error word into
 * *error_bits (may be NULL) and maps it to MLA_OK, MLA_ERR_DEVICE_TIMEOUT
 * (timeout bit set) or MLA_ERR_DEVICE_BOUNDS (any other bit). */
MLA_API mla_status_t mla_get_error(const void* plan, uint32_t* error_bits, mla_stream_t stream);

/* Merge of decode results computed over disjoint token sets of the same
 * rows: the combine step of decode context parallelism, where each of N
 * ranks holds a shard of every sequence's cache, decodes over it, and the
 * ranks' (out, lse) are gathered (the beaiera.top DeepSeek tag page, the
 * abstract on DCP: the KV cache sharded along the sequence across ranks).
 * The same LSE merge as mla_combine, over whole shard results:
 *
 *   lse = ln sum_i exp(lse_i),   out = sum_i exp(lse_i - lse) * out_i
 *
 * parts with lse_i = -inf (no visible token in that shard) weigh nothing;
 * a row empty in every part gets out = 0, lse = -inf.
 *   part_out  bf16 [parts, rows, 512] (each part's mla_decode output, rows = B * Sq * H)
 *   part_lse  fp32 [parts, rows]
 *   out       bf16 [rows, 512]     lse  fp32 [rows]
 * part_out and out 16-byte aligned. One kernel, asynchronous on `stream`,
 * no allocation. */
typedef struct {
  int32_t parts;    /* N >= 1 */
  int32_t d_latent; /* must be 512 */
  int64_t rows;     /* rows per part, >= 0 */
} mla_merge_desc_t;

MLA_API mla_status_t mla_merge(const mla_merge_desc_t* desc, const void* part_out, const float* part_lse, void* out,
                               float* lse, mla_stream_t stream);

/* Decode step with no device allocation by anyone: plan + decode + combine as
 * above, with the plan and the split partials kept in a fixed 32 MiB array of
 * device memory that the library itself defines (every device that loads
 * libmla holds it until the process exits). For callers that cannot call
 * cudaMalloc, for example code running where a caching allocator owns all
 * device memory, or an embedding that forbids allocation while serving.
 * The caller passes inputs and outputs as for mla_decode_plan / mla_decode.
 * No source page describes it; this is an interface convenience.
 *
 * - The first call on a device sets up the scratch's device address and the
 *   kernel attributes (with that device current); make that first call before
 *   any stream capture.
 * - The plan and the partials are rewritten by every call before they are
 *   read, so nothing has to start at zero; the array keeps the last call's
 *   contents. All calls share it: calls that overlap on the GPU (other
 *   streams, other threads) race and give wrong results. Serialise them.
 * - Limit: with T = batch * q_len query tokens, the call fits when
 *     round_up(mla_plan_bytes(desc), 256) + (T + 1) * H * 2056 <= 32 MiB
 *   (the plan, then one fp32 partial slot of H x 512 outputs and 2 x H LSEs
 *   per task plus one per worker). Beyond it the call returns
 *   MLA_ERR_WORKSPACE_TOO_SMALL before touching the device (126 query tokens
 *   of 128 heads fit, 127 do not); within it, fewer workers are used when
 *   the worst-case partials of all of them would not fit.
 * - Device-side errors are handled as in mla_decode (bad tokens skipped) but
 *   the error word is not reachable by the caller; use the allocating entry
 *   points to read it. */
MLA_API mla_status_t mla_decode_noalloc(const mla_decode_desc_t* desc, const int32_t* seq_lens, const void* q,
                                        const void* kv_cache, const int32_t* block_table,
                                        const int32_t* topk_indices, void* out, float* lse, mla_stream_t stream);

/* ---------------------------------------------------------------------------
 * Cache insert: the step before decode that fills the paged cache.
 *
 * For each new token n (sequence b = seq_ids[n], position p = positions[n]):
 *
 *   x      = kv[n, 0:512]   (the latent c_kv)        r = kv[n, 512:576]  (k_pe)
 *   xn     = bf16( x / sqrt(mean(x^2) + eps) )        (computed in float32)
 *   row    = kv_cache[block_table[b][p / 64]][p % 64]
 *   row[0:512]        = bf16( weight * xn )
 *   row[512 + 2i]     = bf16( r[2i] cos[p][i] - r[2i+1] sin[p][i] )
 *   row[512 + 2i + 1] = bf16( r[2i] sin[p][i] + r[2i+1] cos[p][i] )   i < 32
 *
 * The latent is kv_norm'd and k_pe rotated before they are cached, as in the
 * absorbed branch of "深度解读DeepSeek：源码解读 DeepSeek-V3", section "MLA";
 * the RMSNorm's float32 arithmetic, cast and weight order follow
 * "DeepSeek-V2-Lite 模型结构详解", section "四、RMSNorm". The rotation pairs
 * consecutive elements; the cos/sin tables (the model's RoPE frequencies,
 * evaluated at each position) are the caller's.
 *
 *   kv          bf16 [N, 576]   (16-byte aligned, dense)
 *   weight      bf16 [512]      kv_norm weight (16-byte aligned)
 *   cos_table, sin_table  fp32 [max_positions, 32]
 *   seq_ids, positions    int32 [N]
 *   block_table int32 [batch, max_pages_per_seq]
 *   kv_cache    bf16 [num_pages, 64, 576]   rows are overwritten in place
 *   error_word  device uint32 or NULL: bits are OR-ed in, never cleared
 *
 * A token whose sequence id or position is out of range (b outside
 * [0, batch), p outside [0, min(max_pages_per_seq * 64, max_positions)))
 * sets MLA_DEVERR_POSITION, one whose page id is outside [0, num_pages) sets
 * MLA_DEVERR_PAGE_ID; either is skipped and the others are written. Two
 * tokens that address the same row race: which one lands is unspecified.
 * One kernel, asynchronous on `stream`, no allocation. */
typedef struct {
  int32_t num_tokens;        /* N >= 0 */
  int32_t batch;             /* rows of block_table, >= 0 */
  int32_t max_pages_per_seq; /* block_table row stride (entries), >= 1 */
  int32_t num_pages;         /* physical pages in kv_cache, >= 1 */
  int32_t max_positions;     /* rows of cos_table / sin_table, >= 1 */
  int32_t d_latent;          /* must be 512 */
  int32_t d_rope;            /* must be 64 */
  int32_t page_size;         /* must be 64 */
  float eps;                 /* RMSNorm epsilon, finite, >= 0 */
} mla_insert_desc_t;

MLA_API mla_status_t mla_cache_insert(const mla_insert_desc_t* desc, const void* kv, const void* weight,
                                      const float* cos_table, const float* sin_table, const int32_t* seq_ids,
                                      const int32_t* positions, const int32_t* block_table, void* kv_cache,
                                      uint32_t* error_word, mla_stream_t stream);

/* mla_cache_insert writing the fp8 cache format of mla_decode_fp8: the same
 * bf16 latent bf16(weight * bf16(x / rms)) and rotated k_pe, then per token
 * s = amax / 448 over the 512 latent values (float32 quotient; s = 1 for an
 * all-zero latent) and code[j] = e4m3(latent[j] / s) (float32 quotient, round
 * to nearest even, saturating at 448), written with k_pe, s and the zero
 * tail into the token's 656-byte row of kv_cache_fp8 [num_pages, 64, 656].
 * Same descriptor, errors and ordering rules as mla_cache_insert. */
MLA_API mla_status_t mla_cache_insert_fp8(const mla_insert_desc_t* desc, const void* kv, const void* weight,
                                          const float* cos_table, const float* sin_table, const int32_t* seq_ids,
                                          const int32_t* positions, const int32_t* block_table, void* kv_cache_fp8,
                                          uint32_t* error_word, mla_stream_t stream);

/* ---------------------------------------------------------------------------
 * Absorb / un-absorb: the per-head projections around the latent decode.
 *
 * wkv_b is the model's kv up-projection viewed as [H, 256, 512] bf16: rows
 * [0, 128) of head h are W_UK[h] and rows [128, 256) are W_UV[h]
 * ("深度解读DeepSeek：源码解读 DeepSeek-V3", section "MLA", absorbed branch;
 * "DeepSeek-V2-Lite 模型结构详解", section "五、MLA：注意力", the two absorption
 * identities). For T tokens (T = B * Sq of a decode step):
 *
 *   mla_absorb_query:    q_abs[t, h, 0:512]   = sum_d q[t, h, d] * W_UK[h][d, 0:512]   (d < 128)
 *                        q_abs[t, h, 512:576] = q[t, h, 128:192]                       (q_pe, copied)
 *   mla_unabsorb_output: out[t, h, v]         = sum_c W_UV[h][v, c] * o_lat[t, h, c]   (v < 128, c < 512)
 *
 * so that q_abs is mla_decode's query and o_lat its latent output. bf16 in
 * and out, fp32 accumulation on the tensor cores, one kernel each.
 *
 *   q      bf16 [T, H, 192]  (q_nope[128] || q_pe[64], as the q projection emits it)
 *   q_abs  bf16 [T, H, 576]  o_lat bf16 [T, H, 512]  out bf16 [T, H, 128]
 *   wkv_b  bf16 [H, 256, 512]
 * All pointers 16-byte aligned, densely packed; error_word: device uint32 or
 * NULL, MLA_DEVERR_TIMEOUT is OR-ed in if a bounded device wait ran out
 * (results then invalid). Asynchronous on `stream`, no allocation. */
typedef struct {
  int32_t num_tokens; /* T >= 0 */
  int32_t num_heads;  /* H: 1..128 */
  int32_t d_nope;     /* must be 128 (qk_nope_head_dim) */
  int32_t d_rope;     /* must be 64 (qk_rope_head_dim) */
  int32_t d_latent;   /* must be 512 (kv_lora_rank) */
  int32_t d_v;        /* must be 128 (v_head_dim) */
} mla_absorb_desc_t;

MLA_API mla_status_t mla_absorb_query(const mla_absorb_desc_t* desc, const void* q, const void* wkv_b, void* q_abs,
                                      uint32_t* error_word, mla_stream_t stream);
MLA_API mla_status_t mla_unabsorb_output(const mla_absorb_desc_t* desc, const void* o_lat, const void* wkv_b,
                                         void* out, uint32_t* error_word, mla_stream_t stream);

/* ---------------------------------------------------------------------------
 * Sparse-attention indexer: index scores and their top-k positions, the step
 * that picks the tokens a sparse decode (desc->topk > 0) attends to.
 *
 * "DeepSeek-V3.2-Exp unboxing", the Indexer section: the indexer scores the
 * cached keys of each sequence for each query token and keeps the
 * highest-scoring positions. Its scoring kernel takes fp8_index(q [b, m, h, d]
 * fp8, q_s [b, m, h] fp32, k [b, n, d] fp8, k_s [b, n] fp32) -> o [b, m, n]
 * fp32, with the model's per-head weights passed as q_s and the fp8 key
 * cache's per-token scales as k_s (shapes seen there: q [2, 128, 64, 128],
 * k [2, 128, 128]). The page does not print the kernel body; the score here
 * is the plain reading, a ReLU of each head's dot product weighted by q_s and
 * summed over heads, times the key's scale:
 *
 *   scores[b, i, t] = k_s[b, t] * sum_h q_s[b, i, h] * max(0, sum_d q[b, i, h, d] * k[b, t, d])
 *
 *   q       e4m3 (1 byte: sign, 4 exponent bits with bias 7, 3 mantissa bits;
 *           no infinities) [b, m, h, 128], 16-byte aligned
 *   q_s     fp32 [b, m, h], 16-byte aligned
 *   k       e4m3 [b, n, 128] (each sequence's keys contiguous), 16-byte aligned
 *   k_s     fp32 [b, n]
 *   scores  fp32 [b, m, n] (written for every t < n; no masking: the top-k
 *           call below takes each row's valid length)
 *   error_word  device uint32 or NULL: MLA_DEVERR_TIMEOUT is OR-ed in if a
 *           bounded device wait ran out (scores then invalid)
 * Products of two e4m3 values are exact in fp32; the sums over d (tensor
 * cores) and over h are fp32. h must be a multiple of 16, at most 256; d must
 * be 128. One kernel, asynchronous on `stream`, no allocation. */
typedef struct {
  int32_t batch;     /* b >= 0 */
  int32_t q_len;     /* m >= 1: query tokens per sequence */
  int32_t num_heads; /* h: index heads, a multiple of 16 in [16, 256] */
  int32_t head_dim;  /* d: must be 128 */
  int32_t num_keys;  /* n >= 0: keys per sequence */
} mla_index_desc_t;

MLA_API mla_status_t mla_index_scores(const mla_index_desc_t* desc, const void* q, const float* q_s, const void* k,
                                      const float* k_s, float* scores, uint32_t* error_word, mla_stream_t stream);

/* Top-k positions of each row of a score matrix, exactly (no approximation).
 *   scores      fp32 [rows, n] (for the indexer: rows = b * m)
 *   valid_lens  int32 [rows] or NULL: row r considers positions t < valid_lens[r]
 *               (clamped to [0, n]); NULL = all n. For a decode step this is
 *               seq_lens[b], or seq_lens[b] - Sq + i + 1 for causal query i.
 *   indices     int32 [rows, k]: the k positions with the largest scores in
 *               increasing order, equal scores at the cut going to the
 *               smaller positions (-0.0 and +0.0 are equal); when fewer than
 *               k positions are eligible, all of them and then -1. This is
 *               mla_decode's topk_indices layout (-1 = skip).
 * Scores must not be NaN (a NaN ranks above every number). Rows are
 * independent; one kernel (a cluster of up to 8 CTAs per row), asynchronous
 * on `stream`, no allocation. */
typedef struct {
  int32_t rows;     /* >= 0 */
  int32_t num_keys; /* n >= 0: scores per row (the row stride) */
  int32_t k;        /* >= 1: positions kept per row */
} mla_topk_desc_t;

MLA_API mla_status_t mla_topk(const mla_topk_desc_t* desc, const float* scores, const int32_t* valid_lens,
                              int32_t* indices, mla_stream_t stream);

/* Static string for a status code. */
MLA_API const char* mla_status_string(mla_status_t status);

#ifdef __cplusplus
}
#endif

#endif /* LIBMLA_MLA_H_ */
