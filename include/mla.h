/*
 * mla.h — C ABI of a B200 (sm_100a) library for Multi-head Latent Attention
 * (MLA) decoding over a paged latent KV cache.
 *
 * What the library computes (for request b, query token i < s_q, head h):
 *   s_t  = softmax_scale * <q[b,i,h,0:576], row(t)[0:576]>      (K = whole row)
 *   out  = sum_t softmax(s)_t * row(t)[0:512]                    (V = first 512)
 *   lse  = ln sum_t exp(s_t)                                     (natural log)
 * over the key set t of the request: all cached tokens (t < cache_seqlens[b]),
 * restricted by the causal mask t <= seqlen - s_q + i when `causal` is set,
 * or, for sparse decoding, the token positions listed in `indices[b,i,:]`
 * (entries equal to -1 are ignored). An empty key set gives out = 0 and
 * lse = -inf. Optional: a per-head attention sink (one more logit with a
 * zero value, mla_decode_args.sink). With MLA_KV_NVFP4 the rows are 512
 * values that are both K and V (d_qk = d_v = 512) and the query is NVFP4 too.
 *
 * Sources (web pages on FlashMLA):
 *   - "Qu'est-ce que FlashMLA ?" (topnet.top), sections "Obtenir les
 *     métadonnées MLA" and "Exécuter le décodage MLA": the two-call shape
 *     get_mla_metadata(cache_seqlens, s_q*h_q//h_kv, h_kv) ->
 *     (tile_scheduler_metadata, num_splits), computed once per decode step
 *     and reused by every layer's flash_mla_with_kvcache(q, kvcache,
 *     block_table, cache_seqlens, dv, metadata, num_splits, causal).
 *   - "DeepSeek, FlashMLA 오픈소스 공개" (GeekNews), Summary: BF16, paged
 *     KV cache with block size 64, variable-length serving.
 *   - "[flashinfer] FlashInfer, NVFP4를 활용한 DeepSeek-V4 디코딩 성능 최적화",
 *     section 2 (nvfp4_mla_decode README): one latent row per token is both
 *     K and V; 64-token pages; causal mask inside the query block against the
 *     request's last tokens; BF16 out and natural-log FP32 LSE; tensor table
 *     (block_tables [batch, max_pages] int32, seq_lens [batch] int32);
 *     caller-owned workspace buffer; section 3: split-KV combine kernel.
 *   - deepseek-ai/FlashMLA (agentlenshq), "기술적 세부 사항": FP8 latent
 *     cache stores quantised values plus scale factors dequantised on the
 *     fly; sparse decoding takes an indices tensor whose -1 entries are
 *     ignored.
 *
 * Conventions for every entry point:
 *   - Pointers documented "device" must point to memory of the current CUDA
 *     device; "host" pointers to host memory. The caller owns every buffer;
 *     the library allocates no memory and keeps no per-call state.
 *   - Work is enqueued asynchronously on `stream` (a cudaStream_t; NULL = the
 *     legacy default stream). Host-side argument checks run synchronously
 *     before any launch and return an error code without launching.
 *   - Device-side problems (a page id outside [0, num_pages), a request longer
 *     than its block-table row, a wait that exceeded its time limit) never
 *     trap: the kernel skips the bad item and ORs a bit into a status word
 *     kept in the workspace; read it with mla_query_device_status().
 *   - Only h_kv == 1 (the MLA latent cache), d_qk == 576 (512 for NVFP4
 *     rows), d_v == 512 and a page size of 64 are implemented.
 */
#ifndef MLA_B200_H_
#define MLA_B200_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* mla_stream_t; /* identical to cudaStream_t */

typedef enum {
  MLA_OK = 0,
  MLA_ERR_INVALID_ARG = 1,         /* null/misaligned pointer, bad size or shape */
  MLA_ERR_UNSUPPORTED = 2,         /* valid request outside what is implemented */
  MLA_ERR_WORKSPACE_TOO_SMALL = 3, /* workspace_bytes < mla_workspace_size(...) */
  MLA_ERR_CUDA = 4,                /* a CUDA runtime/driver call failed */
  MLA_ERR_DEVICE_TIMEOUT = 5,      /* status word: a device wait hit its limit */
  MLA_ERR_DEVICE_BOUNDS = 6        /* status word: an index/page was out of range */
} mla_status_t;

/* KV cache storage formats (mla_decode_args.kv_format). */
enum {
  /* bf16 [num_pages, 64, 1, 576]; token row = 512 latent + 64 RoPE dims. */
  MLA_KV_BF16 = 0,
  /* uint8 [num_pages, 64, 656] token records, byte layout
   *   [0,512)   512 e4m3 latent codes (OCP FP8 E4M3, no infinities)
   *   [512,528) 4 fp32 scales, scale k applies to latent dims [128k,128k+128)
   *   [528,656) 64 bf16 RoPE dims
   * dequantised value = bf16_rne(fp32(e4m3) * scale), product rounded to
   * nearest in fp32; the RoPE dims are used as stored. */
  MLA_KV_FP8_E4M3 = 1,
  /* NVFP4 rows of 512 values that are both K and V (d_qk = d_v = 512; the
   * FlashInfer page's nvfp4_mla_decode README, section 2): the cache is
   * uint8 [num_pages, 64, 256] packed E2M1 (element 2i in the low nibble of
   * byte i, 2i+1 in the high nibble) with UE4M3 scales uint8 [num_pages, 64,
   * 32] in mla_decode_args.kv_scale, scale byte j for elements [16j, 16j+16);
   * the query is packed the same way, uint8 [batch, s_q, h_q, 256], with
   * scales [batch, s_q, h_q, 32] in q_scale. value = e2m1 * ue4m3 (UE4M3:
   * E4M3 without a sign; bit 7 is ignored), exact in bf16, which the tensor
   * cores then use. Paged decoding only. */
  MLA_KV_NVFP4 = 2
};

/* Bits of the device status word kept at the start of the workspace. */
enum {
  MLA_DEVICE_STATUS_TIMEOUT = 1u, /* an mbarrier wait exceeded timeout_ns */
  MLA_DEVICE_STATUS_BOUNDS = 2u   /* page id, block-table slot or index out of range */
};

/* Test and timing hooks for mla_decode_args.debug_flags (0 in normal use). */
enum {
  /* The MMA issuer withholds its first "scores ready" signal, so the
   * softmax warps' bounded wait runs out: exercises the timeout path. */
  MLA_DEBUG_WITHHOLD_SCORES = 1u,
  /* mla_decode_* enqueue only the decode kernel; the caller enqueues
   * mla_combine afterwards (lets a profiler or timer separate the two). */
  MLA_DEBUG_SKIP_COMBINE = 2u
};

#define MLA_D_QK 576
#define MLA_D_V 512
#define MLA_PAGE_SIZE 64
#define MLA_TILE_MD_INTS 8 /* int32 entries per scheduler part */
#define MLA_MAX_ROWS 128   /* max query rows of one work unit */

/* Human-readable name of a status code (static string, never NULL). */
const char* mla_status_string(mla_status_t status);

/* Work units of a decode problem (host-only, pure function of the sizes).
 * Paged decoding (topk == 0): the R = s_q*h_q/h_kv query rows of a request,
 * laid out [query token][head], are cut into the fewest equal blocks of at
 * most MLA_MAX_ROWS rows (the smallest count n >= ceil(R/128) that divides
 * R); every block is a unit of R/n rows that reads the request's whole key
 * set (FlashInfer README: q_len query tokens per request, six for
 * DeepSeek-V4, so R reaches 6*64 = 384 rows). Sparse decoding (topk > 0):
 * one unit per (request, query token) of h_q/h_kv rows. The units of a
 * request are consecutive: unit u is rows [u*rows, (u+1)*rows) of the
 * flattened [batch*s_q*h_q] row axis of q, out and lse.
 * Writes *units_per_request (units = batch * units_per_request) and
 * *rows_per_unit. Errors: INVALID_ARG (null outputs, non-positive sizes),
 * UNSUPPORTED (h_kv != 1; sparse h_q > MLA_MAX_ROWS; s_q*h_q > 2^20). */
mla_status_t mla_decode_geometry(int s_q, int h_q, int h_kv, int topk, int* units_per_request,
                                 int* rows_per_unit);

/* Number of scheduler parts for a problem on `device` (host-only query).
 * rows = the rows per unit of mla_decode_geometry. One part is processed by
 * ceil(rows/64) CTAs, one per SM, so parts = floor(num_SMs / ceil(rows/64))
 * (for two CTAs per part, no more than the CTA pairs that fit at once).
 * Writes *num_sm_parts. */
mla_status_t mla_get_num_sm_parts(int device, int s_q, int h_q, int h_kv, int topk, int* num_sm_parts);

/* Split-KV tile scheduler ("get_mla_metadata" in the pages' API).
 *
 * Work units (mla_decode_geometry): a paged unit of request b has
 * ceil(cache_seqlens[b]/128) blocks of 128 tokens (two pages); a sparse
 * unit (b, i), i < s_q, has ceil(topk/128) blocks of 128 index slots. Every unit costs its blocks plus a fixed
 * overhead of 3 blocks; the units are laid end to end and cut into ranges of
 * equal cost, so one part covers a contiguous run of (unit, block) pairs and
 * a unit may be split across parts. The range length is
 * ceil(total / num_sm_parts), raised to the largest unit's cost when that is
 * at most 8 blocks more (equal units then take one part each and are not
 * split; the trailing parts get no work). The total cost must stay below 2^31.
 * One exception: when every unit has the same n > 0 blocks, a unit holds
 * more than 64 query rows, and num_sm_parts >= 2 * units, each unit is cut
 * into k = min(num_sm_parts / units, ceil(n / 2)) pieces of whole pairs of
 * blocks (their lengths differ by at most one pair), piece j of unit u goes
 * to part u*k + j, and the parts past k * units get no work (their range
 * begins and ends at {units, 0}). Cost per part is then reported as k.
 *
 *   cache_seqlens  device int32 [batch]; read only when topk == 0 (may be
 *                  NULL when topk > 0).
 *   tile_md        device int32 [num_sm_parts * MLA_TILE_MD_INTS], written:
 *                  per part {begin_unit, begin_block, end_unit, end_block
 *                  (exclusive, lexicographic), workspace index of the
 *                  part's first piece, cost per part, 0, 0}.
 *   num_splits     device int32 [units + 1], written: exclusive prefix sum
 *                  of the number of parts touching each unit (a unit with
 *                  no blocks has 0 splits).
 * Both outputs are reusable by every layer of the same decode step.
 * Errors: INVALID_ARG for null outputs or non-positive sizes, topk % 64 != 0;
 * UNSUPPORTED for h_kv != 1 or s_q*h_q > 2^20. */
mla_status_t mla_get_metadata(const int32_t* cache_seqlens, int batch, int s_q, int h_q, int h_kv,
                              int topk, int num_sm_parts, int32_t* tile_md, int32_t* num_splits,
                              mla_stream_t stream);

/* The same scheduler run on the host: all pointers are host pointers and the
 * call is synchronous. Produces exactly what mla_get_metadata produces. */
mla_status_t mla_get_metadata_host(const int32_t* cache_seqlens, int batch, int s_q, int h_q, int h_kv,
                                   int topk, int num_sm_parts, int32_t* tile_md, int32_t* num_splits);

/* Bytes of caller-owned workspace a decode call needs (units and rows as
 * given by mla_decode_geometry):
 *   256-byte header (the device status word at offset 0), then
 *   partial LSE  fp32 [units + num_sm_parts][rows]          (256-B aligned)
 *   partial O    fp32 [units + num_sm_parts][rows][512]     (256-B aligned)
 * Split s of unit u is entry num_splits[u] + s of the partial arrays; each
 * partial O is already divided by its own softmax denominator. Returns 0 for
 * invalid sizes. A fresh workspace must have its status word cleared once
 * (mla_clear_device_status) before its first use. */
size_t mla_workspace_size(int batch, int s_q, int h_q, int h_kv, int topk, int num_sm_parts);

typedef struct {
  const void* q;                /* device bf16 [batch, s_q, h_q, 576], 16-B aligned
                                   (MLA_KV_NVFP4: uint8 [batch, s_q, h_q, 256]) */
  const void* kcache;           /* device, format per kv_format, 16-B aligned */
  const int32_t* block_table;   /* device int32 [batch, block_table_stride]; entry
                                   j of row b = physical page of tokens [64j, 64j+64) */
  const int32_t* cache_seqlens; /* device int32 [batch] */
  const int32_t* tile_md;       /* device, from mla_get_metadata (same sizes) */
  const int32_t* num_splits;    /* device, from mla_get_metadata */
  void* out;                    /* device bf16 [batch, s_q, h_q, 512], written */
  float* lse;                   /* device fp32 [batch, s_q, h_q], written */
  void* workspace;              /* device, >= mla_workspace_size(...) bytes */
  size_t workspace_bytes;
  int batch, s_q, h_q, h_kv;
  int d_qk, d_v;                /* must be 576 (512 for MLA_KV_NVFP4) and 512 */
  int page_size;                /* must be 64 */
  int num_pages;                /* physical pages in kcache */
  int block_table_stride;       /* int32 elements between block-table rows */
  int num_sm_parts;             /* the value passed to mla_get_metadata */
  float softmax_scale;          /* multiplies q.k before the softmax */
  int causal;                   /* nonzero: causal mask inside the s_q block */
  int kv_format;                /* MLA_KV_BF16, MLA_KV_FP8_E4M3 or MLA_KV_NVFP4 */
  uint64_t timeout_ns;          /* limit of every device wait; 0 = 2 s */
  uint32_t debug_flags;         /* MLA_DEBUG_* test hooks; 0 normally */
  const float* sink;            /* device fp32 [h_q], 4-B aligned, or NULL: per-head
                                   attention-sink logits (FlashInfer page, section 2,
                                   "sinks [num_heads] float32"). sink[h] joins the
                                   softmax denominator of every row of head h as one
                                   more logit, in the units of softmax_scale * q.k,
                                   whose value vector is zero:
                                     lse = ln(sum_t e^(s_t) + e^sink[h]),
                                     out = sum_t e^(s_t - lse) v_t.
                                   An empty key set then gives out 0, lse = sink[h];
                                   sink[h] = -inf is the same as no sink. */
  const void* q_scale;          /* MLA_KV_NVFP4 only: device uint8 [batch, s_q, h_q, 32]
                                   UE4M3 query scales; ignored otherwise */
  const void* kv_scale;         /* MLA_KV_NVFP4 only: device uint8 [num_pages, 64, 32]
                                   UE4M3 cache scales, 16-B aligned; ignored otherwise */
} mla_decode_args;

/* Paged decoding: enqueues the decode kernel and the split combine.
 * Output rows of units processed in one piece are written by the decode
 * kernel; split units and empty units are finished by the combine. Errors:
 * INVALID_ARG (null or misaligned pointers, d_qk/d_v/page_size mismatch,
 * non-positive sizes, bad kv_format), UNSUPPORTED (h_kv != 1, s_q*h_q >
 * 2^20), WORKSPACE_TOO_SMALL, CUDA (launch failure). */
mla_status_t mla_decode_paged(const mla_decode_args* args, mla_stream_t stream);

/* Paged decoding with a built-in workspace (the pages have no counterpart:
 * this entry point exists for callers that cannot allocate device memory
 * when they decode, such as a server that reserved all device memory for its
 * own pool at start-up, or a latency-critical step that must not pay for the
 * implicit synchronisation and latency of cudaMalloc/cudaFree).
 *
 * Same computation and arguments as mla_decode_paged, except that
 * args->workspace must be NULL and args->workspace_bytes 0: the split-KV
 * partials and the device status word live in a file-scope device array of
 * MLA_NOALLOC_WORKSPACE_BYTES held by every GPU that loads the library until
 * the process exits. Nothing is allocated by the call.
 *   - The first call on a device looks up the array's device address (once
 *     per device, with that device current); make that first call before any
 *     stream capture.
 *   - All calls on a device share the array and it keeps the last call's
 *     contents; calls whose work overlaps on the GPU race on it.
 *   - Each call zeroes the status word before enqueueing the decode; device
 *     status bits are not reported through mla_query_device_status (the
 *     caller has no workspace pointer to pass).
 * Errors: as mla_decode_paged; INVALID_ARG when a workspace is passed;
 * WORKSPACE_TOO_SMALL when mla_workspace_size(...) of the problem exceeds
 * MLA_NOALLOC_WORKSPACE_BYTES (use fewer num_sm_parts or mla_decode_paged). */
#define MLA_NOALLOC_WORKSPACE_BYTES (48u << 20)
mla_status_t mla_decode_paged_noalloc(const mla_decode_args* args, mla_stream_t stream);

/* Token-sparse decoding. indices: device int32 [batch, s_q, topk], logical
 * token positions of request b resolved through its block-table row; -1
 * entries are ignored; other values outside [0, cache_seqlens[b]) are ignored
 * and set MLA_DEVICE_STATUS_BOUNDS; duplicates count as often as they occur.
 * topk must be a positive multiple of 64; `causal` is ignored. Both cache
 * formats are accepted: with MLA_KV_FP8_E4M3 the indexed token records are
 * gathered and dequantised as for paged decoding (the FP8 token-sparse
 * combination of the pages' sparse-decoding figures). tile_md/num_splits
 * come from mla_get_metadata(..., topk).
 * Errors as for mla_decode_paged; UNSUPPORTED also for h_q/h_kv >
 * MLA_MAX_ROWS and for MLA_KV_NVFP4. */
mla_status_t mla_decode_sparse(const mla_decode_args* args, const int32_t* indices, int topk,
                               mla_stream_t stream);

/* ---------------------------------------------------------------------------
 * The steps on either side of the attention ("deepseek-ai/FlashMLA"
 * (agentlenshq), feature list: a fused kernel runs Q-norm, RoPE, the
 * attention, the output-side conjugate RoPE and the final FP8 cast in one
 * launch; the page names the steps, not their arithmetic). Query rows are
 * [batch, s_q, h_q, d_qk] and output rows [batch, s_q, h_q, 512], row
 * r = (b*s_q + i)*h_q + h; query token t = b*s_q + i. rope_cos/rope_sin:
 * device fp32 [batch*s_q][32], cos/sin of the angle of RoPE pair p at query
 * token t (the caller derives them from the token's position). Both calls
 * are asynchronous on `stream`, allocate nothing and keep no state.
 * ------------------------------------------------------------------------- */

/* q_out = RMS-norm of each query row over its d_qk values times gamma,
 * q / sqrt(mean(q^2) + eps) * gamma, then its last 64 dims (the RoPE part:
 * 512..575 of a 576-dim row, 448..511 of a 512-dim row) rotated pair-wise,
 * (x[2p], x[2p+1]) -> (x0 cos - x1 sin, x0 sin + x1 cos). Computed in fp32,
 * rounded to bf16 (nearest even).
 * q, q_out: device bf16 [rows][d_qk], 16-byte aligned; q_out may equal q.
 * gamma: device fp32 [d_qk], 8-byte aligned. eps >= 0.
 * Errors: INVALID_ARG for null or misaligned pointers, d_qk not 576 or 512,
 * eps < 0, non-positive sizes; UNSUPPORTED above 2^31 rows; CUDA. */
mla_status_t mla_q_norm_rope(const void* q, void* q_out, int batch, int s_q, int h_q, int d_qk,
                             const float* gamma, float eps, const float* rope_cos, const float* rope_sin,
                             mla_stream_t stream);

/* Output epilogue: the output's RoPE part (the dims of V inside the last 64
 * dims of d_qk: none when d_qk = 576, dims 448..511 when d_qk = 512) rotated
 * back by the query token's angle, (x0 cos + x1 sin, x1 cos - x0 sin); then
 * each 128-value tile cast to e4m3: scale = amax / 448 (1 when amax = 0),
 * code = round-to-nearest-even(value / scale) saturated to +-448. Every
 * product, sum and quotient is rounded once in fp32 (no contraction).
 * out: device bf16 [rows][512], 16-byte aligned (the decode output).
 * out_fp8: device uint8 [rows][512], 16-byte aligned; out_scale: device fp32
 * [rows][4]. rope_cos/rope_sin may be NULL when d_qk = 576.
 * Errors: INVALID_ARG for null or misaligned pointers, d_qk not 576 or 512,
 * non-positive sizes; UNSUPPORTED above 2^31 rows; CUDA. */
mla_status_t mla_out_rope_fp8(const void* out, int batch, int s_q, int h_q, int d_qk, const float* rope_cos,
                              const float* rope_sin, void* out_fp8, float* out_scale, mla_stream_t stream);

/* Split-KV combine alone (mla_decode_* call it already). For every unit u
 * with n = num_splits[u+1] - num_splits[u]:
 *   n >= 2: lse = ln sum_s exp(lse_s), out = sum_s exp(lse_s - lse) * o_s
 *           over the workspace partials (fp32), out rounded to bf16;
 *   n == 0: out = 0, lse = -inf;   n == 1: nothing is written.
 * out/lse rows of unit u start at row u*rows_per_unit (units and rows as
 * given by mla_decode_geometry). */
mla_status_t mla_combine(const void* workspace, size_t workspace_bytes, const int32_t* num_splits,
                         int num_units, int rows_per_unit, int num_sm_parts, void* out, float* lse,
                         mla_stream_t stream);

/* mla_combine with a per-head attention sink (see mla_decode_args.sink):
 * after the splits are merged, row r of unit u, whose head is
 * h = (u*rows_per_unit + r) % h_q, takes
 *   lse' = ln(e^lse + e^sink[h]),  out *= e^(lse - lse'),
 * and a unit with n == 0 gets out = 0, lse = sink[h]. Units with n == 1 are
 * left alone (their decode piece folded the sink in already).
 * sink: device fp32 [h_q], 4-B aligned, or NULL (then identical to
 * mla_combine and h_q is ignored). Errors as mla_combine; INVALID_ARG also
 * when sink is given and h_q <= 0 or sink is misaligned. */
mla_status_t mla_combine_sink(const void* workspace, size_t workspace_bytes, const int32_t* num_splits,
                              int num_units, int rows_per_unit, int num_sm_parts, int h_q, const float* sink,
                              void* out, float* lse, mla_stream_t stream);

/* Reads the device status word (blocks until `stream` reaches this point).
 * Returns MLA_OK, MLA_ERR_DEVICE_TIMEOUT or MLA_ERR_DEVICE_BOUNDS (timeout
 * wins when both are set) and stores the raw bits in *status_bits when
 * status_bits is not NULL. The word stays set until cleared. */
mla_status_t mla_query_device_status(const void* workspace, uint32_t* status_bits, mla_stream_t stream);

/* Zeroes the device status word (asynchronous on `stream`). */
mla_status_t mla_clear_device_status(void* workspace, mla_stream_t stream);

#ifdef __cplusplus
}
#endif
#endif /* MLA_B200_H_ */
