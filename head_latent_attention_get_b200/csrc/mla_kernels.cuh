// Kernel parameter block and launchers shared by the host API and the kernels.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>

#include "mla_common.cuh"

namespace mla {

// Cache format x key-set kind: BF16 paged, FP8 paged, BF16 token-sparse,
// FP8 token-sparse, NVFP4 paged (512-value rows, NVFP4 query).
enum KvMode : int { kModeBf16 = 0, kModeFp8 = 1, kModeSparse = 2, kModeFp8Sparse = 3, kModeNvfp4 = 4 };
__host__ __device__ constexpr bool mode_fp8(int mode) { return mode == kModeFp8 || mode == kModeFp8Sparse; }
__host__ __device__ constexpr bool mode_sparse(int mode) { return mode == kModeSparse || mode == kModeFp8Sparse; }

struct DecodeParams {
  int units, rows, h_q, s_q, causal, topk;  // rows = query rows per unit
  int upr;                                  // units per request (unit u -> request u / upr)
  float scale, scale_log2;                  // softmax scale, and scale * log2(e)
  int num_pages, bt_stride;
  const int32_t* block_table;
  const int32_t* seqlens;
  const int32_t* indices;                   // sparse mode
  const uint8_t* kcache_fp8;                // FP8 mode: token records
  const void* kcache;                       // cache base (L2 prefetch, sparse gather)
  const int32_t* tile_md;
  const int32_t* split_ptr;
  void* out;                                // bf16 [units*rows][512]
  float* lse;                               // [units*rows]
  float* ws_lse;                            // workspace partial LSE
  float* ws_o;                              // workspace partial O
  uint32_t* status;                         // device status word
  uint64_t timeout_ns;
  uint32_t debug_flags;
  const float* sink;                        // per-head sink logits [h_q], or null
  const uint8_t* q_nvfp4;                   // NVFP4 mode: packed E2M1 query rows [units*rows][256]
  const uint8_t* q_scale;                   // NVFP4 mode: UE4M3 query scales [units*rows][32]
  const uint8_t* kv_scale;                  // NVFP4 mode: UE4M3 cache scales [pages*64][32]
};

#ifdef __CUDACC__
// Attention sink ("[flashinfer] ...", section 2: an optional per-head sink,
// sinks [num_heads] float32): one more logit sigma per head that joins the
// softmax denominator with a zero value vector. Folded into a finished
// softmax with log-sum-exp `lse` (-inf for an empty key set):
//   L = ln(e^lse + e^sigma),  out *= e^(lse - L),  lse = L.
// Returns the factor on the output and replaces lse by L; written with
// max + log1p so that no exponential overflows.
__device__ __forceinline__ float fold_sink(float& lse, float sigma) {
  if (lse == -INFINITY) {
    lse = sigma;
    return 0.f;
  }
  const float L = fmaxf(lse, sigma) + log1pf(expf(-fabsf(lse - sigma)));
  const float f = expf(lse - L);
  lse = L;
  return f;
}
#endif

// Launch with programmatic stream serialization: the kernel may start while
// the previous kernel of the stream finishes (it calls griddep_wait before
// touching global memory), which hides the launch gap between the scheduler,
// decode and combine kernels of a step.
template <typename... Params, typename... Args>
cudaError_t launch_pdl(void (*kern)(Params...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                       Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, static_cast<Args&&>(args)...);
}

// tkv: the bf16 cache as [tokens][576] in 64 x 64 boxes; tv: the same bytes as
// [64-dim halves of the row][tokens][64 dims] in 2 x 64 x 64 boxes (a V slot
// of 128 value dims in one copy). Both unused by the FP8 / NVFP4 / sparse modes.
cudaError_t launch_decode(int rows_per_cta, int mode, const CUtensorMap& tq, const CUtensorMap& tkv,
                          const CUtensorMap& tv, const DecodeParams& p, int parts, int row_groups,
                          cudaStream_t stream);
// FP8 or NVFP4 paged cache (mode kModeFp8 / kModeNvfp4): each page fetched by
// bulk copies and converted once (no cache tensor map; NVFP4 needs no tq).
cudaError_t launch_decode_page(int mode, int rows_per_cta, const CUtensorMap& tq, const DecodeParams& p, int parts,
                               int row_groups, cudaStream_t stream);
// Units of more than 64 rows, BF16 cache (paged, or token-sparse when `sparse`):
// CTA pairs (clusters of two), one per part.
cudaError_t launch_decode_pair(const CUtensorMap& tq, const CUtensorMap& tkv, const CUtensorMap& tv,
                               const DecodeParams& p, int parts, bool sparse, cudaStream_t stream);
// How many CTA pairs of the pair kernel can be resident at once on the current device (0 if unknown).
int max_pair_clusters();
// Unit u reads seqlens[u / upr] (paged decoding; upr = units per request);
// rows = query rows per unit.
mla_status_t launch_metadata(const int32_t* seqlens, int U, int upr, int topk, int parts, int rows,
                             int32_t* tile_md, int32_t* num_splits, cudaStream_t stream);
// `sink` (device fp32 [h_q] or null): the head of row r of a unit is r % h_q.
mla_status_t launch_combine(const void* workspace, int units, int rows, int parts, const int32_t* split_ptr,
                            int h_q, const float* sink, void* out, float* lse, cudaStream_t stream);

}  // namespace mla
