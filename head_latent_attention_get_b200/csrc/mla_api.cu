// Host side of the C ABI declared in include/mla.h: argument checks, TMA
// tensor maps, and the launches of the scheduler, decode and combine kernels.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstring>
#include <mutex>

#include "mla_kernels.cuh"

using namespace mla;

namespace {

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*,
                                  CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                  CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(f);
  });
  return fn;
}

// 2-D bf16 view [rows][cols] with the given row pitch, 128-B swizzled boxes.
bool make_map(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols, uint64_t pitch_bytes,
              uint32_t box_cols, uint32_t box_rows) {
  EncodeTiledFn enc = get_encode();
  if (!enc) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {pitch_bytes};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t es[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// The bf16 cache seen as [9 halves of 64 dims][rows][64 dims]: element
// (e, t, h) at byte 1152 t + 128 h + 2 e (the row stride is larger than the
// half stride; the driver accepts the order). A 64 x 64 x 2 box is the
// 128-value-dim V slot of one page in a single copy, landing as two 8 KB
// 128-B-swizzled halves, exactly the layout of two 64 x 64 boxes.
bool make_map_v(CUtensorMap* m, const void* base, uint64_t rows) {
  EncodeTiledFn enc = get_encode();
  if (!enc) return false;
  cuuint64_t dims[3] = {64, rows, (cuuint64_t)(kDqk / 64)};
  cuuint64_t strides[2] = {(cuuint64_t)kDqk * 2, 128};
  cuuint32_t box[3] = {64, 64, 2};
  cuuint32_t es[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// {units per request, rows per unit}; rows 0 when the sizes are out of range.
Geometry geometry_of(int s_q, int h_q, int h_kv, int topk) {
  Geometry g{0, 0};
  if (!unit_geometry(s_q, h_q, h_kv, topk, &g)) g = Geometry{0, 0};
  return g;
}

mla_status_t check_common(const mla_decode_args* a, int topk) {
  if (!a) return MLA_ERR_INVALID_ARG;
  if (!a->q || !a->kcache || !a->block_table || !a->cache_seqlens || !a->tile_md || !a->num_splits ||
      !a->out || !a->lse || !a->workspace)
    return MLA_ERR_INVALID_ARG;
  if (!aligned16(a->q) || !aligned16(a->kcache) || !aligned16(a->out) || !aligned16(a->workspace))
    return MLA_ERR_INVALID_ARG;
  if (a->batch <= 0 || a->s_q <= 0 || a->h_q <= 0 || a->h_kv <= 0 || a->num_pages <= 0 ||
      a->block_table_stride <= 0 || a->num_sm_parts <= 0)
    return MLA_ERR_INVALID_ARG;
  if (a->kv_format != MLA_KV_BF16 && a->kv_format != MLA_KV_FP8_E4M3 && a->kv_format != MLA_KV_NVFP4)
    return MLA_ERR_INVALID_ARG;
  const bool nvfp4 = a->kv_format == MLA_KV_NVFP4;
  if (a->d_qk != (nvfp4 ? kNvfp4D : kDqk) || a->d_v != kDv || a->page_size != kPage) return MLA_ERR_INVALID_ARG;
  if (nvfp4 && (!a->q_scale || !a->kv_scale || !aligned16(a->kv_scale))) return MLA_ERR_INVALID_ARG;
  if (nvfp4 && topk > 0) return MLA_ERR_UNSUPPORTED;
  if (!(a->softmax_scale > 0.f) || !std::isfinite(a->softmax_scale)) return MLA_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(a->sink) & 3u) != 0) return MLA_ERR_INVALID_ARG;
  if (a->h_kv != 1) return MLA_ERR_UNSUPPORTED;
  const Geometry g = geometry_of(a->s_q, a->h_q, a->h_kv, topk);
  const int rows = g.rows;
  if (rows <= 0 || rows > MLA_MAX_ROWS) return MLA_ERR_UNSUPPORTED;
  if ((long long)a->batch * g.units_per_req > 0x7fffffff) return MLA_ERR_UNSUPPORTED;
  const int U = a->batch * g.units_per_req;
  if (a->workspace_bytes < ws_layout(U, rows, a->num_sm_parts).total) return MLA_ERR_WORKSPACE_TOO_SMALL;
  if ((size_t)U * rows > (size_t)0x7fffffff / kDqk || (size_t)a->num_pages * kPage > 0x7fffffffu)
    return MLA_ERR_UNSUPPORTED;
  return MLA_OK;
}

mla_status_t run_decode(const mla_decode_args* a, const int32_t* indices, int topk, cudaStream_t stream) {
  const Geometry g = geometry_of(a->s_q, a->h_q, a->h_kv, topk);
  const int rows = g.rows;
  const int U = a->batch * g.units_per_req;
  const bool fp8 = a->kv_format == MLA_KV_FP8_E4M3;
  const int mode = a->kv_format == MLA_KV_NVFP4 ? kModeNvfp4
                   : topk > 0                  ? (fp8 ? kModeFp8Sparse : kModeSparse)
                                               : (fp8 ? kModeFp8 : kModeBf16);
  // Q rows of every unit (not NVFP4: its query is dequantised by the kernel),
  // and (bf16 paged cache only) the cache as [pages*64 tokens][576 dims];
  // boxes of 64 x 64 with 128-B swizzle. The FP8 and NVFP4 paged modes copy
  // whole pages with cp.async.bulk, the sparse modes gather rows with
  // cp.async: none of them needs a cache map.
  CUtensorMap tq, tkv, tv;
  std::memset(&tq, 0, sizeof(tq));
  std::memset(&tkv, 0, sizeof(tkv));
  std::memset(&tv, 0, sizeof(tv));
  if (mode != kModeNvfp4 && !make_map(&tq, a->q, (uint64_t)U * rows, kDqk, kDqk * 2, 64, 64)) return MLA_ERR_CUDA;
  const int row_groups = (rows + kRowsPerCta - 1) / kRowsPerCta;
  // more than 64 rows on the BF16 cache (paged or sparse): one CTA pair per
  // part shares each cache tile between the two row halves
  const bool pair = row_groups == 2 && (mode == kModeBf16 || mode == kModeSparse);
  if (mode == kModeBf16 &&
      (!make_map(&tkv, a->kcache, (uint64_t)a->num_pages * kPage, kDqk, kDqk * 2, 64, 64) ||
       !make_map_v(&tv, a->kcache, (uint64_t)a->num_pages * kPage)))
    return MLA_ERR_CUDA;
  const WsLayout w = ws_layout(U, rows, a->num_sm_parts);
  char* ws = static_cast<char*>(a->workspace);
  DecodeParams p;
  std::memset(&p, 0, sizeof(p));
  p.units = U;
  p.rows = rows;
  p.upr = g.units_per_req;
  p.h_q = a->h_q;
  p.s_q = a->s_q;
  p.causal = (topk == 0 && a->causal) ? 1 : 0;
  p.topk = topk;
  p.scale = a->softmax_scale;
  p.scale_log2 = a->softmax_scale * 1.4426950408889634f;
  p.num_pages = a->num_pages;
  p.bt_stride = a->block_table_stride;
  p.block_table = a->block_table;
  p.seqlens = a->cache_seqlens;
  p.indices = indices;
  p.kcache_fp8 = static_cast<const uint8_t*>(a->kcache);
  p.kcache = a->kcache;
  p.tile_md = a->tile_md;
  p.split_ptr = a->num_splits;
  p.out = a->out;
  p.lse = a->lse;
  p.ws_lse = reinterpret_cast<float*>(ws + w.lse_off);
  p.ws_o = reinterpret_cast<float*>(ws + w.o_off);
  p.status = reinterpret_cast<uint32_t*>(ws);
  p.timeout_ns = a->timeout_ns ? a->timeout_ns : 2000000000ull;
  p.debug_flags = a->debug_flags;
  p.sink = a->sink;
  p.q_nvfp4 = static_cast<const uint8_t*>(a->q);
  p.q_scale = static_cast<const uint8_t*>(a->q_scale);
  p.kv_scale = static_cast<const uint8_t*>(a->kv_scale);
  const int rows_per_cta = rows < kRowsPerCta ? rows : kRowsPerCta;
  const cudaError_t e =
      pair               ? launch_decode_pair(tq, tkv, tv, p, a->num_sm_parts, mode == kModeSparse, stream)
      : (mode == kModeFp8 || mode == kModeNvfp4)
          ? launch_decode_page(mode, rows_per_cta, tq, p, a->num_sm_parts, row_groups, stream)
                         : launch_decode(rows_per_cta, mode, tq, tkv, tv, p, a->num_sm_parts, row_groups, stream);
  if (e != cudaSuccess) return MLA_ERR_CUDA;
  if (a->debug_flags & MLA_DEBUG_SKIP_COMBINE) return MLA_OK;
  return launch_combine(a->workspace, U, rows, a->num_sm_parts, a->num_splits, a->h_q, a->sink, a->out, a->lse,
                        stream);
}

}  // namespace

extern "C" {

const char* mla_status_string(mla_status_t s) {
  switch (s) {
    case MLA_OK: return "MLA_OK";
    case MLA_ERR_INVALID_ARG: return "MLA_ERR_INVALID_ARG";
    case MLA_ERR_UNSUPPORTED: return "MLA_ERR_UNSUPPORTED";
    case MLA_ERR_WORKSPACE_TOO_SMALL: return "MLA_ERR_WORKSPACE_TOO_SMALL";
    case MLA_ERR_CUDA: return "MLA_ERR_CUDA";
    case MLA_ERR_DEVICE_TIMEOUT: return "MLA_ERR_DEVICE_TIMEOUT";
    case MLA_ERR_DEVICE_BOUNDS: return "MLA_ERR_DEVICE_BOUNDS";
  }
  return "MLA_ERR_UNKNOWN";
}

mla_status_t mla_get_num_sm_parts(int device, int s_q, int h_q, int h_kv, int topk, int* num_sm_parts) {
  if (!num_sm_parts || s_q <= 0 || h_q <= 0 || h_kv <= 0 || topk < 0) return MLA_ERR_INVALID_ARG;
  if (h_kv != 1) return MLA_ERR_UNSUPPORTED;
  const int rows = geometry_of(s_q, h_q, h_kv, topk).rows;
  if (rows <= 0 || rows > MLA_MAX_ROWS) return MLA_ERR_UNSUPPORTED;
  int sms = 0;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, device) != cudaSuccess || sms <= 0)
    return MLA_ERR_CUDA;
  const int groups = (rows + kRowsPerCta - 1) / kRowsPerCta;
  int parts = sms / groups > 0 ? sms / groups : 1;
  if (groups == 2) {  // two CTAs per part: no more parts than CTA pairs that fit at once
    int cur = 0;
    if (cudaGetDevice(&cur) != cudaSuccess) return MLA_ERR_CUDA;
    if (cur != device && cudaSetDevice(device) != cudaSuccess) return MLA_ERR_CUDA;
    const int fit = max_pair_clusters();
    if (cur != device) cudaSetDevice(cur);
    if (fit > 0 && fit < parts) parts = fit;
  }
  *num_sm_parts = parts;
  return MLA_OK;
}

mla_status_t mla_get_metadata(const int32_t* cache_seqlens, int batch, int s_q, int h_q, int h_kv, int topk,
                              int num_sm_parts, int32_t* tile_md, int32_t* num_splits, mla_stream_t stream) {
  if (!tile_md || !num_splits || batch <= 0 || s_q <= 0 || h_q <= 0 || h_kv <= 0 || num_sm_parts <= 0)
    return MLA_ERR_INVALID_ARG;
  if (topk < 0 || (topk > 0 && topk % 64 != 0)) return MLA_ERR_INVALID_ARG;
  if (topk == 0 && !cache_seqlens) return MLA_ERR_INVALID_ARG;
  if (h_kv != 1) return MLA_ERR_UNSUPPORTED;
  const Geometry g = geometry_of(s_q, h_q, h_kv, topk);
  if (g.rows <= 0 || (long long)batch * g.units_per_req > 0x7fffffff) return MLA_ERR_UNSUPPORTED;
  return launch_metadata(cache_seqlens, batch * g.units_per_req, g.units_per_req, topk, num_sm_parts, g.rows, tile_md,
                         num_splits, reinterpret_cast<cudaStream_t>(stream));
}

size_t mla_workspace_size(int batch, int s_q, int h_q, int h_kv, int topk, int num_sm_parts) {
  if (batch <= 0 || s_q <= 0 || h_q <= 0 || h_kv <= 0 || topk < 0 || num_sm_parts <= 0) return 0;
  const Geometry g = geometry_of(s_q, h_q, h_kv, topk);
  if (g.rows <= 0 || (long long)batch * g.units_per_req > 0x7fffffff) return 0;
  return ws_layout(batch * g.units_per_req, g.rows, num_sm_parts).total;
}

mla_status_t mla_decode_geometry(int s_q, int h_q, int h_kv, int topk, int* units_per_request,
                                 int* rows_per_unit) {
  if (!units_per_request || !rows_per_unit || s_q <= 0 || h_q <= 0 || h_kv <= 0 || topk < 0)
    return MLA_ERR_INVALID_ARG;
  if (h_kv != 1) return MLA_ERR_UNSUPPORTED;
  const Geometry g = geometry_of(s_q, h_q, h_kv, topk);
  if (g.rows <= 0 || g.rows > MLA_MAX_ROWS) return MLA_ERR_UNSUPPORTED;
  *units_per_request = g.units_per_req;
  *rows_per_unit = g.rows;
  return MLA_OK;
}

mla_status_t mla_decode_paged(const mla_decode_args* args, mla_stream_t stream) {
  mla_status_t st = check_common(args, 0);
  if (st != MLA_OK) return st;
  return run_decode(args, nullptr, 0, reinterpret_cast<cudaStream_t>(stream));
}

mla_status_t mla_decode_sparse(const mla_decode_args* args, const int32_t* indices, int topk,
                               mla_stream_t stream) {
  if (!indices || topk <= 0 || topk % 64 != 0) return MLA_ERR_INVALID_ARG;
  mla_status_t st = check_common(args, topk);
  if (st != MLA_OK) return st;
  return run_decode(args, indices, topk, reinterpret_cast<cudaStream_t>(stream));
}

mla_status_t mla_combine_sink(const void* workspace, size_t workspace_bytes, const int32_t* num_splits,
                              int num_units, int rows_per_unit, int num_sm_parts, int h_q, const float* sink,
                              void* out, float* lse, mla_stream_t stream) {
  if (!workspace || !num_splits || !out || !lse || num_units <= 0 || rows_per_unit <= 0 || num_sm_parts <= 0)
    return MLA_ERR_INVALID_ARG;
  if (!aligned16(out) || !aligned16(workspace)) return MLA_ERR_INVALID_ARG;
  if (sink && (h_q <= 0 || (reinterpret_cast<uintptr_t>(sink) & 3u) != 0))
    return MLA_ERR_INVALID_ARG;
  if ((long long)num_units * rows_per_unit > 0x7fffffffLL / kDqk) return MLA_ERR_UNSUPPORTED;
  if (workspace_bytes < ws_layout(num_units, rows_per_unit, num_sm_parts).total)
    return MLA_ERR_WORKSPACE_TOO_SMALL;
  return launch_combine(workspace, num_units, rows_per_unit, num_sm_parts, num_splits, sink ? h_q : 1, sink, out,
                        lse, reinterpret_cast<cudaStream_t>(stream));
}

mla_status_t mla_combine(const void* workspace, size_t workspace_bytes, const int32_t* num_splits, int num_units,
                         int rows_per_unit, int num_sm_parts, void* out, float* lse, mla_stream_t stream) {
  return mla_combine_sink(workspace, workspace_bytes, num_splits, num_units, rows_per_unit, num_sm_parts, 1,
                          nullptr, out, lse, stream);
}

mla_status_t mla_query_device_status(const void* workspace, uint32_t* status_bits, mla_stream_t stream) {
  if (!workspace) return MLA_ERR_INVALID_ARG;
  uint32_t bits = 0;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (cudaMemcpyAsync(&bits, workspace, sizeof(bits), cudaMemcpyDeviceToHost, s) != cudaSuccess)
    return MLA_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return MLA_ERR_CUDA;
  if (status_bits) *status_bits = bits;
  if (bits & MLA_DEVICE_STATUS_TIMEOUT) return MLA_ERR_DEVICE_TIMEOUT;
  if (bits & MLA_DEVICE_STATUS_BOUNDS) return MLA_ERR_DEVICE_BOUNDS;
  return MLA_OK;
}

mla_status_t mla_clear_device_status(void* workspace, mla_stream_t stream) {
  if (!workspace) return MLA_ERR_INVALID_ARG;
  return cudaMemsetAsync(workspace, 0, sizeof(uint32_t), reinterpret_cast<cudaStream_t>(stream)) == cudaSuccess
             ? MLA_OK
             : MLA_ERR_CUDA;
}

}  // extern "C"
