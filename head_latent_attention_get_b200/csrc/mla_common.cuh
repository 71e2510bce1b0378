// Constants and layouts shared by the host API and the kernels.
#pragma once
#include <cstddef>
#include <cstdint>

#include "../../include/mla.h"

namespace mla {

constexpr int kDqk = MLA_D_QK;          // 576 = 512 latent + 64 RoPE
constexpr int kDv = MLA_D_V;            // 512
constexpr int kPage = MLA_PAGE_SIZE;    // 64 tokens per page
constexpr int kTile = 128;              // tokens per scheduler block / kernel tile (2 pages)
constexpr int kRowsPerCta = 64;         // query rows handled by one CTA
constexpr int kSchedOverhead = 3;       // fixed cost of a piece, in tiles
constexpr int kFp8RecordBytes = 656;    // 512 e4m3 + 4 fp32 scales + 64 bf16
constexpr int kNvfp4D = 512;            // NVFP4 rows: 512 values, K and V
constexpr int kNvfp4RowBytes = 256;     // packed E2M1, two per byte
constexpr int kNvfp4ScaleBytes = 32;    // one UE4M3 per 16 values
constexpr size_t kWsHeaderBytes = 256;  // device status word lives at offset 0

__host__ __device__ inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Workspace layout (see mla_workspace_size in mla.h).
struct WsLayout {
  size_t lse_off, o_off, total;
  int max_splits;
};
__host__ __device__ inline WsLayout ws_layout(int units, int rows, int num_parts) {
  WsLayout w;
  w.max_splits = units + num_parts;
  w.lse_off = kWsHeaderBytes;
  w.o_off = align_up(w.lse_off + (size_t)w.max_splits * rows * sizeof(float), 256);
  w.total = align_up(w.o_off + (size_t)w.max_splits * rows * kDv * sizeof(float), 256);
  return w;
}

// Work-unit geometry. Sparse decoding has one unit per (request, query
// token) of h_q/h_kv rows (at most MLA_MAX_ROWS). Paged decoding cuts the
// R = s_q*h_q/h_kv query rows of a request into the fewest equal blocks of at
// most MLA_MAX_ROWS rows (the smallest count >= ceil(R/128) that divides R);
// each block is a unit, and the units of a request are consecutive, so unit u
// covers rows [u*rows, (u+1)*rows) of the flattened [batch*s_q*h_q] row axis
// and belongs to request u / units_per_req. Returns false for sizes out of
// range (R above 2^20 rows).
struct Geometry {
  int units_per_req, rows;
};
__host__ __device__ inline bool unit_geometry(int s_q, int h_q, int h_kv, int topk, Geometry* g) {
  if (s_q <= 0 || h_q <= 0 || h_kv <= 0 || (long long)s_q * h_q > (1 << 20)) return false;
  if (topk > 0) {
    g->units_per_req = s_q;
    g->rows = h_q / h_kv;
    return true;
  }
  const int R = s_q * h_q / h_kv;
  int n = (R + MLA_MAX_ROWS - 1) / MLA_MAX_ROWS;
  while (R % n != 0) ++n;
  g->units_per_req = n;
  g->rows = R / n;
  return true;
}

// Scheduler part descriptor, MLA_TILE_MD_INTS int32 per part.
struct PartMd {
  int32_t begin_unit, begin_tile, end_unit, end_tile, first_ws_idx, payload, pad0, pad1;
};
static_assert(sizeof(PartMd) == MLA_TILE_MD_INTS * 4, "tile_md entry size");

}  // namespace mla
