// Device helpers shared by the decode kernels: walking a scheduler part's
// pieces, page-table and sparse-index lookups, key validity, FP8 conversion
// and 128-byte-swizzle addressing.
#pragma once
#include <cuda_bf16.h>
#include <cuda_fp4.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>

#include "mla_kernels.cuh"
#include "sm100_ptx.cuh"

namespace mla {

struct Piece {
  int unit, t0, t1, ws_idx, single;
};

// Walks the pieces of one scheduler part in order; returns false when done.
struct PieceIter {
  PartMd md;
  int u, t, first;
  const DecodeParams* p;
  __device__ void init(const DecodeParams& prm, int part) {
    p = &prm;
    md = *reinterpret_cast<const PartMd*>(prm.tile_md + part * MLA_TILE_MD_INTS);
    u = md.begin_unit;
    t = md.begin_tile;
    first = 1;
  }
  __device__ int tiles_of(int unit) const {
    if (p->topk > 0) return (p->topk + kTile - 1) / kTile;
    int L = p->seqlens[unit / p->upr];
    return L > 0 ? (L + kTile - 1) / kTile : 0;
  }
  __device__ bool next(Piece& pc) {
    while (u < p->units && (u < md.end_unit || (u == md.end_unit && t < md.end_tile))) {
      const int n = tiles_of(u);
      const int tend = (u == md.end_unit) ? min(md.end_tile, n) : n;
      if (t < tend) {
        pc.unit = u;
        pc.t0 = t;
        pc.t1 = tend;
        const int s0 = p->split_ptr[u];
        pc.single = (p->split_ptr[u + 1] - s0) == 1;
        pc.ws_idx = first ? md.first_ws_idx : s0;
        first = 0;
        u += 1;
        t = 0;
        return true;
      }
      first = 0;
      u += 1;
      t = 0;
    }
    return false;
  }
};

// Before a TMA producer exits (normally or after an abort) it waits, with a
// bound, for the copies it issued into its last `nslots` ring slots, so no TMA
// write can land in shared memory after the CTA has finished.
__device__ __forceinline__ void drain_issued(uint64_t* full, int nslots, int issued, uint64_t timeout_ns) {
  for (int i = issued > nslots ? issued - nslots : 0; i < issued; ++i)
    mbar_wait(&full[i % nslots], (uint32_t)((i / nslots) & 1), timeout_ns);
}

// Physical page of logical page j of a request (dense); -1 when j is past the
// request's pages. Out-of-range ids are reported and replaced by page 0.
__device__ __forceinline__ int page_of(const DecodeParams& p, int req, int j, int npages_req) {
  if (j >= npages_req) return -1;
  if (j >= p.bt_stride) {
    atomicOr(p.status, (uint32_t)MLA_DEVICE_STATUS_BOUNDS);
    return 0;
  }
  int pg = p.block_table[(size_t)req * p.bt_stride + j];
  if (pg < 0 || pg >= p.num_pages) {
    atomicOr(p.status, (uint32_t)MLA_DEVICE_STATUS_BOUNDS);
    return 0;
  }
  return pg;
}

// Sparse slot -> physical cache row, or -1 if the slot is ignored.
__device__ __forceinline__ int sparse_row(const DecodeParams& p, int unit, int slot, bool report) {
  if (slot >= p.topk) return -1;
  const int b = unit / p.s_q;
  const int idx = p.indices[(size_t)unit * p.topk + slot];
  const int L = p.seqlens[b];
  if (idx < 0 || idx >= L) {
    if (report && idx != -1) atomicOr(p.status, (uint32_t)MLA_DEVICE_STATUS_BOUNDS);
    return -1;
  }
  const int j = idx / kPage;
  if (j >= p.bt_stride) {
    if (report) atomicOr(p.status, (uint32_t)MLA_DEVICE_STATUS_BOUNDS);
    return -1;
  }
  const int pg = p.block_table[(size_t)b * p.bt_stride + j];
  if (pg < 0 || pg >= p.num_pages) {
    if (report) atomicOr(p.status, (uint32_t)MLA_DEVICE_STATUS_BOUNDS);
    return -1;
  }
  return pg * kPage + (idx % kPage);
}

__device__ __forceinline__ int unit_req(const DecodeParams& p, int unit) { return unit / p.upr; }

// Query token index (0..s_q-1) of row r of a unit: rows are laid out
// [request][query token][head] on one flattened axis.
__device__ __forceinline__ int row_query(const DecodeParams& p, int unit, int r) {
  return ((unit * p.rows + r) / p.h_q) % p.s_q;
}

// Head of row r of a unit (the index into the per-head sink).
__device__ __forceinline__ int row_head(const DecodeParams& p, int unit, int r) {
  return (unit * p.rows + r) % p.h_q;
}

// Number of valid keys of tile k for a row limit (dense): tokens [128k, 128k+128).
__device__ __forceinline__ int dense_tile_valid(int limit, int k) {
  return max(0, min(kTile, limit - k * kTile));
}

// fp8 e4m3 x16 + fp32 scale -> 16 bf16 (two 16-byte chunks), x = bf16(f32(e4m3) * s)
__device__ __forceinline__ void dequant16(const uint4 raw, float s, uint4& lo, uint4& hi) {
  const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
  uint32_t o[8];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const __nv_fp8x2_storage_t pair = (__nv_fp8x2_storage_t)((w[i] >> (16 * h)) & 0xFFFFu);
      const __half2_raw hr = __nv_cvt_fp8x2_to_halfraw2(pair, __NV_E4M3);
      const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&hr));
      o[2 * i + h] = pack_bf16x2(f.x * s, f.y * s);
    }
  }
  lo = make_uint4(o[0], o[1], o[2], o[3]);
  hi = make_uint4(o[4], o[5], o[6], o[7]);
}

// NVFP4: 8 bytes of packed E2M1 (16 values, element 2i in the low nibble of
// byte i) and their UE4M3 scale -> 16 bf16 (two 16-byte chunks). Every
// E2M1 x UE4M3 product is exact in f16 and in bf16, so the f16 product and
// the conversions lose nothing.
__device__ __forceinline__ void dequant_nvfp4_16(const uint2 raw, uint32_t scale_byte, uint4& lo, uint4& hi) {
  const __half_raw sr = __nv_cvt_fp8_to_halfraw((__nv_fp8_storage_t)(scale_byte & 0x7Fu), __NV_E4M3);
  const __half2 s2 = __half2half2(*reinterpret_cast<const __half*>(&sr));
  const uint32_t w[2] = {raw.x, raw.y};
  uint32_t o[8];
#pragma unroll
  for (int i = 0; i < 2; ++i) {
#pragma unroll
    for (int b = 0; b < 4; ++b) {
      const __half2_raw hr = __nv_cvt_fp4x2_to_halfraw2((__nv_fp4x2_storage_t)((w[i] >> (8 * b)) & 0xFFu), __NV_E2M1);
      const float2 f = __half22float2(__hmul2(*reinterpret_cast<const __half2*>(&hr), s2));
      o[4 * i + b] = pack_bf16x2(f.x, f.y);
    }
  }
  lo = make_uint4(o[0], o[1], o[2], o[3]);
  hi = make_uint4(o[4], o[5], o[6], o[7]);
}

// Address of 16-byte chunk c (0..7) of 128-B row `row` of a 128-B-swizzled tile.
__device__ __forceinline__ uint8_t* sw128(uint8_t* tile, int row, int c) {
  return tile + row * 128 + ((c ^ (row & 7)) << 4);
}

__device__ __forceinline__ float pick4(const float4 v, int i) {
  return i == 0 ? v.x : i == 1 ? v.y : i == 2 ? v.z : v.w;
}
__device__ __forceinline__ uint32_t pick4u(const uint4 v, int i) {
  return i == 0 ? v.x : i == 1 ? v.y : i == 2 ? v.z : v.w;
}

}  // namespace mla
