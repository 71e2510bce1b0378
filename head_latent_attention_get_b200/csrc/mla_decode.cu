// MLA decode kernel for sm_100a (tcgen05 + TMEM + TMA).
//
// Computes, per work unit (request, or (request, query token) when sparse),
// softmax(scale * Q K^T) V over the unit's keys, with K = whole 576-dim latent
// row and V = its first 512 dims ("[flashinfer] ... NVFP4 DeepSeek-V4
// decoding", README section: one latent row per token is both K and V;
// FlashMLA-ETAP summary, core mechanism: S = QK^T, P = softmax(S), O = PV).
//
// One CTA = one scheduler part x one group of <= 64 query rows. Per tile of
// 128 tokens (two 64-token pages):
//   S   = Q K^T  tcgen05 M=64 (query rows) x N=128 (tokens) x K=576, both
//                operands K-major in 128-B-swizzled smem; fp32 in TMEM.
//   softmax      one thread per query row reads its 128 scores from TMEM;
//                online max / sum in fp32 with lazily rescaled O.
//   O^T += V^T P^T  tcgen05 M=128 (4 chunks of the 512 value dims) x N=rows x
//                K=128 tokens; V^T is the MN-major view of the token-major V
//                tile, P^T (bf16) is written K-major by the row threads.
// The O accumulator is transposed (value dims on TMEM lanes) so 64 rows x 512
// dims fit in 256 TMEM columns next to two S buffers (2 x 128 columns).
// K slices and V chunks stream through separate smem rings (V is read again
// from L2 for the PV product) so the ring stays several slots deep.
//
// Warp roles (256 threads; 384 with the FP8 cache):
//   0 K producer (Q + K slices via TMA)     1 S issuer (+ TMEM alloc)
//   2 O issuer                              3 V producer (V chunks via TMA)
//   4-7 softmax + epilogue (row r = 16*(warp-4) + lane, lanes 0-15)
//   8-9 FP8 dequant of K slices 0-7         10-11 FP8 dequant of V chunks
// Every mbarrier wait is bounded; on timeout the CTA records
// MLA_DEVICE_STATUS_TIMEOUT, stops issuing work and exits normally.
#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>

#include "mla_kernels.cuh"
#include "sm100_ptx.cuh"

namespace mla {

constexpr int kNK = 3;                 // K ring slots (16 KB: 128 tokens x 64 dims)
constexpr int kNV = 2;                 // V ring slots (32 KB: 128 tokens x 128 dims)
constexpr int kQBytes = 9 * 8192;      // 64 rows x 576 dims
constexpr int kKSlot = 16384;
constexpr int kVSlot = 32768;
constexpr int kTmemCols = 512;
constexpr int kTmemS = 256;            // S buffers at columns 256 and 384
constexpr float kRescaleLog2 = 8.0f;   // rescale O only when the max grows by > 2^8

template <int NR>
struct Smem {
  static constexpr int q = 0;
  static constexpr int k = q + kQBytes;
  static constexpr int v = k + kNK * kKSlot;
  static constexpr int pt = v + kNV * kVSlot;
  static constexpr int pt_bytes = NR * 256;  // [NR rows][128 tokens] bf16
  static constexpr int ctrl = pt + 2 * pt_bytes;
  static constexpr int total = ctrl + 1024;
};

struct Ctrl {
  uint64_t q_full, q_empty;
  uint64_t k_full[kNK], k_empty[kNK];
  uint64_t v_full[kNV], v_empty[kNV];
  uint64_t s_full[2], s_empty[2], p_full[2], o_done[2], o_free, drain_s, drain_o;
  uint64_t grp_sm, grp_k, grp_v;   // bounded group barriers (softmax 128, dequant 64 + 64)
  uint32_t tmem_base;
  int abort_flag;
  int rescale_flag[2];
  float alpha[64];
  float inv_l[64];
};
static_assert(sizeof(Ctrl) <= 1024, "control block");

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
    int L = p->seqlens[unit];
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

__device__ __forceinline__ bool timed_wait(Ctrl* c, uint64_t* bar, uint32_t parity, const DecodeParams& p) {
  if (*(volatile int*)&c->abort_flag) return false;
  if (mbar_wait(bar, parity, p.timeout_ns)) return true;
  atomicOr(p.status, (uint32_t)MLA_DEVICE_STATUS_TIMEOUT);
  *(volatile int*)&c->abort_flag = 1;
  return false;
}

// Barrier among the threads of one warp group, built on an mbarrier so the
// wait is bounded (a named barrier would hang if a member gave up).
__device__ __forceinline__ bool group_sync(Ctrl* c, uint64_t* bar, uint32_t& phase, const DecodeParams& p) {
  mbar_arrive(bar);
  const bool ok = timed_wait(c, bar, phase & 1, p);
  ++phase;
  return ok;
}

// Before a producer exits (normally or after an abort) it waits, with a bound,
// for the copies it issued into its last `nslots` ring slots, so no TMA write
// can land in shared memory after the CTA has finished.
__device__ __forceinline__ void drain_issued(uint64_t* full, int nslots, int issued, uint64_t timeout_ns) {
  for (int i = issued > nslots ? issued - nslots : 0; i < issued; ++i)
    mbar_wait(&full[i % nslots], (uint32_t)((i / nslots) & 1), timeout_ns);
}

// Physical page of logical page j of unit u (dense); -1 when j is past the
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

__device__ __forceinline__ int unit_req(const DecodeParams& p, int unit) {
  return p.topk > 0 ? unit / p.s_q : unit;
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

// Store 16 bytes at chunk c (0..7) of 128-B row `row` of a 128-B-swizzled tile.
__device__ __forceinline__ void st_sw128(uint8_t* tile, int row, int c, uint4 v) {
  *reinterpret_cast<uint4*>(tile + row * 128 + ((c ^ (row & 7)) << 4)) = v;
}

template <int NR, int MODE>
__global__ void __launch_bounds__(MODE == kModeFp8 ? 384 : 256, 1)
    mla_decode_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_kv,
                      const __grid_constant__ CUtensorMap tm_aux, const DecodeParams p) {
  using L = Smem<NR>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem + L::q;
  uint8_t* sK = smem + L::k;
  uint8_t* sV = smem + L::v;
  uint8_t* sP = smem + L::pt;
  Ctrl* c = reinterpret_cast<Ctrl*>(smem + L::ctrl);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int part = blockIdx.x, rg = blockIdx.y;
  const int row0 = rg * kRowsPerCta;                    // first row of this CTA within a unit
  const int rows_here = min(kRowsPerCta, p.rows - row0);

  if (threadIdx.x == 0) {
    mbar_init(&c->q_full, 1);
    mbar_init(&c->q_empty, 1);
    for (int i = 0; i < kNK; ++i) { mbar_init(&c->k_full[i], 1); mbar_init(&c->k_empty[i], 1); }
    for (int i = 0; i < kNV; ++i) { mbar_init(&c->v_full[i], 1); mbar_init(&c->v_empty[i], 1); }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&c->s_full[i], 1);
      mbar_init(&c->s_empty[i], 128);
      mbar_init(&c->p_full[i], 128);
      mbar_init(&c->o_done[i], 1);
    }
    mbar_init(&c->o_free, 128);
    mbar_init(&c->drain_s, 1);
    mbar_init(&c->drain_o, 1);
    mbar_init(&c->grp_sm, 128);
    mbar_init(&c->grp_k, 64);
    mbar_init(&c->grp_v, 64);
    c->abort_flag = 0;
    c->rescale_flag[0] = 0;
    c->rescale_flag[1] = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tm_q);
    if (MODE == kModeBf16) tma_prefetch_desc(&tm_kv);  // the other map is left unencoded
    else tma_prefetch_desc(&tm_aux);
  }
  if (warp == 1) {
    tmem_alloc(&c->tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = c->tmem_base;

  PieceIter it;
  it.init(p, part);
  Piece pc;

  if (warp == 0) {
    // ------------------------------------------------------------ K producer
    int kc = 0, pi = 0, q_issued = 0;
    bool stop = false;
    while (!stop && it.next(pc)) {
      if (lane == 0) {
        if (!timed_wait(c, &c->q_empty, (pi & 1) ^ 1, p)) {
          stop = true;
        } else {
          mbar_arrive_expect_tx(&c->q_full, kQBytes);
          const int qy = pc.unit * p.rows + row0;
          for (int j = 0; j < 9; ++j) tma_load_2d(sQ + j * 8192, &tm_q, &c->q_full, 64 * j, qy);
          ++q_issued;
        }
      }
      stop = __shfl_sync(0xffffffffu, stop ? 1 : 0, 0) != 0;
      if (stop) break;
      const int req = unit_req(p, pc.unit);
      const int npg = (MODE == kModeSparse) ? 0 : (p.seqlens[req] + kPage - 1) / kPage;
      for (int k = pc.t0; k < pc.t1 && !stop; ++k) {
        int pa = 0, pb = 0;
        if (MODE != kModeSparse && lane == 0) {
          pa = page_of(p, req, 2 * k, npg);
          pb = page_of(p, req, 2 * k + 1, npg);
          if (pb < 0) pb = pa;      // half tile: reload page A, its keys are masked
        }
        // sparse: lane l gathers slots 4l..4l+3 of this tile (ignored slots load
        // row 0; their scores are masked and their value rows zeroed later)
        int r4[4] = {0, 0, 0, 0};
        if (MODE == kModeSparse) {
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const int rr = sparse_row(p, pc.unit, k * kTile + 4 * lane + q, true);
            r4[q] = rr < 0 ? 0 : rr;
          }
        }
        if (MODE == kModeFp8) continue;  // the dequant group is the only producer of K slots
        for (int j = 0; j < 9; ++j, ++kc) {
          const int slot = kc % kNK;
          uint8_t* dst = sK + slot * kKSlot;
          if (lane == 0) {
            if (!timed_wait(c, &c->k_empty[slot], ((kc / kNK) & 1) ^ 1, p)) { stop = true; }
            else if (MODE == kModeSparse) mbar_arrive_expect_tx(&c->k_full[slot], kKSlot);
          }
          stop = __shfl_sync(0xffffffffu, stop ? 1 : 0, 0) != 0;
          if (stop) break;
          if (MODE == kModeSparse) {
            __syncwarp();
            tma_gather4(dst + lane * 512, &tm_aux, &c->k_full[slot], 64 * j, r4[0], r4[1], r4[2], r4[3]);
          } else if (lane == 0) {
            mbar_arrive_expect_tx(&c->k_full[slot], kKSlot);
            tma_load_2d(dst, &tm_kv, &c->k_full[slot], 64 * j, pa * kPage);
            tma_load_2d(dst + 8192, &tm_kv, &c->k_full[slot], 64 * j, pb * kPage);
          }
          __syncwarp();
        }
      }
      ++pi;
    }
    if (lane == 0) {
      if (q_issued > 0) mbar_wait(&c->q_full, (uint32_t)((q_issued - 1) & 1), p.timeout_ns);
      if (MODE != kModeFp8) drain_issued(c->k_full, kNK, kc, p.timeout_ns);
    }
    __syncwarp();
  } else if (warp == 3 && MODE != kModeFp8) {
    // ------------------------------------------------------------ V producer
    int vc = 0;
    bool stop = false;
    while (!stop && it.next(pc)) {
      const int req = unit_req(p, pc.unit);
      const int npg = (MODE == kModeSparse) ? 0 : (p.seqlens[req] + kPage - 1) / kPage;
      for (int k = pc.t0; k < pc.t1 && !stop; ++k) {
        int pa = 0, pb = 0;
        if (MODE != kModeSparse && lane == 0) {
          pa = page_of(p, req, 2 * k, npg);
          pb = page_of(p, req, 2 * k + 1, npg);
          if (pb < 0) pb = pa;
        }
        int r4[4];
        if (MODE == kModeSparse) {
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const int rr = sparse_row(p, pc.unit, k * kTile + 4 * lane + q, false);
            r4[q] = rr < 0 ? 0 : rr;
          }
        }
        for (int m = 0; m < 4; ++m, ++vc) {
          const int slot = vc % kNV;
          uint8_t* dst = sV + slot * kVSlot;
          if (lane == 0) {
            if (!timed_wait(c, &c->v_empty[slot], ((vc / kNV) & 1) ^ 1, p)) stop = true;
            else mbar_arrive_expect_tx(&c->v_full[slot], kVSlot);
          }
          stop = __shfl_sync(0xffffffffu, stop ? 1 : 0, 0) != 0;
          if (stop) break;
          __syncwarp();
          if (MODE == kModeSparse) {
            tma_gather4(dst + lane * 512, &tm_aux, &c->v_full[slot], 128 * m, r4[0], r4[1], r4[2], r4[3]);
            tma_gather4(dst + 16384 + lane * 512, &tm_aux, &c->v_full[slot], 128 * m + 64, r4[0], r4[1],
                        r4[2], r4[3]);
          } else if (lane == 0) {
            tma_load_2d(dst, &tm_kv, &c->v_full[slot], 128 * m, pa * kPage);
            tma_load_2d(dst + 8192, &tm_kv, &c->v_full[slot], 128 * m, pb * kPage);
            tma_load_2d(dst + 16384, &tm_kv, &c->v_full[slot], 128 * m + 64, pa * kPage);
            tma_load_2d(dst + 24576, &tm_kv, &c->v_full[slot], 128 * m + 64, pb * kPage);
          }
          __syncwarp();
        }
      }
    }
    if (lane == 0) drain_issued(c->v_full, kNV, vc, p.timeout_ns);
    __syncwarp();
  } else if (MODE == kModeFp8 && warp >= 8) {
    // ------------------------------------------------------------ FP8 dequant
    const bool kgroup = warp < 10;
    const int gt = threadIdx.x - (kgroup ? 256 : 320);  // 0..63 within the group
    uint64_t* grp = kgroup ? &c->grp_k : &c->grp_v;
    uint32_t gph = 0;
    int kc = 0, vc = 0;
    bool stop = false;
    while (!stop && it.next(pc)) {
      const int req = pc.unit;
      const int npg = (p.seqlens[req] + kPage - 1) / kPage;
      for (int k = pc.t0; k < pc.t1 && !stop; ++k) {
        // this thread converts tokens gt and gt + 64 of the tile
        const uint8_t* rec[2];
        int pgs[2];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          int pg = page_of(p, req, 2 * k + h, npg);
          if (pg < 0) pg = page_of(p, req, 2 * k, npg);
          pgs[h] = pg;
          rec[h] = p.kcache_fp8 + ((size_t)pg * kPage + gt) * kFp8RecordBytes;
        }
        if (kgroup) {
          // this group is the only producer of the K ring (one producer keeps every
          // empty-barrier wait at most one phase behind)
          for (int j = 0; j < 9; ++j, ++kc) {
            const int slot = kc % kNK;
            uint8_t* dst = sK + slot * kKSlot;
            if (j == 8) {  // RoPE slice straight from the records (bytes 528..655) by TMA
              if (gt == 0) {
                if (!timed_wait(c, &c->k_empty[slot], ((kc / kNK) & 1) ^ 1, p)) {
                  stop = true;
                } else {
                  mbar_arrive_expect_tx(&c->k_full[slot], kKSlot);
                  tma_load_2d(dst, &tm_aux, &c->k_full[slot], 264, pgs[0] * kPage);
                  tma_load_2d(dst + 8192, &tm_aux, &c->k_full[slot], 264, pgs[1] * kPage);
                }
              }
              continue;
            }
            if (gt == 0 && !timed_wait(c, &c->k_empty[slot], ((kc / kNK) & 1) ^ 1, p)) stop = true;
            if (!group_sync(c, grp, gph, p) || *(volatile int*)&c->abort_flag) { stop = true; break; }
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              const float s = reinterpret_cast<const float*>(rec[h] + 512)[j >> 1];
              const uint4* src = reinterpret_cast<const uint4*>(rec[h] + 64 * j);
#pragma unroll
              for (int q = 0; q < 4; ++q) {
                uint4 lo, hi;
                dequant16(__ldg(src + q), s, lo, hi);
                st_sw128(dst, gt + 64 * h, 2 * q, lo);
                st_sw128(dst, gt + 64 * h, 2 * q + 1, hi);
              }
            }
            fence_proxy_async_smem();
            if (!group_sync(c, grp, gph, p)) { stop = true; break; }
            if (gt == 0) mbar_arrive(&c->k_full[slot]);
          }
        } else {
          for (int m = 0; m < 4; ++m, ++vc) {
            const int slot = vc % kNV;
            uint8_t* dst = sV + slot * kVSlot;
            if (gt == 0 && !timed_wait(c, &c->v_empty[slot], ((vc / kNV) & 1) ^ 1, p)) stop = true;
            if (!group_sync(c, grp, gph, p) || *(volatile int*)&c->abort_flag) { stop = true; break; }
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              const float s = reinterpret_cast<const float*>(rec[h] + 512)[m];
              const uint4* src = reinterpret_cast<const uint4*>(rec[h] + 128 * m);
#pragma unroll
              for (int q = 0; q < 8; ++q) {
                uint4 lo, hi;
                dequant16(__ldg(src + q), s, lo, hi);
                uint8_t* half = dst + (q >> 2) * 16384;   // dims 0-63 / 64-127 of the chunk
                st_sw128(half, gt + 64 * h, 2 * (q & 3), lo);
                st_sw128(half, gt + 64 * h, 2 * (q & 3) + 1, hi);
              }
            }
            fence_proxy_async_smem();
            if (!group_sync(c, grp, gph, p)) { stop = true; break; }
            if (gt == 0) mbar_arrive(&c->v_full[slot]);
          }
        }
      }
    }
    if (kgroup && gt == 0) drain_issued(c->k_full, kNK, kc, p.timeout_ns);
  } else if (warp == 1) {
    // ------------------------------------------------------------ S issuer
    const uint32_t idesc = idesc_bf16(64, 128, false, false);
    int kc = 0, gt = 0, pi = 0;
    bool stop = false;
    while (!stop && it.next(pc)) {
      if (lane == 0 && !timed_wait(c, &c->q_full, pi & 1, p)) stop = true;
      for (int k = pc.t0; k < pc.t1 && !stop; ++k, ++gt) {
        const int b = gt & 1;
        if (lane == 0) {
          if (!timed_wait(c, &c->s_empty[b], ((gt >> 1) & 1) ^ 1, p)) { stop = true; }
          tc_fence_after();
          const uint32_t d = tmem + kTmemS + 128 * b;
          for (int j = 0; j < 9 && !stop; ++j, ++kc) {
            const int slot = kc % kNK;
            if (!timed_wait(c, &c->k_full[slot], (kc / kNK) & 1, p)) { stop = true; break; }
            tc_fence_after();
            const uint32_t qa = smem_u32(sQ + j * 8192), kb = smem_u32(sK + slot * kKSlot);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              mma_bf16_ss(d, sdesc(qa + kk * 32, 16, 1024), sdesc(kb + kk * 32, 16, 1024), idesc,
                          (j | kk) != 0 ? 1u : 0u);
            mma_commit(&c->k_empty[slot]);
          }
          if (!stop && !(gt == 0 && (p.debug_flags & MLA_DEBUG_WITHHOLD_SCORES))) mma_commit(&c->s_full[b]);
        }
        stop = __shfl_sync(0xffffffffu, stop ? 1 : 0, 0) != 0;
      }
      if (lane == 0 && !stop) mma_commit(&c->q_empty);
      ++pi;
    }
    if (lane == 0) {  // drain every MMA this thread issued before TMEM is released
      mma_commit(&c->drain_s);
      mbar_wait(&c->drain_s, 0, p.timeout_ns);
    }
  } else if (warp == 2) {
    // ------------------------------------------------------------ O issuer
    const uint32_t idesc = idesc_bf16(128, NR, true, false);
    int vc = 0, gt = 0, pi = 0;
    bool stop = false;
    while (!stop && it.next(pc)) {
      const int req = unit_req(p, pc.unit);
      for (int k = pc.t0; k < pc.t1 && !stop; ++k, ++gt) {
        const int b = gt & 1;
        const bool first = (k == pc.t0);
        if (lane == 0) {
          if (first && pi > 0 && !timed_wait(c, &c->o_free, (pi - 1) & 1, p)) stop = true;
          if (!stop && !timed_wait(c, &c->p_full[b], (gt >> 1) & 1, p)) stop = true;
        }
        stop = __shfl_sync(0xffffffffu, stop ? 1 : 0, 0) != 0;
        if (stop) break;
        // keys of this tile whose value rows must read as zero
        int nvalid = kTile;
        uint32_t bad = 0;  // sparse: bit i of lane l -> slot 4l + i ignored
        if (MODE == kModeSparse) {
#pragma unroll
          for (int q = 0; q < 4; ++q)
            if (sparse_row(p, pc.unit, k * kTile + 4 * lane + q, false) < 0) bad |= 1u << q;
        } else {
          nvalid = dense_tile_valid(p.seqlens[req], k);
        }
        const uint32_t pt = smem_u32(sP + b * L::pt_bytes);
        for (int m = 0; m < 4 && !stop; ++m, ++vc) {
          const int slot = vc % kNV;
          uint8_t* vs = sV + slot * kVSlot;
          if (lane == 0 && !timed_wait(c, &c->v_full[slot], (vc / kNV) & 1, p)) stop = true;
          stop = __shfl_sync(0xffffffffu, stop ? 1 : 0, 0) != 0;
          if (stop) break;
          if (MODE == kModeSparse ? __any_sync(0xffffffffu, bad != 0) : nvalid < kTile) {
            const uint4 z = make_uint4(0, 0, 0, 0);
            if (MODE == kModeSparse) {
              for (int q = 0; q < 4; ++q)
                if (bad & (1u << q))
                  for (int h = 0; h < 2; ++h)
                    for (int ch = 0; ch < 8; ++ch)
                      *reinterpret_cast<uint4*>(vs + h * 16384 + (4 * lane + q) * 128 + ch * 16) = z;
            } else {
              for (int i = nvalid * 16 + lane; i < kTile * 16; i += 32) {  // 16 chunks per token row
                const int tok = i >> 4, ch = i & 15;
                *reinterpret_cast<uint4*>(vs + (ch >> 3) * 16384 + tok * 128 + (ch & 7) * 16) = z;
              }
            }
            fence_proxy_async_smem();
            __syncwarp();
          }
          if (lane == 0) {
            tc_fence_after();
            const uint32_t va = smem_u32(vs);
            const uint32_t d = tmem + 64 * m;
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
              mma_bf16_ss(d, sdesc(va + kk * 2048, 16384, 1024),
                          sdesc(pt + (kk >> 2) * (NR * 128) + (kk & 3) * 32, 16, 1024), idesc,
                          (first && kk == 0) ? 0u : 1u);
            mma_commit(&c->v_empty[slot]);
          }
          __syncwarp();
        }
        if (lane == 0 && !stop) mma_commit(&c->o_done[b]);
      }
      ++pi;
    }
    if (lane == 0) {
      mma_commit(&c->drain_o);
      mbar_wait(&c->drain_o, 0, p.timeout_ns);
    }
  } else if (warp >= 4 && warp < 8) {
    // ------------------------------------------------------------ softmax + epilogue
    const int q4 = warp - 4;
    const int r = 16 * q4 + lane;                        // query row of this CTA (lanes 0-15)
    const bool owner = lane < 16;
    const bool rvalid = owner && r < rows_here;
    const uint32_t lane_base = (uint32_t)(32 * q4) << 16;
    const float thresh = kRescaleLog2 / p.scale_log2;    // raw-score units
    uint32_t gph = 0;
    int gt = 0;
    bool stop = false;
    while (!stop && it.next(pc)) {
      const int req = unit_req(p, pc.unit);
      const int grow = row0 + r;                          // row within the unit
      int limit = 0;
      if (MODE != kModeSparse) {
        const int Ls = p.seqlens[req];
        limit = Ls;
        if (p.causal) limit = Ls - p.s_q + grow / p.h_q + 1;
      }
      float m_used = -INFINITY, l_sum = 0.f;
      int last_b = 0, last_gt = -1;
      for (int k = pc.t0; k < pc.t1 && !stop; ++k, ++gt) {
        const int b = gt & 1;
        if (!timed_wait(c, &c->s_full[b], (gt >> 1) & 1, p)) { stop = true; break; }
        tc_fence_after();
        const uint32_t s_addr = tmem + lane_base + kTmemS + 128 * b;
        // validity of the 128 keys of this tile for this row
        uint32_t vmask[4];
        if (MODE == kModeSparse) {
#pragma unroll
          for (int w = 0; w < 4; ++w) {
            uint32_t mw = 0;
            for (int i = 0; i < 32; ++i)
              if (sparse_row(p, pc.unit, k * kTile + 32 * w + i, false) >= 0) mw |= 1u << i;
            vmask[w] = mw;
          }
        } else {
          const int nv = dense_tile_valid(limit, k);
#pragma unroll
          for (int w = 0; w < 4; ++w) {
            const int nb = min(32, max(0, nv - 32 * w));
            vmask[w] = nb >= 32 ? 0xffffffffu : ((1u << nb) - 1u);
          }
        }
        // pass 1: tile max
        float tmax = -INFINITY;
#pragma unroll 1
        for (int w = 0; w < 4; ++w) {
          uint32_t sv[32];
          tmem_ld32(s_addr + 32 * w, sv);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 32; ++i)
            if (vmask[w] & (1u << i)) tmax = fmaxf(tmax, __uint_as_float(sv[i]));
        }
        if (!rvalid) tmax = -INFINITY;
        float alpha = 1.f;
        int need = 0;
        if (tmax > m_used + thresh || (m_used == -INFINITY && tmax > -INFINITY)) {
          const float m_new = tmax;
          alpha = (m_used == -INFINITY) ? 0.f : ex2_approx((m_used - m_new) * p.scale_log2);
          need = (k != pc.t0) && (m_used != -INFINITY);
          m_used = m_new;
          l_sum *= alpha;
        }
        if (owner) c->alpha[r] = alpha;
        if (need) c->rescale_flag[gt & 1] = 1;
        if (!group_sync(c, &c->grp_sm, gph, p)) { stop = true; break; }
        const bool do_rescale = *(volatile int*)&c->rescale_flag[gt & 1] != 0;
        if (do_rescale) {
          // O^T of the previous tile must be complete before it is rescaled
          const int pb = (gt - 1) & 1;
          if (!timed_wait(c, &c->o_done[pb], ((gt - 1) >> 1) & 1, p)) { stop = true; }
          if (!stop) {
            tc_fence_after();
#pragma unroll
            for (int m = 0; m < 4; ++m) {
#pragma unroll
              for (int c16 = 0; c16 < NR / 16; ++c16) {
                uint32_t ov[16];
                const uint32_t a = tmem + lane_base + 64 * m + 16 * c16;
                tmem_ld16(a, ov);
                tmem_ld_wait();
#pragma unroll
                for (int i = 0; i < 16; ++i) ov[i] = __float_as_uint(__uint_as_float(ov[i]) * c->alpha[16 * c16 + i]);
                tmem_st16(a, ov);
              }
            }
            tmem_st_wait();
          }
          if (!group_sync(c, &c->grp_sm, gph, p)) stop = true;
          if (threadIdx.x == 128) c->rescale_flag[gt & 1] = 0;
        }
        if (stop) break;
        // P^T buffer b was last read by the O MMAs of tile gt-2
        if (gt >= 2 && !timed_wait(c, &c->o_done[b], ((gt - 2) >> 1) & 1, p)) { stop = true; break; }
        // pass 2: probabilities -> bf16 P^T (K-major [NR rows][128 tokens]), row sum
        uint8_t* ptile = sP + b * L::pt_bytes;
        const float mc = (m_used == -INFINITY ? 0.f : m_used) * p.scale_log2;
#pragma unroll 1
        for (int w = 0; w < 4; ++w) {
          uint32_t sv[32];
          tmem_ld32(s_addr + 32 * w, sv);
          tmem_ld_wait();
          if (owner && r < NR) {
            uint32_t pk[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              float p0 = (rvalid && (vmask[w] >> (2 * i)) & 1u) ? ex2_approx(__uint_as_float(sv[2 * i]) * p.scale_log2 - mc) : 0.f;
              float p1 = (rvalid && (vmask[w] >> (2 * i + 1)) & 1u) ? ex2_approx(__uint_as_float(sv[2 * i + 1]) * p.scale_log2 - mc) : 0.f;
              pk[i] = pack_bf16x2(p0, p1);
              l_sum += p0 + p1;
            }
            // tokens 32w..32w+31 -> slice (w>>1), chunks 4*(w&1) .. +3
            uint8_t* slice = ptile + (w >> 1) * (NR * 128);
            uint8_t* rowp = slice + (r >> 3) * 1024 + (r & 7) * 128;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const int ch = 4 * (w & 1) + q;
              *reinterpret_cast<uint4*>(rowp + ((ch ^ (r & 7)) << 4)) =
                  make_uint4(pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
            }
          }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(&c->s_empty[b]);
        mbar_arrive(&c->p_full[b]);
        last_b = b;
        last_gt = gt;
      }
      if (stop) break;
      // ---------------- epilogue of the piece
      if (last_gt >= 0 && !timed_wait(c, &c->o_done[last_b], (last_gt >> 1) & 1, p)) { stop = true; break; }
      tc_fence_after();
      if (owner) {
        float inv = 0.f, lse = -INFINITY;
        if (l_sum > 0.f) {
          inv = 1.f / l_sum;
          lse = m_used * p.scale + logf(l_sum);
        }
        c->inv_l[r] = inv;
        if (rvalid) {
          const size_t grow_all = (size_t)pc.unit * p.rows + row0 + r;
          if (pc.single) p.lse[grow_all] = lse;
          else p.ws_lse[(size_t)pc.ws_idx * p.rows + row0 + r] = lse;
        }
      }
      if (!group_sync(c, &c->grp_sm, gph, p)) { stop = true; break; }
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        const int d = 128 * m + 32 * q4 + lane;
#pragma unroll
        for (int c16 = 0; c16 < NR / 16; ++c16) {
          uint32_t ov[16];
          tmem_ld16(tmem + lane_base + 64 * m + 16 * c16, ov);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const int rr = 16 * c16 + i;
            if (rr < rows_here) {
              const float val = __uint_as_float(ov[i]) * c->inv_l[rr];
              if (pc.single)
                static_cast<__nv_bfloat16*>(p.out)[((size_t)pc.unit * p.rows + row0 + rr) * kDv + d] = __float2bfloat16_rn(val);
              else
                p.ws_o[((size_t)pc.ws_idx * p.rows + row0 + rr) * kDv + d] = val;
            }
          }
        }
      }
      tc_fence_before();
      if (!group_sync(c, &c->grp_sm, gph, p)) { stop = true; break; }
      mbar_arrive(&c->o_free);
    }
  }

  // ---------------------------------------------------------------- teardown
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, kTmemCols);
}

// ---------------------------------------------------------------- host side
template <int NR, int MODE>
static cudaError_t launch_one(const CUtensorMap& tq, const CUtensorMap& tkv, const CUtensorMap& taux,
                              const DecodeParams& p, int parts, int row_groups, cudaStream_t stream) {
  constexpr int smem = Smem<NR>::total + 1024;
  auto kern = mla_decode_kernel<NR, MODE>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  dim3 grid(parts, row_groups);
  kern<<<grid, MODE == kModeFp8 ? 384 : 256, smem, stream>>>(tq, tkv, taux, p);
  return cudaGetLastError();
}

cudaError_t launch_decode(int rows_per_cta, int mode, const CUtensorMap& tq, const CUtensorMap& tkv,
                          const CUtensorMap& taux, const DecodeParams& p, int parts, int row_groups,
                          cudaStream_t stream) {
#define MLA_DISPATCH(NRV)                                                                              \
  if (mode == kModeBf16) return launch_one<NRV, kModeBf16>(tq, tkv, taux, p, parts, row_groups, stream); \
  if (mode == kModeFp8) return launch_one<NRV, kModeFp8>(tq, tkv, taux, p, parts, row_groups, stream);   \
  return launch_one<NRV, kModeSparse>(tq, tkv, taux, p, parts, row_groups, stream);
  if (rows_per_cta <= 16) { MLA_DISPATCH(16) }
  if (rows_per_cta <= 32) { MLA_DISPATCH(32) }
  if (rows_per_cta <= 48) { MLA_DISPATCH(48) }
  MLA_DISPATCH(64)
#undef MLA_DISPATCH
}

}  // namespace mla
