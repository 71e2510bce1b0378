// MLA decode kernel for sm_100a (tcgen05 + TMEM + TMA).
//
// Computes, per work unit (a block of <= 128 query rows of a request, or
// (request, query token) when sparse), softmax(scale * Q K^T) V over the
// unit's keys, with K = whole 576-dim latent row and V = its first 512 dims
// ("[flashinfer] ... NVFP4 DeepSeek-V4 decoding", README section: one latent
// row per token is both K and V;
// FlashMLA-ETAP summary, core mechanism: S = QK^T, P = softmax(S), O = PV).
//
// One CTA = one scheduler part x one group of <= 64 query rows. Per tile of
// 128 tokens (two 64-token pages):
//   S   = Q K^T  tcgen05 M=64 (query rows) x N=128 (tokens) x K=576, both
//                operands K-major in 128-B-swizzled smem; fp32 in TMEM.
//   softmax      one thread per query row reads its 128 scores from TMEM;
//                online max / sum in fp32 with lazily rescaled O.
//   O^T += V^T P^T  tcgen05 M=128 (4 chunks of the 512 value dims) x N=rows x
//                K=64 tokens per V slot; V^T is the MN-major view of the
//                token-major V tile, P^T (bf16) is written K-major by the row
//                threads.
// The O accumulator is transposed (value dims on TMEM lanes) so 64 rows x 512
// dims fit in 256 TMEM columns next to two S buffers (2 x 128 columns).
// K slices (128 tokens x 64 dims) and V slots (64 tokens x 128 dims) stream
// through separate 4-slot smem rings; V is read a second time (from L2) for
// the PV product rather than held across the softmax, which keeps the rings
// deep enough to cover the load latency.
//
// Serves the BF16 paged cache and token-sparse indices over the BF16 or FP8
// cache (the FP8 and NVFP4 paged caches have the page kernel).
//
// Warp roles (256 threads for the bf16 paged cache; 512 with sparse indices):
//   0 Q (and, bf16 paged, K slices) via TMA   1 S issuer (+ TMEM alloc)
//   2 O issuer                                 3 V slots via TMA (bf16 paged)
//   4-7 softmax + epilogue (row r = 16*(warp-4) + lane, lanes 0-15)
//   8-11 K gather warps, 12-15 V gather warps (sparse): cp.async copies
//       software-pipelined two slots deep; FP8 codes are converted to bf16 in
//       place.
// Every mbarrier wait is bounded; on timeout the CTA records
// MLA_DEVICE_STATUS_TIMEOUT, stops issuing work, waits (bounded) for its own
// copies in flight and exits normally. Every ring has exactly one producer
// role so that no parity wait can fall two phases behind.
#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>

#include "mla_decode_util.cuh"

namespace mla {

constexpr int kNK = 4;                 // K ring slots: 128 tokens x 64 dims (16 KB)
constexpr int kNV = 4;                 // V ring slots: 64 tokens x 128 dims (16 KB)
constexpr int kSlot = 16384;
constexpr int kLag = 2;                // gather groups retire a slot 2 slots after issuing it
constexpr int kQBytes = 9 * 8192;      // 64 rows x 576 dims
constexpr int kTmemCols = 512;
constexpr int kTmemS = 256;            // S buffers at columns 256 and 384
constexpr float kRescaleLog2 = 8.0f;   // rescale O only when the max grows by > 2^8
static_assert(kLag < kNK && kLag < kNV, "a gather group must retire a slot before reusing it");


template <int NR>
struct Smem {
  static constexpr int q = 0;
  static constexpr int k = q + kQBytes;
  static constexpr int v = k + kNK * kSlot;
  static constexpr int pt = v + kNV * kSlot;
  static constexpr int pt_bytes = NR * 256;  // [NR rows][128 tokens] bf16
  static constexpr int ctrl = pt + pt_bytes;
  static constexpr int total = ctrl + 1024;
};

struct Ctrl {
  uint64_t q_full, q_empty;
  uint64_t k_full[kNK], k_empty[kNK];
  uint64_t v_full[kNV], v_empty[kNV];
  uint64_t s_full[2], s_empty[2];
  uint64_t p_full, o_done, o_free, drain_s, drain_o;
  uint64_t grp_sm;  // bounded barrier of the 128 softmax threads
  uint32_t tmem_base;
  int abort_flag;
  int rescale_flag[2];
  float alpha[64];
  float inv_l[64];
};
static_assert(sizeof(Ctrl) <= 1024, "control block");

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

// ============================================================================ gather groups
// Sparse modes: four warps fill the K ring and four the V ring with
// 16-byte cp.async copies. Warp lw of a group owns a quarter of every slot's
// rows (K: tile rows 32lw..32lw+31; V: page rows 16lw..16lw+15), lane t the
// source row of one of them; the copies put 4-16 lanes on each row (row
// pointers by shuffle), FP8 codes are converted in place with four lanes per
// row. Each warp issues a slot's copies, commits them as one group and retires
// the slot it issued kLag slots earlier: wait for that group, convert it
// (FP8), fence the generic-proxy writes for the tensor core, and one
// lane arrives on the slot's full barrier (count: 4 warps).
constexpr int kGatherWarps = 4;
constexpr int kGatherThreads = 32 * kGatherWarps;

struct GatherRing {
  uint64_t* full;
  uint64_t* empty;
  uint8_t* base;
  int nslots;
};

// Pointer held by lane `src` of the warp.
__device__ __forceinline__ const uint8_t* shfl_ptr(const uint8_t* v, int src) {
  return reinterpret_cast<const uint8_t*>(
      __shfl_sync(0xffffffffu, reinterpret_cast<unsigned long long>(v), src));
}

// FP8: converts this warp's rows of a retired slot in place, four lanes per
// row (every lane reads a row before any lane overwrites it).
template <int MODE, bool KGROUP>
__device__ __forceinline__ void retire_slot(const GatherRing& g, int seq, int lw, int t) {
  const int slot = seq % g.nslots;
  uint8_t* s = g.base + slot * kSlot;
  if (mode_fp8(MODE)) {
    __syncwarp();  // every lane's copies of this slot are complete and visible
    if (KGROUP) {
      const int j = seq % 9;
      if (j != 8) {  // latent slice: codes in bytes [0,64) and scales in [64,80) of each row
        // all reads first (independent loads in flight), one warp barrier,
        // then every write: the rows are converted in place
        uint4 cw[4];
        float sc[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int r = 32 * lw + 8 * i + (t >> 2), cc = t & 3;
          cw[i] = *reinterpret_cast<const uint4*>(s + r * 128 + 16 * cc);
          sc[i] = reinterpret_cast<const float*>(s + r * 128 + 64)[j >> 1];
        }
        __syncwarp();
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int r = 32 * lw + 8 * i + (t >> 2), cc = t & 3;
          uint4 lo, hi;
          dequant16(cw[i], sc[i], lo, hi);
          *reinterpret_cast<uint4*>(sw128(s, r, 2 * cc)) = lo;
          *reinterpret_cast<uint4*>(sw128(s, r, 2 * cc + 1)) = hi;
        }
      }
    } else {  // V slot: codes in the half-0 row, scales at the start of the half-1 row
      const int m = (seq >> 1) & 3;
      uint4 cw0[2], cw1[2];
      float sc[2];
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        const int r = 16 * lw + 8 * i + (t >> 2), c4 = t & 3;  // codes 32*c4 .. 32*c4+31 of row r
        cw0[i] = *reinterpret_cast<const uint4*>(s + r * 128 + 32 * c4);
        cw1[i] = *reinterpret_cast<const uint4*>(s + r * 128 + 32 * c4 + 16);
        sc[i] = reinterpret_cast<const float*>(s + 8192 + r * 128)[m];
      }
      __syncwarp();
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        const int r = 16 * lw + 8 * i + (t >> 2), c4 = t & 3;
        uint8_t* half = s + (c4 >> 1) * 8192;
        const int c0 = 4 * (c4 & 1);
        uint4 lo, hi;
        dequant16(cw0[i], sc[i], lo, hi);
        *reinterpret_cast<uint4*>(sw128(half, r, c0)) = lo;
        *reinterpret_cast<uint4*>(sw128(half, r, c0 + 1)) = hi;
        dequant16(cw1[i], sc[i], lo, hi);
        *reinterpret_cast<uint4*>(sw128(half, r, c0 + 2)) = lo;
        *reinterpret_cast<uint4*>(sw128(half, r, c0 + 3)) = hi;
      }
    }
  }
  fence_proxy_async_smem();  // this lane's rows -> the tensor core
  __syncwarp();
  if (t == 0) mbar_arrive(&g.full[slot]);  // one arrival per warp (a per-thread one costs more)
}

// Source row of tile-relative slot tt of index tile k (bf16 cache row or FP8
// record; the gather warps run only with token-sparse indices; ok = 0 for an
// ignored slot, whose copies zero-fill: codes and scales
// 0 dequantise to 0 as well).
template <int MODE, bool KGROUP>
__device__ __forceinline__ const uint8_t* gather_src(const DecodeParams& p, int unit, int k, int tt, uint32_t& ok) {
  const int row = sparse_row(p, unit, k * kTile + tt, KGROUP);
  ok = row >= 0 ? 16u : 0u;
  const size_t rb = MODE == kModeSparse ? (size_t)kDqk * 2 : (size_t)kFp8RecordBytes;
  return static_cast<const uint8_t*>(p.kcache) + (size_t)(row >= 0 ? row : 0) * rb;
}

template <int MODE, bool KGROUP>
__device__ void gather_group(const DecodeParams& p, Ctrl* c, PieceIter& it, const GatherRing& g, int lw, int t) {
  int seq = 0;       // slots issued
  int retired = 0;   // slots retired
  bool stop = false;
  Piece pc;
  while (!stop && it.next(pc)) {
    const int unit = pc.unit;
    for (int k = pc.t0; k < pc.t1 && !stop; ++k) {
      // K: lane t owns tile row 32lw + t; V: lane t (< 16) owns row 16lw + t
      // of page h, i.e. tile row 64h + 16lw + t
      uint32_t ok = 0, ok0 = 0, ok1 = 0;
      const uint8_t* srcK = nullptr;
      const uint8_t* srcV0 = nullptr;
      const uint8_t* srcV1 = nullptr;
      if (KGROUP) {
        srcK = gather_src<MODE, KGROUP>(p, unit, k, 32 * lw + t, ok);
      } else {
        srcV0 = gather_src<MODE, KGROUP>(p, unit, k, 16 * lw + (t & 15), ok0);
        srcV1 = gather_src<MODE, KGROUP>(p, unit, k, 64 + 16 * lw + (t & 15), ok1);
      }
      const int slots_per_tile = KGROUP ? 9 : 8;
      for (int j = 0; j < slots_per_tile; ++j, ++seq) {
        const int slot = seq % g.nslots;
        uint8_t* s = g.base + slot * kSlot;
        if (!timed_wait(c, &g.empty[slot], ((seq / g.nslots) & 1) ^ 1, p)) { stop = true; break; }
        if (KGROUP) {
          if (MODE == kModeSparse || j == 8) {  // bf16 128-B row slice: 8 lanes per row
            const int off = MODE == kModeSparse ? 128 * j : 528;
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              const int r = 4 * i + (t >> 3), ch = t & 7;
              const uint32_t nb = __shfl_sync(0xffffffffu, ok, r);
              cp_async16(sw128(s, 32 * lw + r, ch), shfl_ptr(srcK, r) + off + 16 * ch, nb);
            }
          } else {  // FP8 latent slice j: codes (64 B, 4 lanes per row) and scales, converted at retire
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const int r = 8 * i + (t >> 2), cc = t & 3;
              const uint32_t nb = __shfl_sync(0xffffffffu, ok, r);
              cp_async16(s + (32 * lw + r) * 128 + 16 * cc, shfl_ptr(srcK, r) + 64 * j + 16 * cc, nb);
            }
            cp_async16(s + (32 * lw + t) * 128 + 64, srcK + 512, ok);
          }
        } else {  // V slot j: value dims 128*(j/2).., page half h = j%2
          const int m = j >> 1;
          const uint8_t* sv = (j & 1) ? srcV1 : srcV0;
          const uint32_t okv = (j & 1) ? ok1 : ok0;
          if (MODE == kModeSparse) {  // 256 B per row in two 128-B halves: 16 lanes per row
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              const int r = 2 * i + (t >> 4), hh = (t >> 3) & 1, ch = t & 7;
              const uint32_t nb = __shfl_sync(0xffffffffu, okv, r);
              cp_async16(sw128(s + hh * 8192, 16 * lw + r, ch), shfl_ptr(sv, r) + 256 * m + 128 * hh + 16 * ch, nb);
            }
          } else {  // FP8: codes (128 B, 8 lanes per row) in the half-0 row, scales at the half-1 row start
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const int r = 4 * i + (t >> 3), ch = t & 7;
              const uint32_t nb = __shfl_sync(0xffffffffu, okv, r);
              cp_async16(s + (16 * lw + r) * 128 + 16 * ch, shfl_ptr(sv, r) + 128 * m + 16 * ch, nb);
            }
            if (t < 16) cp_async16(s + 8192 + (16 * lw + t) * 128, sv + 512, okv);
          }
        }
        cp_async_commit();
        if (seq + 1 - retired > kLag) {
          cp_async_wait<kLag>();
          retire_slot<MODE, KGROUP>(g, retired, lw, t);
          ++retired;
        }
      }
    }
  }
  cp_async_wait<0>();  // no copy may land after the CTA has finished
  if (!stop) {
    while (retired < seq) {
      retire_slot<MODE, KGROUP>(g, retired, lw, t);
      ++retired;
    }
  }
}

// ============================================================================ kernel
template <int NR, int MODE>
__global__ void __launch_bounds__(MODE == kModeBf16 ? 256 : 256 + 2 * kGatherThreads, 1)
    mla_decode_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_kv,
                      const __grid_constant__ CUtensorMap tm_v, const DecodeParams p) {
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
  constexpr uint32_t kFullCount = MODE == kModeBf16 ? 1 : kGatherWarps;  // TMA producer, or one per gather warp

  if (threadIdx.x == 0) {
    mbar_init(&c->q_full, 1);
    mbar_init(&c->q_empty, 1);
    for (int i = 0; i < kNK; ++i) { mbar_init(&c->k_full[i], kFullCount); mbar_init(&c->k_empty[i], 1); }
    for (int i = 0; i < kNV; ++i) { mbar_init(&c->v_full[i], kFullCount); mbar_init(&c->v_empty[i], 1); }
    for (int i = 0; i < 2; ++i) { mbar_init(&c->s_full[i], 1); mbar_init(&c->s_empty[i], 128); }
    mbar_init(&c->p_full, 128);
    mbar_init(&c->o_done, 1);
    mbar_init(&c->o_free, 128);
    mbar_init(&c->drain_s, 1);
    mbar_init(&c->drain_o, 1);
    mbar_init(&c->grp_sm, 128);
    c->abort_flag = 0;
    c->rescale_flag[0] = 0;
    c->rescale_flag[1] = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tm_q);
    if (MODE == kModeBf16) {  // encoded only for the bf16 paged cache
      tma_prefetch_desc(&tm_kv);
      tma_prefetch_desc(&tm_v);
    }
  }
  if (warp == 1) {
    tmem_alloc(&c->tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = c->tmem_base;
  griddep_wait();  // the scheduler's output (and every input) is ready

  PieceIter it;
  it.init(p, part);
  Piece pc;

  if (warp == 0) {
    // ------------------------------------------------------------ Q (+ K slices, bf16)
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
        if (MODE == kModeBf16 && !stop) {
          const int req = unit_req(p, pc.unit);
          const int npg = (p.seqlens[req] + kPage - 1) / kPage;
          for (int k = pc.t0; k < pc.t1 && !stop; ++k) {
            int pa = page_of(p, req, 2 * k, npg);
            int pb = page_of(p, req, 2 * k + 1, npg);
            if (pb < 0) pb = pa;  // half tile: reload page A, its keys are masked
            for (int j = 0; j < 9; ++j, ++kc) {
              const int slot = kc % kNK;
              uint8_t* dst = sK + slot * kSlot;
              if (!timed_wait(c, &c->k_empty[slot], ((kc / kNK) & 1) ^ 1, p)) { stop = true; break; }
              mbar_arrive_expect_tx(&c->k_full[slot], kSlot);
              tma_load_2d_hint(dst, &tm_kv, &c->k_full[slot], 64 * j, pa * kPage, l2_policy_evict_last());
              tma_load_2d_hint(dst + 8192, &tm_kv, &c->k_full[slot], 64 * j, pb * kPage, l2_policy_evict_last());
            }
          }
        }
      }
      stop = __shfl_sync(0xffffffffu, stop ? 1 : 0, 0) != 0;
      ++pi;
    }
    if (lane == 0) {
      if (q_issued > 0) mbar_wait(&c->q_full, (uint32_t)((q_issued - 1) & 1), p.timeout_ns);
      if (MODE == kModeBf16) drain_issued(c->k_full, kNK, kc, p.timeout_ns);
    }
    __syncwarp();
  } else if (warp == 3 && MODE == kModeBf16) {
    // ------------------------------------------------------------ V slots (bf16)
    if (lane == 0) {
      int vc = 0;
      bool stop = false;
      while (!stop && it.next(pc)) {
        const int req = unit_req(p, pc.unit);
        const int npg = (p.seqlens[req] + kPage - 1) / kPage;
        for (int k = pc.t0; k < pc.t1 && !stop; ++k) {
          int pg[2];
          pg[0] = page_of(p, req, 2 * k, npg);
          pg[1] = page_of(p, req, 2 * k + 1, npg);
          if (pg[1] < 0) pg[1] = pg[0];
          for (int j = 0; j < 8; ++j, ++vc) {  // slot j: value dims 128*(j/2).., page half j%2
            const int slot = vc % kNV;
            uint8_t* dst = sV + slot * kSlot;
            if (!timed_wait(c, &c->v_empty[slot], ((vc / kNV) & 1) ^ 1, p)) { stop = true; break; }
            mbar_arrive_expect_tx(&c->v_full[slot], kSlot);
            const int m = j >> 1, y = pg[j & 1] * kPage;
            tma_load_3d_hint(dst, &tm_v, &c->v_full[slot], 0, y, 2 * m, l2_policy_evict_first());
          }
        }
      }
      drain_issued(c->v_full, kNV, vc, p.timeout_ns);
    }
    __syncwarp();
  } else if (MODE != kModeBf16 && warp >= 8) {
    // ------------------------------------------------------------ gather groups
    if (warp < 8 + kGatherWarps) {
      const GatherRing g{c->k_full, c->k_empty, sK, kNK};
      gather_group<MODE, true>(p, c, it, g, warp - 8, lane);
    } else {
      const GatherRing g{c->v_full, c->v_empty, sV, kNV};
      gather_group<MODE, false>(p, c, it, g, warp - 8 - kGatherWarps, lane);
    }
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
            const uint32_t qa = smem_u32(sQ + j * 8192), kb = smem_u32(sK + slot * kSlot);
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
        const bool first = (k == pc.t0);
        if (lane == 0) {
          if (first && pi > 0 && !timed_wait(c, &c->o_free, (pi - 1) & 1, p)) stop = true;
          if (!stop && !timed_wait(c, &c->p_full, gt & 1, p)) stop = true;
        }
        stop = __shfl_sync(0xffffffffu, stop ? 1 : 0, 0) != 0;
        if (stop) break;
        // dense: value rows of keys past the request's end must read as zero
        // (ignored sparse slots are zero-filled by the gather already)
        const int nvalid = mode_sparse(MODE) ? kTile : dense_tile_valid(p.seqlens[req], k);
        const uint32_t pt = smem_u32(sP);
        for (int j = 0; j < 8 && !stop; ++j, ++vc) {
          const int slot = vc % kNV;
          const int m = j >> 1, h = j & 1;
          uint8_t* vs = sV + slot * kSlot;
          if (lane == 0 && !timed_wait(c, &c->v_full[slot], (vc / kNV) & 1, p)) stop = true;
          stop = __shfl_sync(0xffffffffu, stop ? 1 : 0, 0) != 0;
          if (stop) break;
          const int nv_slot = min(64, max(0, nvalid - 64 * h));
          if (nv_slot < 64) {
            const uint4 z = make_uint4(0, 0, 0, 0);
            for (int i = nv_slot * 16 + lane; i < 64 * 16; i += 32) {  // 16 chunks per token row
              const int tok = i >> 4, ch = i & 15;
              *reinterpret_cast<uint4*>(vs + (ch >> 3) * 8192 + tok * 128 + (ch & 7) * 16) = z;
            }
            fence_proxy_async_smem();
            __syncwarp();
          }
          if (lane == 0) {
            tc_fence_after();
            const uint32_t va = smem_u32(vs);
            const uint32_t d = tmem + 64 * m;
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              mma_bf16_ss(d, sdesc(va + kk * 2048, 8192, 1024),
                          sdesc(pt + h * (NR * 128) + kk * 32, 16, 1024), idesc,
                          (first && h == 0 && kk == 0) ? 0u : 1u);
            mma_commit(&c->v_empty[slot]);
          }
          __syncwarp();
        }
        if (lane == 0 && !stop) mma_commit(&c->o_done);
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
      if (!mode_sparse(MODE)) {
        const int Ls = p.seqlens[req];
        limit = Ls;
        if (p.causal) limit = Ls - p.s_q + row_query(p, pc.unit, grow) + 1;
      }
      float m_used = -INFINITY, l_sum = 0.f;
      int last_gt = -1;
      for (int k = pc.t0; k < pc.t1 && !stop; ++k, ++gt) {
        const int b = gt & 1;
        // validity of the 128 keys of this tile for this row (bit i of word w = key 32w + i)
        uint4 vmask;
        if (mode_sparse(MODE)) {
          vmask.x = __ballot_sync(0xffffffffu, sparse_row(p, pc.unit, k * kTile + lane, false) >= 0);
          vmask.y = __ballot_sync(0xffffffffu, sparse_row(p, pc.unit, k * kTile + 32 + lane, false) >= 0);
          vmask.z = __ballot_sync(0xffffffffu, sparse_row(p, pc.unit, k * kTile + 64 + lane, false) >= 0);
          vmask.w = __ballot_sync(0xffffffffu, sparse_row(p, pc.unit, k * kTile + 96 + lane, false) >= 0);
        } else {
          const int nv = dense_tile_valid(limit, k);
          auto word = [nv](int w) {
            const int nb = min(32, max(0, nv - 32 * w));
            return nb >= 32 ? 0xffffffffu : ((1u << nb) - 1u);
          };
          vmask = make_uint4(word(0), word(1), word(2), word(3));
        }
        if (!timed_wait(c, &c->s_full[b], (gt >> 1) & 1, p)) { stop = true; break; }
        tc_fence_after();
        const uint32_t s_addr = tmem + lane_base + kTmemS + 128 * b;
        // pass 1: tile max
        float tmax = -INFINITY;
#pragma unroll 1
        for (int w = 0; w < 4; ++w) {
          uint32_t sv[32];
          tmem_ld32(s_addr + 32 * w, sv);
          tmem_ld_wait();
          const uint32_t mw = pick4u(vmask, w);
#pragma unroll
          for (int i = 0; i < 32; ++i)
            tmax = fmaxf(tmax, ((mw >> i) & 1u) ? __uint_as_float(sv[i]) : -INFINITY);
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
        // pass 2: probabilities (masked by select, never by branch) -> bf16, staged
        // in TMEM over the S columns already read (tokens 32w.. -> columns 16w..)
        const float mc = (m_used == -INFINITY ? 0.f : m_used) * p.scale_log2;
        float part = 0.f;
#pragma unroll 1
        for (int w = 0; w < 4; ++w) {
          uint32_t sv[32];
          tmem_ld32(s_addr + 32 * w, sv);
          tmem_ld_wait();
          const uint32_t mw = rvalid ? pick4u(vmask, w) : 0u;
          uint32_t pk[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const float e0 = ex2_approx(fmaf(__uint_as_float(sv[2 * i]), p.scale_log2, -mc));
            const float e1 = ex2_approx(fmaf(__uint_as_float(sv[2 * i + 1]), p.scale_log2, -mc));
            const float p0 = ((mw >> (2 * i)) & 1u) ? e0 : 0.f;
            const float p1 = ((mw >> (2 * i + 1)) & 1u) ? e1 : 0.f;
            pk[i] = pack_bf16x2(p0, p1);
            part += p0 + p1;
          }
          tmem_st16(s_addr + 16 * w, pk);
        }
        tmem_st_wait();
        l_sum += part;
        if (owner) c->alpha[r] = alpha;
        if (need) c->rescale_flag[gt & 1] = 1;
        if (!group_sync(c, &c->grp_sm, gph, p)) { stop = true; break; }
        const bool do_rescale = *(volatile int*)&c->rescale_flag[gt & 1] != 0;
        // the O MMAs of the previous tile must be complete before O^T is
        // rescaled and before P^T (which they read) is overwritten
        if (gt >= 1 && !timed_wait(c, &c->o_done, (gt - 1) & 1, p)) { stop = true; break; }
        tc_fence_after();
        if (do_rescale) {
#pragma unroll 1
          for (int m = 0; m < 4; ++m) {
#pragma unroll 1
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
          if (!group_sync(c, &c->grp_sm, gph, p)) { stop = true; break; }
          if (threadIdx.x == 128) c->rescale_flag[gt & 1] = 0;
        }
        // P^T, K-major [NR rows][128 tokens]: tokens 64h.. in slice h, 8 tokens per 16-B chunk
#pragma unroll 1
        for (int w = 0; w < 4; ++w) {
          uint32_t pk[16];
          tmem_ld16(s_addr + 16 * w, pk);
          tmem_ld_wait();
          if (owner && r < NR) {
            uint8_t* rowp = sP + (w >> 1) * (NR * 128) + (r >> 3) * 1024 + (r & 7) * 128;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const int ch = 4 * (w & 1) + q;
              *reinterpret_cast<uint4*>(rowp + ((ch ^ (r & 7)) << 4)) =
                  make_uint4(pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
            }
          }
        }
        tc_fence_before();
        mbar_arrive(&c->s_empty[b]);  // scores and staged probabilities of this buffer are consumed
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(&c->p_full);
        last_gt = gt;
      }
      if (stop) break;
      // ---------------- epilogue of the piece
      if (last_gt >= 0 && !timed_wait(c, &c->o_done, last_gt & 1, p)) { stop = true; break; }
      tc_fence_after();
      if (owner) {
        float inv = 0.f, lse = -INFINITY;
        if (l_sum > 0.f) {
          inv = 1.f / l_sum;
          lse = m_used * p.scale + logf(l_sum);
        }
        if (pc.single && rvalid && p.sink != nullptr) inv *= fold_sink(lse, p.sink[row_head(p, pc.unit, row0 + r)]);
        c->inv_l[r] = inv;
        if (rvalid) {
          const size_t grow_all = (size_t)pc.unit * p.rows + row0 + r;
          if (pc.single) p.lse[grow_all] = lse;
          else p.ws_lse[(size_t)pc.ws_idx * p.rows + row0 + r] = lse;
        }
      }
      if (!group_sync(c, &c->grp_sm, gph, p)) { stop = true; break; }
#pragma unroll 1
      for (int m = 0; m < 4; ++m) {
        const int d = 128 * m + 32 * q4 + lane;
#pragma unroll 1
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
                static_cast<__nv_bfloat16*>(p.out)[((size_t)pc.unit * p.rows + row0 + rr) * kDv + d] =
                    __float2bfloat16_rn(val);
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
  griddep_launch_dependents();  // the combine may be scheduled (it waits for this grid)
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, kTmemCols);
}

// ---------------------------------------------------------------- host side
template <int NR, int MODE>
static cudaError_t launch_one(const CUtensorMap& tq, const CUtensorMap& tkv, const CUtensorMap& tv,
                              const DecodeParams& p, int parts,
                              int row_groups, cudaStream_t stream) {
  constexpr int smem = Smem<NR>::total + 1024;
  auto kern = mla_decode_kernel<NR, MODE>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  e = launch_pdl(kern, dim3(parts, row_groups), dim3(MODE == kModeBf16 ? 256 : 256 + 2 * kGatherThreads), smem,
                 stream, tq, tkv, tv, p);
  return e != cudaSuccess ? e : cudaGetLastError();
}

cudaError_t launch_decode(int rows_per_cta, int mode, const CUtensorMap& tq, const CUtensorMap& tkv,
                          const CUtensorMap& tv, const DecodeParams& p, int parts, int row_groups,
                          cudaStream_t stream) {
#define MLA_DISPATCH(NRV)                                                                         \
  if (mode == kModeBf16) return launch_one<NRV, kModeBf16>(tq, tkv, tv, p, parts, row_groups, stream); \
  if (mode == kModeSparse) return launch_one<NRV, kModeSparse>(tq, tkv, tv, p, parts, row_groups, stream); \
  return launch_one<NRV, kModeFp8Sparse>(tq, tkv, tv, p, parts, row_groups, stream);
  // <= 16 rows run in the 32-row kernel: the extra P^T rows are written as
  // zeros and their output rows are never stored
  if (rows_per_cta <= 32) { MLA_DISPATCH(32) }
  if (rows_per_cta <= 48) { MLA_DISPATCH(48) }
  MLA_DISPATCH(64)
#undef MLA_DISPATCH
}

}  // namespace mla
