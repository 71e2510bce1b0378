// MLA decode over a quantised paged cache (FP8 records or NVFP4 rows) for
// sm_100a: every page is fetched once by bulk copies and converted once.
//
// FP8: each cached token is one 656-byte record of 512 e4m3 latent codes,
// four fp32 scales (one per 128 codes) and the 64 RoPE dims in bf16
// ("deepseek-ai/FlashMLA", technical details: an FP8 KV cache dequantised on
// the fly); x = bf16(f32(e4m3) * scale). The 64 records of a page are one
// contiguous 41,984-byte run.
// NVFP4 ("[flashinfer] ... NVFP4 DeepSeek-V4 decoding", README: one 512-value
// row per token is both K and V, E2M1 codes two per byte with a UE4M3 scale
// per 16 values, and an NVFP4 query): a page is 16 KB of codes and 2 KB of
// scales, each contiguous; x = e2m1 * ue4m3, exact in bf16.
// Bulk copies put a page's bytes at the tail of a 72 KB page slot, and eight
// converter warps expand them in place into 64-token x 64-dim bf16 slices
// (128-B swizzled): nine for FP8 (576 dims), eight for NVFP4 (512). The same
// slices feed both products of the page:
//   S    = Q K^T     tcgen05 M=64 rows x N=64 tokens x K=576 or 512 (the
//                    slices as the K-major B operand)
//   O^T += V^T P^T   M=128 value dims (slices 2m and 2m+1, read MN-major) x
//                    N=rows x K=64 tokens
// so no cache byte crosses from L2 twice and none is converted twice. Q takes
// 72 KB (64 KB for NVFP4), which leaves room for two page slots: one page is
// fetched and converted while the other is multiplied.
//
// Warp roles (512 threads):
//   0 Q (TMA, or dequantised from NVFP4 by the warp) and the page copies
//   1 S issuer (+ TMEM alloc)          2 O issuer          3 idle
//   4-7 softmax + epilogue (row r = 16*(warp-4) + lane, lanes 0-15)
//   8-15 converters: thread (token 8*(warp-8) + lane%8, quarter lane/8 of the
//        token's latent values)
// The softmax, the lazily rescaled O^T accumulator and the split epilogue are
// those of the bf16 row-group kernel, on 64-token pages. Every wait is
// bounded; on a timeout the CTA records MLA_DEVICE_STATUS_TIMEOUT, stops
// issuing work, waits (bounded) for its own copies and MMAs, and exits.
#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>

#include "mla_decode_util.cuh"

namespace mla {
namespace {

constexpr int kSlotB = 9 * 8192;                         // one page: up to nine 64 x 64 bf16 slices
constexpr int kQMax = 9 * 8192;                          // 64 rows x 576 dims
// 64-dim slices per row, raw page bytes, where they land in the slot
__host__ __device__ constexpr int slices_of(int mode) { return mode == kModeNvfp4 ? 8 : 9; }
__host__ __device__ constexpr int raw_bytes(int mode) {
  return mode == kModeNvfp4 ? kPage * (kNvfp4RowBytes + kNvfp4ScaleBytes) : kPage * kFp8RecordBytes;
}
__host__ __device__ constexpr int raw_off(int mode) { return kSlotB - raw_bytes(mode); }
constexpr int kCvWarps = 8;
constexpr int kThreads = 256 + 32 * kCvWarps;
constexpr int kTmemCols = 512;
constexpr int kTmemS = 256;                              // S buffers at columns 256 and 320
constexpr float kRescaleLog2 = 8.0f;                     // rescale O only when the max grows by > 2^8
static_assert(raw_off(kModeFp8) % 16 == 0 && raw_bytes(kModeFp8) % 16 == 0, "bulk copy alignment");
static_assert(raw_off(kModeNvfp4) % 16 == 0 && (kPage * kNvfp4RowBytes) % 16 == 0, "bulk copy alignment");

template <int NR>
struct Smem {
  static constexpr int q = 0;
  static constexpr int slot = q + kQMax;
  static constexpr int pt = slot + 2 * kSlotB;
  static constexpr int pt_bytes = NR * 128;              // P^T: [NR rows][64 tokens] bf16
  static constexpr int ctrl = pt + pt_bytes;
  static constexpr int total = ctrl + 1024;
};
static_assert(Smem<64>::total + 1024 <= 232448, "shared memory budget");

struct Ctrl {
  uint64_t q_full, q_empty;
  uint64_t raw_full[2], page_full[2], page_empty[2];
  uint64_t s_full[2], s_empty[2];
  uint64_t p_full, o_done, o_free, drain_s, drain_o;
  uint64_t grp_sm, grp_cv;
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

// Bounded barrier of a thread group, built on an mbarrier.
__device__ __forceinline__ bool group_sync(Ctrl* c, uint64_t* bar, uint32_t& phase, const DecodeParams& p) {
  mbar_arrive(bar);
  const bool ok = timed_wait(c, bar, phase & 1, p);
  ++phase;
  return ok;
}

// Logical pages [2*t0, end) of a piece: its 128-token tiles, cut at the request's last page.
__device__ __forceinline__ int piece_page_end(const Piece& pc, int npg) { return min(2 * pc.t1, npg); }

template <int NR, int MODE>
__global__ void __launch_bounds__(kThreads, 1)
    mla_decode_page_kernel(const __grid_constant__ CUtensorMap tm_q, const DecodeParams p) {
  constexpr int kSl = slices_of(MODE);
  constexpr int kRawB = raw_bytes(MODE);
  constexpr int kRawOff = raw_off(MODE);
  using L = Smem<NR>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem + L::q;
  uint8_t* sS = smem + L::slot;
  uint8_t* sP = smem + L::pt;
  Ctrl* c = reinterpret_cast<Ctrl*>(smem + L::ctrl);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int part = blockIdx.x, rg = blockIdx.y;
  const int row0 = rg * kRowsPerCta;
  const int rows_here = min(kRowsPerCta, p.rows - row0);

  if (threadIdx.x == 0) {
    mbar_init(&c->q_full, 1);
    mbar_init(&c->q_empty, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&c->raw_full[i], 1);
      mbar_init(&c->page_full[i], kCvWarps);
      mbar_init(&c->page_empty[i], 1);
      mbar_init(&c->s_full[i], 1);
      mbar_init(&c->s_empty[i], 128);
    }
    mbar_init(&c->p_full, 128);
    mbar_init(&c->o_done, 1);
    mbar_init(&c->o_free, 128);
    mbar_init(&c->drain_s, 1);
    mbar_init(&c->drain_o, 1);
    mbar_init(&c->grp_sm, 128);
    mbar_init(&c->grp_cv, kCvWarps);
    c->abort_flag = 0;
    c->rescale_flag[0] = 0;
    c->rescale_flag[1] = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0 && MODE != kModeNvfp4) tma_prefetch_desc(&tm_q);
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
    // ------------------------------------------------------------ Q and page copies
    int gp = 0, pi = 0, q_issued = 0;
    bool stop = false;
    while (!stop && it.next(pc)) {
      if (lane == 0 && !timed_wait(c, &c->q_empty, (pi & 1) ^ 1, p)) stop = true;
      stop = __shfl_sync(0xffffffffu, stop ? 1 : 0, 0) != 0;
      if (stop) break;
      if (MODE == kModeNvfp4) {
        // the warp dequantises the query rows: lane l converts values
        // 16l..16l+15 of each row into slice l/4, chunks 2(l%4) and 2(l%4)+1;
        // rows past this CTA's rows are zero
        const size_t qrow0 = (size_t)pc.unit * p.rows + row0;
        uint8_t* box = sQ + (lane >> 2) * 8192;
#pragma unroll 1
        for (int r0 = 0; r0 < kRowsPerCta; r0 += 8) {
          uint2 cw[8];
          uint32_t sb[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const bool live = r0 + i < rows_here;
            const size_t qr = qrow0 + (live ? r0 + i : 0);
            cw[i] = live ? *reinterpret_cast<const uint2*>(p.q_nvfp4 + qr * kNvfp4RowBytes + 8 * lane) : make_uint2(0, 0);
            sb[i] = live ? p.q_scale[qr * kNvfp4ScaleBytes + lane] : 0u;
          }
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            uint4 lo, hi;
            dequant_nvfp4_16(cw[i], sb[i], lo, hi);
            *reinterpret_cast<uint4*>(sw128(box, r0 + i, 2 * (lane & 3))) = lo;
            *reinterpret_cast<uint4*>(sw128(box, r0 + i, 2 * (lane & 3) + 1)) = hi;
          }
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&c->q_full);
      } else if (lane == 0) {
        mbar_arrive_expect_tx(&c->q_full, kSl * 8192);
        const int qy = pc.unit * p.rows + row0;
        for (int j = 0; j < kSl; ++j) tma_load_2d(sQ + j * 8192, &tm_q, &c->q_full, 64 * j, qy);
        ++q_issued;
      }
      if (lane == 0) {
        const int req = unit_req(p, pc.unit);
        const int npg = (p.seqlens[req] + kPage - 1) / kPage;
        const int pend = piece_page_end(pc, npg);
        for (int pj = 2 * pc.t0; pj < pend; ++pj) {
          const int slot = gp & 1;
          if (!timed_wait(c, &c->page_empty[slot], ((gp >> 1) & 1) ^ 1, p)) { stop = true; break; }
          const size_t pg = (size_t)page_of(p, req, pj, npg);
          uint8_t* dst = sS + slot * kSlotB + kRawOff;
          mbar_arrive_expect_tx(&c->raw_full[slot], kRawB);
          if (MODE == kModeNvfp4) {  // codes, then scales
            bulk_load(dst, p.kcache_fp8 + pg * (kPage * kNvfp4RowBytes), kPage * kNvfp4RowBytes, &c->raw_full[slot]);
            bulk_load(dst + kPage * kNvfp4RowBytes, p.kv_scale + pg * (kPage * kNvfp4ScaleBytes),
                      kPage * kNvfp4ScaleBytes, &c->raw_full[slot]);
          } else {
            bulk_load(dst, p.kcache_fp8 + pg * kRawB, kRawB, &c->raw_full[slot]);
          }
          ++gp;
        }
      }
      stop = __shfl_sync(0xffffffffu, stop ? 1 : 0, 0) != 0;
      ++pi;
    }
    if (lane == 0) {
      if (q_issued > 0) mbar_wait(&c->q_full, (uint32_t)((q_issued - 1) & 1), p.timeout_ns);
      drain_issued(c->raw_full, 2, gp, p.timeout_ns);
    }
    __syncwarp();
  } else if (warp >= 8) {
    // ------------------------------------------------------------ converters
    const int tk = 8 * (warp - 8) + (lane & 7);  // token row of the page
    const int qq = lane >> 3;                    // latent values 128qq..128qq+127 (FP8: + RoPE chunks 2qq, 2qq+1)
    uint32_t cph = 0;
    int gp = 0;
    bool stop = false;
    while (!stop && it.next(pc)) {
      const int req = unit_req(p, pc.unit);
      const int Ls = p.seqlens[req];
      const int npg = (Ls + kPage - 1) / kPage;
      const int pend = piece_page_end(pc, npg);
      for (int pj = 2 * pc.t0; pj < pend; ++pj, ++gp) {
        const int slot = gp & 1;
        uint8_t* s = sS + slot * kSlotB;
        if (!timed_wait(c, &c->raw_full[slot], (gp >> 1) & 1, p)) { stop = true; break; }
        // every converter reads its raw bytes before any slice row
        // overwrites them (the slices overlap the raw area)
        const bool live = kPage * pj + tk < Ls;  // rows past the request's end are written as zeros
        const uint4 z = make_uint4(0, 0, 0, 0);
        if (MODE == kModeNvfp4) {
          // 64 code bytes (4 x 16) and 8 scale bytes; the 16-byte chunks are
          // read in an order rotated by the token (the 256-byte row pitch
          // would put 8 tokens on one bank group)
          const uint8_t* codes = s + kRawOff + tk * kNvfp4RowBytes + 64 * qq;
          uint4 cw[4];
#pragma unroll
          for (int i = 0; i < 4; ++i) cw[i] = *reinterpret_cast<const uint4*>(codes + 16 * ((i + tk) & 3));
          const uint2 scw = *reinterpret_cast<const uint2*>(s + kRawOff + kPage * kNvfp4RowBytes +
                                                            tk * kNvfp4ScaleBytes + 8 * qq);
          const unsigned long long sc8 = ((unsigned long long)scw.y << 32) | scw.x;
          __syncwarp();
          if (lane == 0) mbar_arrive(&c->grp_cv);
          if (!timed_wait(c, &c->grp_cv, cph & 1, p)) { stop = true; break; }
          ++cph;
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            // chunk ch: values 128qq + 32ch .. +31 -> slice 2qq + ch/2, 16-B chunks 4(ch%2) .. 4(ch%2)+3
            const int ch = (i + tk) & 3;
            uint8_t* slice = s + (2 * qq + (ch >> 1)) * 8192;
            const uint32_t sb = (uint32_t)(sc8 >> (16 * ch));
            uint4 lo, hi;
            dequant_nvfp4_16(make_uint2(cw[i].x, cw[i].y), sb & 0xFFu, lo, hi);
            *reinterpret_cast<uint4*>(sw128(slice, tk, 4 * (ch & 1))) = live ? lo : z;
            *reinterpret_cast<uint4*>(sw128(slice, tk, 4 * (ch & 1) + 1)) = live ? hi : z;
            dequant_nvfp4_16(make_uint2(cw[i].z, cw[i].w), (sb >> 8) & 0xFFu, lo, hi);
            *reinterpret_cast<uint4*>(sw128(slice, tk, 4 * (ch & 1) + 2)) = live ? lo : z;
            *reinterpret_cast<uint4*>(sw128(slice, tk, 4 * (ch & 1) + 3)) = live ? hi : z;
          }
        } else {
          // 164 record bytes (8 lanes on 8 tokens per 16-byte access: the
          // 656-byte stride puts them on distinct banks)
          const uint8_t* rec = s + kRawOff + tk * kFp8RecordBytes;
          uint4 cw[8], rope[2];
#pragma unroll
          for (int i = 0; i < 8; ++i) cw[i] = *reinterpret_cast<const uint4*>(rec + 128 * qq + 16 * i);
          const float sc = reinterpret_cast<const float*>(rec + 512)[qq];
          rope[0] = *reinterpret_cast<const uint4*>(rec + 528 + 32 * qq);
          rope[1] = *reinterpret_cast<const uint4*>(rec + 528 + 32 * qq + 16);
          __syncwarp();
          if (lane == 0) mbar_arrive(&c->grp_cv);
          if (!timed_wait(c, &c->grp_cv, cph & 1, p)) { stop = true; break; }
          ++cph;
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            uint8_t* slice = s + (2 * qq + (i >> 2)) * 8192;
            uint4 lo, hi;
            dequant16(cw[i], sc, lo, hi);
            *reinterpret_cast<uint4*>(sw128(slice, tk, 2 * (i & 3))) = live ? lo : z;
            *reinterpret_cast<uint4*>(sw128(slice, tk, 2 * (i & 3) + 1)) = live ? hi : z;
          }
          *reinterpret_cast<uint4*>(sw128(s + 8 * 8192, tk, 2 * qq)) = live ? rope[0] : z;
          *reinterpret_cast<uint4*>(sw128(s + 8 * 8192, tk, 2 * qq + 1)) = live ? rope[1] : z;
        }
        fence_proxy_async_smem();  // this thread's slice rows -> the tensor core
        __syncwarp();
        if (lane == 0) mbar_arrive(&c->page_full[slot]);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ S issuer
    const uint32_t idesc = idesc_bf16(64, 64, false, false);
    int gp = 0, pi = 0;
    bool stop = false;
    while (!stop && it.next(pc)) {
      if (lane == 0 && !timed_wait(c, &c->q_full, pi & 1, p)) stop = true;
      stop = __shfl_sync(0xffffffffu, stop ? 1 : 0, 0) != 0;
      const int npg = (p.seqlens[unit_req(p, pc.unit)] + kPage - 1) / kPage;
      const int pend = piece_page_end(pc, npg);
      for (int pj = 2 * pc.t0; pj < pend && !stop; ++pj, ++gp) {
        const int b = gp & 1;
        if (lane == 0) {
          if (!timed_wait(c, &c->s_empty[b], ((gp >> 1) & 1) ^ 1, p) ||
              !timed_wait(c, &c->page_full[b], (gp >> 1) & 1, p)) {
            stop = true;
          } else {
            tc_fence_after();
            const uint32_t d = tmem + kTmemS + 64 * b;
            const uint32_t qa = smem_u32(sQ), kb = smem_u32(sS + b * kSlotB);
            for (int j = 0; j < kSl; ++j) {
#pragma unroll
              for (int kk = 0; kk < 4; ++kk)
                mma_bf16_ss(d, sdesc(qa + j * 8192 + kk * 32, 16, 1024), sdesc(kb + j * 8192 + kk * 32, 16, 1024),
                            idesc, (j | kk) != 0 ? 1u : 0u);
            }
            if (!(gp == 0 && (p.debug_flags & MLA_DEBUG_WITHHOLD_SCORES))) mma_commit(&c->s_full[b]);
          }
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
    int gp = 0, pi = 0;
    bool stop = false;
    while (!stop && it.next(pc)) {
      const int npg = (p.seqlens[unit_req(p, pc.unit)] + kPage - 1) / kPage;
      const int pend = piece_page_end(pc, npg);
      for (int pj = 2 * pc.t0; pj < pend && !stop; ++pj, ++gp) {
        const bool first = pj == 2 * pc.t0;
        if (lane == 0) {
          if (first && pi > 0 && !timed_wait(c, &c->o_free, (pi - 1) & 1, p)) stop = true;
          if (!stop && !timed_wait(c, &c->p_full, gp & 1, p)) stop = true;
          if (!stop) {
            tc_fence_after();
            const int slot = gp & 1;
            const uint32_t va = smem_u32(sS + slot * kSlotB), pt = smem_u32(sP);
#pragma unroll
            for (int m = 0; m < 4; ++m) {
#pragma unroll
              for (int kk = 0; kk < 4; ++kk)
                mma_bf16_ss(tmem + 64 * m, sdesc(va + 16384 * m + kk * 2048, 8192, 1024),
                            sdesc(pt + kk * 32, 16, 1024), idesc, (first && kk == 0) ? 0u : 1u);
            }
            mma_commit(&c->page_empty[slot]);  // the page slot may be refilled
            mma_commit(&c->o_done);
          }
        }
        stop = __shfl_sync(0xffffffffu, stop ? 1 : 0, 0) != 0;
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
    int gp = 0;
    bool stop = false;
    while (!stop && it.next(pc)) {
      const int req = unit_req(p, pc.unit);
      const int Ls = p.seqlens[req];
      const int npg = (Ls + kPage - 1) / kPage;
      const int pend = piece_page_end(pc, npg);
      int limit = Ls;
      if (p.causal) limit = Ls - p.s_q + row_query(p, pc.unit, row0 + r) + 1;
      float m_used = -INFINITY, l_sum = 0.f;
      int last_gp = -1;
      for (int pj = 2 * pc.t0; pj < pend && !stop; ++pj, ++gp) {
        const int b = gp & 1;
        // validity of the 64 keys of this page for this row (bit i of word w = key 32w + i)
        const int nv = max(0, min(kPage, limit - kPage * pj));
        const uint32_t vw0 = nv >= 32 ? 0xffffffffu : ((1u << max(nv, 0)) - 1u);
        const uint32_t vw1 = nv >= 64 ? 0xffffffffu : (nv <= 32 ? 0u : ((1u << (nv - 32)) - 1u));
        if (!timed_wait(c, &c->s_full[b], (gp >> 1) & 1, p)) { stop = true; break; }
        tc_fence_after();
        const uint32_t s_addr = tmem + lane_base + kTmemS + 64 * b;
        // pass 1: page max
        float tmax = -INFINITY;
#pragma unroll 1
        for (int w = 0; w < 2; ++w) {
          uint32_t sv[32];
          tmem_ld32(s_addr + 32 * w, sv);
          tmem_ld_wait();
          const uint32_t mw = w == 0 ? vw0 : vw1;
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
          need = (pj != 2 * pc.t0) && (m_used != -INFINITY);
          m_used = m_new;
          l_sum *= alpha;
        }
        // pass 2: probabilities (masked by select) -> bf16, staged in TMEM over
        // the S columns already read (tokens 32w.. -> columns 16w..)
        const float mc = (m_used == -INFINITY ? 0.f : m_used) * p.scale_log2;
        float part = 0.f;
#pragma unroll 1
        for (int w = 0; w < 2; ++w) {
          uint32_t sv[32];
          tmem_ld32(s_addr + 32 * w, sv);
          tmem_ld_wait();
          const uint32_t mw = rvalid ? (w == 0 ? vw0 : vw1) : 0u;
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
        if (need) c->rescale_flag[gp & 1] = 1;
        if (!group_sync(c, &c->grp_sm, gph, p)) { stop = true; break; }
        const bool do_rescale = *(volatile int*)&c->rescale_flag[gp & 1] != 0;
        // the O MMAs of the previous page must be complete before O^T is
        // rescaled and before P^T (which they read) is overwritten
        if (gp >= 1 && !timed_wait(c, &c->o_done, (gp - 1) & 1, p)) { stop = true; break; }
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
          if (threadIdx.x == 128) c->rescale_flag[gp & 1] = 0;
        }
        // P^T, K-major [NR rows][64 tokens], 8 tokens per 16-B chunk
#pragma unroll 1
        for (int w = 0; w < 2; ++w) {
          uint32_t pk[16];
          tmem_ld16(s_addr + 16 * w, pk);
          tmem_ld_wait();
          if (owner && r < NR) {
            uint8_t* rowp = sP + (r >> 3) * 1024 + (r & 7) * 128;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const int ch = 4 * w + q;
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
        last_gp = gp;
      }
      if (stop) break;
      // ---------------- epilogue of the piece
      if (last_gp >= 0 && !timed_wait(c, &c->o_done, last_gp & 1, p)) { stop = true; break; }
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

template <int NR, int MODE>
cudaError_t launch_page(const CUtensorMap& tq, const DecodeParams& p, int parts, int row_groups,
                        cudaStream_t stream) {
  constexpr int smem = Smem<NR>::total + 1024;
  auto kern = mla_decode_page_kernel<NR, MODE>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  e = launch_pdl(kern, dim3(parts, row_groups), dim3(kThreads), smem, stream, tq, p);
  return e != cudaSuccess ? e : cudaGetLastError();
}

template <int MODE>
cudaError_t launch_rows(int rows_per_cta, const CUtensorMap& tq, const DecodeParams& p, int parts, int row_groups,
                        cudaStream_t stream) {
  // <= 16 rows run in the 32-row kernel: the extra P^T rows are written as
  // zeros and their output rows are never stored
  if (rows_per_cta <= 32) return launch_page<32, MODE>(tq, p, parts, row_groups, stream);
  if (rows_per_cta <= 48) return launch_page<48, MODE>(tq, p, parts, row_groups, stream);
  return launch_page<64, MODE>(tq, p, parts, row_groups, stream);
}

}  // namespace

cudaError_t launch_decode_page(int mode, int rows_per_cta, const CUtensorMap& tq, const DecodeParams& p, int parts,
                               int row_groups, cudaStream_t stream) {
  if (mode == kModeNvfp4) return launch_rows<kModeNvfp4>(rows_per_cta, tq, p, parts, row_groups, stream);
  return launch_rows<kModeFp8>(rows_per_cta, tq, p, parts, row_groups, stream);
}

}  // namespace mla
