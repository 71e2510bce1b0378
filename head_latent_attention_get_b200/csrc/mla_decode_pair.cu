// MLA decode for units of 65-128 query rows (e.g. 128 heads, or a 128-row
// block of a request with more rows) on the BF16 cache, paged or
// token-sparse: one CTA pair (cluster of 2 CTAs on two SMs) per scheduler part.
//
// Same computation as mla_decode.cu -- per unit, softmax(scale * Q K^T) V with
// K = the 576-dim latent row and V = its first 512 dims ([flashinfer] ...
// NVFP4 DeepSeek-V4 decoding, README section; FlashMLA-ETAP summary, core
// mechanism) -- organised so that a 128-row unit is served by two SMs that
// share every cache byte instead of each reading all of it:
//
//   step = two consecutive 128-token tiles (256 tokens); CTA r loads
//          K of tile r (all 576 dims) and V of all 256 tokens for its value
//          dims {256j + 128r + [0,128) : j = 0,1}.
//   S = Q K^T   pair MMA M=128 (64 rows per CTA) x N=256 (128 tokens per CTA)
//               x K=576. Each CTA's TMEM receives its 64 rows x 256 tokens:
//               lanes 0-63 hold tokens 0-127, lanes 64-127 tokens 128-255.
//   softmax     thread (row, half) of the CTA reads its row's 128 scores of
//               token half `half`; the row max is agreed between the two
//               threads of a row through shared memory, once per step. The
//               probabilities go straight to the P buffer once the
//               previous step's O product has read it.
//   O = P V     pair MMA M=128 x N=256 (value dims, 128 per CTA) x K=256
//               tokens, twice (dims 0-255 and 256-511). P is this CTA's 64
//               rows (K-major); V is read MN-major straight from the
//               token-major cache rows. O stays in this CTA's TMEM (rows on
//               lanes), so rescaling is thread-local.
// TMEM per CTA: O 2 x 128 columns + S 2 x 128 columns = 512.
//
// Loads: one ring of 16 KB slots filled by TMA in exactly the order the MMA
// issuer consumes them -- K of step 0, then per step g: K of step g+1, V of
// step g -- so whichever product is being issued sees the whole ring as
// look-ahead. The MMA issuer follows the same order: S(0), S(1), O(0), S(2),
// O(1), ...
//
// Warp roles (256 threads per CTA; 320 with sparse indices):
//   0 Q (and, paged, K and V) via TMA (both CTAs; completion counted on the
//     even CTA's barriers)
//   1 TMEM allocation (both) and MMA issue (even CTA); sparse: forwarding of
//     the odd CTA's slot completions (odd CTA)
//   2, 3, 8, 9 sparse: row gathers with cp.async (both CTAs); a TMA row gather
//     moves only ~7 B/clk per SM, cp.async from four warps about 20
//   4-7 softmax + epilogue (both): thread i = (row i % 64, token half i / 64)
// All waits are bounded; a timeout sets MLA_DEVICE_STATUS_TIMEOUT, raises the
// abort flag of both CTAs, and every role winds down to the final cluster
// barrier, which both CTAs always reach.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "mla_decode_util.cuh"

namespace mla {
namespace pair {

constexpr int kN = 7;                // ring slots of 16 KB: a K slice (128 tokens x 64 dims)
                                     // or a V slot (64 tokens x 128 value dims, two 8 KB halves)
constexpr int kSlot = 16384;
constexpr int kThreads = 256;         // paged
constexpr int kThreadsSparse = 320;   // + four cp.async loader warps (2, 3, 8, 9)
constexpr int kQBytes = 9 * 8192;    // 64 rows x 576 dims
constexpr int kPBytes = 4 * 8192;    // 64 rows x 256 tokens (one buffer)
constexpr int kTmemCols = 512;
constexpr int kTmemS = 256;          // S buffers at columns 256 and 384; O at 0 and 128
constexpr float kRescaleLog2 = 8.0f;

struct Smem {
  static constexpr int q = 0;
  static constexpr int ring = q + kQBytes;
  static constexpr int pt = ring + kN * kSlot;
  static constexpr int ctrl = pt + kPBytes;
  static constexpr int total = ctrl + 2048;
};

struct Ctrl {
  // barriers counted on the even CTA (the MMA issuer) ...
  uint64_t q_full;                     // 1 arrival (+ both CTAs' Q bytes)
  uint64_t full[kN];                   // 1 arrival (+ both CTAs' bytes of the slot)
  uint64_t p_full[2], o_free;          // 8 arrivals: 4 softmax warps x 2 CTAs
  uint64_t drain;
  // ... and in each CTA
  uint64_t q_empty, empty[kN];         // pair-MMA commits
  uint64_t s_full[2], o_done[2];       // pair-MMA commits; o_done[g & 1] completes O of step g
  uint64_t v_fix;                      // local loads of partial pages
  uint64_t m_full[4];                  // sparse: key-validity mask of a step written (4 loader warps)
  uint64_t v_loc[kN];                  // sparse, odd CTA: its 128 loader threads
  uint64_t grp_sm;                     // 128 softmax threads
  uint32_t tmem_base;
  int abort_flag;
  float mx[2][2][64];                  // [step parity][token half][row]: per-half tile max
  float lx[2][64];                     // [token half][row]: per-half row sum
  __align__(16) uint32_t vmask[4][8];  // sparse: [step % 4][tile half * 4 + word]: bit s = key 32*word + s valid
};
static_assert(sizeof(Ctrl) <= 2048, "control block");

struct Pair {
  uint32_t rank;
  bool leader;
  Ctrl* c;
  uint32_t peer_abort;                 // cluster address of the other CTA's abort flag
};

__device__ __forceinline__ void raise_abort(const Pair& pr, const DecodeParams& p) {
  atomicOr(p.status, (uint32_t)MLA_DEVICE_STATUS_TIMEOUT);
  *(volatile int*)&pr.c->abort_flag = 1;
  st_cluster_u32(pr.peer_abort, 1u);
}

__device__ __forceinline__ bool aborted(const Pair& pr) { return *(volatile int*)&pr.c->abort_flag != 0; }

// Bounded wait with cluster-scope acquire (several barriers receive arrivals
// from the other CTA or pair-MMA commits).
__device__ __forceinline__ bool pwait(const Pair& pr, uint64_t* bar, uint32_t parity, const DecodeParams& p) {
  if (aborted(pr)) return false;
  if (mbar_wait_cluster(bar, parity, p.timeout_ns)) return true;
  raise_abort(pr, p);
  return false;
}

__device__ __forceinline__ bool group_sync(const Pair& pr, uint32_t& phase, const DecodeParams& p) {
  mbar_arrive(&pr.c->grp_sm);
  const bool ok = pwait(pr, &pr.c->grp_sm, phase & 1, p);
  ++phase;
  return ok;
}

// Arrive on barrier `bar` of the even CTA (a local arrive there, a remote one from the odd CTA).
__device__ __forceinline__ void arrive_leader(const Pair& pr, uint64_t* bar) {
  if (pr.leader) mbar_arrive(bar);
  else mbar_arrive_cluster(map_to_rank(smem_u32(bar), 0));
}

// Ring order of a piece of n steps: h = 0 -> K of step 0; h = 2g+1 -> K of
// step g+1 (only if g+1 < n); h = 2g+2 -> V of step g.
__device__ __forceinline__ bool ring_entry_exists(int h, int nsteps) { return !((h & 1) && (h >> 1) + 1 >= nsteps); }
__device__ __forceinline__ bool ring_entry_is_k(int h) { return h == 0 || (h & 1); }
__device__ __forceinline__ int ring_entry_step(int h) { return h == 0 ? 0 : (h & 1) ? (h >> 1) + 1 : (h >> 1) - 1; }

// Page ids of a request for one warp: lane l holds the id of logical page
// base + l, so a page is one shuffle away instead of a dependent global load.
// Every call is made by all 32 lanes with the same arguments.
struct PageWindow {
  int base = -1 << 30, mine = -1;
  __device__ __forceinline__ void cover(const DecodeParams& p, int req, int lo, int hi, int npg, int lane) {
    if (lo < base || hi > base + 32) {
      base = lo;
      mine = page_of(p, req, base + lane, npg);
    }
  }
  __device__ __forceinline__ int get(const DecodeParams& p, int req, int j, int npg, int lane) const {
    const int v = __shfl_sync(0xffffffffu, mine, (j - base) & 31);
    return (j >= base && j < base + 32) ? v : page_of(p, req, j, npg);
  }
};

// Sparse: cache row of index slot `slot` of unit `unit` (request b, whose
// cache holds L tokens), or -1 when the slot is ignored: -1 entries (silently),
// out-of-range indices and page ids (reported in the status word), slots past
// topk and slots of tiles outside the piece [.., t1).
__device__ __forceinline__ int sparse_slot_row(const DecodeParams& p, int unit, int b, int L, int slot, int t1) {
  if (slot / kTile >= t1 || slot >= p.topk) return -1;
  const int idx = p.indices[(size_t)unit * p.topk + slot];
  if (idx == -1) return -1;
  const int j = idx / kPage;
  if (idx < 0 || idx >= L || j >= p.bt_stride) {
    atomicOr(p.status, (uint32_t)MLA_DEVICE_STATUS_BOUNDS);
    return -1;
  }
  const int pg = p.block_table[(size_t)b * p.bt_stride + j];
  if (pg < 0 || pg >= p.num_pages) {
    atomicOr(p.status, (uint32_t)MLA_DEVICE_STATUS_BOUNDS);
    return -1;
  }
  return pg * kPage + idx % kPage;
}

template <bool SPARSE>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(SPARSE ? kThreadsSparse : kThreads, 1)
    mla_decode_pair_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_kv,
                           const __grid_constant__ CUtensorMap tm_v, const DecodeParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem + Smem::q;
  uint8_t* sRing = smem + Smem::ring;
  uint8_t* sP = smem + Smem::pt;
  Ctrl* c = reinterpret_cast<Ctrl*>(smem + Smem::ctrl);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  Pair pr;
  pr.rank = cluster_rank();
  pr.leader = pr.rank == 0;
  pr.c = c;
  pr.peer_abort = map_to_rank(smem_u32(&c->abort_flag), pr.rank ^ 1u);
  const int part = blockIdx.x >> 1;
  const int row0 = 64 * (int)pr.rank;   // first row of this CTA within a unit

  if (threadIdx.x == 0) {
    mbar_init(&c->q_full, 1);
    // paged: the even CTA's producer arrives with both CTAs' TMA bytes;
    // sparse: this CTA's 128 loader threads (cp.async) + one forward from the odd CTA
    for (int i = 0; i < kN; ++i) mbar_init(&c->full[i], SPARSE ? 129 : 1);
    for (int i = 0; i < 2; ++i) mbar_init(&c->p_full[i], 8);
    mbar_init(&c->o_free, 8);
    mbar_init(&c->drain, 1);
    mbar_init(&c->q_empty, 1);
    for (int i = 0; i < kN; ++i) mbar_init(&c->empty[i], 1);
    for (int i = 0; i < 2; ++i) mbar_init(&c->s_full[i], 1);
    for (int i = 0; i < 2; ++i) mbar_init(&c->o_done[i], 1);
    mbar_init(&c->v_fix, 1);
    for (int i = 0; i < 4; ++i) mbar_init(&c->m_full[i], 4);
    for (int i = 0; i < kN; ++i) mbar_init(&c->v_loc[i], 128);
    mbar_init(&c->grp_sm, 128);
    c->abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tm_q);
    if (!SPARSE) {  // the sparse path gathers rows with cp.async
      tma_prefetch_desc(&tm_kv);
      tma_prefetch_desc(&tm_v);
    }
  }
  if (warp == 1) {
    tmem_alloc_pair(&c->tmem_base, kTmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync_all();  // barriers initialised and TMEM allocated in both CTAs
  tc_fence_after();
  const uint32_t tmem = c->tmem_base;
  griddep_wait();  // the scheduler's output (and every input) is ready

  PieceIter it;
  it.init(p, part);
  Piece pc;

  if (warp == 0) {
    // ------------------------------------------------------------ producer: Q, then the ring in order
    int sc = 0, pi = 0, q_issued = 0, fixc = 0;
    bool stop = false;
    while (!stop && it.next(pc)) {
      if (lane == 0) {
        if (!pwait(pr, &c->q_empty, (pi & 1) ^ 1, p)) {
          stop = true;
        } else {
          const uint32_t qbar = map_to_rank(smem_u32(&c->q_full), 0);
          if (pr.leader) mbar_arrive_expect_tx(&c->q_full, 2 * kQBytes);
          const int qy = pc.unit * p.rows + row0;
          for (int j = 0; j < 9; ++j) tma_load_2d_pair(sQ + j * 8192, &tm_q, qbar, 64 * j, qy);
          ++q_issued;
        }
      }
      stop = __shfl_sync(0xffffffffu, stop ? 1 : 0, 0) != 0;
      const int req = unit_req(p, pc.unit);
      const int Ls = p.seqlens[req];
      const int npg = (Ls + kPage - 1) / kPage;
      const int nsteps = SPARSE ? 0 : (pc.t1 - pc.t0 + 1) >> 1;  // sparse rows: loader warps
      PageWindow pw;
      for (int h = 0; nsteps > 0 && h <= 2 * nsteps && !stop; ++h) {
        if (!ring_entry_exists(h, nsteps)) continue;
        const int k = pc.t0 + 2 * ring_entry_step(h);
        if (ring_entry_is_k(h)) {
          // own tile; past the piece's end the pair's other tile is loaded
          // again (its keys are masked)
          const int t = (k + (int)pr.rank < pc.t1) ? k + (int)pr.rank : k;
          // pages of the previous step's V through the next steps' K (no L2
          // prefetch: it would occupy this SM's TMA engine ahead of the loads)
          pw.cover(p, req, max(0, 2 * k - 4), 2 * k + 8, npg, lane);
          int pa = pw.get(p, req, 2 * t, npg, lane);
          int pb = pw.get(p, req, 2 * t + 1, npg, lane);
          if (pb < 0) pb = pa;
          for (int j = 0; j < 9; ++j, ++sc) {
            const int slot = sc % kN;
            uint8_t* dst = sRing + slot * kSlot;
            bool ok = true;
            if (lane == 0) {
              ok = pwait(pr, &c->empty[slot], ((sc / kN) & 1) ^ 1, p);
              if (ok) {
                const uint32_t bar = map_to_rank(smem_u32(&c->full[slot]), 0);
                if (pr.leader) mbar_arrive_expect_tx(&c->full[slot], 2 * kSlot);
                tma_load_2d_pair_hint(dst, &tm_kv, bar, 64 * j, pa * kPage, l2_policy_evict_last());
                tma_load_2d_pair_hint(dst + 8192, &tm_kv, bar, 64 * j, pb * kPage, l2_policy_evict_last());
              }
            }
            ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
            if (!ok) { stop = true; break; }
          }
        } else {
          // V: slot (q, jd) = page q of the step (tile k + q/2, page half
          // q%2), value dims 256*jd + 128*rank + [0,128) as two 64-dim halves
          for (int q = 0; q < 4 && !stop; ++q) {
            const int tile = k + (q >> 1), pj = 2 * tile + (q & 1);
            const int nv = tile < pc.t1 ? max(0, min(kPage, Ls - kPage * pj)) : 0;
            const int pg = nv > 0 ? pw.get(p, req, pj, npg, lane) : 0;
            for (int jd = 0; jd < 2; ++jd, ++sc) {
              const int slot = sc % kN;
              uint8_t* dst = sRing + slot * kSlot;
              bool ok = true;
              if (lane == 0) ok = pwait(pr, &c->empty[slot], ((sc / kN) & 1) ^ 1, p);
              ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
              if (!ok) { stop = true; break; }
              const int x0 = 256 * jd + 128 * (int)pr.rank;
              const uint32_t bar = map_to_rank(smem_u32(&c->full[slot]), 0);
              // the even CTA expects both CTAs' bytes of every slot
              if (lane == 0 && pr.leader) mbar_arrive_expect_tx(&c->full[slot], 2 * kSlot);
              if (nv == kPage) {
                if (lane == 0) {
                  tma_load_3d_pair_hint(dst, &tm_v, bar, 0, pg * kPage, x0 / 64, l2_policy_evict_first());
                }
              } else {
                // keys past the request's end have zero probability, but their
                // cache rows may hold anything (0 x NaN = NaN): load locally,
                // zero those rows, then report the slot's bytes as delivered
                if (nv > 0) {
                  if (lane == 0) {
                    mbar_arrive_expect_tx(&c->v_fix, kSlot);
                    tma_load_3d(dst, &tm_v, &c->v_fix, 0, pg * kPage, x0 / 64);
                    ok = pwait(pr, &c->v_fix, fixc & 1, p);
                  }
                  ++fixc;
                  ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
                  if (!ok) { stop = true; break; }
                }
                const uint4 z = make_uint4(0, 0, 0, 0);
                for (int i = nv * 8 + lane; i < kPage * 8; i += 32) {  // 8 chunks of 16 B per 128-B row
                  *reinterpret_cast<uint4*>(dst + i * 16) = z;
                  *reinterpret_cast<uint4*>(dst + 8192 + i * 16) = z;
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) {
                  fence_acq_rel_cluster();
                  mbar_complete_tx_cluster(bar, kSlot);
                }
              }
            }
          }
        }
      }
      ++pi;
    }
    if (lane == 0 && pr.leader) {  // the even CTA's barriers count both CTAs' copies
      if (q_issued > 0) mbar_wait_cluster(&c->q_full, (uint32_t)((q_issued - 1) & 1), p.timeout_ns);
      for (int i = sc > kN ? sc - kN : 0; i < sc; ++i)
        mbar_wait_cluster(&c->full[i % kN], (uint32_t)((i / kN) & 1), p.timeout_ns);
    }
    __syncwarp();
  } else if (SPARSE && (warp == 2 || warp == 3 || warp >= 8)) {
    // ------------------------------------------------------------ sparse: cp.async row gathers
    // Thread lt (0..127) owns index slot lt of each 128-slot tile: it copies
    // that key's row into the K slices of this CTA's tile and, for the V
    // slots, the keys 64q..64q+63 of the step that include it. Ignored slots
    // are zero-filled. Ring order as for the paged cache.
    const int lw = warp < 4 ? warp - 2 : warp - 6;
    const int lt = 32 * lw + lane;
    const uint8_t* cache = static_cast<const uint8_t*>(p.kcache);
    int sc = 0, gk = 0, gv = 0;
    int ra0 = -1, rb0 = -1, ra1 = -1, rb1 = -1;  // rows of tiles k, k+1 of steps with even / odd gk
    bool stop = false;
    while (!stop && it.next(pc)) {
      const int b = unit_req(p, pc.unit);
      const int L = p.seqlens[b];
      const int nsteps = (pc.t1 - pc.t0 + 1) >> 1;
      for (int h = 0; h <= 2 * nsteps && !stop; ++h) {
        if (!ring_entry_exists(h, nsteps)) continue;
        const int k = pc.t0 + 2 * ring_entry_step(h);
        if (ring_entry_is_k(h)) {
          const int ra = sparse_slot_row(p, pc.unit, b, L, kTile * k + lt, pc.t1);
          const int rb = sparse_slot_row(p, pc.unit, b, L, kTile * (k + 1) + lt, pc.t1);
          if (gk & 1) { ra1 = ra; rb1 = rb; } else { ra0 = ra; rb0 = rb; }
          const uint32_t va = __ballot_sync(0xffffffffu, ra >= 0), vb = __ballot_sync(0xffffffffu, rb >= 0);
          if (lane == 0) {
            c->vmask[gk & 3][lw] = va;
            c->vmask[gk & 3][4 + lw] = vb;
            mbar_arrive(&c->m_full[gk & 3]);  // the softmax of this step reads the mask
          }
          // K slice j of this CTA's tile: this warp copies its 32 keys' rows,
          // 8 lanes per 128-B row (row pointers of key 4i + lane/8 by shuffle)
          const int row = pr.rank ? rb : ra;
          const int ch = lane & 7;
          for (int j = 0; j < 9; ++j, ++sc) {
            const int slot = sc % kN;
            bool ok = true;
            if (lane == 0) ok = pwait(pr, &c->empty[slot], ((sc / kN) & 1) ^ 1, p);
            ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
            if (!ok) { stop = true; break; }
            uint8_t* base = sRing + slot * kSlot + (32 * lw) * 128;
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              const int key = 4 * i + (lane >> 3);  // key within this warp's 32
              const int r = __shfl_sync(0xffffffffu, row, key);
              const uint8_t* src = cache + (size_t)(r >= 0 ? r : 0) * (kDqk * 2) + 128 * j + 16 * ch;
              cp_async16(base + key * 128 + ((ch ^ (key & 7)) << 4), src, r >= 0 ? 16u : 0u);
            }
            cp_async_commit();
            cp_async_mbar_arrive_noinc(pr.leader ? &c->full[slot] : &c->v_loc[slot]);
          }
          ++gk;
        } else {
          const int ra = (gv & 1) ? ra1 : ra0, rb = (gv & 1) ? rb1 : rb0;
          for (int q = 0; q < 4 && !stop; ++q) {
            // V slot (q, jd): keys 64q..64q+63 of the step belong to warps
            // 2(q%2) and 2(q%2)+1 (lw); 16 lanes per key row (two 128-B halves)
            const bool mine = (lw >> 1) == (q & 1);
            const int row = (q >> 1) ? rb : ra;
            const int ch = lane & 7, hh = (lane >> 3) & 1;
            for (int jd = 0; jd < 2; ++jd, ++sc) {
              const int slot = sc % kN;
              bool ok = true;
              if (lane == 0) ok = pwait(pr, &c->empty[slot], ((sc / kN) & 1) ^ 1, p);
              ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
              if (!ok) { stop = true; break; }
              if (mine) {
                uint8_t* base = sRing + slot * kSlot + hh * 8192 + (32 * (lw & 1)) * 128;
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                  const int key = 2 * i + (lane >> 4);  // key within this warp's 32
                  const int r = __shfl_sync(0xffffffffu, row, key);
                  const uint8_t* src = cache + (size_t)(r >= 0 ? r : 0) * (kDqk * 2) + 256 * (int)pr.rank + 512 * jd +
                                       128 * hh + 16 * ch;
                  const int vrow = 32 * (lw & 1) + key;  // row within the 64-key slot
                  cp_async16(base + key * 128 + ((ch ^ (vrow & 7)) << 4), src, r >= 0 ? 16u : 0u);
                }
                cp_async_commit();
              }
              cp_async_mbar_arrive_noinc(pr.leader ? &c->full[slot] : &c->v_loc[slot]);
            }
          }
          ++gv;
        }
      }
    }
    cp_async_commit();
    cp_async_wait<0>();  // no copy may land after the CTA has finished
  } else if (SPARSE && warp == 1 && !pr.leader) {
    // ------------------------------------------------------------ sparse, odd CTA: forward slot completions
    if (lane == 0) {
      int sc = 0;
      bool stop = false;
      while (!stop && it.next(pc)) {
        const int nslots = 17 * ((pc.t1 - pc.t0 + 1) >> 1);  // 9 K slices + 8 V slots per step
        for (int i = 0; i < nslots; ++i, ++sc) {
          if (!pwait(pr, &c->v_loc[sc % kN], (sc / kN) & 1, p)) { stop = true; break; }
          // relaxed: a release arrive would first wait for this thread's
          // earlier memory operations (~0.8K clk after cp.async traffic
          // instead of ~0.1K); the data it signals has landed (v_loc)
          mbar_arrive_relaxed_cluster(map_to_rank(smem_u32(&c->full[sc % kN]), 0));
        }
      }
    }
    __syncwarp();
  } else if (warp == 1 && pr.leader) {
    // ------------------------------------------------------------ MMA issuer: S(0), S(1), O(0), S(2), O(1), ...
    const uint32_t idesc_s = idesc_bf16(128, 256, false, false);
    const uint32_t idesc_o = idesc_bf16(128, 256, false, true);
    int sc = 0, gs = 0, go = 0, pi = 0;
    bool stop = false;
    if (lane == 0) {
      while (!stop && it.next(pc)) {
        if (!pwait(pr, &c->q_full, pi & 1, p)) { stop = true; break; }
        const int nsteps = (pc.t1 - pc.t0 + 1) >> 1;
        for (int h = 0; h <= 2 * nsteps && !stop; ++h) {
          if (!ring_entry_exists(h, nsteps)) continue;
          const int g = ring_entry_step(h);
          if (ring_entry_is_k(h)) {
            // S buffer b was last read by the softmax of step gs - 2, whose
            // P the O product of step gs - 2 (issued just before) waited for
            const int b = gs & 1;
            tc_fence_after();
            const uint32_t d = tmem + kTmemS + 128 * b;
            for (int j = 0; j < 9; ++j, ++sc) {
              const int slot = sc % kN;
              if (!pwait(pr, &c->full[slot], (sc / kN) & 1, p)) { stop = true; break; }
              tc_fence_after();
              const uint32_t qa = smem_u32(sQ + j * 8192), kb = smem_u32(sRing + slot * kSlot);
#pragma unroll
              for (int kk = 0; kk < 4; ++kk)
                mma_bf16_ss_pair(d, sdesc(qa + kk * 32, 16, 1024), sdesc(kb + kk * 32, 16, 1024), idesc_s,
                                 (j | kk) != 0 ? 1u : 0u);
              mma_commit_pair(&c->empty[slot]);
            }
            if (stop) break;
            if (!(gs == 0 && (p.debug_flags & MLA_DEBUG_WITHHOLD_SCORES))) mma_commit_pair(&c->s_full[b]);
            ++gs;
            if (g == nsteps - 1) mma_commit_pair(&c->q_empty);  // Q is free once the last S completes
          } else {
            const bool first = g == 0;
            if (first && pi > 0 && !pwait(pr, &c->o_free, (pi - 1) & 1, p)) { stop = true; break; }
            if (!pwait(pr, &c->p_full[go & 1], (go >> 1) & 1, p)) { stop = true; break; }
            const uint32_t pt = smem_u32(sP);
            for (int q = 0; q < 4 && !stop; ++q) {
              for (int jd = 0; jd < 2; ++jd, ++sc) {
                const int slot = sc % kN;
                if (!pwait(pr, &c->full[slot], (sc / kN) & 1, p)) { stop = true; break; }
                tc_fence_after();
                const uint32_t va = smem_u32(sRing + slot * kSlot);
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                  mma_bf16_ss_pair(tmem + 128 * jd, sdesc(pt + q * 8192 + kk * 32, 16, 1024),
                                   sdesc(va + kk * 2048, 8192, 1024), idesc_o, (first && q == 0 && kk == 0) ? 0u : 1u);
                mma_commit_pair(&c->empty[slot]);
              }
            }
            if (stop) break;
            mma_commit_pair(&c->o_done[go & 1]);
            ++go;
          }
        }
        ++pi;
      }
      mma_commit_pair(&c->drain);  // every MMA this thread issued has completed before teardown
      mbar_wait(&c->drain, 0, p.timeout_ns);
    }
    __syncwarp();
  } else if (warp >= 4) {
    // ------------------------------------------------------------ softmax + epilogue
    const int ti = threadIdx.x - 128;                     // TMEM lane of this thread
    const int row = ti & 63, half = ti >> 6;
    const int grow = row0 + row;                          // row within the unit
    const bool rvalid = grow < p.rows;
    const uint32_t lane_base = (uint32_t)(32 * (warp - 4)) << 16;
    const float thresh = kRescaleLog2 / p.scale_log2;     // raw-score units
    uint32_t gph = 0;
    int gt = 0;
    bool stop = false;
    while (!stop && it.next(pc)) {
      const int req = unit_req(p, pc.unit);
      const int Ls = p.seqlens[req];
      const int limit = p.causal ? Ls - p.s_q + row_query(p, pc.unit, grow) + 1 : Ls;
      float m_used = -INFINITY, l_sum = 0.f;
      int last_gt = -1;
      for (int k = pc.t0; k < pc.t1 && !stop; k += 2, ++gt) {
        const int b = gt & 1;
        // validity of this thread's 128 keys: bit i of word w = key 32w + i
        uint4 vm;
        if (SPARSE) {
          if (!pwait(pr, &c->m_full[gt & 3], (gt >> 2) & 1, p)) { stop = true; break; }
          vm = rvalid ? *reinterpret_cast<const uint4*>(&c->vmask[gt & 3][4 * half]) : make_uint4(0, 0, 0, 0);
        } else {
          const int tile = k + half;
          const int nv = (rvalid && tile < pc.t1) ? dense_tile_valid(limit, tile) : 0;
          auto word = [nv](int w) {
            const int nb = min(32, max(0, nv - 32 * w));
            return nb >= 32 ? 0xffffffffu : ((1u << nb) - 1u);
          };
          vm = make_uint4(word(0), word(1), word(2), word(3));
        }
        if (!pwait(pr, &c->s_full[b], (gt >> 1) & 1, p)) { stop = true; break; }
        tc_fence_after();
        const uint32_t s_addr = tmem + lane_base + kTmemS + 128 * b;
        // pass 1: max over this thread's 128 keys
        float tmax = -INFINITY;
#pragma unroll 1
        for (int w = 0; w < 4; ++w) {
          uint32_t sv[32];
          tmem_ld32(s_addr + 32 * w, sv);
          tmem_ld_wait();
          const uint32_t mw = pick4u(vm, w);
#pragma unroll
          for (int i = 0; i < 32; ++i) tmax = fmaxf(tmax, ((mw >> i) & 1u) ? __uint_as_float(sv[i]) : -INFINITY);
        }
        c->mx[gt & 1][half][row] = tmax;
        if (!group_sync(pr, gph, p)) { stop = true; break; }
        tmax = fmaxf(tmax, c->mx[gt & 1][half ^ 1][row]);
        // both threads of a row take the same decision from the same values
        float alpha = 1.f;
        bool need = false;
        if (tmax > m_used + thresh || (m_used == -INFINITY && tmax > -INFINITY)) {
          alpha = (m_used == -INFINITY) ? 0.f : ex2_approx((m_used - tmax) * p.scale_log2);
          need = (k != pc.t0) && (m_used != -INFINITY);
          m_used = tmax;
          l_sum *= alpha;
        }
        // pass 2: probabilities (masked by select) -> bf16 -> the P buffer,
        // K-major [64 rows][64 keys] per slice: keys 64s.. in slice s; this
        // thread's keys are 128*half + [0,128), slices 2*half and 2*half + 1.
        // The single P buffer was last read by the O product of step gt - 1,
        // which must also be complete before O is rescaled. (O of step gt + 1,
        // the next completion of the same barrier, needs this thread's P, so
        // the parity wait never falls two phases behind.) Half of the
        // probabilities are computed into registers while that product runs.
        const float mc = (m_used == -INFINITY ? 0.f : m_used) * p.scale_log2;
        float part = 0.f;
        auto probs = [&](int w, uint32_t (&pk)[16]) {
          uint32_t sv[32];
          tmem_ld32(s_addr + 32 * w, sv);
          tmem_ld_wait();
          const uint32_t mw = pick4u(vm, w);
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const float e0 = ex2_approx(fmaf(__uint_as_float(sv[2 * i]), p.scale_log2, -mc));
            const float e1 = ex2_approx(fmaf(__uint_as_float(sv[2 * i + 1]), p.scale_log2, -mc));
            const float p0 = ((mw >> (2 * i)) & 1u) ? e0 : 0.f;
            const float p1 = ((mw >> (2 * i + 1)) & 1u) ? e1 : 0.f;
            pk[i] = pack_bf16x2(p0, p1);
            part += p0 + p1;
          }
        };
        auto store = [&](int w, const uint32_t (&pk)[16]) {
          uint8_t* rowp = sP + (2 * half + (w >> 1)) * 8192 + (row >> 3) * 1024 + (row & 7) * 128;
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const int ch = 4 * (w & 1) + q;
            *reinterpret_cast<uint4*>(rowp + ((ch ^ (row & 7)) << 4)) =
                make_uint4(pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
          }
        };
        {
          uint32_t pk[2][16];
#pragma unroll
          for (int w = 0; w < 2; ++w) probs(w, pk[w]);
          if (gt >= 1 && !pwait(pr, &c->o_done[(gt - 1) & 1], ((gt - 1) >> 1) & 1, p)) { stop = true; break; }
#pragma unroll
          for (int w = 0; w < 2; ++w) store(w, pk[w]);
#pragma unroll 1
          for (int w = 2; w < 4; ++w) {
            probs(w, pk[0]);
            store(w, pk[0]);
          }
        }
        tc_fence_after();
        l_sum += part;
        if (need) {
          // O holds every product up to step gt - 1 (waited for above)
#pragma unroll 1
          for (int c16 = 0; c16 < 16; ++c16) {  // 2 x 128 columns of this row
            uint32_t ov[16];
            const uint32_t a = tmem + lane_base + 16 * c16;
            tmem_ld16(a, ov);
            tmem_ld_wait();
#pragma unroll
            for (int i = 0; i < 16; ++i) ov[i] = __float_as_uint(__uint_as_float(ov[i]) * alpha);
            tmem_st16(a, ov);
          }
          tmem_st_wait();
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) arrive_leader(pr, &c->p_full[b]);  // P written, O rescaled, scores consumed
        last_gt = gt;
      }
      if (stop) break;
      // ---------------- epilogue of the piece
      c->lx[half][row] = l_sum;
      if (!group_sync(pr, gph, p)) { stop = true; break; }
      const float l_tot = l_sum + c->lx[half ^ 1][row];
      if (last_gt >= 0 && !pwait(pr, &c->o_done[last_gt & 1], (last_gt >> 1) & 1, p)) { stop = true; break; }
      tc_fence_after();
      float inv = 0.f, lse = -INFINITY;
      if (l_tot > 0.f) {
        inv = 1.f / l_tot;
        lse = m_used * p.scale + logf(l_tot);
      }
      if (pc.single && rvalid && p.sink != nullptr) inv *= fold_sink(lse, p.sink[row_head(p, pc.unit, grow)]);
      const size_t orow = (size_t)pc.unit * p.rows + grow;
      if (rvalid && half == 0) {
        if (pc.single) p.lse[orow] = lse;
        else p.ws_lse[(size_t)pc.ws_idx * p.rows + grow] = lse;
      }
#pragma unroll 1
      for (int jd = 0; jd < 2; ++jd) {
        const int d0 = 256 * jd + 128 * half;
#pragma unroll 1
        for (int c16 = 0; c16 < 8; ++c16) {
          uint32_t ov[16];
          tmem_ld16(tmem + lane_base + 128 * jd + 16 * c16, ov);
          tmem_ld_wait();
          if (rvalid) {
            if (pc.single) {
              uint32_t pk[8];
#pragma unroll
              for (int i = 0; i < 8; ++i)
                pk[i] = pack_bf16x2(__uint_as_float(ov[2 * i]) * inv, __uint_as_float(ov[2 * i + 1]) * inv);
              uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.out) + orow * kDv + d0 + 16 * c16);
              dst[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
              dst[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
            } else {
              float4* dst = reinterpret_cast<float4*>(p.ws_o + ((size_t)pc.ws_idx * p.rows + grow) * kDv + d0 + 16 * c16);
#pragma unroll
              for (int i = 0; i < 4; ++i)
                dst[i] = make_float4(__uint_as_float(ov[4 * i]) * inv, __uint_as_float(ov[4 * i + 1]) * inv,
                                     __uint_as_float(ov[4 * i + 2]) * inv, __uint_as_float(ov[4 * i + 3]) * inv);
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) arrive_leader(pr, &c->o_free);
    }
  }

  // ---------------------------------------------------------------- teardown
  // In a normal exit every copy has landed: each slot and Q phase was
  // consumed by the MMA issuer, and the producer drained its last phases.
  // After an abort (a bounded wait ran out), a copy this CTA issued may still
  // be in flight, and when its completion is counted on the other CTA's
  // barrier no wait here can observe it. Such copies read resident cache
  // pages and land within microseconds, so the CTA holds its shared memory
  // for a fixed 200 us of wall time (%globaltimer, not a sleep hint that may
  // return early) before the final cluster barrier; this bounds the window,
  // it does not prove every copy landed.
  if (aborted(pr)) {
    const uint64_t t0 = global_timer_ns();
    while (global_timer_ns() - t0 < 200000) {
    }
  }
  griddep_launch_dependents();  // the combine may be scheduled (it waits for this grid)
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // no pair MMA, copy or remote arrive of either CTA is still pending
  tc_fence_after();
  if (warp == 1) tmem_dealloc_pair(tmem, kTmemCols);
}

}  // namespace pair

cudaError_t launch_decode_pair(const CUtensorMap& tq, const CUtensorMap& tkv, const CUtensorMap& tv,
                               const DecodeParams& p, int parts, bool sparse, cudaStream_t stream) {
  constexpr int smem = pair::Smem::total + 1024;
  auto kern = sparse ? pair::mla_decode_pair_kernel<true> : pair::mla_decode_pair_kernel<false>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  e = launch_pdl(kern, dim3(2 * parts), dim3(sparse ? pair::kThreadsSparse : pair::kThreads), smem, stream, tq, tkv, tv, p);
  return e != cudaSuccess ? e : cudaGetLastError();
}

int max_pair_clusters() {
  constexpr int smem = pair::Smem::total + 1024;
  auto kern = pair::mla_decode_pair_kernel<false>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess) return 0;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2, 1, 1);
  cfg.blockDim = dim3(pair::kThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cudaLaunchAttribute attr;
  attr.id = cudaLaunchAttributeClusterDimension;
  attr.val.clusterDim.x = 2;
  attr.val.clusterDim.y = 1;
  attr.val.clusterDim.z = 1;
  cfg.attrs = &attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess) return 0;
  return n;
}

}  // namespace mla
