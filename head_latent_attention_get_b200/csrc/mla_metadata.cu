// Split-KV tile scheduler ("get_mla_metadata": "Qu'est-ce que FlashMLA ?",
// section "Obtenir les métadonnées MLA" — computed once per decode step from
// cache_seqlens and reused by every layer).
//
// Every work unit (a block of at most 128 query rows of a request for paged
// decoding, a (request, query token) pair for sparse decoding) costs n_u tiles of 128 tokens plus a fixed
// overhead of kSchedOverhead tiles (loading Q, writing a partial result,
// combining). Units are laid end to end on a cost axis [0, total); part p
// takes the cost range [p*payload, (p+1)*payload) with payload =
// ceil(total / parts). Tile k of unit u sits at cost position
// C_u + overhead + k, so it belongs to part floor(position / payload): every
// tile lands in exactly one part, parts are contiguous in (unit, tile)
// order, and the number of parts touching unit u follows in closed form.
// A piece of a split unit costs more than the fixed overhead suggests (its
// partial result is written in fp32 and merged by the combine pass, and the
// pipeline refills), so when the largest unit costs at most kSplitPenalty
// tiles more than an even share, the payload is raised to that unit's cost:
// equal units then map one to a part and are never split.
// The cost axis is int32 (the prefix is stored in num_splits), so the sum of
// all tile counts plus overheads must stay below 2^31.
#include <cuda_runtime.h>

#include "mla_kernels.cuh"
#include "sm100_ptx.cuh"

namespace mla {

__host__ __device__ inline int unit_tiles(const int32_t* seqlens, int u, int upr, int topk) {
  if (topk > 0) return (topk + kTile - 1) / kTile;
  int L = seqlens[u / upr];
  return L > 0 ? (L + kTile - 1) / kTile : 0;
}

// position on the cost axis -> {unit, tile} of the first tile at or after it
__host__ __device__ inline int2 cost_to_tile(const int32_t* C, int U, int total, int x) {
  if (x >= total) return make_int2(U, 0);
  int lo = 0, hi = U - 1;  // last u with C[u] <= x (C non-decreasing, C[0] = 0)
  while (lo < hi) {
    int mid = (lo + hi + 1) >> 1;
    if (C[mid] <= x) lo = mid; else hi = mid - 1;
  }
  // zero-cost units share C with the next unit; the binary search lands on the
  // last unit with C[u] <= x, which is the one whose cost range contains x.
  const int local = x - C[lo] - kSchedOverhead;
  return make_int2(lo, local > 0 ? (int)local : 0);
}

constexpr int kSplitPenalty = 8;  // tiles

__host__ __device__ inline int choose_payload(int total, int parts, int max_cost) {
  if (total <= 0) return 1;
  const int even = (total + parts - 1) / parts;
  return (max_cost > even && max_cost <= even + kSplitPenalty) ? max_cost : even;
}

__host__ __device__ inline int first_part_of(int Cu, int payload) {
  return (int)((Cu + kSchedOverhead) / payload);
}

// Equal units of more than 64 rows. Their kernels (the CTA pair, or two
// row-group CTAs) run the keys in steps of two tiles, and every piece pays a
// pipeline fill and a partial-result write. When every unit has the same n
// tiles and there are at least two parts per unit, the cost-axis cut would
// hand some parts a run that ends half a step into a unit plus a second
// piece; instead each unit is cut into k = min(parts / units, ceil(n / 2))
// pieces of whole steps (as equal as steps allow), one piece per part, and
// the parts past k * units get no work. Returns k, or 0 when the cost-axis
// plan applies.
__host__ __device__ inline int equal_unit_pieces(int U, int parts, int rows, int n_min, int n_max) {
  if (rows <= 64 || U <= 0 || n_min != n_max || n_min <= 0) return 0;
  const int k = min(parts / U, (n_min + 1) / 2);
  return k >= 2 ? k : 0;
}
// Part p of the equal-unit plan: piece p % k of unit p / k, tiles
// [2 floor(j s / k), min(2 floor((j+1) s / k), n)) with s = ceil(n / 2) steps.
__host__ __device__ inline void equal_unit_part(int p, int U, int k, int n, int32_t* md) {
  const int steps = (n + 1) / 2;
  if (p >= U * k) {
    md[0] = U; md[1] = 0; md[2] = U; md[3] = 0; md[4] = 0;
  } else {
    const int u = p / k, j = p - u * k;
    md[0] = u; md[1] = 2 * (int)((long long)j * steps / k);
    md[2] = u; md[3] = min(n, 2 * (int)((long long)(j + 1) * steps / k));
    md[4] = p;  // the unit's splits are u*k .. u*k + k-1
  }
  md[5] = k; md[6] = 0; md[7] = 0;
}

// ---------------------------------------------------------------- host twin
extern "C" mla_status_t mla_get_metadata_host(const int32_t* cache_seqlens, int batch, int s_q, int h_q,
                                              int h_kv, int topk, int num_sm_parts, int32_t* tile_md,
                                              int32_t* num_splits) {
  if (!tile_md || !num_splits || batch <= 0 || s_q <= 0 || h_q <= 0 || h_kv <= 0 || num_sm_parts <= 0)
    return MLA_ERR_INVALID_ARG;
  if (topk < 0 || (topk > 0 && topk % 64 != 0)) return MLA_ERR_INVALID_ARG;
  if (topk == 0 && !cache_seqlens) return MLA_ERR_INVALID_ARG;
  if (h_kv != 1) return MLA_ERR_UNSUPPORTED;
  Geometry g;
  if (!unit_geometry(s_q, h_q, h_kv, topk, &g)) return MLA_ERR_UNSUPPORTED;
  const int U = batch * g.units_per_req;
  int n_min = 0x7fffffff, n_max = 0;
  for (int u = 0; u < U; ++u) {
    const int n = unit_tiles(cache_seqlens, u, g.units_per_req, topk);
    n_min = n < n_min ? n : n_min;
    n_max = n > n_max ? n : n_max;
  }
  const int k = equal_unit_pieces(U, num_sm_parts, g.rows, n_min, n_max);
  if (k > 0) {
    for (int p = 0; p < num_sm_parts; ++p) equal_unit_part(p, U, k, n_max, tile_md + p * MLA_TILE_MD_INTS);
    for (int u = 0; u <= U; ++u) num_splits[u] = u * k;
    return MLA_OK;
  }
  // cost prefix C[0..U] kept in num_splits first, then replaced by split pointers
  int total = 0, max_cost = 0;
  for (int u = 0; u < U; ++u) {
    num_splits[u] = (int32_t)total;
    int n = unit_tiles(cache_seqlens, u, g.units_per_req, topk);
    const int cost = n > 0 ? n + kSchedOverhead : 0;
    total += cost;
    max_cost = cost > max_cost ? cost : max_cost;
  }
  num_splits[U] = (int32_t)total;
  const int payload = choose_payload(total, num_sm_parts, max_cost);
  for (int p = 0; p < num_sm_parts; ++p) {
    const int2 b = cost_to_tile(num_splits, U, total, p * payload);
    const int2 e = cost_to_tile(num_splits, U, total, (p + 1) * payload);
    int32_t* md = tile_md + p * MLA_TILE_MD_INTS;
    md[0] = b.x; md[1] = b.y; md[2] = e.x; md[3] = e.y;
    md[4] = b.x < U ? p - first_part_of(num_splits[b.x], payload) : 0;
    md[5] = (int32_t)payload; md[6] = 0; md[7] = 0;
  }
  int32_t acc = 0;
  for (int u = 0; u < U; ++u) {
    const int Cu = num_splits[u];
    const int n = unit_tiles(cache_seqlens, u, g.units_per_req, topk);
    int ns = 0;
    if (n > 0) ns = (int)((Cu + kSchedOverhead + n - 1) / payload) - first_part_of(Cu, payload) + 1;
    num_splits[u] = acc;
    acc += ns;
  }
  num_splits[U] = acc;
  for (int p = 0; p < num_sm_parts; ++p) {
    int32_t* md = tile_md + p * MLA_TILE_MD_INTS;
    if (md[0] < U) md[4] += num_splits[md[0]];
  }
  return MLA_OK;
}

// ---------------------------------------------------------------- device kernel
constexpr int kMetaThreads = 256;

// returns {exclusive prefix of v over the block, block total}
__device__ int2 block_exclusive_scan(int v) {
  __shared__ int warp_sums[kMetaThreads / 32];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) warp_sums[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int w = lane < kMetaThreads / 32 ? warp_sums[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int y = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += y;
    }
    if (lane < kMetaThreads / 32) warp_sums[lane] = w;  // inclusive
  }
  __syncthreads();
  const int before = (warp > 0 ? warp_sums[warp - 1] : 0) + x - v;
  const int total = warp_sums[kMetaThreads / 32 - 1];
  __syncthreads();
  return make_int2(before, total);
}

__device__ int block_max(int v) {
  __shared__ int warp_max[kMetaThreads / 32];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = max(v, __shfl_xor_sync(0xffffffffu, v, o));
  if (lane == 0) warp_max[warp] = v;
  __syncthreads();
  int m = warp_max[0];
#pragma unroll
  for (int i = 1; i < kMetaThreads / 32; ++i) m = max(m, warp_max[i]);
  __syncthreads();
  return m;
}

// Equal-unit plan on the device (every thread of the block takes the same
// branch: n_min and n_max are block-wide). Returns true if it wrote the plan.
__device__ bool equal_unit_plan(const int32_t* seqlens, int U, int upr, int topk, int parts, int rows, int u0, int u1,
                                int32_t* tile_md, int32_t* num_splits) {
  int lo = 0x7fffffff, hi = 0;
  for (int u = u0; u < u1; ++u) {
    const int n = unit_tiles(seqlens, u, upr, topk);
    lo = min(lo, n);
    hi = max(hi, n);
  }
  const int n_max = block_max(hi);
  const int n_min = -block_max(-lo);
  const int k = equal_unit_pieces(U, parts, rows, n_min, n_max);
  if (k == 0) return false;
  for (int p = threadIdx.x; p < parts; p += kMetaThreads) equal_unit_part(p, U, k, n_max, tile_md + p * MLA_TILE_MD_INTS);
  for (int u = threadIdx.x; u <= U; u += kMetaThreads) num_splits[u] = u * k;
  return true;
}

__global__ void __launch_bounds__(kMetaThreads) mla_metadata_kernel(const int32_t* __restrict__ seqlens,
                                                                   int U, int upr, int topk, int parts, int rows,
                                                                   int32_t* __restrict__ tile_md,
                                                                   int32_t* __restrict__ num_splits) {
  griddep_launch_dependents();  // the decode kernel may start its set-up (it waits for this grid)
  griddep_wait();  // launched early behind the previous kernel: its reads of tile_md / num_splits are done
  __shared__ int s_payload;
  const int t = threadIdx.x;
  const int per = (U + kMetaThreads - 1) / kMetaThreads;
  const int u0 = min(U, t * per), u1 = min(U, u0 + per);
  if (equal_unit_plan(seqlens, U, upr, topk, parts, rows, u0, u1, tile_md, num_splits)) return;
  // 1. cost prefix C[u] -> num_splits[u], total -> num_splits[U]
  int my = 0, my_max = 0;
  for (int u = u0; u < u1; ++u) {
    int n = unit_tiles(seqlens, u, upr, topk);
    const int cost = n > 0 ? n + kSchedOverhead : 0;
    my += cost;
    my_max = max(my_max, cost);
  }
  const int max_cost = block_max(my_max);
  const int2 sc = block_exclusive_scan(my);
  const int total = sc.y;
  int c = sc.x;
  for (int u = u0; u < u1; ++u) {
    num_splits[u] = c;
    int n = unit_tiles(seqlens, u, upr, topk);
    c += n > 0 ? n + kSchedOverhead : 0;
  }
  if (t == 0) {
    num_splits[U] = total;
    s_payload = choose_payload(total, parts, max_cost);
  }
  __syncthreads();
  const int payload = s_payload;
  // 2. part boundaries (binary search on C)
  for (int p = t; p < parts; p += kMetaThreads) {
    const int2 b = cost_to_tile(num_splits, U, total, p * payload);
    const int2 e = cost_to_tile(num_splits, U, total, (p + 1) * payload);
    int32_t* md = tile_md + p * MLA_TILE_MD_INTS;
    md[0] = b.x; md[1] = b.y; md[2] = e.x; md[3] = e.y;
    md[4] = b.x < U ? p - first_part_of(num_splits[b.x], payload) : 0;
    md[5] = (int32_t)payload; md[6] = 0; md[7] = 0;
  }
  __syncthreads();
  // 3. splits per unit -> exclusive prefix in num_splits
  int mys = 0;
  for (int u = u0; u < u1; ++u) {
    const int Cu = num_splits[u];
    const int n = unit_tiles(seqlens, u, upr, topk);
    if (n > 0) mys += (int)((Cu + kSchedOverhead + n - 1) / payload) - first_part_of(Cu, payload) + 1;
  }
  const int2 ss = block_exclusive_scan(mys);
  const int tot_splits = ss.y;
  int sp = ss.x;
  for (int u = u0; u < u1; ++u) {
    const int Cu = num_splits[u];  // read before overwriting this slot
    const int n = unit_tiles(seqlens, u, upr, topk);
    int ns = 0;
    if (n > 0) ns = (int)((Cu + kSchedOverhead + n - 1) / payload) - first_part_of(Cu, payload) + 1;
    num_splits[u] = sp;
    sp += ns;
  }
  __syncthreads();
  if (t == 0) num_splits[U] = tot_splits;
  __syncthreads();
  // 4. workspace index of each part's first piece
  for (int p = t; p < parts; p += kMetaThreads) {
    int32_t* md = tile_md + p * MLA_TILE_MD_INTS;
    if (md[0] < U) md[4] += num_splits[md[0]];
  }
}

// Up to kMetaSmemUnits units, the cost prefix C and the split prefix S live
// in shared memory: the part boundaries are binary searches there, and every
// output is written once. Larger problems use the same steps with C kept in
// num_splits (global memory).
constexpr int kMetaSmemUnits = 4096;

__global__ void __launch_bounds__(kMetaThreads) mla_metadata_smem_kernel(const int32_t* __restrict__ seqlens,
                                                                        int U, int upr, int topk, int parts, int rows,
                                                                        int32_t* __restrict__ tile_md,
                                                                        int32_t* __restrict__ num_splits) {
  griddep_launch_dependents();  // the decode kernel may start its set-up (it waits for this grid)
  griddep_wait();  // launched early behind the previous kernel: its reads of tile_md / num_splits are done
  __shared__ int32_t C[kMetaSmemUnits + 1];  // cost prefix
  __shared__ int32_t S[kMetaSmemUnits + 1];  // split prefix
  __shared__ int s_payload;
  const int t = threadIdx.x;
  const int per = (U + kMetaThreads - 1) / kMetaThreads;
  const int u0 = min(U, t * per), u1 = min(U, u0 + per);
  if (equal_unit_plan(seqlens, U, upr, topk, parts, rows, u0, u1, tile_md, num_splits)) return;
  // 1. cost prefix C[0..U]
  int my = 0, my_max = 0;
  for (int u = u0; u < u1; ++u) {
    const int n = unit_tiles(seqlens, u, upr, topk);
    const int cost = n > 0 ? n + kSchedOverhead : 0;
    C[u] = cost;
    my += cost;
    my_max = max(my_max, cost);
  }
  const int max_cost = block_max(my_max);
  const int2 sc = block_exclusive_scan(my);
  int c = sc.x;
  for (int u = u0; u < u1; ++u) {
    const int cost = C[u];
    C[u] = c;
    c += cost;
  }
  if (t == 0) {
    C[U] = sc.y;
    s_payload = choose_payload(sc.y, parts, max_cost);
  }
  __syncthreads();
  const int total = sc.y, payload = s_payload;
  // 2. split counts -> split prefix S[0..U] (also the num_splits output)
  int mys = 0;
  for (int u = u0; u < u1; ++u) {
    const int n = C[u + 1] - C[u] - kSchedOverhead;  // tiles of unit u (cost 0: no tiles)
    const int ns = n > 0 ? (int)((C[u] + kSchedOverhead + n - 1) / payload) - first_part_of(C[u], payload) + 1 : 0;
    S[u] = ns;
    mys += ns;
  }
  const int2 ss = block_exclusive_scan(mys);
  int sp = ss.x;
  for (int u = u0; u < u1; ++u) {
    const int ns = S[u];
    S[u] = sp;
    num_splits[u] = sp;
    sp += ns;
  }
  if (t == 0) {
    S[U] = ss.y;
    num_splits[U] = ss.y;
  }
  __syncthreads();
  // 3. parts: boundaries by binary search on C, workspace index of the first piece
  for (int p = t; p < parts; p += kMetaThreads) {
    const int2 b = cost_to_tile(C, U, total, p * payload);
    const int2 e = cost_to_tile(C, U, total, (p + 1) * payload);
    const int ws = b.x < U ? p - first_part_of(C[b.x], payload) + S[b.x] : 0;
    int32_t* md = tile_md + p * MLA_TILE_MD_INTS;
    md[0] = b.x; md[1] = b.y; md[2] = e.x; md[3] = e.y;
    md[4] = ws; md[5] = payload; md[6] = 0; md[7] = 0;
  }
}

mla_status_t launch_metadata(const int32_t* seqlens, int U, int upr, int topk, int parts, int rows,
                             int32_t* tile_md, int32_t* num_splits, cudaStream_t stream) {
  // programmatic dependent launch: the block is scheduled while the previous
  // kernel of the stream (e.g. the last step's combine) finishes, and waits
  // for it before reading or writing anything
  const cudaError_t e =
      U <= kMetaSmemUnits
          ? launch_pdl(mla_metadata_smem_kernel, dim3(1), dim3(kMetaThreads), 0, stream, seqlens, U, upr, topk, parts,
                       rows, tile_md, num_splits)
          : launch_pdl(mla_metadata_kernel, dim3(1), dim3(kMetaThreads), 0, stream, seqlens, U, upr, topk, parts, rows,
                       tile_md, num_splits);
  return (e == cudaSuccess && cudaGetLastError() == cudaSuccess) ? MLA_OK : MLA_ERR_CUDA;
}

}  // namespace mla
