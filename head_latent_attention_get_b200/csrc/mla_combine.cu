// Split-KV combine ("[flashinfer] ... NVFP4 DeepSeek-V4 decoding", section 3,
// cake_backend: a combine kernel merges the partial results of CTAs that split
// one request's KV). Each split s of a unit holds its own softmax-normalised
// partial output o_s and log-sum-exp lse_s over a disjoint subset of the keys:
//   lse = ln sum_s exp(lse_s),   out = sum_s exp(lse_s - lse) * o_s.
// With a per-head attention sink sigma (an extra logit with a zero value,
// "[flashinfer] ...", section 2), it joins here once per row, after the
// splits: lse' = ln(e^lse + e^sigma), out *= e^(lse - lse'); a unit with no
// split at all gets out 0 and lse sigma.
// One warp merges one output row: every lane walks the row's splits in order
// (the lse values are broadcast loads) and owns 16 of the 512 dims, so each
// split's partial row is read with coalesced 16-byte loads (the first two
// splits' rows are requested together with the lse values); a row whose unit
// was not split (its piece wrote the output directly) costs one read. A fixed
// grid of 8 blocks per SM strides over the rows. The kernel is launched with
// programmatic stream serialization and waits for the decode grid first.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "mla_kernels.cuh"
#include "sm100_ptx.cuh"

namespace mla {

constexpr int kCombineThreads = 256;                 // 8 warps: 8 rows at a time
constexpr int kCombineRowsPerBlock = kCombineThreads / 32;
constexpr int kCombineBlocksPerSm = 8;

__global__ void __launch_bounds__(kCombineThreads) mla_combine_kernel(
    const float* __restrict__ part_lse, const float* __restrict__ part_o, const int32_t* __restrict__ split_ptr,
    int units, int rows, int h_q, const float* __restrict__ sink, __nv_bfloat16* __restrict__ out,
    float* __restrict__ lse) {
  griddep_wait();  // the decode grid's partial results are complete and visible
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int total = units * rows;  // < 2^31: the host rejects larger problems
  for (int gr = blockIdx.x * kCombineRowsPerBlock + warp; gr < total; gr += gridDim.x * kCombineRowsPerBlock) {
    const int u = gr / rows, r = gr - u * rows;
    const int s0 = split_ptr[u], n = split_ptr[u + 1] - s0;
    if (n == 1) continue;  // written directly by the decode kernel
    float4 acc[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) acc[i] = make_float4(0.f, 0.f, 0.f, 0.f);
    float L = -INFINITY;  // no split at all: an empty key set (out 0, lse -inf)
    if (n >= 2) {
      // split s of the row: lse at lse_u[s * rows], partial row at o_u[s * o_stride]
      const float* lse_u = part_lse + (size_t)s0 * rows + r;
      const float4* o_u = reinterpret_cast<const float4*>(part_o + ((size_t)s0 * rows + r) * kDv) + lane;
      const size_t o_stride = (size_t)rows * (kDv / 4);
      // the first two partial rows are requested with the lse values (most
      // split units have two pieces), not after the weights are known
      float4 o0[4], o1[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        o0[i] = o_u[32 * i];
        o1[i] = o_u[o_stride + 32 * i];
      }
      float m = -INFINITY;
      for (int s = 0; s < n; ++s) m = fmaxf(m, lse_u[(size_t)s * rows]);
      if (m != -INFINITY) {
        float sum = 0.f;
        for (int s = 0; s < n; ++s) sum += expf(lse_u[(size_t)s * rows] - m);
        L = m + logf(sum);
        // splits in order, acc += w_s o_s from zero
        const float w0 = expf(lse_u[0] - L), w1 = expf(lse_u[rows] - L);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          acc[i].x += w0 * o0[i].x; acc[i].y += w0 * o0[i].y; acc[i].z += w0 * o0[i].z; acc[i].w += w0 * o0[i].w;
          acc[i].x += w1 * o1[i].x; acc[i].y += w1 * o1[i].y; acc[i].z += w1 * o1[i].z; acc[i].w += w1 * o1[i].w;
        }
        for (int s = 2; s < n; ++s) {
          const float w = expf(lse_u[(size_t)s * rows] - L);
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const float4 o = o_u[s * o_stride + 32 * i];
            acc[i].x += w * o.x; acc[i].y += w * o.y; acc[i].z += w * o.z; acc[i].w += w * o.w;
          }
        }
      }
    }
    if (sink != nullptr) {
      const float f = fold_sink(L, sink[(int)(gr % h_q)]);
#pragma unroll
      for (int i = 0; i < 4; ++i) { acc[i].x *= f; acc[i].y *= f; acc[i].z *= f; acc[i].w *= f; }
    }
    uint2* dst = reinterpret_cast<uint2*>(out + (size_t)gr * kDv);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      __nv_bfloat162 lo = __floats2bfloat162_rn(acc[i].x, acc[i].y);
      __nv_bfloat162 hi = __floats2bfloat162_rn(acc[i].z, acc[i].w);
      dst[lane + 32 * i] = make_uint2(*reinterpret_cast<uint32_t*>(&lo), *reinterpret_cast<uint32_t*>(&hi));
    }
    if (lane == 0) lse[gr] = L;
  }
}

mla_status_t launch_combine(const void* workspace, int units, int rows, int parts, const int32_t* split_ptr,
                            int h_q, const float* sink, void* out, float* lse, cudaStream_t stream) {
  const WsLayout w = ws_layout(units, rows, parts);
  const char* ws = static_cast<const char*>(workspace);
  int sms = 148;
  int dev = 0;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const long long blocks_needed = ((long long)units * rows + kCombineRowsPerBlock - 1) / kCombineRowsPerBlock;
  const long long cap = (long long)kCombineBlocksPerSm * (sms > 0 ? sms : 148);
  const int blocks = (int)(blocks_needed < cap ? blocks_needed : cap);
  const cudaError_t e = launch_pdl(mla_combine_kernel, dim3(blocks > 0 ? blocks : 1), dim3(kCombineThreads), 0, stream,
                                   reinterpret_cast<const float*>(ws + w.lse_off),
                                   reinterpret_cast<const float*>(ws + w.o_off), split_ptr, units, rows, h_q, sink,
                                   static_cast<__nv_bfloat16*>(out), lse);
  return (e == cudaSuccess && cudaGetLastError() == cudaSuccess) ? MLA_OK : MLA_ERR_CUDA;
}

}  // namespace mla
