// Split-KV combine ("[flashinfer] ... NVFP4 DeepSeek-V4 decoding", section 3,
// cake_backend: a combine kernel merges the partial results of CTAs that split
// one request's KV). Each split s of a unit holds its own softmax-normalised
// partial output o_s and log-sum-exp lse_s over a disjoint subset of the keys:
//   lse = ln sum_s exp(lse_s),   out = sum_s exp(lse_s - lse) * o_s.
// With a per-head attention sink sigma (an extra logit with a zero value,
// "[flashinfer] ...", section 2), it joins here once per row, after the
// splits: lse' = ln(e^lse + e^sigma), out *= e^(lse - lse'); a unit with no
// split at all gets out 0 and lse sigma.
// Work items are (unit, chunk of 4 rows); a fixed grid of blocks strides over
// them, and an item whose unit was not split (its piece wrote the output
// directly) costs one read. Each half-block of 128 threads merges one row at
// a time, each thread owning 4 of the 512 dims. The kernel is launched with
// programmatic stream serialization and waits for the decode grid first.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "mla_kernels.cuh"
#include "sm100_ptx.cuh"

namespace mla {

constexpr int kCombineThreads = 256;
constexpr int kCombineRows = 4;  // rows per work item
constexpr int kCombineMaxBlocks = 8 * 148;

__global__ void __launch_bounds__(kCombineThreads) mla_combine_kernel(
    const float* __restrict__ part_lse, const float* __restrict__ part_o, const int32_t* __restrict__ split_ptr,
    int units, int rows, int h_q, const float* __restrict__ sink, __nv_bfloat16* __restrict__ out,
    float* __restrict__ lse) {
  griddep_wait();  // the decode grid's partial results are complete and visible
  const int half = threadIdx.x >> 7;
  const int d = (threadIdx.x & 127) * 4;
  const int chunks = (rows + kCombineRows - 1) / kCombineRows;
  for (int item = blockIdx.x; item < units * chunks; item += gridDim.x) {
    const int u = item / chunks, chunk = item - u * chunks;
    const int s0 = split_ptr[u], n = split_ptr[u + 1] - s0;
    if (n == 1) continue;  // written directly by the decode kernel
    const int r1 = min(rows, (chunk + 1) * kCombineRows);
    for (int r = chunk * kCombineRows + half; r < r1; r += 2) {
      const size_t orow = (size_t)u * rows + r;
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
      float L = -INFINITY;  // no split at all: an empty key set (out 0, lse -inf)
      if (n >= 2) {
        float m = -INFINITY;
        for (int s = 0; s < n; ++s) m = fmaxf(m, part_lse[(size_t)(s0 + s) * rows + r]);
        if (m != -INFINITY) {
          float sum = 0.f;
          for (int s = 0; s < n; ++s) sum += expf(part_lse[(size_t)(s0 + s) * rows + r] - m);
          L = m + logf(sum);
          for (int s = 0; s < n; ++s) {
            const float w = expf(part_lse[(size_t)(s0 + s) * rows + r] - L);
            const float4 o = *reinterpret_cast<const float4*>(part_o + ((size_t)(s0 + s) * rows + r) * kDv + d);
            acc.x += w * o.x; acc.y += w * o.y; acc.z += w * o.z; acc.w += w * o.w;
          }
        }
      }
      if (sink != nullptr) {
        const float f = fold_sink(L, sink[(int)(orow % h_q)]);
        acc.x *= f; acc.y *= f; acc.z *= f; acc.w *= f;
      }
      __nv_bfloat162 lo = __floats2bfloat162_rn(acc.x, acc.y);
      __nv_bfloat162 hi = __floats2bfloat162_rn(acc.z, acc.w);
      uint2 packed;
      packed.x = *reinterpret_cast<uint32_t*>(&lo);
      packed.y = *reinterpret_cast<uint32_t*>(&hi);
      *reinterpret_cast<uint2*>(out + orow * kDv + d) = packed;
      if ((threadIdx.x & 127) == 0) lse[orow] = L;
    }
  }
}

mla_status_t launch_combine(const void* workspace, int units, int rows, int parts, const int32_t* split_ptr,
                            int h_q, const float* sink, void* out, float* lse, cudaStream_t stream) {
  const WsLayout w = ws_layout(units, rows, parts);
  const char* ws = static_cast<const char*>(workspace);
  const long long items = (long long)units * ((rows + kCombineRows - 1) / kCombineRows);
  const int blocks = (int)(items < kCombineMaxBlocks ? items : kCombineMaxBlocks);
  const cudaError_t e = launch_pdl(mla_combine_kernel, dim3(blocks), dim3(kCombineThreads), 0, stream,
                                   reinterpret_cast<const float*>(ws + w.lse_off),
                                   reinterpret_cast<const float*>(ws + w.o_off), split_ptr, units, rows, h_q, sink,
                                   static_cast<__nv_bfloat16*>(out), lse);
  return (e == cudaSuccess && cudaGetLastError() == cudaSuccess) ? MLA_OK : MLA_ERR_CUDA;
}

}  // namespace mla
