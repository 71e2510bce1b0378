// The steps on either side of the attention ("deepseek-ai/FlashMLA"
// (agentlenshq), feature list: one fused launch runs Q-norm, RoPE, the
// attention, the output-side conjugate RoPE and the final FP8 cast):
//
//   mla_q_norm_rope   q' = RMS-norm(q) * gamma, then the last 64 dims of each
//                     query row rotated pair-wise, (x[2i], x[2i+1]) by the
//                     query token's angle theta_i: (x0 c - x1 s, x0 s + x1 c).
//   mla_out_rope_fp8  the output's RoPE part (the dims of V inside the last 64
//                     of d_qk: none for 576-dim rows, 448..511 for 512-dim
//                     rows) rotated back by theta_i, then cast to e4m3 per
//                     128-value tile: scale = amax / 448 (1 if amax = 0),
//                     code = RNE(value / scale) saturated to +-448. Products,
//                     sums and quotients are rounded once each in fp32 (no
//                     contraction), so the codes are a function of the inputs.
//
// Both are HBM-bound row maps: one warp per row, coalesced 4-byte (query) and
// 32-byte (output) accesses per lane.
#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>

#include "mla_kernels.cuh"

namespace mla {

constexpr int kRopeDims = 64;
constexpr int kPrePostThreads = 256;  // 8 rows per block

// ---------------------------------------------------------------- query: RMS-norm + RoPE
// Lane l holds pairs l + 32 k (k < d/64) of its row: for d = 576 the last of
// them (pairs 256..287) is the RoPE part, for d = 512 pairs 224..255; either
// way lane l's last pair is RoPE pair l.
template <int D>
__global__ void __launch_bounds__(kPrePostThreads) q_norm_rope_kernel(
    const __nv_bfloat162* __restrict__ q, __nv_bfloat162* __restrict__ q_out, int rows, int rows_per_token,
    const float* __restrict__ gamma, float eps, const float* __restrict__ cos_t, const float* __restrict__ sin_t) {
  constexpr int kPairs = D / 64;  // pairs per lane
  const int lane = threadIdx.x & 31;
  const int row = blockIdx.x * (kPrePostThreads / 32) + (threadIdx.x >> 5);
  if (row >= rows) return;
  const __nv_bfloat162* src = q + (size_t)row * (D / 2);
  float2 v[kPairs];
  float ss = 0.f;
#pragma unroll
  for (int k = 0; k < kPairs; ++k) {
    v[k] = __bfloat1622float2(src[lane + 32 * k]);
    ss = fmaf(v[k].x, v[k].x, fmaf(v[k].y, v[k].y, ss));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  const float r = rsqrtf(ss / (float)D + eps);
  const float2* g2 = reinterpret_cast<const float2*>(gamma);
  __nv_bfloat162* dst = q_out + (size_t)row * (D / 2);
  const int tok = row / rows_per_token;  // [batch * s_q] query token of this row
#pragma unroll
  for (int k = 0; k < kPairs; ++k) {
    const float2 g = g2[lane + 32 * k];
    float y0 = v[k].x * r * g.x, y1 = v[k].y * r * g.y;
    if (k == kPairs - 1) {
      const float c = cos_t[tok * (kRopeDims / 2) + lane], s = sin_t[tok * (kRopeDims / 2) + lane];
      const float t0 = y0 * c - y1 * s;
      y1 = y0 * s + y1 * c;
      y0 = t0;
    }
    dst[lane + 32 * k] = __floats2bfloat162_rn(y0, y1);
  }
}

// ---------------------------------------------------------------- output: conjugate RoPE + e4m3 cast
// Lane l holds dims 16l..16l+15 of its 512-dim row; tile j = lanes 8j..8j+7.
__global__ void __launch_bounds__(kPrePostThreads) out_rope_fp8_kernel(
    const uint4* __restrict__ out, int rows, int rows_per_token, int rope_lo, const float* __restrict__ cos_t,
    const float* __restrict__ sin_t, uint4* __restrict__ out_fp8, float* __restrict__ out_scale) {
  const int lane = threadIdx.x & 31;
  const int row = blockIdx.x * (kPrePostThreads / 32) + (threadIdx.x >> 5);
  if (row >= rows) return;
  const uint4* src = out + (size_t)row * (kDv * 2 / 16) + 2 * lane;
  const uint4 a = src[0], b = src[1];
  const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
  float y[16];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[i]));
    y[2 * i] = f.x;
    y[2 * i + 1] = f.y;
  }
  const int d0 = 16 * lane;
  if (d0 >= rope_lo) {  // conjugate rotation: (x0 c + x1 s, x1 c - x0 s)
    const int tok = row / rows_per_token;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int pr = (d0 - rope_lo) / 2 + i;
      const float c = cos_t[tok * (kRopeDims / 2) + pr], s = sin_t[tok * (kRopeDims / 2) + pr];
      const float x0 = y[2 * i], x1 = y[2 * i + 1];
      y[2 * i] = __fadd_rn(__fmul_rn(x0, c), __fmul_rn(x1, s));
      y[2 * i + 1] = __fsub_rn(__fmul_rn(x1, c), __fmul_rn(x0, s));
    }
  }
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(y[i]));
#pragma unroll
  for (int o = 1; o < 8; o <<= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  const float scale = amax > 0.f ? __fdiv_rn(amax, 448.f) : 1.f;
  uint32_t pk[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    uint32_t v = 0;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const __nv_fp8_storage_t c8 = __nv_cvt_float_to_fp8(__fdiv_rn(y[4 * i + j], scale), __NV_SATFINITE, __NV_E4M3);
      v |= (uint32_t)c8 << (8 * j);
    }
    pk[i] = v;
  }
  out_fp8[(size_t)row * (kDv / 16) + lane] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
  if ((lane & 7) == 0) out_scale[(size_t)row * (kDv / 128) + (lane >> 3)] = scale;
}

}  // namespace mla

using namespace mla;

namespace {
bool al16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
}  // namespace

extern "C" mla_status_t mla_q_norm_rope(const void* q, void* q_out, int batch, int s_q, int h_q, int d_qk,
                                        const float* gamma, float eps, const float* rope_cos,
                                        const float* rope_sin, mla_stream_t stream) {
  if (!q || !q_out || !gamma || !rope_cos || !rope_sin || batch <= 0 || s_q <= 0 || h_q <= 0)
    return MLA_ERR_INVALID_ARG;
  if (d_qk != kDqk && d_qk != kNvfp4D) return MLA_ERR_INVALID_ARG;
  if (!al16(q) || !al16(q_out) || (reinterpret_cast<uintptr_t>(gamma) & 7u) != 0 || !(eps >= 0.f))
    return MLA_ERR_INVALID_ARG;
  if ((long long)batch * s_q * h_q > 0x7fffffff) return MLA_ERR_UNSUPPORTED;
  const int rows = batch * s_q * h_q;
  const dim3 grid((rows + kPrePostThreads / 32 - 1) / (kPrePostThreads / 32));
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const auto* qi = static_cast<const __nv_bfloat162*>(q);
  auto* qo = static_cast<__nv_bfloat162*>(q_out);
  if (d_qk == kDqk)
    q_norm_rope_kernel<kDqk><<<grid, kPrePostThreads, 0, s>>>(qi, qo, rows, h_q, gamma, eps, rope_cos, rope_sin);
  else
    q_norm_rope_kernel<kNvfp4D><<<grid, kPrePostThreads, 0, s>>>(qi, qo, rows, h_q, gamma, eps, rope_cos, rope_sin);
  return cudaGetLastError() == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
}

extern "C" mla_status_t mla_out_rope_fp8(const void* out, int batch, int s_q, int h_q, int d_qk,
                                         const float* rope_cos, const float* rope_sin, void* out_fp8,
                                         float* out_scale, mla_stream_t stream) {
  if (!out || !out_fp8 || !out_scale || batch <= 0 || s_q <= 0 || h_q <= 0) return MLA_ERR_INVALID_ARG;
  if (d_qk != kDqk && d_qk != kNvfp4D) return MLA_ERR_INVALID_ARG;
  const int rope_lo = d_qk - kRopeDims;  // 512 (no RoPE dims in the output) or 448
  if (rope_lo < kDv && (!rope_cos || !rope_sin)) return MLA_ERR_INVALID_ARG;
  if (!al16(out) || !al16(out_fp8) || (reinterpret_cast<uintptr_t>(out_scale) & 3u) != 0)
    return MLA_ERR_INVALID_ARG;
  if ((long long)batch * s_q * h_q > 0x7fffffff) return MLA_ERR_UNSUPPORTED;
  const int rows = batch * s_q * h_q;
  const dim3 grid((rows + kPrePostThreads / 32 - 1) / (kPrePostThreads / 32));
  out_rope_fp8_kernel<<<grid, kPrePostThreads, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      static_cast<const uint4*>(out), rows, h_q, rope_lo, rope_cos, rope_sin, static_cast<uint4*>(out_fp8),
      out_scale);
  return cudaGetLastError() == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
}
