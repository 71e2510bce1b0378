// Paged decoding with a built-in workspace, for callers that cannot allocate
// device memory when they decode.
//
// Some callers cannot call cudaMalloc at the point where they decode: a
// serving process that reserved all device memory for its own pool at start-up
// and forbids further allocations, or a latency-critical step that must not
// pay for cudaMalloc/cudaFree (their implicit device synchronisation and
// unpredictable latency). mla_decode_paged_noalloc gives them the same paged
// decode without a caller-owned workspace: the split-KV partial results and
// the device status word live in one file-scope device array of fixed size.
//
// The array is held by every GPU that loads this library until the process
// exits. It is shared by all calls on a device and keeps the contents of the
// last call; calls whose work overlaps on the GPU (different streams without
// ordering between them) race on it. Each call zeroes the status word it uses
// before the decode is enqueued.
#include <cuda_runtime.h>

#include <mutex>

#include "mla_kernels.cuh"

namespace {

constexpr size_t kStaticWsBytes = size_t(48) << 20;  // MLA_NOALLOC_WORKSPACE_BYTES in mla.h
static_assert(kStaticWsBytes == MLA_NOALLOC_WORKSPACE_BYTES, "keep the header in step");

static __device__ __align__(256) unsigned char g_static_workspace[kStaticWsBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mutex;
void* g_ws_ptr[kMaxDevices] = {};

// Device address of the array for the current device, looked up once per
// device (the host-side symbol is only a stand-in, never a device address).
mla_status_t static_workspace(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) return MLA_ERR_CUDA;
  if (dev >= kMaxDevices) return MLA_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_mutex);
  if (!g_ws_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_static_workspace) != cudaSuccess || !p) return MLA_ERR_CUDA;
    g_ws_ptr[dev] = p;
  }
  *out = g_ws_ptr[dev];
  return MLA_OK;
}

}  // namespace

extern "C" mla_status_t mla_decode_paged_noalloc(const mla_decode_args* args, mla_stream_t stream) {
  if (!args) return MLA_ERR_INVALID_ARG;
  if (args->workspace != nullptr || args->workspace_bytes != 0) return MLA_ERR_INVALID_ARG;
  const size_t need =
      mla_workspace_size(args->batch, args->s_q, args->h_q, args->h_kv, 0, args->num_sm_parts);
  if (need == 0) return MLA_ERR_INVALID_ARG;
  if (need > kStaticWsBytes) return MLA_ERR_WORKSPACE_TOO_SMALL;
  void* ws = nullptr;
  const mla_status_t st = static_workspace(&ws);
  if (st != MLA_OK) return st;
  mla_decode_args a = *args;
  a.workspace = ws;
  a.workspace_bytes = kStaticWsBytes;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(ws, 0, sizeof(uint32_t), s) != cudaSuccess) return MLA_ERR_CUDA;  // status word
  return mla_decode_paged(&a, stream);
}
