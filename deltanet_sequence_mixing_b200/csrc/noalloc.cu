// deltanet_chunk_fwd_noalloc: the chunked forward for callers that cannot
// allocate device memory, with its scratch in a static device array.
//
// Some callers have no way to obtain device memory at the call site: code that
// runs inside another framework's allocator or memory-pool hooks (where calling
// cudaMalloc would re-enter the allocator), plug-ins and embedded runtimes whose
// device memory is fully budgeted up front, and code paths that must not call
// cudaMalloc because it synchronises the device.  They still own their inputs
// and outputs, but cannot provide the workspace deltanet_chunk_fwd asks for.
// This variant takes its workspace from a file-scope device array instead.
#include <cuda_runtime.h>

#include <mutex>

#include "deltanet.h"

namespace {

// The scratch: the device status word plus, for bf16 problems, the per-chunk
// WY factors of the pre-pass (16.25 KB per (b, h, 64-token chunk)), up to this
// many bytes; larger problems are rejected.  Every device that loads the
// library holds one copy until the process exits.
constexpr size_t kNoAllocScratchBytes = 1u << 20;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_setup_mutex;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device.  Resolved once per
// device (the array's name is only a host-side stand-in for it in host code) and
// kept: a device reset after the first call would leave a stale address, which
// the public header rules out.
cudaError_t scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  if (!g_scratch_ptr[dev]) {
    void* ptr = nullptr;
    e = cudaGetSymbolAddress(&ptr, g_noalloc_scratch);
    if (e != cudaSuccess) return e;
    if (!ptr) return cudaErrorInvalidSymbol;
    g_scratch_ptr[dev] = ptr;
  }
  *out = g_scratch_ptr[dev];
  return cudaSuccess;
}

}  // namespace

extern "C" int deltanet_chunk_fwd_noalloc(const void* q, const void* k, const void* v,
                                          const float* beta, const float* alpha,
                                          const float* S0, void* o, float* S_out, int B,
                                          int H, int T, int Dk, int Dv, int C, dn_dtype dt,
                                          void* cuda_stream) {
  const size_t need = deltanet_workspace_bytes(B, H, T, Dk, Dv, C, dt);
  if (need == 0) {
    // Same answers as deltanet_chunk_fwd for the sizes it rejects.
    if (B < 0 || H < 0 || T < 0) return DN_ERR_INVALID_ARG;
    return DN_ERR_UNSUPPORTED;
  }
  if (need > kNoAllocScratchBytes) return DN_ERR_WORKSPACE;  // beyond the static scratch
  void* scratch = nullptr;
  if (scratch_address(&scratch) != cudaSuccess) return DN_ERR_CUDA;
  cudaStream_t st = static_cast<cudaStream_t>(cuda_stream);
  // The status word (first 256 bytes) must start at zero for this call; the rest
  // of the scratch is fully written by the call before it is read.
  if (cudaMemsetAsync(scratch, 0, 256, st) != cudaSuccess) return DN_ERR_CUDA;
  return deltanet_chunk_fwd(q, k, v, beta, alpha, S0, o, S_out, B, H, T, Dk, Dv, C, dt, scratch,
                            kNoAllocScratchBytes, cuda_stream);
}
