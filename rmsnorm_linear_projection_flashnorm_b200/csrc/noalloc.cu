// fn_norm_proj_static: the fused norm + projection for callers that cannot
// allocate device memory.
//
// Some callers have no way to provide a workspace: code that records work
// while a CUDA stream capture is active (cudaMalloc is not permitted during
// a global-mode capture), plug-ins that run inside a host application which
// owns every device allocation, and latency-critical loops that must never
// call cudaMalloc because it can synchronise the device.  For them the
// scratch memory of the call (the status word and the per-CTA split-K
// partial sums of the decode path, the activations split once per call of the
// fp8 decode path) lives in a fixed-size array inside this library instead of
// a caller-provided workspace.
//
// The array is a file-scope __device__ variable: every GPU that loads the
// library holds kStaticScratchBytes of it until the process exits.  Global
// device variables without an initialiser are zero when the module loads, so
// the status word starts at zero without any set-up copy.  In host code the
// array's name is only a host-side stand-in, so its device address is
// fetched with cudaGetSymbolAddress once per device, with that device
// current, on the first call made on that device; that first call must
// therefore come before any stream capture.  All calls on a device share the
// array and it keeps the last call's contents (every call overwrites the
// partials it reads, so nothing else has to start at zero); calls that may
// overlap on the GPU, on any streams, race on it.  A device-side wait that
// runs out of time records itself in the array's status word, which
// fn_query_static_status reads and clears.
#include <cstdint>
#include <mutex>

#include <cuda_runtime.h>

#include "flashnorm.h"
#include "internal.h"

namespace {

constexpr size_t kStaticScratchBytes = size_t{8} << 20;   // 8 MiB per device

__device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device (fetched on
// first use; no memory is allocated or written).
fn_status static_scratch(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    cudaGetLastError();
    return FN_ERR_CUDA;
  }
  std::lock_guard<std::mutex> lock(g_mu);
  if (g_scratch_ptr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess || p == nullptr) {
      cudaGetLastError();
      return FN_ERR_CUDA;
    }
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return FN_OK;
}

}  // namespace

extern "C" fn_status fn_norm_proj_static(const void* x, int64_t M, int64_t d, const void* Wp, const float* scales,
                                         fn_wtype wt, int64_t N, float eps, void* y, fn_stream_t stream) {
  if (M == 0) return fn_norm_proj(x, M, d, Wp, scales, wt, N, eps, y, nullptr, 0, stream);
  // sizes whose scratch would not fit the static array are rejected up front
  const size_t need = fn_workspace_size(M, d, N, wt, 0);
  if (M > 0 && d > 0 && N > 0 && need > kStaticScratchBytes) return FN_ERR_WORKSPACE;
  void* scratch = nullptr;
  if (M > 0 && d > 0 && N > 0) {
    const fn_status st = static_scratch(&scratch);
    if (st != FN_OK) return st;
  }
  return fn_norm_proj(x, M, d, Wp, scales, wt, N, eps, y, scratch, kStaticScratchBytes, stream);
}

extern "C" fn_status fn_query_static_status(unsigned int* detail, fn_stream_t stream) {
  void* scratch = nullptr;
  const fn_status st = static_scratch(&scratch);
  if (st != FN_OK) return st;
  return fn_query_device_status(scratch, detail, stream);
}
