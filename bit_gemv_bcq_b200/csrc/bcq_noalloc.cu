// bcq_noalloc.cu -- bcq_gemm_noalloc: the matmul for callers that cannot
// allocate device memory (code running inside an allocator or memory pool, a
// plug-in whose host framework owns all device allocations, a loop that must
// not block on the driver's allocator).  The split-K scratch that bcq_gemm
// takes from its caller comes from a static array of this library instead.
//
// The array lives in this translation unit.  Host code sees only a host-side
// stand-in under its name, so its device address is looked up here, with the
// call's device current, and passed to the kernels as the workspace pointer
// of bcq_gemm.
#include <cuda_runtime.h>

#include <cstddef>
#include <mutex>

#include "bcq.h"
#include "bcq_launch.h"

namespace {

constexpr size_t kScratchBytes = BCQ_NOALLOC_SCRATCH_BYTES;
constexpr int kMaxDevices = 64;

// Zero at module load; every call clears the bytes it uses before its kernels.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kScratchBytes];

std::mutex g_scratch_mu;
void* g_scratch_addr[kMaxDevices] = {};

// Device address of g_noalloc_scratch on the current device: looked up on
// every call (cheap, and right again after a device or context reset loads
// the module anew) except while `stream` is capturing a graph, when the last
// address found on this device is used.
bcq_status scratch_address(cudaStream_t stream, void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return BCQ_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return BCQ_ERR_UNSUPPORTED;
  cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(stream, &cap) != cudaSuccess) return BCQ_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (cap == cudaStreamCaptureStatusNone || !g_scratch_addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return BCQ_ERR_CUDA;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return BCQ_OK;
}

}  // namespace

extern "C" bcq_status bcq_gemm_noalloc(const uint16_t* x, const uint32_t* planes,
                                       const uint16_t* const alpha[4], const uint16_t* z,
                                       int p, const int32_t* p_row, int M, int N, int K,
                                       int p_H, int group, uint16_t* y, void* stream) {
  const size_t need = (M > 0) ? bcq_workspace_bytes(M, N, K) : 0;
  void* ws = nullptr;
  if (need > 0) {
    bcq_status s = scratch_address(static_cast<cudaStream_t>(stream), &ws);
    if (s != BCQ_OK) return s;
  }
  // bcq_gemm's checks, with the scratch standing in for the workspace, so
  // that a rejected call (BCQ_ERR_SCRATCH included) launches nothing.
  bcq_status s = bcq::check_gemm_args(x, planes, alpha, z, p, p_row, M, N, K, p_H, group, y,
                                      ws, need);
  if (s != BCQ_OK || M == 0) return s;
  if (need > kScratchBytes) return BCQ_ERR_SCRATCH;
  if (need > 0 &&
      cudaMemsetAsync(ws, 0, need, static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return BCQ_ERR_CUDA;
  return bcq_gemm(x, planes, alpha, z, p, p_row, M, N, K, p_H, group, y, ws, need, stream);
}
