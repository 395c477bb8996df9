// noalloc.cu - mxq_linear_noalloc: the quantised linear layer for callers
// that cannot allocate device memory.
//
// mxq_linear needs a workspace for the quantised activation (codes, block
// scales, amax and the per-tensor scale).  Normally the caller allocates it.
// Some callers cannot: a host whose device-memory budget is fixed when it
// starts and that forbids allocations afterwards, or a latency-critical loop
// where cudaMalloc (which may synchronise the device and whose latency is
// unbounded) is not acceptable.  For them this file keeps the workspace in a
// file-scope device array and passes its address to the unchanged mxq_linear
// path.  Nothing here calls cudaMalloc, cudaFree or any allocating routine.
//
// Costs and rules of use:
//   * The array is MXQ_NOALLOC_SCRATCH_BYTES (64 MiB) on every GPU that loads
//     this library, held until the process exits, whether the entry point is
//     used or not.
//   * The first call on a device (with that device current) looks up the
//     array's device address with cudaGetSymbolAddress and caches it; make
//     that first call before any stream capture.
//   * All calls on a device share the one array and it keeps the previous
//     call's contents.  mxq_linear needs no value of its workspace to start
//     at zero: codes and scales are fully rewritten and the quantiser's amax
//     exchange is valid from any contents.  Calls whose work can overlap on
//     the GPU (different streams, or several host threads without ordering)
//     race on the array: serialise them, e.g. on one stream.
#include <cuda_runtime.h>

#include <mutex>

#include "../../include/mxq.h"

namespace {

// The workspace.  Host code must not use this name as an address: on the host
// it is only a stand-in for the device symbol (a kernel handed it would fault,
// or silently touch the wrong memory where the GPU can reach host memory).
// Host code uses the address from cudaGetSymbolAddress instead.
static __device__ __align__(256) unsigned char g_noalloc_scratch[MXQ_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
void* g_scratch_addr[kMaxDevices] = {};
std::mutex g_scratch_mu;

// Device address of the scratch array on the current device (looked up once
// per device, with that device current).
mxq_status scratch_address(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return MXQ_ERR_ARCH;
  }
  if (dev < 0 || dev >= kMaxDevices) return MXQ_ERR_ARCH;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (g_scratch_addr[dev] == nullptr) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || p == nullptr) {
      cudaGetLastError();
      return MXQ_ERR_CUDA;
    }
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return MXQ_OK;
}

}  // namespace

extern "C" mxq_status mxq_linear_noalloc(const mxq_weight* w, const void* x_bf16, int64_t M,
                                         void* y_bf16, const mxq_linear_opts* opts,
                                         mxq_stream_t stream) {
  if (w == nullptr || M < 0) return MXQ_ERR_INVALID_ARG;
  const int path = mxq_linear_path(w, M, opts);
  if (path == MXQ_BF16) {
    // the bf16 GEMM needs no workspace
    return mxq_linear(w, x_bf16, M, y_bf16, nullptr, 0, opts, stream);
  }
  const size_t need = mxq_linear_workspace_bytes(M, w->K, static_cast<mxq_format>(path));
  if (need > static_cast<size_t>(MXQ_NOALLOC_SCRATCH_BYTES)) return MXQ_ERR_WORKSPACE;
  void* scratch = nullptr;
  const mxq_status st = scratch_address(&scratch);
  if (st != MXQ_OK) return st;
  return mxq_linear(w, x_bf16, M, y_bf16, scratch, static_cast<size_t>(MXQ_NOALLOC_SCRATCH_BYTES),
                    opts, stream);
}
