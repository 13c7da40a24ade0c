// moe_forward_static: the forward pass for callers that cannot allocate device
// memory.  It runs exactly the kernels of moe_forward, with the scratch they
// need (routing tables and expert-sorted activations) taken from a fixed
// array compiled into this library instead of a caller-provided workspace.
//
// Who needs it: code that has no way to obtain device memory of its own, for
// example a plug-in running inside a host framework that owns every device
// allocation and exposes no workspace to its extensions, or a latency-critical
// serving loop that is not allowed to enter an allocator on its hot path.
//
// Limits and behaviour (also stated in include/moe.h):
//   * the scratch is kStaticScratchBytes = 32 MiB per device; a call whose
//     moe_workspace_bytes() is larger is rejected with MOE_ERR_UNSUPPORTED;
//   * the array lives in device memory of every GPU that loads this library,
//     for as long as the process runs;
//   * the first call on a device looks up the array's device address
//     (cudaGetSymbolAddress) with that device current; make that first call
//     before any stream capture;
//   * all calls share the one array: calls whose executions overlap on the
//     GPU (different streams, or several host threads) race on it; the last
//     call's contents stay there;
//   * nothing in the scratch has to start at zero: every value the kernels
//     read is written earlier in the same call (rows of a tile past the end
//     of an expert's group are read but only feed output rows never stored);
//   * this file calls no cudaMalloc, cudaFree or other allocating routine.
#include <cuda_runtime.h>

#include <mutex>
#include <string>

#include "internal.h"
#include "moe.h"

namespace {

constexpr size_t kStaticScratchBytes = static_cast<size_t>(32) << 20;

static __device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

constexpr int kMaxDevices = 64;
void* g_scratch_addr[kMaxDevices];
std::mutex g_scratch_mu;

// Device address of the scratch array on the current device (set up once per device).
cudaError_t scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lk(g_scratch_mu);
  if (g_scratch_addr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_static_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return cudaSuccess;
}

}  // namespace

extern "C" int moe_forward_static(moe_handle h, int64_t T, const void* x, const float* W_r, const float* b_r,
                                  const void* W1, const void* W3, const void* W2, void* y, int32_t* expert_counts,
                                  int32_t* dropped, float* aux_loss, float* z_loss, void* stream) {
  if (h == nullptr || T < 0) {
    moe::set_error_message("moe_forward_static: NULL handle or T < 0");
    return MOE_ERR_INVALID_ARG;
  }
  const size_t need = moe_workspace_bytes(h, T);
  if (need > kStaticScratchBytes) {
    moe::set_error_message(("moe_forward_static: this layer needs " + std::to_string(need) +
                            " bytes of scratch for T = " + std::to_string(T) +
                            "; the static scratch holds " + std::to_string(kStaticScratchBytes) +
                            " bytes (use moe_forward with a caller workspace)").c_str());
    return MOE_ERR_UNSUPPORTED;
  }
  void* scratch = nullptr;
  const cudaError_t e = scratch_address(&scratch);
  if (e != cudaSuccess) {
    moe::set_error_message((std::string("moe_forward_static: cudaGetSymbolAddress failed: ") +
                            cudaGetErrorString(e)).c_str());
    return MOE_ERR_CUDA;
  }
  return moe_forward(h, T, x, W_r, b_r, W1, W3, W2, y, expert_counts, dropped, aux_loss, z_loss, scratch,
                     kStaticScratchBytes, nullptr, stream);
}
