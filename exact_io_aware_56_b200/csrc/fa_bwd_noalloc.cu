// fa_bwd_noalloc: the backward pass with its workspace in a fixed device
// array owned by this library, for callers that cannot allocate device memory.
//
// Some hosts hand a kernel library only its input and output buffers: a
// plugin interface with a fixed signature and no workspace argument, or a
// runtime that budgets every byte of device memory itself and forbids its
// plugins to call cudaMalloc (which also synchronises the device, a stall
// that latency-bound loops cannot take). fa_bwd needs an fp32 workspace (row
// sums D and the dQ accumulator); this entry point takes it from a
// file-scope device array instead of from the caller.
//
// The array is allocated when the module is loaded and every GPU that loads
// it keeps it until the process exits. Every call shares it: the kernels
// rewrite all of it that they read (D and a zeroed dQ accumulator) before
// use, so a call never depends on what a previous call left there, but two
// calls whose kernels overlap on the GPU (other streams, other host threads)
// race on it and give wrong results.

#include <mutex>

#include "../../include/fa.h"
#include "fa_internal.h"

namespace {

constexpr size_t kScratchBytes = FA_BWD_NOALLOC_SCRATCH_BYTES;
constexpr int kMaxDevices = 64;

// In host code this name is only a stand-in for the device array: its
// device address comes from cudaGetSymbolAddress below.
static __device__ __align__(256) unsigned char g_bwd_scratch[kScratchBytes];

// Device address of the array per device. Only a successful lookup is
// kept; a failed one is retried by the next call.
std::mutex g_addr_mu;
void* g_addr[kMaxDevices] = {};

}  // namespace

extern "C" int fa_bwd_noalloc(const void* q, const void* k, const void* v, const void* o, const void* dout,
                              const float* lse, void* dq, void* dk, void* dv, int B, int Hq, int Hkv, int N, int d,
                              int causal, float scale, void* stream) {
  const size_t need = fa_bwd_workspace_bytes(B, Hq, Hkv, N, d);
  if (need == 0) {
    // The shape itself is invalid (non-positive sizes) or unsupported
    // (head dim, head ratio or size limits of fa_bwd).
    return (B <= 0 || Hq <= 0 || Hkv <= 0 || N <= 0) ? FA_ERR_INVALID_ARGUMENT : FA_ERR_UNSUPPORTED;
  }
  if (need > kScratchBytes) return FA_ERR_UNSUPPORTED;
  // The device check of every entry point comes first, so that a device
  // this library has no kernels for reports FA_ERR_UNSUPPORTED.
  int rc = fa::check_current_device();
  if (rc != FA_OK) return rc;
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fa::record_cuda_error(e);
  if (dev < 0 || dev >= kMaxDevices) return FA_ERR_UNSUPPORTED;
  // Set-up, once per device, with that device current: the device address
  // of the array.
  void* ptr = nullptr;
  {
    std::lock_guard<std::mutex> lock(g_addr_mu);
    if (g_addr[dev] == nullptr) {
      e = cudaGetSymbolAddress(&ptr, g_bwd_scratch);
      if (e != cudaSuccess || ptr == nullptr) {
        cudaGetLastError();  // clear the last-error state; the next call retries the lookup
        return fa::record_cuda_error(e != cudaSuccess ? e : cudaErrorInvalidSymbol);
      }
      g_addr[dev] = ptr;
    }
    ptr = g_addr[dev];
  }
  return fa_bwd(q, k, v, o, dout, lse, dq, dk, dv, B, Hq, Hkv, N, d, causal, scale, ptr, kScratchBytes, stream);
}
