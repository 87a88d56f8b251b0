// moe_noalloc.cu -- moe_layer_forward_noalloc: the fused layer running on a
// scratch area that belongs to the library itself, for callers that must not
// allocate device memory.
//
// Who needs it: a caller that runs under a fixed device-memory budget, or in
// a loop where allocating is not allowed (cudaMalloc can synchronise the
// device and can fail under memory pressure), and that does not want to keep
// a workspace of its own.  Instead of a caller workspace, the call uses
// g_scratch below: a file-scope device array of MOE_NOALLOC_SCRATCH_BYTES that
// is part of the loaded module, so no allocation ever happens.
//
// Set-up: the first call on a device (with that device current) looks up the
// array's address with cudaGetSymbolAddress and zeroes its first 256 bytes
// (the kernel's grid counters and error word, which must start at zero).
// Those two calls are synchronous, so make the first call on each device
// before any stream capture.  The kernel returns its grid counters to zero
// when it exits, but not the error word (a failing launch leaves its code
// there), so every call first clears the error word on its stream: one
// call's device-side failure (a wait that expired, a bad expert pointer)
// leaves that call's outputs unspecified and can be read with
// moe_noalloc_device_error before the next call, and the next call starts
// clean.  Every call on a device shares the one scratch: calls that may
// overlap in time (on different streams or host threads) race on it and must
// be serialised by the caller.
#include <cuda_runtime.h>

#include <cstdio>
#include <mutex>

#include "../../include/moe.h"

namespace moe {
moe_status abi_fail(moe_status s, const char* msg);
size_t fused_workspace_bytes(const moe_config* cfg, int T);
moe_status layer_forward_on(const moe_config* cfg, const moe_layer_weights* wts, const void* x_bf16,
                            const void* residual_bf16, int T, void* h_out_bf16, void* y_norm_bf16,
                            int32_t* idx_out, float* w_out, void* workspace, size_t ws_bytes,
                            cudaStream_t stream);
}  // namespace moe

namespace {

constexpr size_t kScratchBytes = MOE_NOALLOC_SCRATCH_BYTES;
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_scratch[kScratchBytes];

constexpr size_t kErrOffset = 64;  // the kernel's error word inside the first 256 bytes

std::mutex g_mu;
void* g_scratch_ptr[kMaxDevices];  // per device, set on first use

// The device address of g_scratch on device `dev` (current), looked up and
// its first 256 bytes zeroed on first use.
moe_status scratch_of(int dev, void** out) {
  std::lock_guard<std::mutex> lock(g_mu);
  if (g_scratch_ptr[dev] == nullptr) {
    void* p = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&p, g_scratch);
    if (e != cudaSuccess) return moe::abi_fail(MOE_ERR_CUDA, cudaGetErrorString(e));
    e = cudaMemset(p, 0, 256);
    if (e != cudaSuccess) return moe::abi_fail(MOE_ERR_CUDA, cudaGetErrorString(e));
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return MOE_OK;
}

}  // namespace

extern "C" moe_status moe_layer_forward_noalloc(const moe_config* cfg, const moe_layer_weights* wts,
                                                const void* x_bf16, const void* residual_bf16, int T,
                                                void* h_out_bf16, void* y_norm_bf16, int32_t* idx_out,
                                                float* w_out, cudaStream_t stream) {
  if (!cfg) return moe::abi_fail(MOE_ERR_INVALID_ARG, "cfg is NULL");
  if (T < 0) return moe::abi_fail(MOE_ERR_INVALID_ARG, "T < 0");
  const size_t need = moe::fused_workspace_bytes(cfg, T);
  if (need == 0)
    return moe::abi_fail(MOE_ERR_UNSUPPORTED,
                         "unsupported shape (bits 2 or 4, group 64, hidden and inter positive multiples of 64)");
  if (need > kScratchBytes) {
    char msg[256];
    snprintf(msg, sizeof(msg),
             "this shape needs %zu bytes of scratch; the built-in scratch holds %zu "
             "(use moe_layer_forward with a workspace of your own)",
             need, kScratchBytes);
    return moe::abi_fail(MOE_ERR_WORKSPACE, msg);
  }
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return moe::abi_fail(MOE_ERR_CUDA, cudaGetErrorString(e));
  if (dev < 0 || dev >= kMaxDevices) return moe::abi_fail(MOE_ERR_UNSUPPORTED, "device index out of range");
  void* scratch = nullptr;
  const moe_status st = scratch_of(dev, &scratch);
  if (st != MOE_OK) return st;
  if (T > 0) {
    // the previous call's error code must not outlive it (see the top of the file)
    e = cudaMemsetAsync(static_cast<unsigned char*>(scratch) + kErrOffset, 0, 4, stream);
    if (e != cudaSuccess) return moe::abi_fail(MOE_ERR_CUDA, cudaGetErrorString(e));
  }
  return moe::layer_forward_on(cfg, wts, x_bf16, residual_bf16, T, h_out_bf16, y_norm_bf16, idx_out, w_out,
                               scratch, kScratchBytes, stream);
}

extern "C" moe_status moe_noalloc_device_error(uint32_t* detail, cudaStream_t stream) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return moe::abi_fail(MOE_ERR_CUDA, cudaGetErrorString(e));
  if (dev < 0 || dev >= kMaxDevices) return moe::abi_fail(MOE_ERR_UNSUPPORTED, "device index out of range");
  void* scratch = nullptr;
  const moe_status st = scratch_of(dev, &scratch);
  if (st != MOE_OK) return st;
  return moe_device_error(scratch, detail, stream);
}
