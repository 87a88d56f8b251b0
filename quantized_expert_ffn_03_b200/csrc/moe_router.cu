// moe_router.cu -- stand-alone router: logits GEMV over bf16 [E][H], then
// top-K with renormalised softmax weights (one warp per token).  The fused
// layer kernel runs the same phase functions inside its single launch.
#include "moe_kernels.h"
#include "moe_phases.cuh"

namespace moe {

constexpr int kR = 4;

__global__ void __launch_bounds__(kThreads, 1)
    router_logits_kernel(const uint16_t* x, const uint16_t* wr, const float* bias, int T, int H,
                         int E, int tw, float* logits) {
  __shared__ float red[2 * kWarps * kR];
  phase_router<kR>(wr, bias, x, T, H, E, tw, logits, red);
}

__global__ void topk_kernel(const float* logits, int T, int E, int K, int32_t* idx, float* w) {
  const int t = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (t >= T) return;
  warp_topk(logits + (size_t)t * E, E, K, idx + (size_t)t * K, w + (size_t)t * K);
}

cudaError_t launch_router_logits(const uint16_t* x, const uint16_t* wr, const float* bias, int T,
                                 int H, int E, int tw, int grid, float* logits, cudaStream_t st) {
  router_logits_kernel<<<grid, kThreads, 0, st>>>(x, wr, bias, T, H, E, tw, logits);
  return cudaGetLastError();
}

cudaError_t launch_topk(const float* logits, int T, int E, int K, int32_t* idx, float* w,
                        cudaStream_t st) {
  const int warps = 4;
  topk_kernel<<<(T + warps - 1) / warps, 32 * warps, 0, st>>>(logits, T, E, K, idx, w);
  return cudaGetLastError();
}

}  // namespace moe
