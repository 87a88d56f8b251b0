// moe_router.cu -- stand-alone router: logits GEMV over bf16 [E][H], then
// top-K with renormalised softmax weights (one warp per token).  The fused
// layer kernel computes the same logits and top-K inside its single launch.
#include "moe_kernels.h"
#include "moe_device.cuh"

namespace moe {

// logits[t][e] = sum_h x[t][h] * wr[e][h] + bias[e].  One warp per expert
// row; tokens go in groups of 8 so a weight chunk is read once per group.
// Lane l owns columns 256*k + 8*l .. +7 (H is a multiple of 64).
__global__ void __launch_bounds__(512) router_logits_kernel(const uint16_t* x, const uint16_t* wr,
                                                            const float* bias, int T, int H, int E,
                                                            float* logits) {
  const int lane = threadIdx.x & 31;
  const int nwarps = (int)((gridDim.x * blockDim.x) >> 5);
  for (int e = (int)((blockIdx.x * blockDim.x + threadIdx.x) >> 5); e < E; e += nwarps) {
    const uint16_t* w = wr + (size_t)e * H;
    for (int t0 = 0; t0 < T; t0 += 8) {
      const int nt = min(8, T - t0);
      float acc[8];
#pragma unroll
      for (int tt = 0; tt < 8; ++tt) acc[tt] = 0.f;
      for (int c0 = 8 * lane; c0 < H; c0 += 256) {
        float wv[8];
        unpack_bf16x8(__ldg(reinterpret_cast<const uint4*>(w + c0)), wv);
#pragma unroll
        for (int tt = 0; tt < 8; ++tt) {
          if (tt < nt) {
            float xv[8];
            unpack_bf16x8(__ldg(reinterpret_cast<const uint4*>(x + (size_t)(t0 + tt) * H + c0)), xv);
#pragma unroll
            for (int k = 0; k < 8; ++k) acc[tt] = fmaf(wv[k], xv[k], acc[tt]);
          }
        }
      }
#pragma unroll
      for (int tt = 0; tt < 8; ++tt) {
        if (tt < nt) {
          const float v = warp_sum(acc[tt]);
          if (lane == 0) logits[(size_t)(t0 + tt) * E + e] = v + (bias ? bias[e] : 0.f);
        }
      }
    }
  }
}

__global__ void topk_kernel(const float* logits, int T, int E, int K, int32_t* idx, float* w) {
  const int t = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (t >= T) return;
  warp_topk(logits + (size_t)t * E, E, K, idx + (size_t)t * K, w + (size_t)t * K);
}

cudaError_t launch_router_logits(const uint16_t* x, const uint16_t* wr, const float* bias, int T,
                                 int H, int E, int grid, float* logits, cudaStream_t st) {
  router_logits_kernel<<<grid, 512, 0, st>>>(x, wr, bias, T, H, E, logits);
  return cudaGetLastError();
}

cudaError_t launch_topk(const float* logits, int T, int E, int K, int32_t* idx, float* w,
                        cudaStream_t st) {
  const int warps = 4;
  topk_kernel<<<(T + warps - 1) / warps, 32 * warps, 0, st>>>(logits, T, E, K, idx, w);
  return cudaGetLastError();
}

}  // namespace moe
