// moe_router.cu -- stand-alone router: logits GEMV over bf16 [E][H], then
// top-K with renormalised softmax weights (one warp per token).  The fused
// layer kernel computes the same logits and top-K inside its single launch.
#include "moe_kernels.h"
#include "moe_device.cuh"

namespace moe {

// logits[t][e] = sum_h x[t][h] * wr[e][h] + bias[e].  A block takes 4 expert
// rows; each row is split into 4 column parts, one warp each (16 warps), so
// a 4096-column row is 4 loads of 16 bytes per lane, all in flight at once,
// and ceil(E/4) blocks spread the weights over the SMs.  The 4 parts are
// summed in part order (a fixed order).  Tokens go in groups of 8 so a
// weight chunk is read once per group.  Lane l of part p owns columns
// 256*k + 8*l .. +7 for k = p, p + 4, ... (H is a multiple of 64).
constexpr int kRouterRows = 4, kRouterParts = 4;
__global__ void __launch_bounds__(512) router_logits_kernel(const uint16_t* __restrict__ x,
                                                            const uint16_t* __restrict__ wr,
                                                            const float* __restrict__ bias, int T, int H, int E,
                                                            float* __restrict__ logits) {
  __shared__ float red[kRouterRows * kRouterParts][8];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int rl = warp / kRouterParts, part = warp - rl * kRouterParts;
  const int e = blockIdx.x * kRouterRows + rl;
  const int nchunk = H / 256;  // whole 256-column chunks; a tail of 64..192 columns is chunk nchunk
  const int tail = H - 256 * nchunk;
  const uint16_t* w = wr + (size_t)(e < E ? e : 0) * H;
#pragma unroll 1
  for (int t0 = 0; t0 < T; t0 += 8) {
    const int nt = min(8, T - t0);
    float acc[8];
#pragma unroll
    for (int tt = 0; tt < 8; ++tt) acc[tt] = 0.f;
    if (e < E) {
#pragma unroll 1
      for (int k0 = part; k0 <= nchunk; k0 += 4 * kRouterParts) {
        // up to 4 chunks of this part: loads first, then the FMAs
        uint4 wq[4];
        bool in[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int k = k0 + q * kRouterParts;
          const int c = 256 * k + 8 * lane;
          in[q] = k < nchunk || (k == nchunk && 8 * lane < tail);
          wq[q] = in[q] ? __ldg(reinterpret_cast<const uint4*>(w + c)) : make_uint4(0u, 0u, 0u, 0u);
        }
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          if (!in[q]) continue;
          const int c = 256 * (k0 + q * kRouterParts) + 8 * lane;
          float wv[8];
          unpack_bf16x8(wq[q], wv);
#pragma unroll
          for (int tt = 0; tt < 8; ++tt) {
            if (tt < nt) {
              float xv[8];
              unpack_bf16x8(__ldg(reinterpret_cast<const uint4*>(x + (size_t)(t0 + tt) * H + c)), xv);
#pragma unroll
              for (int i = 0; i < 8; ++i) acc[tt] = fmaf(wv[i], xv[i], acc[tt]);
            }
          }
        }
      }
    }
#pragma unroll
    for (int tt = 0; tt < 8; ++tt) {
      const float v = warp_sum(acc[tt]);
      if (lane == 0) red[warp][tt] = v;
    }
    __syncthreads();
    if (threadIdx.x < kRouterRows * 8) {
      const int r = threadIdx.x >> 3, tt = threadIdx.x & 7;
      const int er = blockIdx.x * kRouterRows + r;
      if (er < E && tt < nt) {
        float v = 0.f;
        for (int p = 0; p < kRouterParts; ++p) v += red[r * kRouterParts + p][tt];
        logits[(size_t)(t0 + tt) * E + er] = v + (bias ? bias[er] : 0.f);
      }
    }
    __syncthreads();
  }
}
__global__ void topk_kernel(const float* logits, int T, int E, int K, int32_t* idx, float* w) {
  const int t = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (t >= T) return;
  warp_topk(logits + (size_t)t * E, E, K, idx + (size_t)t * K, w + (size_t)t * K);
}

cudaError_t launch_router_logits(const uint16_t* x, const uint16_t* wr, const float* bias, int T,
                                 int H, int E, int grid, float* logits, cudaStream_t st) {
  (void)grid;  // one block per 4 rows
  router_logits_kernel<<<(E + kRouterRows - 1) / kRouterRows, 512, 0, st>>>(x, wr, bias, T, H, E, logits);
  return cudaGetLastError();
}

cudaError_t launch_topk(const float* logits, int T, int E, int K, int32_t* idx, float* w,
                        cudaStream_t st) {
  const int warps = 4;
  topk_kernel<<<(T + warps - 1) / warps, 32 * warps, 0, st>>>(logits, T, E, K, idx, w);
  return cudaGetLastError();
}

}  // namespace moe
