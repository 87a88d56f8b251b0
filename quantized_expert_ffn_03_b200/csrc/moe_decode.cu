// moe_decode.cu -- the fused single-launch MoE layer for decode (T <= 8).
//
// One persistent cooperative launch, one block per SM, runs the whole layer:
//   phase 0  router logits (all blocks), then the shared expert's gate/up
//   phase 1  top-K (every block, redundantly), L2 prefetch of this block's
//            share of the chosen experts, routed gate/up + SwiGLU
//   phase 2  shared expert down for this block's output rows, then the
//            routed experts' down rows, combine + residual, sum of squares
//   phase 3  RMSNorm of this block's rows
// Blocks meet at four split-phase grid counters (router, shared, expert,
// down); each wait is bounded and comes after independent work, so the
// latency of a barrier is mostly hidden.  This is the single-kernel version
// of the pages' pipeline: the router projection with the shared expert
// (CMD2), top-K, the expert reads and the deferred expert forward with
// combine + residual + norm (CMD3), with no return to the host
// ("Flash-MoE: ラップトップでの397Bパラメータモデルの実行", section
// "パイプライン概要"; "Streaming experts: как запустить триллионную модель на
// MacBook", section "Оптимизации, которые сработали").
#include <cuda_bf16.h>

#include "moe_kernels.h"
#include "moe_phases.cuh"

namespace moe {

constexpr int kRouterR = 4;
constexpr int kSharedR = 4;
constexpr int kGateUpR = 4;
constexpr int kDownR = 8;

// Shared-memory plan (bytes) for T tokens, K experts, nrows output rows.
struct DecodeSmem {
  size_t red, tk_w, tk_i, eptr, ypart, ys, hacc, inv, total;
};

__host__ __device__ inline size_t align16(size_t n) { return (n + 15) & ~size_t(15); }

__host__ __device__ inline DecodeSmem decode_smem_plan(int T, int K, int nrows) {
  DecodeSmem s;
  size_t pos = 0;
  const int rmax = 8;  // largest R*NM of any phase
  s.red = pos;
  pos = align16(pos + sizeof(float) * 2 * kWarps * rmax);
  s.tk_w = pos;
  pos = align16(pos + sizeof(float) * T * K);
  s.tk_i = pos;
  pos = align16(pos + sizeof(int) * T * K);
  s.eptr = pos;
  pos = align16(pos + sizeof(void*) * T * K);
  s.ypart = pos;
  pos = align16(pos + sizeof(float) * T * K * nrows);
  s.ys = pos;
  pos = align16(pos + sizeof(float) * T * nrows);
  s.hacc = pos;
  pos = align16(pos + sizeof(float) * T * nrows);
  s.inv = pos;
  pos = align16(pos + sizeof(float) * T);
  s.total = pos;
  return s;
}

size_t decode_smem_bytes(int T, int K, int nrows) { return decode_smem_plan(T, K, nrows).total; }

template <int FMT>
__global__ void __launch_bounds__(kThreads, 1) moe_decode_kernel(const DecodeParams p) {
  extern __shared__ __align__(16) uint8_t smem[];
  __shared__ int s_flag;
  const Layout& L = p.L;
  const int T = p.T, K = L.K, H = L.H, I = L.I, E = L.E;
  const int G = gridDim.x, c = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int r0 = (int)((long long)H * c / G), r1 = (int)((long long)H * (c + 1) / G);
  const int nrows = r1 - r0;
  const int nrows_max = (H + G - 1) / G;
  const DecodeSmem sp = decode_smem_plan(T, K, nrows_max);
  float* red = reinterpret_cast<float*>(smem + sp.red);
  float* tk_w = reinterpret_cast<float*>(smem + sp.tk_w);
  int* tk_i = reinterpret_cast<int*>(smem + sp.tk_i);
  const uint8_t** eptr = reinterpret_cast<const uint8_t**>(smem + sp.eptr);
  float* ypart = reinterpret_cast<float*>(smem + sp.ypart);
  float* ys = reinterpret_cast<float*>(smem + sp.ys);
  float* hacc = reinterpret_cast<float*>(smem + sp.hacc);
  float* inv = reinterpret_cast<float*>(smem + sp.inv);
  uint32_t* ctr = p.ctr;

  // ---- prefetch this block's phase-0 rows into L2 -------------------------
  if (threadIdx.x == 0) {
    int cb, ce;
    chunk_range((E + kRouterR - 1) / kRouterR, cb, ce);
    const int e0 = cb * kRouterR, e1 = min(E, ce * kRouterR);
    if (e1 > e0) l2_prefetch(p.wr + (size_t)e0 * H, (size_t)(e1 - e0) * H * 2);
    if (L.has_shared) {
      chunk_range(I / kSharedR, cb, ce);
      const size_t i0 = (size_t)cb * kSharedR, n = (size_t)(ce - cb) * kSharedR;
      l2_prefetch(p.sg + i0 * H, n * H * 2);
      l2_prefetch(p.su + i0 * H, n * H * 2);
    }
  }

  // ---- phase 0: router logits, shared gate/up ------------------------------
  phase_router<kRouterR>(p.wr, p.bias, p.x, T, H, E, p.tw_h, p.logits, red);
  grid_arrive(&ctr[0]);
  if (L.has_shared) phase_shared_gateup<kSharedR>(p.sg, p.su, p.x, T, H, I, p.tw_h, p.hs, red);
  grid_arrive(&ctr[1]);

  // ---- phase 1: top-K, routed gate/up --------------------------------------
  bool ok = grid_wait(&ctr[0], G, &ctr[5], p.err, p.timeout_ns, &s_flag);
  if (ok) {
    if (warp < T) warp_topk(p.logits + (size_t)warp * E, E, K, tk_i + warp * K, tk_w + warp * K);
    __syncthreads();
    for (int j = threadIdx.x; j < T * K; j += kThreads) {
      const int e = tk_i[j];
      const void* b = (e >= 0 && e < E) ? p.expert_ptr[e] : nullptr;
      if (b == nullptr || (reinterpret_cast<uintptr_t>(b) & 255u)) {
        atomicCAS(p.err, 0u, 2u);
        atomicExch(&ctr[5], 1u);
        b = nullptr;
      }
      eptr[j] = reinterpret_cast<const uint8_t*>(b);
      if (c == 0) {
        if (p.idx_out) p.idx_out[j] = e;
        if (p.w_out) p.w_out[j] = tk_w[j];
      }
    }
    __syncthreads();
    for (int j = 0; j < T * K; ++j) ok = ok && eptr[j] != nullptr;
  }
  if (ok && threadIdx.x == 0) {
    // this block's routed gate/up rows, its down rows of every chosen expert,
    // and its rows of the shared down projection
    const int cpp = I / kGateUpR;
    int cb, ce;
    chunk_range(T * K * cpp, cb, ce);
    for (int pair = cb / cpp; pair < T * K && pair * cpp < ce; ++pair) {
      const int a = max(cb, pair * cpp) - pair * cpp, b = min(ce, (pair + 1) * cpp) - pair * cpp;
      const size_t i0 = (size_t)a * kGateUpR, n = (size_t)(b - a) * kGateUpR;
      const uint8_t* blob = eptr[pair];
      for (int m = 0; m < 2; ++m) {
        l2_prefetch(blob + L.off_codes[m] + i0 * L.code_row_bytes[m], n * L.code_row_bytes[m]);
        l2_prefetch(blob + L.off_scales[m] + i0 * L.scale_row_bytes[m], n * L.scale_row_bytes[m]);
      }
    }
    if (L.has_shared) l2_prefetch(p.sd + (size_t)r0 * I, (size_t)nrows * I * 2);
    for (int pair = 0; pair < T * K; ++pair) {
      const uint8_t* blob = eptr[pair];
      l2_prefetch(blob + L.off_codes[2] + (size_t)r0 * L.code_row_bytes[2], (size_t)nrows * L.code_row_bytes[2]);
      l2_prefetch(blob + L.off_scales[2] + (size_t)r0 * L.scale_row_bytes[2], (size_t)nrows * L.scale_row_bytes[2]);
    }
  }
  if (ok) phase_expert_gateup<FMT, kGateUpR>(eptr, L, p.x, T, p.tw_h, p.he, red);
  grid_arrive(&ctr[2]);

  // ---- phase 2: shared down, routed down, combine ---------------------------
  if (L.has_shared) {
    ok = ok && grid_wait(&ctr[1], G, &ctr[5], p.err, p.timeout_ns, &s_flag);
    if (ok) phase_shared_down<kDownR>(p.sd, p.hs, T, H, I, p.tw_i, r0, r1, ys, red);
  }
  ok = ok && grid_wait(&ctr[2], G, &ctr[5], p.err, p.timeout_ns, &s_flag);
  if (ok) {
    phase_expert_down<FMT, kDownR>(eptr, L, p.he, T, p.tw_i, r0, r1, ypart, red);
    __syncthreads();
    for (int q = threadIdx.x; q < T * nrows; q += kThreads) {
      const int t = q / nrows, j = q - t * nrows;
      float acc = 0.f;
      for (int k = 0; k < K; ++k) acc = fmaf(tk_w[t * K + k], ypart[(t * K + k) * nrows + j], acc);
      const float res = __bfloat162float(__ushort_as_bfloat16(p.res[(size_t)t * H + r0 + j]));
      float h = res + acc;
      if (L.has_shared) h += ys[t * nrows + j];
      hacc[t * nrows + j] = h;
      p.h_out[(size_t)t * H + r0 + j] = __bfloat16_as_ushort(__float2bfloat16_rn(h));
    }
    __syncthreads();
    if (warp < T) {
      float s = 0.f;
      for (int j = lane; j < nrows; j += 32) s = fmaf(hacc[warp * nrows + j], hacc[warp * nrows + j], s);
      s = warp_sum(s);
      if (lane == 0) p.ss[(size_t)c * T + warp] = s;
    }
  }
  grid_arrive(&ctr[3]);

  // ---- phase 3: RMSNorm -----------------------------------------------------
  ok = ok && grid_wait(&ctr[3], G, &ctr[5], p.err, p.timeout_ns, &s_flag);
  if (ok) {
    if (warp < T) {
      float s = 0.f;
      for (int b = lane; b < G; b += 32) s += __ldcg(p.ss + (size_t)b * T + warp);
      s = warp_sum(s);
      if (lane == 0) inv[warp] = 1.f / sqrtf(s / (float)H + L.eps);
    }
    __syncthreads();
    for (int q = threadIdx.x; q < T * nrows; q += kThreads) {
      const int t = q / nrows, j = q - t * nrows;
      const float gm = __bfloat162float(__ushort_as_bfloat16(p.gamma[r0 + j]));
      p.y_norm[(size_t)t * H + r0 + j] = __bfloat16_as_ushort(__float2bfloat16_rn(hacc[t * nrows + j] * inv[t] * gm));
    }
  }

  // ---- exit: the last block out resets the counters for the next launch -----
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    const uint32_t old = atomicAdd(&ctr[4], 1u);
    if (old == (uint32_t)G - 1u) {
      for (int i = 0; i < 6; ++i) atomicExch(&ctr[i], 0u);
      __threadfence();
    }
  }
}

template <int FMT>
static cudaError_t launch_one(const DecodeParams& p, int grid, size_t smem, cudaStream_t st) {
  static bool attr_set[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && !attr_set[dev]) {
    cudaError_t e = cudaFuncSetAttribute(moe_decode_kernel<FMT>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024);
    if (e != cudaSuccess) return e;
    attr_set[dev] = true;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, moe_decode_kernel<FMT>, p);
}

cudaError_t launch_decode(const DecodeParams& p, int grid, size_t smem, cudaStream_t st) {
  return p.L.bits == 4 ? launch_one<FMT_Q4>(p, grid, smem, st) : launch_one<FMT_Q2>(p, grid, smem, st);
}

cudaError_t decode_occupancy(int bits, size_t smem, int* blocks_per_sm) {
  if (bits == 4)
    return cudaOccupancyMaxActiveBlocksPerMultiprocessor(blocks_per_sm, moe_decode_kernel<FMT_Q4>, kThreads, smem);
  return cudaOccupancyMaxActiveBlocksPerMultiprocessor(blocks_per_sm, moe_decode_kernel<FMT_Q2>, kThreads, smem);
}

// A stand-alone bounded wait on a counter that nothing increments: checks the
// timeout path of grid_wait (it must record the timeout and return) without
// a fault or a hang.
__global__ void barrier_timeout_probe_kernel(uint32_t* ctr, uint32_t* err, uint64_t timeout_ns) {
  __shared__ int s_flag;
  grid_wait(&ctr[0], 0xffffffffu, &ctr[5], err, timeout_ns, &s_flag);
  __syncthreads();
  if (threadIdx.x == 0) {
    const uint32_t old = atomicAdd(&ctr[4], 1u);
    if (old == gridDim.x - 1u)
      for (int i = 0; i < 6; ++i) atomicExch(&ctr[i], 0u);
  }
}

cudaError_t launch_barrier_timeout_probe(uint32_t* ctr, uint32_t* err, uint64_t timeout_ns, cudaStream_t st) {
  barrier_timeout_probe_kernel<<<2, 64, 0, st>>>(ctr, err, timeout_ns);
  return cudaGetLastError();
}

}  // namespace moe
