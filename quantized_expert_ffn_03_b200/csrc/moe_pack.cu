// moe_pack.cu -- expert repacker: fp32 weights -> packed 4/2-bit blobs.
//
// The pages repack the model's experts offline into 4-bit and 2-bit files
// ("Flash-MoE: ラップトップでの397Bパラメータモデルの実行", section
// "プロジェクト構成": repack_experts.py, repack_experts_2bit.py).  Here the
// same group-affine quantiser runs on the host (multi-threaded) and on the
// GPU, and the two give bit-identical blobs: every float step is one IEEE
// single-precision operation in the same order, with no contraction.
//   s = bf16_rne((max - min) / (2^b - 1)),  beta = bf16_rne(min)
//   q = clamp(rint((w - beta) / s), 0, 2^b - 1),  q = 0 when s == 0
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstring>
#include <thread>
#include <vector>

#include "moe_kernels.h"

namespace moe {

__host__ __device__ inline uint16_t bf16_rne_bits(float f) {
  uint32_t u;
#ifdef __CUDA_ARCH__
  u = __float_as_uint(f);
#else
  std::memcpy(&u, &f, 4);
#endif
  if ((u & 0x7f800000u) == 0x7f800000u && (u & 0x007fffffu)) return (uint16_t)((u >> 16) | 0x40u);
  const uint32_t lsb = (u >> 16) & 1u;
  return (uint16_t)((u + 0x7fffu + lsb) >> 16);
}

__host__ __device__ inline float bf16_bits_to_f32(uint16_t h) {
  const uint32_t u = (uint32_t)h << 16;
#ifdef __CUDA_ARCH__
  return __uint_as_float(u);
#else
  float f;
  std::memcpy(&f, &u, 4);
  return f;
#endif
}

// IEEE single operations that the compiler may not fuse or reorder.
__host__ __device__ inline float sub_rn(float a, float b) {
#ifdef __CUDA_ARCH__
  return __fsub_rn(a, b);
#else
  volatile float r = a - b;
  return r;
#endif
}
__host__ __device__ inline float div_rn(float a, float b) {
#ifdef __CUDA_ARCH__
  return __fdiv_rn(a, b);
#else
  volatile float r = a / b;
  return r;
#endif
}

// Quantise one 64-weight group: writes 64*bits/32 code words and returns the
// scale word (scale in bits 0..15, bias in bits 16..31).
__host__ __device__ inline uint32_t quantize_group64(const float* w, int bits, uint32_t* words) {
  float mn = w[0], mx = w[0];
  for (int i = 1; i < 64; ++i) {
    mn = w[i] < mn ? w[i] : mn;
    mx = w[i] > mx ? w[i] : mx;
  }
  const float qmax = (float)((1 << bits) - 1);
  const uint16_t sb = bf16_rne_bits(div_rn(sub_rn(mx, mn), qmax));
  const uint16_t bb = bf16_rne_bits(mn);
  const float s = bf16_bits_to_f32(sb), beta = bf16_bits_to_f32(bb);
  const int per_word = 32 / bits;
  for (int j = 0; j < 64 / per_word; ++j) {
    uint32_t word = 0;
    for (int n = 0; n < per_word; ++n) {
      uint32_t q = 0;
      if (s != 0.f) {
        float r = rintf(div_rn(sub_rn(w[j * per_word + n], beta), s));
        r = r < 0.f ? 0.f : (r > qmax ? qmax : r);
        q = (uint32_t)r;
      }
      word |= q << (n * bits);
    }
    words[j] = word;
  }
  return (uint32_t)sb | ((uint32_t)bb << 16);
}

// ---- device packer: one thread per (expert, matrix, row, group) -------------
__global__ void pack_kernel(Layout L, const float* wg, const float* wu, const float* wd, int e_count,
                            uint8_t* out) {
  const uint64_t gpr_h = L.H / 64, gpr_i = L.I / 64;
  const uint64_t n_gu = (uint64_t)L.I * gpr_h;  // groups in gate (or up)
  const uint64_t n_d = (uint64_t)L.H * gpr_i;
  const uint64_t per_e = 2 * n_gu + n_d;
  const uint64_t gid = (uint64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (gid >= per_e * (uint64_t)e_count) return;
  const uint64_t e = gid / per_e;
  uint64_t rem = gid - e * per_e;
  int m;
  if (rem < n_gu) {
    m = 0;
  } else if (rem < 2 * n_gu) {
    m = 1;
    rem -= n_gu;
  } else {
    m = 2;
    rem -= 2 * n_gu;
  }
  const uint64_t gpr = m == 2 ? gpr_i : gpr_h;
  const uint64_t cols = m == 2 ? L.I : L.H;
  const uint64_t rows = m == 2 ? L.H : L.I;
  const uint64_t row = rem / gpr, g = rem - row * gpr;
  const float* src = (m == 0 ? wg : m == 1 ? wu : wd) + e * rows * cols + row * cols + g * 64;
  float w[64];
  const float4* s4 = reinterpret_cast<const float4*>(src);
  for (int i = 0; i < 16; ++i) {
    const float4 v = s4[i];
    w[4 * i] = v.x;
    w[4 * i + 1] = v.y;
    w[4 * i + 2] = v.z;
    w[4 * i + 3] = v.w;
  }
  uint32_t words[8];
  const uint32_t sw = quantize_group64(w, L.bits, words);
  uint8_t* blob = out + e * L.blob_bytes;
  uint32_t* cdst = reinterpret_cast<uint32_t*>(blob + L.off_codes[m] + row * L.code_row_bytes[m] +
                                               g * (64 * L.bits / 8));
  for (int j = 0; j < 2 * L.bits; ++j) cdst[j] = words[j];
  *reinterpret_cast<uint32_t*>(blob + L.off_scales[m] + row * L.scale_row_bytes[m] + g * 4) = sw;
}

cudaError_t launch_pack(const Layout& L, const float* wg, const float* wu, const float* wd,
                        int e_count, uint8_t* out, cudaStream_t st) {
  const uint64_t per_e = 3ull * L.H * L.I / 64;
  const uint64_t n = per_e * (uint64_t)e_count;
  if (n == 0) return cudaSuccess;
  // padding bytes between sections are part of the format: zero them first
  cudaError_t err = cudaMemsetAsync(out, 0, L.blob_bytes * (size_t)e_count, st);
  if (err != cudaSuccess) return err;
  const int threads = 256;
  pack_kernel<<<(unsigned)((n + threads - 1) / threads), threads, 0, st>>>(L, wg, wu, wd, e_count, out);
  return cudaGetLastError();
}

// ---- host packer --------------------------------------------------------------
static void pack_one_host(const Layout& L, const float* wg, const float* wu, const float* wd,
                          uint8_t* blob) {
  std::memset(blob, 0, L.blob_bytes);
  const float* src[3] = {wg, wu, wd};
  const int rows[3] = {L.I, L.I, L.H};
  const int cols[3] = {L.H, L.H, L.I};
  uint32_t words[8];
  for (int m = 0; m < 3; ++m)
    for (int r = 0; r < rows[m]; ++r)
      for (int g = 0; g < cols[m] / 64; ++g) {
        const uint32_t sw = quantize_group64(src[m] + (size_t)r * cols[m] + (size_t)g * 64, L.bits, words);
        std::memcpy(blob + L.off_codes[m] + (size_t)r * L.code_row_bytes[m] + (size_t)g * (64 * L.bits / 8),
                    words, 8 * L.bits);
        std::memcpy(blob + L.off_scales[m] + (size_t)r * L.scale_row_bytes[m] + (size_t)g * 4, &sw, 4);
      }
}

void pack_host(const Layout& L, const float* wg, const float* wu, const float* wd, int e_begin,
               int e_count, uint8_t* out) {
  const size_t gu = (size_t)L.I * L.H, dn = (size_t)L.H * L.I;
  const unsigned hw = std::max(1u, std::thread::hardware_concurrency());
  const int nthreads = (int)std::min<unsigned>(hw, (unsigned)std::max(e_count, 1));
  std::vector<std::thread> pool;
  for (int w = 0; w < nthreads; ++w) {
    pool.emplace_back([&, w] {
      for (int e = w; e < e_count; e += nthreads) {
        const size_t ge = (size_t)(e_begin + e);
        pack_one_host(L, wg + ge * gu, wu + ge * gu, wd + ge * dn, out + (size_t)e * L.blob_bytes);
      }
    });
  }
  for (auto& t : pool) t.join();
}

}  // namespace moe
