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
// and the codes are stored in the block layout described in moe_layout.h.
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

// Quantise one 64-weight group: writes the 64 codes (column order) to q and
// returns the scale word (scale in bits 0..15, bias in bits 16..31).
__host__ __device__ inline uint32_t quantize_group64(const float* w, int bits, uint8_t* q) {
  float mn = w[0], mx = w[0];
  for (int i = 1; i < 64; ++i) {
    mn = w[i] < mn ? w[i] : mn;
    mx = w[i] > mx ? w[i] : mx;
  }
  const float qmax = (float)((1 << bits) - 1);
  const uint16_t sb = bf16_rne_bits(div_rn(sub_rn(mx, mn), qmax));
  const uint16_t bb = bf16_rne_bits(mn);
  const float s = bf16_bits_to_f32(sb), beta = bf16_bits_to_f32(bb);
  for (int i = 0; i < 64; ++i) {
    uint8_t c = 0;
    if (s != 0.f) {
      float r = rintf(div_rn(sub_rn(w[i], beta), s));
      r = r < 0.f ? 0.f : (r > qmax ? qmax : r);
      c = (uint8_t)r;
    }
    q[i] = c;
  }
  return (uint32_t)sb | ((uint32_t)bb << 16);
}

// Block layout of the codes (see moe_layout.h): the words of row `row`
// (row % 8 = n) for one 64-column group are the lanes 4n + t, t = 0..3;
// lane words hold, per 16-column step s, the columns 16s + 2t + e ("first")
// and 16s + 8 + 2t + e ("second"), e = 0, 1.
// 4-bit: two words per lane; word s/2, nibble 2(s%2) + 4e (first) or
//        2(s%2) + 1 + 4e (second).  2-bit: one word; code 2s + 8e (first) or
//        2s + 1 + 8e (second).
__host__ __device__ inline void group_words(const uint8_t* q, int bits, int t, uint32_t* words) {
  if (bits == 4) {
    for (int h = 0; h < 2; ++h) {
      uint32_t w = 0;
      for (int j = 0; j < 2; ++j) {
        const int s = 2 * h + j;
        for (int e = 0; e < 2; ++e) {
          w |= (uint32_t)q[16 * s + 2 * t + e] << (4 * (2 * j + 4 * e));
          w |= (uint32_t)q[16 * s + 8 + 2 * t + e] << (4 * (2 * j + 1 + 4 * e));
        }
      }
      words[h] = w;
    }
  } else {
    uint32_t w = 0;
    for (int s = 0; s < 4; ++s)
      for (int e = 0; e < 2; ++e) {
        w |= (uint32_t)q[16 * s + 2 * t + e] << (2 * (2 * s + 8 * e));
        w |= (uint32_t)q[16 * s + 8 + 2 * t + e] << (2 * (2 * s + 1 + 8 * e));
      }
    words[0] = w;
  }
}

// Store the codes and scale word of (row, group g) of a [rows][cols] matrix.
__host__ __device__ inline void store_group(uint8_t* codes, uint8_t* scales, int bits, int cols, int row,
                                            int g, const uint8_t* q, uint32_t sw) {
  const size_t block = (size_t)(row / 8) * (cols / 64) + g;
  const int n = row % 8;
  const int wpl = bits == 4 ? 2 : 1;  // words per lane
  uint32_t* blk = reinterpret_cast<uint32_t*>(codes + block * (size_t)(64 * bits));
  for (int t = 0; t < 4; ++t) {
    uint32_t words[2];
    group_words(q, bits, t, words);
    for (int h = 0; h < wpl; ++h) blk[(4 * n + t) * wpl + h] = words[h];
  }
  reinterpret_cast<uint32_t*>(scales)[block * 8 + n] = sw;
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
  uint8_t q[64];
  const uint32_t sw = quantize_group64(w, L.bits, q);
  uint8_t* blob = out + e * L.blob_bytes;
  store_group(blob + L.off_codes[m], blob + L.off_scales[m], L.bits, (int)cols, (int)row, (int)g, q, sw);
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
  uint8_t q[64];
  for (int m = 0; m < 3; ++m)
    for (int r = 0; r < rows[m]; ++r)
      for (int g = 0; g < cols[m] / 64; ++g) {
        const uint32_t sw = quantize_group64(src[m] + (size_t)r * cols[m] + (size_t)g * 64, L.bits, q);
        store_group(blob + L.off_codes[m], blob + L.off_scales[m], L.bits, cols[m], r, g, q, sw);
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
