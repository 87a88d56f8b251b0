// moe_layout.h -- packed-expert layout and launch geometry shared by the host
// side and the kernels of libmoe.  Plain C++ (no CUDA types) so that the host
// packer can use it too.
#pragma once

#include <stddef.h>
#include <stdint.h>

namespace moe {

constexpr int kMaxTokensFused = 8;           // tokens per launch of the fused decode kernel
constexpr int kMaxK = 32;                    // largest top_k

// Where the sections of one packed expert blob live (byte offsets) and how
// many bytes a row takes in each.  Matrix index m: 0 gate [I][H], 1 up [I][H],
// 2 down [H][I].  Sections follow each other in the order gate codes, up
// codes, down codes, gate scales, up scales, down scales, each starting on a
// 256-byte boundary.
//
// Inside a code section the codes come in blocks of 8 rows x 64 columns,
// row-block major then column group (64*b bytes per block); inside a block,
// lane l = 4*(row % 8) + t owns 2*b bytes holding the codes that the
// tensor-core B fragment of an m16n8k16 step takes for t (see moe_pack.cu).
// Scale words are stored [row block][group][row % 8].  So any run of whole
// row blocks is one contiguous byte range in both sections, of
// rows * code_row_bytes and rows * scale_row_bytes bytes.
struct Layout {
  int H, I, E, K, bits;
  int has_shared;
  float eps;
  int prenorm;  // 1: the layer's x is its residual stream, RMS-normalised with a second gamma first
  int sgate;    // 1: the shared expert's output is scaled by sigmoid(x . g), g bf16 [H]
  int spacked;  // 1: the shared expert is a packed blob, run as pair K of every token
  int KP;       // (token, expert) pairs per token: K, or K + 1 with a packed shared expert
  uint32_t off_codes[3];
  uint32_t off_scales[3];
  uint32_t code_row_bytes[3];
  uint32_t scale_row_bytes[3];
  uint64_t blob_bytes;
};

inline uint64_t round_up_256(uint64_t n) { return (n + 255u) & ~uint64_t(255); }

// Fills L from the shape; returns false if the shape is not supported
// (bits not 2/4, group not 64, H or I not a multiple of 64).
inline bool make_layout(int H, int I, int E, int K, int bits, int group, int has_shared,
                        float eps, Layout* L) {
  if (bits != 2 && bits != 4) return false;
  if (group != 64 || H <= 0 || I <= 0 || H % 64 || I % 64) return false;
  L->H = H;
  L->I = I;
  L->E = E;
  L->K = K;
  L->bits = bits;
  L->has_shared = has_shared;
  L->eps = eps;
  L->prenorm = 0;
  L->sgate = 0;
  L->spacked = 0;
  L->KP = K;
  const uint64_t rows[3] = {(uint64_t)I, (uint64_t)I, (uint64_t)H};
  const uint64_t cols[3] = {(uint64_t)H, (uint64_t)H, (uint64_t)I};
  uint64_t pos = 0;
  for (int m = 0; m < 3; ++m) {
    L->code_row_bytes[m] = (uint32_t)(cols[m] * bits / 8);
    L->off_codes[m] = (uint32_t)pos;
    pos = round_up_256(pos + rows[m] * L->code_row_bytes[m]);
  }
  for (int m = 0; m < 3; ++m) {
    L->scale_row_bytes[m] = (uint32_t)(cols[m] / 64 * 4);
    L->off_scales[m] = (uint32_t)pos;
    pos = round_up_256(pos + rows[m] * L->scale_row_bytes[m]);
  }
  L->blob_bytes = pos;
  return true;
}

}  // namespace moe
