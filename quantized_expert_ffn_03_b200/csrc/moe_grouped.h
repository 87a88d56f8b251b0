// moe_grouped.h -- launch parameters of the batched path's GEMM kernel
// (moe_grouped.cu), shared with the host code that sets it up.
#pragma once

#include <stdint.h>

namespace moe {

// Parameters of one GEMM launch.  Output rows are features (M of them), the
// reduction runs over K (a multiple of 64), columns are tokens or slots.
struct GemmParams {
  int M, K;
  int bits;                      // packed A: 4 or 2
  // packed A (routed experts): blob of expert e = expert_ptr[e]; matrix a's
  // codes / scales at the section offsets; G = K / 64 groups per row
  const void* const* expert_ptr;
  uint32_t off_codes[2], off_scales[2];
  // dense A (bf16 [M][K] per matrix)
  const uint16_t* a_dense[2];
  // B: 16-bit rows of length K: row of column c = b_rows ? b_rows[col0 + c] : col0 + c;
  // b2 (if set) is a second B read after b with the same A (K doubled)
  const uint16_t* b;
  const uint16_t* b2;
  const int* b_rows;
  // columns: chunks (expert, first column, count) from the grouping step, or
  // dense chunks of 128 over n_cols
  const int* ch_e;
  const int* ch_c0;
  const int* ch_n;
  const int* n_chunks_dev;
  int n_cols;
  // epilogue
  void* out;       // [column][M] (fp32, or fp16 / bf16 hi for SwiGLU)
  void* out2;      // bf16 lo part (shared gate/up)
  const float* bias;  // [M] added to fp32 outputs (router) or null
  uint32_t* err;
  uint32_t* abort_flag;
  uint64_t timeout_ns;
};


}  // namespace moe
