// moe_kernels.h -- host-side declarations of the kernels' launch wrappers.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "moe_layout.h"

namespace moe {

// Geometry of the packed rows of one matrix with `cols` input columns, as the
// tensor-core dot walks it: the weights are the A operand of m16n8k16 steps
// (16 rows, two 8-row blocks of the packed layout), and the 8 columns of B
// carry a "window" of groups: 8 groups of activations for gate/up (gpw = 8),
// or 4 groups of the intermediate as bf16 hi and lo columns for down
// (gpw = 4).  G groups of 64 columns, nwin windows, W windows per work unit,
// U units per 16-row block (U <= kMaxUnits).
constexpr int kMaxUnits = 8;
constexpr int kRowBlock = 16;  // rows of one routed work unit (the mma's M)
constexpr int kMaxGrid = 256;  // most blocks of a fused-kernel launch (one per SM)
constexpr int kMaxPairsFused = 64;  // tokens x K of one fused-kernel launch (tokens <= 64 / K)
struct RoutedGeo {
  int G, gpw, nwin, W, U;
};

// Device counters of a device-resolved expert-streaming cache: the use
// clock, hits, misses, bytes copied, copy time, the error code, and the fill
// kernel's bookkeeping (blocks done, first and last timestamps, fills).
enum StreamCounter {
  DC_CLOCK = 0, DC_HITS, DC_MISSES, DC_BYTES, DC_FILL_NS, DC_ERROR, DC_FILL_DONE, DC_FILL_T0, DC_FILL_T1,
  DC_FILLS, DC_N
};

// A device-resolved cache as a streamed layer call sees it: the slot table
// [L][E] -> slot (or -1), each slot's key (layer * E + expert, or -1) and
// last use, the counters, the pinned store as the device addresses it
// ([L][E] blobs), and the slots (one blob each).
struct StreamView {
  int32_t* slot_of;
  int32_t* key;
  uint64_t* tick;
  uint64_t* dctr;
  const uint8_t* host;
  uint8_t* slots;
  int S;      // slots
  int layer;  // the layer of this call
};
// A streamed call publishes each pair's slot in 15 bits beside a 16-bit
// expert index, and keeps the slots it holds as a bitmap in the 8 * E bytes
// of the top-K key buffer: S <= 32767, S <= 64 * E, E <= 65535.
constexpr int kStreamMaxSlots = 32767;
constexpr int kStreamMaxExperts = 65535;
__host__ __device__ inline RoutedGeo routed_geo(int cols, int gpw) {
  RoutedGeo g;
  g.G = cols / 64;
  g.gpw = gpw;
  g.nwin = (g.G + gpw - 1) / gpw;
  g.W = (g.nwin + kMaxUnits - 1) / kMaxUnits;
  g.U = (g.nwin + g.W - 1) / g.W;
  return g;
}

// Output rows [r0, r1) of block c of G: whole 16-row blocks, spread evenly.
__host__ __device__ inline void block_rows(int H, int c, int G, int& r0, int& r1) {
  const uint32_t nrb = (uint32_t)H / 16u;  // nrb * G < 2^32
  r0 = (int)(16u * (nrb * (uint32_t)c / (uint32_t)G));
  r1 = (int)(16u * (nrb * (uint32_t)(c + 1) / (uint32_t)G));
}
__host__ __device__ inline int decode_rows_max(int H, int G) { return 16 * ((H / 16 + G - 1) / G); }

// Workspace of a layer call: counters and error word first, then the
// intermediates.  ctr[1] shared gate/up, [2] routed gate/up, [3] blocks that
// finished, [5] abort flag of the running launch, [6] the last launch's
// epoch (each launch publishes its router logits and sums of squares as
// 64-bit words tagged with its own epoch, ctr[6] + 1), [7] blocks done
// copying a streamed call's missed experts.
struct DecodeParams {
  Layout L;
  int T;
  const void* const* expert_ptr;
  const uint16_t* wr;
  const float* bias;
  const uint16_t* sg;
  const uint16_t* su;
  const uint16_t* sd;
  const uint16_t* gamma;
  const uint16_t* gamma_pre;  // L.prenorm: bf16 [H] weight of the RMSNorm applied to x first
  uint16_t* x_out;            // L.prenorm: the normalised x, bf16 [T][H] (block 0 writes it), or null
  const uint16_t* sgate;      // L.sgate: bf16 [H], the shared expert's output gate
  const uint8_t* spacked;     // L.spacked: the shared expert's packed blob (pair K of each token)
  const uint16_t* x;
  const uint16_t* res;
  uint16_t* h_out;
  uint16_t* y_norm;
  int32_t* idx_out;
  float* w_out;
  const int32_t* idx_in;  // routing given ([T][K] expert ids and weights), or null: the kernel routes
  const float* w_in;
  uint32_t* ctr;
  uint32_t* err;
  uint64_t* logits;  // [T][E] router logits as epoch words (epoch << 32 | float bits)
  float* hs;         // [T][I]
  uint8_t* hf;       // routed intermediate as hi/lo bf16 B fragments, 4*T*K*I bytes
  float* hx;         // [T*K][I/16] sums of hi + lo over 16-row blocks
  uint64_t* ss;      // [grid][T] each block's sum of squares of its rows of h, as epoch words
  uint64_t* route;   // [T][K][3] the routing block 0 found (expert index, weight bits, cache slot), as epoch words
  uint64_t* sstot;   // [T] the total sum of squares block 0 found, as epoch words
  uint64_t timeout_ns;
  uint32_t slot_bytes;  // bytes per shared-memory ring slot
  int nslots;           // ring slots (2..4)
  uint64_t* trace;      // optional [grid][64] phase timestamps (ns), or null
  // streamed layer call (expert_ptr null): block 0 looks the chosen experts
  // up in the cache, takes slots for the misses, and every block copies its
  // share of the missed blobs from the store before the routed tiles
  int streamed;
  StreamView sv;
};

constexpr int kDecodeBlockThreads = 512;  // 14 consumer warps, a producer warp, a sync warp
size_t decode_smem_bytes(const Layout& L, int T, int nrows, int nslots, uint32_t slot_bytes);
uint32_t decode_slot_bytes(const Layout& L, int T, int nrows_max, int* nslots);
cudaError_t launch_decode(const DecodeParams& p, int grid, size_t smem, cudaStream_t st);
cudaError_t decode_occupancy(int bits, size_t smem, int* blocks_per_sm);
cudaError_t launch_barrier_timeout_probe(uint32_t* ctr, uint32_t* err, uint64_t timeout_ns,
                                         cudaStream_t st);

// Stand-alone router: logits into `logits` ([T][E]), then top-K.
cudaError_t launch_router_logits(const uint16_t* x, const uint16_t* wr, const float* bias, int T,
                                 int H, int E, int grid, float* logits, cudaStream_t st);
cudaError_t launch_topk(const float* logits, int T, int E, int K, int32_t* idx, float* w,
                        cudaStream_t st);

// Device packer: e_count experts, fp32 weights [e][I][H], [e][I][H], [e][H][I].
cudaError_t launch_pack(const Layout& L, const float* wg, const float* wu, const float* wd,
                        int e_count, uint8_t* out, cudaStream_t st);

// ---- batched path (moe_grouped.cu) ----
struct GemmParams;
size_t grouped_gemm_smem_bytes(int na, bool packed);
// ak: 0 dense bf16 A, 4 / 2 packed A; na: A matrices (2 = gate and up);
// epi: 0 fp32 (+ bias), 1 SwiGLU -> fp16, 2 SwiGLU -> bf16 hi and lo.
cudaError_t launch_grouped_gemm(int ak, int na, int epi, const GemmParams& p, int grid, cudaStream_t st);
cudaError_t launch_set_ptr(const void** dst, const void* v, cudaStream_t st);
cudaError_t launch_prenorm(const uint16_t* h, const uint16_t* gamma, int T, int H, float eps, uint16_t* x,
                           cudaStream_t st);
cudaError_t launch_to_half(const uint16_t* x, void* xh, size_t n, uint32_t* abort_flag, cudaStream_t st);
cudaError_t launch_group(const int32_t* idx, int TK, int E, int K, int* slot_token, int* pair_slot, int* ch_e,
                         int* ch_c0, int* ch_n, int* n_chunks, const void* const* expert_ptr, uint32_t* err,
                         cudaStream_t st);
cudaError_t launch_combine(const float* Y, const float* Ys, const int* pair_slot, const float* w, const uint16_t* res,
                           const uint16_t* gamma, int T, int H, int K, float eps, const uint16_t* x,
                           const uint16_t* sgate, uint16_t* h_out, uint16_t* y_norm, cudaStream_t st);

}  // namespace moe
