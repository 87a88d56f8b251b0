// moe_decode.cu -- the fused single-launch MoE layer for decode (T <= 8).
//
// One persistent cooperative launch, one block per SM.  Each block streams
// exactly the weight bytes it owns through a ring of shared-memory slots:
// a producer warp issues bulk copies (cp.async.bulk, completion counted on an
// mbarrier per slot) and 14 consumer warps compute from shared memory.  A
// sync warp prepares the activations, does the block's grid-wide arrivals and
// waits, runs the router's top-K and stages the intermediates, so consumers
// never stall on a release fence, on polling global memory, or on block-wide
// barriers between tiles.
// The block's byte stream, in order:
//   router rows  -> [arrive R]  shared gate/up rows  -> [arrive S]
//   (sync warp: wait R, top-K, expert pointers; producer waits for them)
//   routed gate/up row blocks of the chosen experts  -> [arrive E]
//   [wait S]  shared down rows of the block's output rows
//   [wait E]  routed down row blocks of the block's output rows
// then combine + residual, a grid-wide sum of squares, and RMSNorm of the
// block's rows.  The copies that follow a wait are already in flight while a
// block waits, so HBM stays busy across the waits.  Phase arrivals and waits
// ride on the data tiles as flags, so they take no ring slot of their own.
//
// bf16 rows (router, shared expert) are dotted on the CUDA cores, one row per
// warp.  Packed expert rows go through the tensor cores: mma.sync m16n8k16
// with the 4/2-bit codes as the B operand (each code becomes the bf16 number
// 128 + q with two logic ops), the activations as the A operand, and the
// group's scale and bias applied to the fp32 result:
//   sum_k x_k (q_k s + beta) = s * D + (beta - 128 s) * X,
//   D = sum_k x_k (128 + q_k),  X = sum_k x_k  over the group's 64 columns.
// A "window" is 8 consecutive groups of one 8-row block: A row m carries the
// activations of group m of the window (zero in the other groups' steps), so
// after the window's 32 mma steps lane group m holds group m's D for 8
// weight rows and the scale epilogue is spread over all 32 lanes.  For the
// down projection the fp32 intermediate is split into bf16 hi + lo parts in
// A rows 0..7 and 8..15, so it enters at about 16 bits of precision.
//
// This is the single-kernel form of the pages' pipeline: router projection
// with the shared expert (CMD2), top-K, the K expert reads and the deferred
// expert forward with combine + residual + norm (CMD3)
// ("Flash-MoE: ラップトップでの397Bパラメータモデルの実行", section
// "パイプライン概要"; "Streaming experts: как запустить триллионную модель на
// MacBook", sections "Flash-MoE: чистый C, Metal и никакого Python" and
// "Оптимизации, которые сработали").
#include <cuda_bf16.h>

#include <mutex>

#include "../../include/moe.h"
#include "moe_kernels.h"
#include "moe_device.cuh"

namespace moe {

// 16 warps in all, 4 per SM sub-partition, so each thread may use up to 128
// registers: 14 consumer warps, the producer warp and the sync warp.
constexpr int kConsumerWarps = 14;
constexpr int kConsumers = kConsumerWarps * 32;  // 448
constexpr int kProducerWarp = kConsumerWarps;    // warp 14
constexpr int kSyncWarp = kConsumerWarps + 1;    // warp 15
constexpr int kDecodeThreads = kConsumers + 64;
static_assert(kDecodeThreads == kDecodeBlockThreads, "block size");
constexpr int kSlots = 4;  // ring slots at most (the launch picks 2..4)
constexpr int kMaxSeg = 8;
constexpr int kMaxSlotBytes = 48 * 1024;
constexpr int kTraceEntries = 128;
// Routed gate/up: at most this many row blocks per tile, and a ring of
// accumulator entries large enough for every row block of kSlots tiles.
constexpr int kMaxRbPerTile = 2;
constexpr int kAccSlots = kSlots * kMaxRbPerTile;
// One-token router and shared gate/up tiles with few rows: each row is dotted
// in up to kMaxParts column parts by different warps (a tile of at most
// kSplitRows rows), and the warp that finishes a row's last part sums the
// parts in order.
constexpr int kSplitRows = 7;
constexpr int kMaxParts = 14;

enum TileType : int { TILE_NONE = 0, TILE_ROUTER, TILE_SHARED_GU, TILE_EXPERT_GU, TILE_SHARED_DOWN, TILE_EXPERT_DOWN };

// flags carried by a tile: waits done before its compute, arrivals after it
enum TileFlag : int {
  F_WAIT_S = 1,
  F_WAIT_E = 2,
  F_ARRIVE_R = 4,
  F_ARRIVE_S = 8,
  F_ARRIVE_E = 16,
  F_END = 32
};

struct Seg {
  int pair;   // (token, expert) pair of routed tiles
  int row0;   // bf16 tiles: first matrix row; routed tiles: first 8-row block
  int nrows;  // bf16 tiles: rows; routed tiles: row blocks
  int u0, u1; // routed tiles: units of each row block held in the slot
  int gbase;  // routed tiles: first group held (0 for whole row blocks)
  int acc;    // routed gate/up: accumulator entry of the first row block
  uint32_t off[8];  // slot byte offset of each range's first valid byte
};

struct TileDesc {
  int type;
  int nseg;
  int pre;   // F_WAIT_* flags
  int post;  // F_ARRIVE_* / F_END flags
  Seg seg[kMaxSeg];
};

// barriers consumers -> sync warp (evt) and sync warp -> consumers (go)
enum { EVT_R = 0, EVT_S, EVT_E, EVT_D, NEVT };
enum { GO_S = 0, GO_E, GO_D, NGO };
// flags[] slots: routing valid; consumer warps past the S tiles; a sum of
// squares that never arrived; this launch's epoch
enum { FLAG_TOPK = NGO, FLAG_SCNT, FLAG_NOSS, FLAG_EPOCH };

// ---- shared-memory plan ------------------------------------------------------
// xf: x as mma A fragments, [token][group][t][8 words]; word 2s is the bf16
//     pair at columns 16s + 2t (+1) of the group, word 2s+1 the pair at 16s + 8 + 2t.
// xsum: per token, the G group sums of x, then (4-bit experts) the G
//     power-of-two scales of x's int8 limbs.
// hf: routed intermediate as A fragments (hi/lo), [pair][group][t][step] x 16 bytes.
// hx: per (pair, 8-row block of I) sum of hi + lo.
struct DecodeSmem {
  size_t ring, bars, desc, xs, xf, xsum, hs, hf, hx, zero, part, cnt, rpart, rcnt, tk_w, tk_i, eptr, tkbuf, res, gam,
      gpre, sgv, ypart, ys, hacc, inv, flags, spin, total;
};

__host__ __device__ inline size_t align_up(size_t n, size_t a) { return (n + a - 1) / a * a; }

// Optional shared-memory regions of a layout: bit 0 the pre-norm, bit 1 the
// shared output gate.
__host__ __device__ inline int smem_opts(const Layout& L) { return (L.prenorm ? 1 : 0) | (L.sgate ? 2 : 0); }

__host__ __device__ inline DecodeSmem decode_smem_plan(int T, int K, int E, int H, int I, int nrows, int nslots,
                                                       uint32_t slot_bytes, int opts) {
  const RoutedGeo gi = routed_geo(I, 4);
  DecodeSmem s;
  size_t pos = 0;
  s.ring = pos;
  pos = align_up(pos + (size_t)nslots * slot_bytes, 128);
  s.bars = pos;  // full[kSlots], empty[kSlots], xbar, xfbar, topkbar, evt[NEVT], go[NGO]
  pos = align_up(pos + 8 * (2 * kSlots + 3 + NEVT + NGO), 16);
  s.desc = pos;
  pos = align_up(pos + sizeof(TileDesc) * kSlots, 16);
  s.xs = pos;
  pos = align_up(pos + 2ull * T * H, 16);
  s.xf = pos;
  pos = align_up(pos + 2ull * T * H, 16);
  s.xsum = pos;
  pos = align_up(pos + 8ull * T * (H / 64), 16);
  s.hs = pos;
  pos = align_up(pos + 4ull * T * I, 16);
  s.hf = pos;
  pos = align_up(pos + 4ull * T * K * I, 16);
  s.hx = pos;
  pos = align_up(pos + 4ull * T * K * (I / 16), 16);
  s.zero = pos;
  pos = align_up(pos + 64, 16);
  s.part = pos;
  pos = align_up(pos + 4ull * kAccSlots * kMaxUnits * 32, 16);
  s.cnt = pos;
  pos = align_up(pos + 4ull * kAccSlots, 16);
  s.rpart = pos;
  pos = align_up(pos + 4ull * kSlots * kSplitRows * kMaxParts * 2, 16);
  s.rcnt = pos;
  pos = align_up(pos + 4ull * kSlots * kSplitRows, 16);
  s.tk_w = pos;
  pos = align_up(pos + sizeof(float) * T * K, 16);
  s.tk_i = pos;
  pos = align_up(pos + sizeof(int) * T * K, 16);
  s.eptr = pos;
  pos = align_up(pos + sizeof(void*) * T * K, 16);
  s.tkbuf = pos;
  pos = align_up(pos + sizeof(uint64_t) * E, 16);
  s.res = pos;
  pos = align_up(pos + 2ull * T * nrows, 16);
  s.gam = pos;
  pos = align_up(pos + 2ull * nrows, 16);
  s.gpre = pos;  // pre-norm gamma [H] and the consumer warps' partial sums of squares [14][T]
  pos = align_up(pos + ((opts & 1) ? 2ull * H + 4ull * kConsumerWarps * T : 0ull), 16);
  s.sgv = pos;  // shared output gate [H], the consumer warps' partial dots [14][T], the gates [T]
  pos = align_up(pos + ((opts & 2) ? 2ull * H + 4ull * (kConsumerWarps + 1) * T : 0ull), 16);
  s.ypart = pos;
  pos = align_up(pos + sizeof(float) * T * K * gi.U * nrows, 16);
  s.ys = pos;
  pos = align_up(pos + sizeof(float) * T * nrows, 16);
  s.hacc = pos;
  pos = align_up(pos + sizeof(float) * T * nrows, 16);
  s.inv = pos;
  pos = align_up(pos + sizeof(float) * T, 16);
  s.flags = pos;
  pos = align_up(pos + 16 * sizeof(int), 16);
  s.spin = pos;
  pos = align_up(pos + 16 * sizeof(uint32_t), 16);
  s.total = pos;
  return s;
}

size_t decode_smem_bytes(const Layout& L, int T, int nrows, int nslots, uint32_t slot_bytes) {
  return decode_smem_plan(T, L.KP, L.E, L.H, L.I, nrows, nslots, slot_bytes, smem_opts(L)).total;
}

// ---- small helpers ----------------------------------------------------------------

__device__ __forceinline__ void consumer_sync() { named_sync(1, kConsumers); }

// Warp-wide bounded wait on an mbarrier phase.  Every lane polls, so the
// warp never diverges around a wait: a warp left split into lane groups after
// a one-lane wait runs its later warp-wide code (shuffles, mma) several times
// slower.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, uint64_t timeout_ns,
                                          uint32_t* spins = nullptr) {
  const bool ok = mbar_wait(bar, parity, timeout_ns, (threadIdx.x & 31) == 0 ? spins : nullptr);
  return __all_sync(0xffffffffu, ok);
}

// Trace stamp k of this block (traced launches only; the untraced kernel
// carries no trace code).
template <bool TRACE>
__device__ __forceinline__ void trace_mark(const DecodeParams& p, int k) {
  if constexpr (TRACE) p.trace[(size_t)blockIdx.x * kTraceEntries + k] = globaltimer_ns();
}

// Share [a, b) of n items for block c of G (n * G < 2^32 for every caller).
__device__ __forceinline__ void range_of(int n, int c, int G, int& a, int& b) {
  a = (int)((uint32_t)n * (uint32_t)c / (uint32_t)G);
  b = (int)((uint32_t)n * (uint32_t)(c + 1) / (uint32_t)G);
}


// One grid wait by the calling thread only.
__device__ __forceinline__ bool grid_wait_thread(const uint32_t* ctr, uint32_t target, uint32_t* abort_flag,
                                                 uint32_t* err, uint64_t timeout_ns, uint32_t* spins = nullptr) {
  const uint64_t t0 = globaltimer_ns();
  bool ok = true;
  uint32_t it = 0;
  for (;; ++it) {
    if (ld_acquire_gpu(ctr) >= target) break;
    if (ld_relaxed_gpu(abort_flag) != 0u) {
      ok = false;
      break;
    }
    if ((it & 63u) == 63u && (globaltimer_ns() - t0 > timeout_ns || it > (1u << 28))) {
      atomicCAS(err, 0u, 1u);
      atomicExch(abort_flag, 1u);
      ok = false;
      break;
    }
  }
  if (spins) atomicAdd(spins, it + 1);
  return ok;
}

// ---- bf16 rows on the CUDA cores -----------------------------------------------------
// Dot of one bf16 weight row w0 (and w1, the up row of a gate/up pair, if not
// null) with up to 4 tokens' activations: bf16 x, or the fp32 shared
// intermediate (xf32).  Lane l owns columns 256k + 8l .. +7, so each 16-byte
// read of a row is contiguous across the warp.  acc[m][t]: lane partial sums.
__device__ __forceinline__ void bf16_dot4(const uint8_t* w0, const uint8_t* w1, int cols, const uint8_t* x,
                                          uint32_t xstride, bool xf32, int nt, float (&acc)[2][4]) {
  const int lane = threadIdx.x & 31;
  float2 a[2][4];
#pragma unroll
  for (int mm = 0; mm < 2; ++mm)
#pragma unroll
    for (int tt = 0; tt < 4; ++tt) a[mm][tt] = make_float2(0.f, 0.f);
#pragma unroll 1
  for (int c = 8 * lane; c < cols; c += 256) {
    uint4 q[2];
    q[0] = *reinterpret_cast<const uint4*>(w0 + 2 * c);
    q[1] = w1 ? *reinterpret_cast<const uint4*>(w1 + 2 * c) : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
    for (int tt = 0; tt < 4; ++tt) {
      if (tt < nt) {
        float xx[8];
        if (xf32) {
          const float4* xp = reinterpret_cast<const float4*>(x + tt * xstride + 4 * c);
          const float4 u = xp[0], v = xp[1];
          xx[0] = u.x, xx[1] = u.y, xx[2] = u.z, xx[3] = u.w, xx[4] = v.x, xx[5] = v.y, xx[6] = v.z, xx[7] = v.w;
        } else {
          unpack_bf16x8(*reinterpret_cast<const uint4*>(x + tt * xstride + 2 * c), xx);
        }
#pragma unroll
        for (int mm = 0; mm < 2; ++mm) {
          if (mm == 0 || w1) {
            const uint32_t w[4] = {q[mm].x, q[mm].y, q[mm].z, q[mm].w};
#pragma unroll
            for (int k = 0; k < 4; ++k)
              a[mm][tt] = __ffma2_rn(make_float2(__uint_as_float(w[k] << 16), __uint_as_float(w[k] & 0xffff0000u)),
                                     make_float2(xx[2 * k], xx[2 * k + 1]), a[mm][tt]);
          }
        }
      }
    }
  }
#pragma unroll
  for (int mm = 0; mm < 2; ++mm)
#pragma unroll
    for (int tt = 0; tt < 4; ++tt) acc[mm][tt] = a[mm][tt].x + a[mm][tt].y;
}

// ---- packed rows on the tensor cores ----------------------------------------------------

// D += A * B for one m16n8k16 step, bf16 inputs, fp32 accumulators.
__device__ __forceinline__ void mma_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                          uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// D += A * B for one m16n8k32 step, unsigned 8-bit A, signed 8-bit B,
// 32-bit integer accumulators (exact).
__device__ __forceinline__ void mma_16832_u8s8(int (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                               uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// B fragments of the four 16-column steps of one block from this lane's
// code bytes: each 16-bit half becomes the bf16 number 128 + q (exponent of
// 128 OR-ed over a code in the low mantissa bits).  Code positions: see the
// block layout in moe_layout.h.
template <int FMT>
struct LaneCodes;
template <>
struct LaneCodes<FMT_Q4> {
  uint2 w;
  static constexpr int kBytes = 8;
  __device__ __forceinline__ void load(const uint8_t* p) { w = *reinterpret_cast<const uint2*>(p); }
  __device__ __forceinline__ void frags(uint32_t (&b)[4][2]) const {
    const uint32_t v[2] = {w.x, w.y};
#pragma unroll
    for (int h = 0; h < 2; ++h)
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        b[2 * h + j][0] = ((v[h] >> (8 * j)) & 0x000F000Fu) | 0x43004300u;
        b[2 * h + j][1] = ((v[h] >> (8 * j + 4)) & 0x000F000Fu) | 0x43004300u;
      }
  }
};
template <>
struct LaneCodes<FMT_Q2> {
  uint32_t w;
  static constexpr int kBytes = 4;
  __device__ __forceinline__ void load(const uint8_t* p) { w = *reinterpret_cast<const uint32_t*>(p); }
  __device__ __forceinline__ void frags(uint32_t (&b)[4][2]) const {
#pragma unroll
    for (int s = 0; s < 4; ++s) {
      b[s][0] = ((w >> (4 * s)) & 0x00030003u) | 0x43004300u;
      b[s][1] = ((w >> (4 * s + 2)) & 0x00030003u) | 0x43004300u;
    }
  }
};

// Shared-memory loads at 32-bit shared addresses (no generic address math).
__device__ __forceinline__ uint4 lds128(uint32_t a) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(a));
  return v;
}
__device__ __forceinline__ uint2 lds64(uint32_t a) {
  uint2 v;
  asm volatile("ld.shared.v2.u32 {%0,%1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(a));
  return v;
}
__device__ __forceinline__ uint32_t lds32(uint32_t a) {
  uint32_t v;
  asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(a));
  return v;
}
__device__ __forceinline__ float lds32f(uint32_t a) { return __uint_as_float(lds32(a)); }

// One token's dot products with NM bf16 rows (NM = 1 or 2) over `cols`
// columns (a multiple of 8): w0, w1 (bf16 rows), x (bf16, or fp32 when XF32)
// and zero (64 zero bytes) are shared-memory addresses.  Each lane keeps four
// 256-column chunks in flight, each with its own accumulator pair; chunks
// past the end read the zero bytes.  Returns this lane's sums (the caller
// reduces over the warp).
template <int NM, bool XF32>
__device__ __forceinline__ void row_dot_t1(uint32_t w0, uint32_t w1, uint32_t x, int cols, uint32_t zero,
                                           float (&out)[NM]) {
  const int lane = threadIdx.x & 31;
  float2 a[NM][4];
#pragma unroll
  for (int m = 0; m < NM; ++m)
#pragma unroll
    for (int k = 0; k < 4; ++k) a[m][k] = make_float2(0.f, 0.f);
#pragma unroll 1
  for (int c = 8 * lane; c < cols; c += 1024) {
    uint4 q[NM][4], xv[4][XF32 ? 2 : 1];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int ck = c + 256 * k;
      const bool in = ck < cols;
      q[0][k] = lds128(in ? w0 + 2u * ck : zero);
      if constexpr (NM == 2) q[1][k] = lds128(in ? w1 + 2u * ck : zero);
      if constexpr (XF32) {
        xv[k][0] = lds128(in ? x + 4u * ck : zero);
        xv[k][XF32 ? 1 : 0] = lds128(in ? x + 4u * ck + 16u : zero + 16u);
      } else {
        xv[k][0] = lds128(in ? x + 2u * ck : zero);
      }
    }
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      float xx[8];
      if constexpr (XF32) {
        const uint4 u = xv[k][0], v = xv[k][XF32 ? 1 : 0];
        xx[0] = __uint_as_float(u.x), xx[1] = __uint_as_float(u.y), xx[2] = __uint_as_float(u.z);
        xx[3] = __uint_as_float(u.w), xx[4] = __uint_as_float(v.x), xx[5] = __uint_as_float(v.y);
        xx[6] = __uint_as_float(v.z), xx[7] = __uint_as_float(v.w);
      } else {
        unpack_bf16x8(xv[k][0], xx);
      }
#pragma unroll
      for (int m = 0; m < NM; ++m) {
        const uint32_t wq[4] = {q[m][k].x, q[m][k].y, q[m][k].z, q[m][k].w};
#pragma unroll
        for (int i = 0; i < 4; ++i)
          a[m][k] = __ffma2_rn(make_float2(__uint_as_float(wq[i] << 16), __uint_as_float(wq[i] & 0xffff0000u)),
                               make_float2(xx[2 * i], xx[2 * i + 1]), a[m][k]);
      }
    }
  }
#pragma unroll
  for (int m = 0; m < NM; ++m)
    out[m] = ((a[m][0].x + a[m][0].y) + (a[m][1].x + a[m][1].y)) + ((a[m][2].x + a[m][2].y) + (a[m][3].x + a[m][3].y));
}

template <int FMT>
__device__ __forceinline__ void load_codes(LaneCodes<FMT>& c, uint32_t a);
template <>
__device__ __forceinline__ void load_codes<FMT_Q4>(LaneCodes<FMT_Q4>& c, uint32_t a) { c.w = lds64(a); }
template <>
__device__ __forceinline__ void load_codes<FMT_Q2>(LaneCodes<FMT_Q2>& c, uint32_t a) { c.w = lds32(a); }

// One unit of a routed tile: windows [u*W, u*W + W) of the 16-row block of the
// segment (its two 8-row halves, codes at sg.off[2m + h], scales at
// sg.off[2*NM + 2m + h] for matrix m and half h).  The weights are the A
// operand: lane (g, t) = (lane / 4, lane % 4) holds rows g and g + 8 of a
// 16-column step, which are exactly its code bytes of the two 8-row halves.
// The activations are the B operand, one window of groups per pass of steps:
// GU: column n of B carries group n of the window (x, from bfrag =
// [group][t][8 words]), zero in the other groups' steps; down: columns 2n and
// 2n + 1 carry the bf16 hi and lo parts of group n of the intermediate (bfrag
// = [group][hi/lo][t][8 words]).  After a window, D[r][n] is group n's code
// dot of row r, and the group's scale and bias are applied to it:
//   sum_k x_k (q_k s + beta) = s * D + (beta - 128 s) * X.
// bsum: GU [group] sums of x; down [16-row block] sums of hi + lo.
// Returns in res[m][0] / res[m][1] the unit's sums of rows g and g + 8 (every
// lane of lane group g holds them).
// A 4-bit gate/up unit on the integer tensor cores: the same 16 rows x one
// window of 8 groups x gate and up as routed_unit, with the codes expanded to
// bytes (one AND for the low nibbles of a code word, a shift and an AND for
// the high ones: the A fragment of an m16n8k32 step is then the 32 columns
// of two 16-column steps in a fixed permutation that x's limb fragments
// follow) and x as its two int8 limbs, each an exact integer dot.  Epilogue
// per group: s * sigma * (256 * D_hi + D_lo) + beta * X, the codes taken as
// q itself (no 128 offset); bsum holds the token's G group sums, then its G
// limb scales.
// 2-bit codes: one 32-bit word per lane and 8x64 block expands into four
// byte registers R_k = (w >> 2k) & 0x03030303; step 0 takes R_0, R_1 and
// step 1 R_2, R_3 (the 64 columns split into two fixed sets of 32).
template <int FMT>
__device__ __forceinline__ void routed_unit_gu_i8(uint32_t sl, const Seg& sg, int u, const RoutedGeo& geo,
                                                  uint32_t bfrag, uint32_t bsum, float (&res)[2][2]) {
  constexpr int GPW = 8;
  constexpr int CB = LaneCodes<FMT>::kBytes;
  constexpr int BB = 32 * CB;  // code bytes of one 8x64 block
  const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
  float acc[2][2] = {{0.f, 0.f}, {0.f, 0.f}};
  const int wa = u * geo.W, wb = min(wa + geo.W, geo.nwin);
  uint32_t cbase[2][2], sbase[2][2];
#pragma unroll
  for (int mm = 0; mm < 2; ++mm)
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      cbase[mm][h] = sl + sg.off[2 * mm + h] + (uint32_t)(lane * CB) - (uint32_t)(sg.gbase * BB);
      sbase[mm][h] = sl + sg.off[4 + 2 * mm + h] + (uint32_t)(g * 4) - (uint32_t)(sg.gbase * 32);
    }
  // this lane's B column: group g of the window
  const int bg = g;
#pragma unroll 1
  for (int w = wa; w < wb; ++w) {
    const int g0 = GPW * w, nv = min(GPW, geo.G - g0);
    uint32_t xb[8];  // word 4 * st + 2 * limb + b of this lane's group
    {
      const uint32_t a = bfrag + (uint32_t)(((g0 + bg) * 4 + t) * 32);
      uint4 v0 = make_uint4(0u, 0u, 0u, 0u), v1 = v0;
      if (bg < nv) {
        v0 = lds128(a);
        v1 = lds128(a + 16);
      }
      xb[0] = v0.x, xb[1] = v0.y, xb[2] = v0.z, xb[3] = v0.w;
      xb[4] = v1.x, xb[5] = v1.y, xb[6] = v1.z, xb[7] = v1.w;
    }
    int dh[2][4], dl[2][4];
#pragma unroll
    for (int mm = 0; mm < 2; ++mm)
#pragma unroll
      for (int k = 0; k < 4; ++k) dh[mm][k] = dl[mm][k] = 0;
#pragma unroll
    for (int j = 0; j < GPW; ++j) {
      if (j < nv) {
        const bool on = bg == j;
        uint32_t bm[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) bm[k] = on ? xb[k] : 0u;
        if constexpr (FMT == FMT_Q4) {
          uint2 c[2][2];
#pragma unroll
          for (int mm = 0; mm < 2; ++mm)
#pragma unroll
            for (int h = 0; h < 2; ++h) c[mm][h] = lds64(cbase[mm][h] + (uint32_t)((g0 + j) * BB));
#pragma unroll
          for (int mm = 0; mm < 2; ++mm)
#pragma unroll
            for (int st = 0; st < 2; ++st) {
              const uint32_t w0 = st ? c[mm][0].y : c[mm][0].x, w1 = st ? c[mm][1].y : c[mm][1].x;
              const uint32_t a0 = w0 & 0x0F0F0F0Fu, a2 = (w0 >> 4) & 0x0F0F0F0Fu;
              const uint32_t a1 = w1 & 0x0F0F0F0Fu, a3 = (w1 >> 4) & 0x0F0F0F0Fu;
              mma_16832_u8s8(dh[mm], a0, a1, a2, a3, bm[4 * st], bm[4 * st + 1]);
              mma_16832_u8s8(dl[mm], a0, a1, a2, a3, bm[4 * st + 2], bm[4 * st + 3]);
            }
        } else {
          uint32_t c[2][2];
#pragma unroll
          for (int mm = 0; mm < 2; ++mm)
#pragma unroll
            for (int h = 0; h < 2; ++h) c[mm][h] = lds32(cbase[mm][h] + (uint32_t)((g0 + j) * BB));
#pragma unroll
          for (int mm = 0; mm < 2; ++mm)
#pragma unroll
            for (int st = 0; st < 2; ++st) {
              const uint32_t a0 = (c[mm][0] >> (4 * st)) & 0x03030303u;
              const uint32_t a2 = (c[mm][0] >> (4 * st + 2)) & 0x03030303u;
              const uint32_t a1 = (c[mm][1] >> (4 * st)) & 0x03030303u;
              const uint32_t a3 = (c[mm][1] >> (4 * st + 2)) & 0x03030303u;
              mma_16832_u8s8(dh[mm], a0, a1, a2, a3, bm[4 * st], bm[4 * st + 1]);
              mma_16832_u8s8(dl[mm], a0, a1, a2, a3, bm[4 * st + 2], bm[4 * st + 3]);
            }
        }
      }
    }
    // epilogue: D[g][2t], D[g][2t+1], D[g+8][2t], D[g+8][2t+1]
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int n = 2 * t + e;
      if (n < nv) {
        const float X = lds32f(bsum + 4u * (uint32_t)(g0 + n));
        const float sig = lds32f(bsum + 4u * (uint32_t)(geo.G + g0 + n));
#pragma unroll
        for (int mm = 0; mm < 2; ++mm)
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const uint32_t sw = lds32(sbase[mm][h] + (uint32_t)((g0 + n) * 32));
            const float sc = __uint_as_float(sw << 16), bi = __uint_as_float(sw & 0xffff0000u);
            const float dot = __int2float_rn(dh[mm][2 * h + e] * 256 + dl[mm][2 * h + e]) * sig;
            acc[mm][h] = fmaf(sc, dot, fmaf(bi, X, acc[mm][h]));
          }
      }
    }
  }
#pragma unroll
  for (int mm = 0; mm < 2; ++mm)
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      float v = acc[mm][h];
      v += __shfl_xor_sync(0xffffffffu, v, 1);
      v += __shfl_xor_sync(0xffffffffu, v, 2);
      res[mm][h] = v;
    }
}

template <int FMT, bool GU>
__device__ __forceinline__ void routed_unit(uint32_t sl, const Seg& sg, int u, const RoutedGeo& geo, uint32_t bfrag,
                                            uint32_t bsum, float (&res)[2][2]) {
  constexpr int NM = GU ? 2 : 1;
  constexpr int GPW = GU ? 8 : 4;
  constexpr int CB = LaneCodes<FMT>::kBytes;
  constexpr int BB = 32 * CB;  // code bytes of one 8x64 block
  const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
  float acc[NM][2];
#pragma unroll
  for (int mm = 0; mm < NM; ++mm) acc[mm][0] = acc[mm][1] = 0.f;
  const int wa = u * geo.W, wb = min(wa + geo.W, geo.nwin);
  uint32_t cbase[NM][2], sbase[NM][2];
#pragma unroll
  for (int mm = 0; mm < NM; ++mm)
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      cbase[mm][h] = sl + sg.off[2 * mm + h] + (uint32_t)(lane * CB) - (uint32_t)(sg.gbase * BB);
      sbase[mm][h] = sl + sg.off[2 * NM + 2 * mm + h] + (uint32_t)(g * 4) - (uint32_t)(sg.gbase * 32);
    }
  // this lane's B column: group bg of the window, part bh (down: 0 hi, 1 lo)
  const int bg = GU ? g : (g >> 1);
#pragma unroll 1
  for (int w = wa; w < wb; ++w) {
    const int g0 = GPW * w, nv = min(GPW, geo.G - g0);
    uint32_t xb[8];
    {
      const uint32_t a = GU ? bfrag + (uint32_t)(((g0 + bg) * 4 + t) * 32)
                            : bfrag + (uint32_t)((((g0 + bg) * 2 + (g & 1)) * 4 + t) * 32);
      uint4 v0 = make_uint4(0u, 0u, 0u, 0u), v1 = v0;
      if (bg < nv) {
        v0 = lds128(a);
        v1 = lds128(a + 16);
      }
      xb[0] = v0.x, xb[1] = v0.y, xb[2] = v0.z, xb[3] = v0.w;
      xb[4] = v1.x, xb[5] = v1.y, xb[6] = v1.z, xb[7] = v1.w;
    }
    float d[NM][4];
#pragma unroll
    for (int mm = 0; mm < NM; ++mm) d[mm][0] = d[mm][1] = d[mm][2] = d[mm][3] = 0.f;
#pragma unroll
    for (int j = 0; j < GPW; ++j) {
      if (j < nv) {
        LaneCodes<FMT> c[NM][2];
#pragma unroll
        for (int mm = 0; mm < NM; ++mm)
#pragma unroll
          for (int h = 0; h < 2; ++h) load_codes<FMT>(c[mm][h], cbase[mm][h] + (uint32_t)((g0 + j) * BB));
        const bool on = bg == j;
#pragma unroll
        for (int mm = 0; mm < NM; ++mm) {
          uint32_t a0[4][2], a1[4][2];
          c[mm][0].frags(a0);
          c[mm][1].frags(a1);
#pragma unroll
          for (int s = 0; s < 4; ++s)
            mma_16816(d[mm], a0[s][0], a1[s][0], a0[s][1], a1[s][1], on ? xb[2 * s] : 0u, on ? xb[2 * s + 1] : 0u);
        }
      }
    }
    // epilogue: D[g][2t], D[g][2t+1], D[g+8][2t], D[g+8][2t+1]
    if constexpr (GU) {
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int n = 2 * t + e;
        if (n < nv) {
          const float X = lds32f(bsum + 4u * (uint32_t)(g0 + n));
#pragma unroll
          for (int mm = 0; mm < NM; ++mm) {
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              const uint32_t sw = lds32(sbase[mm][h] + (uint32_t)((g0 + n) * 32));
              const float sc = __uint_as_float(sw << 16), bi = __uint_as_float(sw & 0xffff0000u);
              acc[mm][h] = fmaf(sc, d[mm][2 * h + e], fmaf(fmaf(-128.f, sc, bi), X, acc[mm][h]));
            }
          }
        }
      }
    } else {
      if (t < nv) {
        const int gq = g0 + t;  // group of columns 2t (hi) and 2t + 1 (lo)
        const uint4 hs4 = lds128(bsum + 16u * (uint32_t)gq);
        const float X = (__uint_as_float(hs4.x) + __uint_as_float(hs4.y)) +
                        (__uint_as_float(hs4.z) + __uint_as_float(hs4.w));
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const uint32_t sw = lds32(sbase[0][h] + (uint32_t)(gq * 32));
          const float sc = __uint_as_float(sw << 16), bi = __uint_as_float(sw & 0xffff0000u);
          acc[0][h] = fmaf(sc, d[0][2 * h] + d[0][2 * h + 1], fmaf(fmaf(-128.f, sc, bi), X, acc[0][h]));
        }
      }
    }
  }
#pragma unroll
  for (int mm = 0; mm < 2; ++mm)
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      float v = mm < NM ? acc[mm < NM ? mm : 0][h] : 0.f;
      v += __shfl_xor_sync(0xffffffffu, v, 1);
      v += __shfl_xor_sync(0xffffffffu, v, 2);
      res[mm][h] = v;
    }
}

// A routed gate/up unit is done: store its partial sums (rows g and g + 8 of
// the 16-row block, from the lanes with t = 0) in accumulator entry e; the
// warp that completes the block's last unit sums the units in order, applies
// SiLU(gate) * up and publishes the 16 intermediate values as bf16 hi and lo
// B fragments of the down projection (layout [pair][group][hi/lo][t][8
// words]: rows 16rb .. 16rb + 15 of I are step rb % 4 of group rb / 4), with
// their sum.
__device__ __noinline__ void gu_unit_done(float g0r, float g8r, float u0r, float u8r, int e, int u, int U,
                                          float* part, int* cnt, int pair, int rb, int I, uint8_t* hf, float* hx) {
  const int lane = threadIdx.x & 31;
  float* pe = part + (size_t)e * kMaxUnits * 32;
  if ((lane & 3) == 0) {
    const int g = lane >> 2;
    *reinterpret_cast<float2*>(pe + u * 32 + 2 * g) = make_float2(g0r, u0r);
    *reinterpret_cast<float2*>(pe + u * 32 + 2 * (g + 8)) = make_float2(g8r, u8r);
    __threadfence_block();
  }
  __syncwarp();
  int last = 0;
  if (lane == 0) {
    __threadfence_block();
    last = atomicAdd(&cnt[e], 1) == U - 1 ? 1 : 0;
  }
  last = __shfl_sync(0xffffffffu, last, 0);
  if (!last) return;
  __threadfence_block();
  // lane v (v = lane % 16; lanes 16..31 repeat rows 0..15 and are dropped)
  // sums row v over the units in order, so the warp does not diverge
  const int v = lane & 15;
  float gs = 0.f, us = 0.f;
  const volatile float* pp = pe + 2 * v;
#pragma unroll 1
  for (int uu = 0; uu < U; ++uu) {
    gs += pp[uu * 32];
    us += pp[uu * 32 + 1];
  }
  if (lane == 0) cnt[e] = 0;  // entry free for a later row block
  const float h = silu_mul(gs, us);
  const __nv_bfloat16 hi = __float2bfloat16_rn(h);
  const __nv_bfloat16 lo = __float2bfloat16_rn(h - __bfloat162float(hi));
  float hsum = lane < 16 ? __bfloat162float(hi) + __bfloat162float(lo) : 0.f;
  hsum += __shfl_xor_sync(0xffffffffu, hsum, 1);
  hsum += __shfl_xor_sync(0xffffffffu, hsum, 2);
  hsum += __shfl_xor_sync(0xffffffffu, hsum, 4);
  hsum += __shfl_xor_sync(0xffffffffu, hsum, 8);
  const uint32_t hb = __bfloat16_as_ushort(hi), lb = __bfloat16_as_ushort(lo);
  // lane L < 8 builds word (t' = L % 4, first/second = L / 4) of hi and of lo:
  // values 8*second + 2t' and 8*second + 2t' + 1 of the 16
  const int tq = lane & 3, sec = (lane >> 2) & 1;
  const int src = 8 * sec + 2 * tq;
  const uint32_t h0 = __shfl_sync(0xffffffffu, hb, src), h1 = __shfl_sync(0xffffffffu, hb, src + 1);
  const uint32_t l0 = __shfl_sync(0xffffffffu, lb, src), l1 = __shfl_sync(0xffffffffu, lb, src + 1);
  const int Gi = I / 64;
  const int gq = rb >> 2, sq = rb & 3;
  if (lane < 8) {
    uint32_t* base = reinterpret_cast<uint32_t*>(hf) + (((size_t)pair * Gi + gq) * 2) * 32;
    base[(0 * 4 + tq) * 8 + 2 * sq + sec] = h0 | (h1 << 16);
    base[(1 * 4 + tq) * 8 + 2 * sq + sec] = l0 | (l1 << 16);
  }
  if (lane == 0) hx[(size_t)pair * (I / 16) + rb] = hsum;
}

// ---- producer ----------------------------------------------------------------------
// One thread (lane 0 of the producer warp) builds each tile's descriptor in
// place in shared memory once the consumers have freed the slot, announces
// each copy's bytes on the slot's "full" barrier and issues it, and finally
// arrives on the barrier, which completes when every copy has landed.  All of
// it is inlined so the producer's state stays in registers: the producer is
// on the critical path of every phase, and out-of-line calls kept this state
// in local memory at a round trip per access.
struct Producer {
  uint8_t* ring;
  uint64_t* full;
  uint64_t* empty;
  TileDesc* descs;
  uint32_t slot_bytes;
  uint32_t slot, phase, nslots;
  uint64_t timeout_ns;
  uint32_t* err;
  uint32_t* abort_flag;
  uint64_t* trace;
  uint32_t* spins;  // [0] empty-slot waits, [1] routing wait (traced launches only)
  int ncommit;
  bool ok;
  bool open;
  int pending_pre;
  int nrb_tile;
  TileDesc* d;
  uint32_t fill;
  uint64_t policy;  // L2 evict-first: weights are read once per launch

  __device__ __forceinline__ void commit() {
    if (!open) return;
    if (trace && ncommit < 16) trace[48 + ncommit] = globaltimer_ns();
    ++ncommit;
    mbar_arrive(&full[slot]);
    if (++slot == nslots) {
      slot = 0;
      phase ^= 1u;
    }
    open = false;
  }
  __device__ __forceinline__ bool begin(int type) {
    commit();
    if (!ok) return false;
    if (!mbar_wait(&empty[slot], phase ^ 1u, timeout_ns, spins)) {
      ok = false;
      atomicCAS(err, 0u, 1u);
      atomicExch(abort_flag, 1u);
      return false;
    }
    d = &descs[slot];
    d->type = type;
    d->nseg = 0;
    d->pre = pending_pre;
    d->post = 0;
    pending_pre = 0;
    fill = 0;
    nrb_tile = 0;
    open = true;
    return true;
  }
  __device__ Seg& seg(int pair, int row0, int nrows) {
    Seg& s = d->seg[d->nseg++];
    s.pair = pair;
    s.row0 = row0;
    s.nrows = nrows;
    s.u0 = 0;
    s.u1 = 0;
    s.gbase = 0;
    s.acc = 0;
    return s;
  }
  // Copy a byte range into the slot; returns the slot offset of its first
  // byte.  The copy is widened to 16-byte boundaries (the widened range stays
  // inside the same 256-byte aligned section).
  __device__ __forceinline__ uint32_t range(const void* p, size_t bytes) {
    const uintptr_t a = reinterpret_cast<uintptr_t>(p);
    const uintptr_t al = a & ~uintptr_t(15);
    const uint32_t pad = (uint32_t)(a - al);
    const uint32_t n = (uint32_t)((pad + bytes + 15) & ~size_t(15));
    mbar_expect_tx(&full[slot], n);
    bulk_g2s_hint(ring + (size_t)slot * slot_bytes + fill, reinterpret_cast<const void*>(al), n, &full[slot],
                  policy);
    const uint32_t off = fill + pad;
    fill += n;
    return off;
  }
  // Attach arrival flags to the current tile (an empty tile if none is open)
  // and publish it.
  __device__ void post(int flag) {
    if (!open && !begin(TILE_NONE)) return;
    d->post |= flag;
    commit();
  }
  // Waits for the consumers to do before the next tile's compute.
  __device__ void pre(int flag) {
    commit();
    pending_pre |= flag;
  }
};

// Routed tiles for row blocks [rb_a, rb_b) of nm matrices of one (token,
// expert) pair (off_codes / off_scales: the matrices' section offsets).  A
// segment is one row block's run of whole units [u0, u1) that fits the open
// tile; a tile takes segments until it is full, holds kMaxSeg of them or
// max_rb row blocks.  Each row block gets the next accumulator entry.
__device__ __forceinline__ void emit_routed(Producer& pr, int type, int bits, const size_t* off_codes,
                                         const size_t* off_scales, const uint8_t* blob, int pair, int rb_a,
                                         int rb_b, int nm, RoutedGeo geo, int max_rb, int* rbseq) {
  const uint32_t bb = 64u * (uint32_t)bits;
  // both 8-row halves of every group of the unit's windows, codes and scales
  const uint32_t per_unit = (uint32_t)(geo.gpw * geo.W) * (uint32_t)nm * 2u * (bb + 32u);
  const uint32_t slack = 64;
#pragma unroll 1
  for (int rb = rb_a; rb < rb_b; ++rb) {
    const int e = (*rbseq)++ % kAccSlots;
#pragma unroll 1
    for (int u = 0; u < geo.U;) {
      if (pr.open && (pr.d->type != type || pr.d->nseg >= kMaxSeg || pr.nrb_tile >= max_rb ||
                      pr.fill + per_unit + slack > pr.slot_bytes))
        pr.commit();
      if (!pr.open && !pr.begin(type)) return;
      const int un = min(geo.U - u, max(1, (int)((pr.slot_bytes - pr.fill - slack) / per_unit)));
      const int ga = geo.gpw * geo.W * u, gb = min(geo.G, geo.gpw * geo.W * (u + un));
      Seg& s = pr.seg(pair, rb, 1);
      s.u0 = u;
      s.u1 = u + un;
      s.gbase = ga;
      s.acc = e;
#pragma unroll
      for (int mm = 0; mm < 2; ++mm) {
        if (mm < nm) {
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const size_t b0 = (size_t)(2 * rb + h) * geo.G + ga;
            s.off[2 * mm + h] = pr.range(blob + off_codes[mm] + b0 * bb, (size_t)(gb - ga) * bb);
            s.off[2 * nm + 2 * mm + h] = pr.range(blob + off_scales[mm] + b0 * 32u, (size_t)(gb - ga) * 32u);
          }
        }
      }
      ++pr.nrb_tile;
      u += un;
    }
  }
}

// bf16 rows [a, b) of one or two row-major matrices (row_bytes each), as many
// rows per tile as fit.
__device__ __forceinline__ void emit_rows(Producer& pr, int type, const uint8_t* m0, const uint8_t* m1,
                                       uint32_t row_bytes, int a, int b) {
  const uint32_t nm = m1 ? 2u : 1u;
  const int cap = max(1, min(1024, (int)((pr.slot_bytes - 16u * nm) / (nm * row_bytes))));
#pragma unroll 1
  for (int r = a; r < b; r += cap) {
    const int n = min(cap, b - r);
    if (!pr.begin(type)) return;
    Seg& s = pr.seg(-1, r, n);
    s.off[0] = pr.range(m0 + (size_t)r * row_bytes, (size_t)n * row_bytes);
    if (m1) s.off[1] = pr.range(m1 + (size_t)r * row_bytes, (size_t)n * row_bytes);
  }
}

// The expert pointer table is staged in shared memory (in the top-K key
// buffer, which the register top-K for E <= 512 leaves unused) when it is
// small and 16-byte aligned.
__device__ __forceinline__ bool ptab_in_smem(const DecodeParams& p) {
  return p.expert_ptr != nullptr && p.L.E <= 512 && (p.L.E & 1) == 0 &&
         (reinterpret_cast<uintptr_t>(p.expert_ptr) & 15u) == 0;
}

// ---- streamed calls: the expert cache -----------------------------------------------
// A pair's cache slot as block 0 publishes it (the high half of its index
// word): the slot, kSlotMiss when its blob is still to be copied in, or
// kNoSlot when the call found no slot (the cache had too few).
constexpr uint32_t kSlotMiss = 0x8000u;
constexpr uint32_t kNoSlot = 0x7fffu;

// Block 0's sync warp, streamed calls: the device resolve's cache policy over
// the call's T*K chosen experts, in order.  A hit marks its slot held and
// touches it; a repeat of an expert already held is neither; a miss takes
// the lowest empty slot that the call does not hold, else the least
// recently used one it does not hold, unmaps that slot's old expert and maps
// the new one.  code[j] gets pair j's slot (| kSlotMiss for a miss).  If no
// slot is left, the call's assignments are undone, MOE_ERR_OOM goes to the
// cache's error counter and every code is kNoSlot.  held: at least S bits of
// shared memory.  Returns false on that failure.  Warp-uniform.  (Fields
// are passed one by one: a reference to the kernel's parameters would make
// the whole kernel keep them in local memory.)
__device__ __noinline__ bool warp_stream_resolve(int32_t* slot_of_, int32_t* key_, uint64_t* tick_, uint64_t* dctr_,
                                                 int S, int layer, int E, uint64_t blob, const int* tk_i, int T,
                                                 int K, int KP, uint32_t* held, uint32_t* code) {
  const int lane = threadIdx.x & 31, n = T * K;
  volatile int32_t* slot_of = slot_of_;
  volatile int32_t* key = key_;
  volatile uint64_t* tick = tick_;
  for (int i = lane; i < (S + 31) / 32; i += 32) held[i] = 0u;
  // every pair's table entry and the use clock in one round trip (lane q
  // looks up pairs q and q + 32); entries are read again only after a miss
  // of this call has changed the table
  auto pair_key = [&](int j) { return layer * E + tk_i[(j / K) * KP + j % K]; };
  const int look0 = lane < n ? slot_of[pair_key(lane)] : -1;
  const int look1 = lane + 32 < n ? slot_of[pair_key(lane + 32)] : -1;
  uint64_t clock = reinterpret_cast<volatile uint64_t*>(dctr_)[DC_CLOCK];
  __syncwarp();
  int nj = 0, nh = 0, j = 0;
  bool fail = false;
#pragma unroll 1
  for (; j < n; ++j) {
    const int kv = pair_key(j);
    int sl = __shfl_sync(0xffffffffu, j < 32 ? look0 : look1, j & 31);
    if (nj > 0) sl = slot_of[kv];
    if (sl >= 0) {  // a hit, or a repeat of an expert this call holds
      if (lane == 0) {
        if (!(held[sl >> 5] >> (sl & 31) & 1u)) {
          held[sl >> 5] |= 1u << (sl & 31);
          tick[sl] = ++clock;
          ++nh;
        }
        code[j] = (uint32_t)sl;
      }
      __syncwarp();
      continue;
    }
    int be = 0x7fffffff;
    unsigned long long bl = ~0ull;
#pragma unroll 1
    for (int q = lane; q < S; q += 32) {
      if (held[q >> 5] >> (q & 31) & 1u) continue;
      if (key[q] < 0) {
        be = min(be, q);
      } else {
        const unsigned long long kk = ((unsigned long long)tick[q] << 24) | (unsigned long long)q;
        bl = kk < bl ? kk : bl;
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      be = min(be, __shfl_xor_sync(0xffffffffu, be, o));
      const unsigned long long ob = __shfl_xor_sync(0xffffffffu, bl, o);
      bl = ob < bl ? ob : bl;
    }
    const int vs = be != 0x7fffffff ? be : (bl != ~0ull ? (int)(bl & 0xffffffull) : -1);
    if (vs < 0) {
      fail = true;
      break;
    }
    if (lane == 0) {
      const int old = key[vs];
      if (old >= 0) slot_of[old] = -1;
      key[vs] = kv;
      slot_of[kv] = vs;
      held[vs >> 5] |= 1u << (vs & 31);
      tick[vs] = ++clock;
      code[j] = (uint32_t)vs | kSlotMiss;
    }
    ++nj;
    __syncwarp();
  }
  if (lane == 0) {
    if (fail) {
      // undo: the slots this call took were never filled (the experts they
      // held before are gone, as with the resolve kernel)
      for (int q = 0; q < j; ++q)
        if (code[q] & kSlotMiss) {
          slot_of[pair_key(q)] = -1;
          key[code[q] & kNoSlot] = -1;
        }
      nj = 0;
      atomicCAS(reinterpret_cast<unsigned long long*>(&dctr_[DC_ERROR]), 0ull, (unsigned long long)MOE_ERR_OOM);
      for (int q = 0; q < n; ++q) code[q] = kNoSlot;
    }
    // the counters: added, not waited for (the next call's clock read is
    // ordered by the kernel boundary)
    atomicAdd(reinterpret_cast<unsigned long long*>(&dctr_[DC_HITS]), (unsigned long long)nh);
    if (nj > 0) {
      atomicAdd(reinterpret_cast<unsigned long long*>(&dctr_[DC_MISSES]), (unsigned long long)nj);
      atomicAdd(reinterpret_cast<unsigned long long*>(&dctr_[DC_BYTES]), (unsigned long long)nj * blob);
      atomicAdd(reinterpret_cast<unsigned long long*>(&dctr_[DC_FILLS]), 1ull);
    }
    reinterpret_cast<volatile uint64_t*>(dctr_)[DC_CLOCK] = clock;
  }
  __syncwarp();
  return !fail;
}

// Every block's sync warp, streamed calls with misses: this block's share
// (1/G of each blob, in 16-byte pieces, four loads in flight per lane) of
// the missed blobs, from the store (host memory the device maps) into their
// slots.
__device__ __noinline__ void warp_fill_share(const uint8_t* host, uint8_t* slots, int layer, int E, uint64_t blob,
                                             const int* tk_i, const uint32_t* code, int T, int K, int KP) {
  const int lane = threadIdx.x & 31, G = gridDim.x, c = blockIdx.x;
  const uint64_t per = blob / 16;  // blob is a multiple of 256
  const uint64_t a = per * (uint64_t)c / (uint64_t)G, b = per * (uint64_t)(c + 1) / (uint64_t)G;
#pragma unroll 1
  for (int j = 0; j < T * K; ++j) {
    if (!(code[j] & kSlotMiss) || code[j] == kNoSlot) continue;
    const int e = tk_i[(j / K) * KP + j % K];
    const uint4* src = reinterpret_cast<const uint4*>(host + (uint64_t)(layer * E + e) * blob);
    uint4* dst = reinterpret_cast<uint4*>(slots + (uint64_t)(code[j] & kNoSlot) * blob);
#pragma unroll 1
    for (uint64_t u = a + lane; u < b; u += 4 * 32) {
      uint4 w[4];
#pragma unroll
      for (int k = 0; k < 4; ++k)
        if (u + 32 * k < b) w[k] = src[u + 32 * k];
#pragma unroll
      for (int k = 0; k < 4; ++k)
        if (u + 32 * k < b) dst[u + 32 * k] = w[k];
    }
  }
}

template <bool TRACE>
__device__ void run_producer(const DecodeParams& p, Producer& pr, uint16_t* xs, uint16_t* res_s, uint16_t* gam_s,
                             uint64_t* xbar, uint64_t* topkbar, const int* flags, const uint8_t* const* eptr,
                             uint64_t* ptab, uint16_t* gpre_s, uint16_t* sgv_s) {
  const Layout& L = p.L;
  const int T = p.T, H = L.H, I = L.I, E = L.E;
  const int G = gridDim.x, c = blockIdx.x;
  int r0, r1;
  block_rows(H, c, G, r0, r1);
  // the token activations, and this block's rows of the residual and of gamma
  const uint32_t xb = (uint32_t)(2ull * T * H);
  const uint32_t rb = (uint32_t)(2 * (r1 - r0));
  // the expert pointer table too, when it fits the top-K key buffer (unused
  // for E <= 512): the routing then finds its blobs without a global round trip
  const uint32_t tb = ptab_in_smem(p) ? (uint32_t)(8 * E) : 0u;
  const uint32_t gb = L.prenorm ? (uint32_t)(2 * H) : 0u;
  const uint32_t sb = L.sgate ? (uint32_t)(2 * H) : 0u;
  mbar_expect_tx(xbar, xb + (uint32_t)(T + 1) * rb + tb + gb + sb);
  bulk_g2s(xs, p.x, xb, xbar);
  if (tb) bulk_g2s(ptab, p.expert_ptr, tb, xbar);
  if (gb) bulk_g2s(gpre_s, p.gamma_pre, gb, xbar);
  if (sb) bulk_g2s(sgv_s, p.sgate, sb, xbar);
  if (rb > 0) {
#pragma unroll 1
    for (int t = 0; t < T; ++t) bulk_g2s(res_s + (size_t)t * (r1 - r0), p.res + (size_t)t * H + r0, rb, xbar);
    bulk_g2s(gam_s, p.gamma + r0, rb, xbar);
  }
  mbar_arrive(xbar);
  int a, b;
  if (!p.idx_in) {  // with the routing given there are no router rows
    range_of(E, c, G, a, b);
    emit_rows(pr, TILE_ROUTER, reinterpret_cast<const uint8_t*>(p.wr), nullptr, 2u * H, a, b);
  }
  pr.post(F_ARRIVE_R);
  const bool bf16_shared = L.has_shared && !L.spacked;
  if (bf16_shared) {
    range_of(I, c, G, a, b);
    emit_rows(pr, TILE_SHARED_GU, reinterpret_cast<const uint8_t*>(p.sg), reinterpret_cast<const uint8_t*>(p.su),
              2u * H, a, b);
  }
  pr.post(F_ARRIVE_S);
  // the routing, from the sync warp
  bool routed = false;
  if (pr.ok) {
    if (mbar_wait(topkbar, 0, p.timeout_ns, pr.spins ? pr.spins + 1 : nullptr)) {
      routed = flags[FLAG_TOPK] != 0;
      // streamed calls: other blocks may have just written the blobs these
      // copies read (their stores, seen through the fill barrier)
      if (p.streamed) fence_proxy_async_global();
    } else {
      pr.ok = false;
      atomicCAS(p.err, 0u, 1u);
      atomicExch(pr.abort_flag, 1u);
    }
  }
  if (pr.trace) pr.trace[9] = globaltimer_ns();
  const RoutedGeo gh = routed_geo(H, 8), gi = routed_geo(I, 4);
  const size_t oc[3] = {L.off_codes[0], L.off_codes[1], L.off_codes[2]};
  const size_t os[3] = {L.off_scales[0], L.off_scales[1], L.off_scales[2]};
  const int nrb_i = I / kRowBlock;
  int rbseq = 0;
  const int KP = L.KP;  // pairs per token (the packed shared expert is pair K)
  if (routed) {
    // routed gate/up: this block's share of the T*KP*(I/16) (pair, row block) items
    range_of(T * KP * nrb_i, c, G, a, b);
#pragma unroll 1
    for (int q = a; q < b && pr.ok;) {
      const int pair = q / nrb_i, rb0 = q - pair * nrb_i;
      const int n = min(b - q, nrb_i - rb0);
      emit_routed(pr, TILE_EXPERT_GU, L.bits, oc, os, eptr[pair], pair, rb0, rb0 + n, 2, gh, kMaxRbPerTile, &rbseq);
      q += n;
    }
  }
  pr.post(F_ARRIVE_E);
  // the shared expert's down rows of this block: every block's shared
  // intermediate (S) was staged while the routing was found, so they run
  // while the routed intermediate (E) is being completed
  if (bf16_shared) {
    pr.pre(F_WAIT_S);
    emit_rows(pr, TILE_SHARED_DOWN, reinterpret_cast<const uint8_t*>(p.sd), nullptr, 2u * I, r0, r1);
  }
  pr.pre(F_WAIT_E);
  if (routed && r1 > r0) {
#pragma unroll 1
    for (int pair = 0; pair < T * KP && pr.ok; ++pair)
      emit_routed(pr, TILE_EXPERT_DOWN, L.bits, oc + 2, os + 2, eptr[pair], pair, r0 / kRowBlock, r1 / kRowBlock, 1, gi, 1 << 20,
                  &rbseq);
  }
  pr.post(F_END);
  if (pr.trace) pr.trace[10] = globaltimer_ns();
}

// ---- sync warp ----------------------------------------------------------------------
// Prepares x as A fragments with its group sums, then does the block's
// grid-wide arrivals (R, S, E, D) and waits (R, S, E, D).  After the R wait it
// runs the top-K and hands the expert pointers to the producer; after the S
// and E waits it stages the shared / routed intermediates into shared memory
// with bulk copies that complete the consumers' "go" barriers.
template <bool TRACE>
__device__ void run_sync(const DecodeParams& p, uint64_t* xbar, uint64_t* xfbar, uint64_t* topkbar, uint64_t* evt,
                         uint64_t* go, int* flags, const uint16_t* xs, uint4* xf, float* xsum, float* hs_s,
                         uint8_t* hf_s, float* hx_s, float* tk_w, int* tk_i, const uint8_t** eptr, uint64_t* tkbuf,
                         uint32_t* spins) {
  const int lane = threadIdx.x & 31;
  const Layout& L = p.L;
  const int T = p.T, K = L.K, KP = L.KP, E = L.E, G = gridDim.x;
  uint32_t* ctr = p.ctr;
  const uint64_t to = p.timeout_ns;
  __shared__ uint32_t s_code[kMaxPairsFused];  // streamed calls: each pair's cache slot code
  uint32_t* sp_evt = spins ? spins + 5 : nullptr;
  uint32_t* sp_grid = spins ? spins + 6 : nullptr;
  bool ok = warp_wait(xbar, 0, to, spins ? spins + 7 : nullptr);
  const uint32_t epoch = (uint32_t)flags[FLAG_EPOCH];
  int good;
  if (p.idx_in) {
    // the routing is given: no router barrier, no top-K
#pragma unroll 1
    for (int j = lane; j < T * K; j += 32) {
      const int t = j / K, k = j - t * K;
      tk_i[t * KP + k] = __ldg(p.idx_in + j);
      tk_w[t * KP + k] = __ldg(p.w_in + j);
    }
    __syncwarp();
    good = __all_sync(0xffffffffu, ok) ? 1 : 0;
  } else {
    // the router logits of every block carry this launch's epoch once they
    // are written: polling them is the router barrier and the top-K's loads
    // in one (warp-uniform, so the top-K runs unsplit)
    // Block 0 alone polls the E logit words and runs the top-K, then
    // publishes the routing as 2*T*K epoch words; every other block polls
    // those few words.  (148 blocks all polling all E words took ~4 us per
    // exchange in a micro kernel, one block polling and the rest polling one
    // result ~1 us.)
    if (lane == 0) trace_mark<TRACE>(p, 65);
    bool gr = ok;
    if (blockIdx.x == 0) {
      // first pass only once this block's own router rows are written: a
      // pass issued during the launch's first burst of weight loads came back
      // ~4 us later and mostly stale, and the next could only start then
      if (gr) gr = warp_wait(&evt[EVT_R], 0, to, sp_evt);
#pragma unroll 1
      for (int t = 0; t < T && gr; ++t)
        gr = warp_topk_poll(p.logits + (size_t)t * E, epoch, E, K, tkbuf, tk_i + t * KP, tk_w + t * KP, &ctr[5],
                            p.err, to, sp_grid, TRACE ? p.trace + 73 : nullptr);
      gr = __all_sync(0xffffffffu, gr);
      __syncwarp();
      if (TRACE && lane == 0) p.trace[78] = globaltimer_ns();
      // a streamed call: the chosen experts' cache slots (the key buffer is
      // free once the top-K is done; it holds the slots' bitmap); a call
      // that finds too few slots still publishes, with no slot for any pair
      if (gr && p.streamed)
        warp_stream_resolve(p.sv.slot_of, p.sv.key, p.sv.tick, p.sv.dctr, p.sv.S, p.sv.layer, E, L.blob_bytes, tk_i,
                            T, K, KP, reinterpret_cast<uint32_t*>(tkbuf), s_code);
      if (gr) {
#pragma unroll 1
        for (int j = lane; j < T * K; j += 32) {
          const int t = j / K, k = j - t * K;
          const uint32_t hi = p.streamed ? s_code[j] << 16 : 0u;
          st_relaxed_gpu_b64(p.route + 2 * j, ((uint64_t)epoch << 32) | hi | (uint32_t)tk_i[t * KP + k]);
          st_relaxed_gpu_b64(p.route + 2 * j + 1, epoch_word(epoch, tk_w[t * KP + k]));
        }
      }
      if (TRACE && lane == 0) p.trace[79] = globaltimer_ns();
    } else if (gr) {
      __shared__ uint32_t rw[2 * kMaxPairsFused];
      gr = warp_poll_words(p.route, 2 * T * K, epoch, rw, &ctr[5], p.err, to);
      __syncwarp();
      if (TRACE && lane == 0) p.trace[(size_t)blockIdx.x * kTraceEntries + 78] = globaltimer_ns();
      if (gr) {
#pragma unroll 1
        for (int j = lane; j < T * K; j += 32) {
          const int t = j / K, k = j - t * K;
          tk_i[t * KP + k] = p.streamed ? (int)(rw[2 * j] & 0xffffu) : (int)rw[2 * j];
          tk_w[t * KP + k] = __uint_as_float(rw[2 * j + 1]);
          if (p.streamed) s_code[j] = rw[2 * j] >> 16;
        }
      }
    }
    good = __all_sync(0xffffffffu, gr) ? 1 : 0;
    __syncwarp();
    if (lane == 0) trace_mark<TRACE>(p, 66);
  }
  if (good) {
#pragma unroll 1
    for (int j = lane; j < T * KP; j += 32) {
      // pair K of a token is the packed shared expert (weight 1: its gate,
      // if any, is applied in the combine)
      const int t = j / KP, k = j - t * KP;
      const bool shp = k == K;
      if (shp) {
        tk_i[j] = -1;
        tk_w[j] = 1.f;
      }
      const int e = shp ? 0 : tk_i[j];
      const uint32_t sc = p.streamed && !shp ? s_code[t * K + k] & kNoSlot : 0u;
      const void* bp = shp ? reinterpret_cast<const void*>(p.spacked)
                       : !(e >= 0 && e < E) ? nullptr
                       : p.streamed ? (sc == kNoSlot ? nullptr : p.sv.slots + (uint64_t)sc * L.blob_bytes)
                       : ptab_in_smem(p) ? reinterpret_cast<const void*>(tkbuf[e])
                                         : p.expert_ptr[e];
      if (bp == nullptr || (reinterpret_cast<uintptr_t>(bp) & 255u)) {
        atomicCAS(p.err, 0u, 2u);
        atomicExch(&ctr[5], 1u);
        bp = nullptr;
        good = 0;
      }
      eptr[j] = reinterpret_cast<const uint8_t*>(bp);
      if (blockIdx.x == 0 && !shp) {
        if (p.idx_out) p.idx_out[t * K + k] = e;
        if (p.w_out) p.w_out[t * K + k] = tk_w[j];
      }
    }
    good = __all_sync(0xffffffffu, good != 0) ? 1 : 0;
  }
  // a streamed call with misses: every block copies its share of the missed
  // blobs into their slots and waits until every block has (its routed
  // tiles read them next; the producer orders its copies after this)
  if (p.streamed && good) {
    bool miss = false;
    for (int j = 0; j < T * K; ++j) miss = miss || (s_code[j] & kSlotMiss) != 0u;
    if (miss) {
      warp_fill_share(p.sv.host, p.sv.slots, p.sv.layer, E, L.blob_bytes, tk_i, s_code, T, K, KP);
      __syncwarp();
      int gf = 1;
      if (lane == 0) {
        __threadfence();
        red_release_add(&ctr[7], 1u);
        gf = grid_wait_thread(&ctr[7], G, &ctr[5], p.err, to, sp_grid) ? 1 : 0;
      }
      good = __shfl_sync(0xffffffffu, gf, 0) ? good : 0;
    }
  }
  // every lane's eptr store must precede lane 0's release to the producer
  __syncwarp();
  if (lane == 0) {
    flags[FLAG_TOPK] = good;
    mbar_arrive(topkbar);
    trace_mark<TRACE>(p, 67);
    // E: arrive once every consumer warp has passed the routed gate/up
    // tiles, wait for every block, stage the routed intermediate, release
    // the consumers (S is handled by the consumer warps themselves)
    if (!mbar_wait(&evt[EVT_E], 0, to, sp_evt)) ok = false;
    red_release_add(&ctr[2], 1u);
    trace_mark<TRACE>(p, 69);
    bool ge = ok && good != 0;
    if (ge) ge = grid_wait_thread(&ctr[2], G, &ctr[5], p.err, to, sp_grid);
    trace_mark<TRACE>(p, 71);
    flags[GO_E] = ge ? 1 : 0;
    if (ge) {
      fence_proxy_async_global();
      const uint32_t hfb = (uint32_t)(4ull * T * KP * L.I), hxb = (uint32_t)(4ull * T * KP * (L.I / 16));
      mbar_expect_tx(&go[GO_E], hfb + hxb);
      bulk_g2s(hf_s, p.hf, hfb, &go[GO_E]);
      bulk_g2s(hx_s, p.hx, hxb, &go[GO_E]);
    }
    mbar_arrive(&go[GO_E]);
  }
  __syncwarp();
}

template <int FMT, bool TRACE>
__global__ void __launch_bounds__(kDecodeThreads, 1) moe_decode_kernel(const DecodeParams p) {
  extern __shared__ __align__(128) uint8_t smem[];
  const Layout& L = p.L;
  const int T = p.T, K = L.K, H = L.H, I = L.I;
  const int G = gridDim.x, c = blockIdx.x;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  int r0, r1;
  block_rows(H, c, G, r0, r1);
  const int nrows = r1 - r0;
  const int nslots = p.nslots;
  const DecodeSmem sp = decode_smem_plan(T, L.KP, L.E, H, I, decode_rows_max(H, G), nslots, p.slot_bytes, smem_opts(L));
  uint8_t* ring = smem + sp.ring;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + sp.bars);
  uint64_t* empty = full + nslots;
  uint64_t* xbar = empty + kSlots;
  uint64_t* xfbar = xbar + 1;
  uint64_t* topkbar = xfbar + 1;
  uint64_t* evt = topkbar + 1;
  uint64_t* go = evt + NEVT;
  TileDesc* descs = reinterpret_cast<TileDesc*>(smem + sp.desc);
  uint16_t* xs = reinterpret_cast<uint16_t*>(smem + sp.xs);
  uint4* xf = reinterpret_cast<uint4*>(smem + sp.xf);
  float* xsum = reinterpret_cast<float*>(smem + sp.xsum);
  float* hs_s = reinterpret_cast<float*>(smem + sp.hs);
  uint8_t* hf_s = smem + sp.hf;
  float* hx_s = reinterpret_cast<float*>(smem + sp.hx);
  uint4* zero4 = reinterpret_cast<uint4*>(smem + sp.zero);
  float* part = reinterpret_cast<float*>(smem + sp.part);
  int* cnt = reinterpret_cast<int*>(smem + sp.cnt);
  float* rpart = reinterpret_cast<float*>(smem + sp.rpart);
  int* rcnt = reinterpret_cast<int*>(smem + sp.rcnt);
  float* tk_w = reinterpret_cast<float*>(smem + sp.tk_w);
  int* tk_i = reinterpret_cast<int*>(smem + sp.tk_i);
  const uint8_t** eptr = reinterpret_cast<const uint8_t**>(smem + sp.eptr);
  uint64_t* tkbuf = reinterpret_cast<uint64_t*>(smem + sp.tkbuf);
  uint16_t* res_s = reinterpret_cast<uint16_t*>(smem + sp.res);
  uint16_t* gam_s = reinterpret_cast<uint16_t*>(smem + sp.gam);
  uint16_t* gpre_s = reinterpret_cast<uint16_t*>(smem + sp.gpre);
  float* wss = reinterpret_cast<float*>(smem + sp.gpre + 2ull * H);
  uint16_t* sgv_s = reinterpret_cast<uint16_t*>(smem + sp.sgv);
  float* sgp = reinterpret_cast<float*>(smem + sp.sgv + 2ull * H);  // [14][T] partial dots, then [T] gates
  float* sgt = sgp + kConsumerWarps * T;
  float* ypart = reinterpret_cast<float*>(smem + sp.ypart);
  float* ys = reinterpret_cast<float*>(smem + sp.ys);
  float* hacc = reinterpret_cast<float*>(smem + sp.hacc);
  float* inv = reinterpret_cast<float*>(smem + sp.inv);
  int* flags = reinterpret_cast<int*>(smem + sp.flags);
  uint32_t* spin_s = reinterpret_cast<uint32_t*>(smem + sp.spin);
  uint32_t* spins = TRACE ? spin_s : nullptr;  // poll counts, traced launches only
  uint32_t* ctr = p.ctr;

  if (tid == 0) {
    for (int s = 0; s < nslots; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kConsumerWarps);
    }
    mbar_init(xbar, 1);
    mbar_init(xfbar, 1);
    mbar_init(topkbar, 1);
    for (int k = 0; k < NEVT; ++k) mbar_init(&evt[k], k == EVT_D ? 1 : kConsumerWarps);
    for (int k = 0; k < NGO; ++k) mbar_init(&go[k], 1);
    mbar_fence_init();
    trace_mark<TRACE>(p, 0);
  }
  if (tid < 16) {
    zero4[tid >> 2] = make_uint4(0u, 0u, 0u, 0u);
    spin_s[tid] = 0u;
    if (tid == FLAG_EPOCH) {
      // this launch's epoch: one past the last launch's (0 is never used)
      const uint32_t ep = ld_relaxed_gpu(ctr + 6) + 1u;
      flags[tid] = (int)(ep == 0u ? 1u : ep);
    } else {
      flags[tid] = 0;
    }
  }
  if (tid < kAccSlots) cnt[tid] = 0;
  if (tid < kSlots * kSplitRows) rcnt[tid] = 0;
  __syncthreads();

  if (warp == kProducerWarp) {
    if (lane == 0) {
      Producer pr;
      pr.ring = ring;
      pr.full = full;
      pr.empty = empty;
      pr.descs = descs;
      pr.slot_bytes = p.slot_bytes;
      pr.slot = 0;
      pr.phase = 0;
      pr.nslots = (uint32_t)nslots;
      pr.timeout_ns = p.timeout_ns;
      pr.err = p.err;
      pr.abort_flag = &ctr[5];
      pr.trace = TRACE ? p.trace + (size_t)c * kTraceEntries : nullptr;
      pr.spins = spins ? spins + 3 : nullptr;
      pr.ncommit = 0;
      pr.ok = true;
      pr.open = false;
      pr.pending_pre = 0;
      pr.nrb_tile = 0;
      pr.d = descs;
      pr.fill = 0;
      pr.policy = l2_policy_evict_first();
      run_producer<TRACE>(p, pr, xs, res_s, gam_s, xbar, topkbar, flags, eptr, tkbuf, gpre_s, sgv_s);
    }
    __syncwarp();
  } else if (warp == kSyncWarp) {
    run_sync<TRACE>(p, xbar, xfbar, topkbar, evt, go, flags, xs, xf, xsum, hs_s, hf_s, hx_s, tk_w, tk_i, eptr, tkbuf,
                    spins);
  } else {
    // ---------------- consumer warps ----------------
    // Every warp walks every tile; the tile's work items (bf16 rows, or units
    // of packed row blocks) are dealt round-robin to the warps, continuing
    // across tiles, and each warp releases a slot on its own.
    const RoutedGeo gh = routed_geo(H, 8), gi = routed_geo(I, 4);
    const uint32_t epoch = (uint32_t)flags[FLAG_EPOCH];
    bool ok = warp_wait(xbar, 0, p.timeout_ns, spins ? spins + 2 : nullptr);
    if (L.prenorm) {
      // x is the residual stream: normalise it first, x = bf16(h / sqrt(mean(h^2) + eps) * gamma_pre),
      // the sum of squares in fixed order (per warp, then over the warps)
      const int np = T * H / 8;
      float part[8];
#pragma unroll
      for (int t = 0; t < 8; ++t) part[t] = 0.f;
#pragma unroll 1
      for (int q = tid; q < np; q += kConsumers) {
        float hv[8];
        unpack_bf16x8(reinterpret_cast<const uint4*>(xs)[q], hv);
        float sq = 0.f;
#pragma unroll
        for (int i = 0; i < 8; ++i) sq = fmaf(hv[i], hv[i], sq);
        const int t = (8 * q) / H;
#pragma unroll
        for (int tt = 0; tt < 8; ++tt)
          if (tt == t) part[tt] += sq;
      }
#pragma unroll
      for (int t = 0; t < 8; ++t) {
        const float v = warp_sum(part[t]);
        if (lane == 0 && t < T) wss[warp * T + t] = v;
      }
      consumer_sync();
      if (tid < T) {
        float ss = 0.f;
        for (int w = 0; w < kConsumerWarps; ++w) ss += wss[w * T + tid];
        inv[tid] = __fdiv_rn(1.f, __fsqrt_rn(__fdiv_rn(ss, (float)H) + L.eps));
      }
      consumer_sync();
#pragma unroll 1
      for (int q = tid; q < np; q += kConsumers) {
        float hv[8], gv[8];
        unpack_bf16x8(reinterpret_cast<const uint4*>(xs)[q], hv);
        const int t = (8 * q) / H, col = 8 * q - t * H;
        unpack_bf16x8(*reinterpret_cast<const uint4*>(gpre_s + col), gv);
        const float iv = inv[t];
        uint32_t o[4];
#pragma unroll
        for (int i = 0; i < 4; ++i)
          o[i] = (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(__fmul_rn(__fmul_rn(hv[2 * i], iv), gv[2 * i]))) |
                 ((uint32_t)__bfloat16_as_ushort(
                      __float2bfloat16_rn(__fmul_rn(__fmul_rn(hv[2 * i + 1], iv), gv[2 * i + 1])))
                  << 16);
        const uint4 xo = make_uint4(o[0], o[1], o[2], o[3]);
        reinterpret_cast<uint4*>(xs)[q] = xo;
        if (c == 0 && p.x_out) reinterpret_cast<uint4*>(p.x_out)[q] = xo;
      }
      consumer_sync();
    }
    {
      // x as the gate/up units' B fragments, with its group sums and scales,
      // built by all consumer threads (piece q is 8 columns of one token):
      // x is rounded to an integer multiple of the group's power-of-two
      // scale sigma = 2^(e - 13) (e the exponent of the group's largest |x|),
      // so |x / sigma| < 2^14, and split as 256 * hi + lo (hi in [-64, 64],
      // lo in [-128, 127]).  The fragment words follow the column order that
      // the units' code expansion gives A: [token][group][t][8 words], word
      // 4 * st + 2 * limb + b holds one limb at four columns of step st; for
      // 4-bit codes 32 st + {2t, 16 + 2t, 2t + 1, 17 + 2t} (b = 0) or
      // 32 st + {8 + 2t, 24 + 2t, 9 + 2t, 25 + 2t} (b = 1); for 2-bit codes
      // 16 st + {2t, 32 + 2t, 2t + 1, 33 + 2t} (b = 0) or
      // 16 st + {8 + 2t, 40 + 2t, 9 + 2t, 41 + 2t} (b = 1).
      const int np = T * H / 8;
      const int Gx = H / 64;
#pragma unroll 1
      for (int q0 = 0; q0 < np; q0 += kConsumers) {
        const int q = q0 + tid;
        float sm = 0.f, mx = 0.f;
        uint4 v = make_uint4(0u, 0u, 0u, 0u);
        float xx[8];
        if (q < np) {
          v = reinterpret_cast<const uint4*>(xs)[q];
          unpack_bf16x8(v, xx);
          sm = ((xx[0] + xx[1]) + (xx[2] + xx[3])) + ((xx[4] + xx[5]) + (xx[6] + xx[7]));
#pragma unroll
          for (int i = 0; i < 8; ++i) mx = fmaxf(mx, fabsf(xx[i]));
        }
        sm += __shfl_xor_sync(0xffffffffu, sm, 1);
        sm += __shfl_xor_sync(0xffffffffu, sm, 2);
        sm += __shfl_xor_sync(0xffffffffu, sm, 4);
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
        if (q < np) {
          const int tg = q >> 3, o8 = q & 7;  // tg = token * Gx + group
          const int tok = tg / Gx, grp = tg - tok * Gx;
          {
            const int ex = max(mx > 0.f ? (int)((__float_as_uint(mx) >> 23) & 0xffu) - 127 : -100, -100);
            const float up = __uint_as_float((uint32_t)(127 + 13 - ex) << 23);  // 1 / sigma
            uint8_t* dst = reinterpret_cast<uint8_t*>(xf) + (size_t)tg * 128;
            // this piece's step, B register and byte offset in the units'
            // column permutation (4-bit: steps of 32 consecutive columns;
            // 2-bit: the 8-column blocks 0, 1, 4, 5 then 2, 3, 6, 7)
            const int st = FMT == FMT_Q4 ? o8 >> 2 : (o8 >> 1) & 1;
            const int b = o8 & 1;
            const int ihi = FMT == FMT_Q4 ? (o8 >> 1) & 1 : o8 >> 2;
#pragma unroll
            for (int r = 0; r < 8; ++r) {
              const int xi = __float2int_rn(xx[r] * up);
              const int hi = (xi + 128) >> 8, lo = xi - (hi << 8);
              const int t4 = r >> 1, i = ihi + 2 * (r & 1);
              uint8_t* w = dst + t4 * 32 + (4 * st + b) * 4 + i;
              w[0] = (uint8_t)(int8_t)hi;  // limb 0: hi
              w[8] = (uint8_t)(int8_t)lo;  // limb 1: lo (two words on)
            }
            if (o8 == 0) {
              xsum[(size_t)tok * 2 * Gx + grp] = sm;
              xsum[(size_t)tok * 2 * Gx + Gx + grp] = __uint_as_float((uint32_t)(127 + ex - 13) << 23);
            }
          }
        }
      }
      consumer_sync();
      if (L.sgate) {
        // the shared output gate of each token: sigmoid(x . g), the dot in
        // fp32 in a fixed order (per thread over its pieces, per warp, then
        // over the warps in order)
        float part[8];
#pragma unroll
        for (int t = 0; t < 8; ++t) part[t] = 0.f;
#pragma unroll 1
        for (int q = tid; q < np; q += kConsumers) {
          float xv[8], gv[8];
          const int t = (8 * q) / H, col = 8 * q - t * H;
          unpack_bf16x8(reinterpret_cast<const uint4*>(xs)[q], xv);
          unpack_bf16x8(*reinterpret_cast<const uint4*>(sgv_s + col), gv);
          float d = 0.f;
#pragma unroll
          for (int i = 0; i < 8; ++i) d = fmaf(xv[i], gv[i], d);
#pragma unroll
          for (int tt = 0; tt < 8; ++tt)
            if (tt == t) part[tt] += d;
        }
#pragma unroll
        for (int t = 0; t < 8; ++t) {
          const float v = warp_sum(part[t]);
          if (lane == 0 && t < T) sgp[warp * T + t] = v;
        }
        consumer_sync();
        if (tid < T) {
          float z = 0.f;
          for (int w = 0; w < kConsumerWarps; ++w) z += sgp[w * T + tid];
          sgt[tid] = 1.f / (1.f + expf(-z));
        }
        // read after the later consumer barriers (the combine)
      }
      if (tid == 0) trace_mark<TRACE>(p, 64);
    }
    int item = 0;  // running count of work items over the compute tiles
    int probed = 0;  // first routed units traced: bit 0 gate/up, bit 1 down
    int nunit = 0;   // routed units done by this warp (traced launches)
    uint32_t slot = 0, phase = 0;
#pragma unroll 1
    for (int ntile = 0;; ++ntile) {
      if (!warp_wait(&full[slot], phase, p.timeout_ns, spins)) {
        if (lane == 0) {
          atomicCAS(p.err, 0u, 1u);
          atomicExch(&ctr[5], 1u);
        }
        ok = false;
        break;
      }
      if (tid == 0 && ntile < 16) trace_mark<TRACE>(p, 16 + 2 * ntile);
      const TileDesc& d = descs[slot];
      const int type = d.type;
      const uint8_t* sl = ring + (size_t)slot * p.slot_bytes;
#pragma unroll 1
      for (int k = 0; k < 2; ++k) {
        if (d.pre & (F_WAIT_S << k)) {
          ok = warp_wait(&go[GO_S + k], 0, p.timeout_ns, spins ? spins + 1 : nullptr) && flags[GO_S + k] != 0 && ok;
          if (tid == 0) trace_mark<TRACE>(p, 4 + k);
        }
      }
      const bool routed_tile = type == TILE_EXPERT_GU || type == TILE_EXPERT_DOWN;
      const bool down = type == TILE_SHARED_DOWN || type == TILE_EXPERT_DOWN;
      const bool work = type != TILE_NONE && (ok || !down);  // down tiles need the staged intermediate
#pragma unroll 1
      for (int si = 0; si < d.nseg; ++si) {
        const Seg& sg = d.seg[si];
        const int nu = sg.u1 - sg.u0;
        // router / shared gate/up rows go through the tensor cores in groups
        // of 16 rows; a tile of one group splits its columns into nparts parts
        // one-token router / shared gate/up rows: nparts column parts per row
        const bool split = T == 1 && (type == TILE_ROUTER || type == TILE_SHARED_GU) && d.nseg == 1 &&
                           sg.nrows <= kSplitRows;
        const int nparts = split ? min(kMaxParts, kConsumerWarps / sg.nrows) : 1;
        const int nitems = routed_tile ? sg.nrows * nu : sg.nrows * nparts;
        if (work) {
#pragma unroll 1
          for (int j = (warp - item % kConsumerWarps + kConsumerWarps) % kConsumerWarps; j < nitems;
               j += kConsumerWarps) {
            if (routed_tile) {
              // ---- one unit of a packed row block: gate/up, or down ----
              const bool gu = type == TILE_EXPERT_GU;
              const int u = sg.u0 + j;  // a routed segment holds one 16-row block
              const int pb = gu ? 1 : 2;
              if (tid == 0 && !(probed & pb)) trace_mark<TRACE>(p, gu ? 11 : 13);
              float r[2][2];
              const uint64_t tu0 = TRACE ? globaltimer_ns() : 0;
              if (gu) {
                const uint32_t xfa = smem_u32(xf + (size_t)(sg.pair / L.KP) * gh.G * 8);
                const uint32_t xsa = smem_u32(xsum + (size_t)(sg.pair / L.KP) * 2 * gh.G);
                routed_unit_gu_i8<FMT>(smem_u32(sl), sg, u, gh, xfa, xsa, r);
              } else {
                routed_unit<FMT, false>(smem_u32(sl), sg, u, gi, smem_u32(hf_s + (size_t)sg.pair * gi.G * 256),
                                        smem_u32(hx_s + (size_t)sg.pair * (I / kRowBlock)), r);
              }
              if (TRACE && tid == 0 && !(probed & pb)) p.trace[(size_t)c * kTraceEntries + (gu ? 100 : 102)] = globaltimer_after(r[0][0]);
              if (TRACE && tid == 0 && nunit < 8) {
                p.trace[(size_t)c * kTraceEntries + 104 + 2 * nunit] = tu0;
                p.trace[(size_t)c * kTraceEntries + 105 + 2 * nunit] = globaltimer_after(r[0][0] + r[1][1]);
              }
              if (TRACE) ++nunit;
              if (gu) {
                gu_unit_done(r[0][0], r[0][1], r[1][0], r[1][1], sg.acc, u, gh.U, part, cnt, sg.pair, sg.row0, I,
                             p.hf, p.hx);
              } else if ((lane & 3) == 0) {
                float* yp = ypart + (size_t)(sg.pair * gi.U + u) * nrows + kRowBlock * sg.row0 - r0;
                yp[lane >> 2] = r[0][0];
                yp[(lane >> 2) + 8] = r[0][1];
              }
              if (tid == 0 && !(probed & pb)) {
                trace_mark<TRACE>(p, gu ? 12 : 14);
                probed |= pb;
              }
            } else {
              // ---- one bf16 row (the gate/up pair for the shared expert) ----
              const int cols = down ? I : H;
              if (split) {
                // part q of row rl: columns [q*chunk, min(cols, (q+1)*chunk))
                const bool probe = TRACE && warp == 0 && type == TILE_SHARED_GU && !(probed & 4);
                if (probe && lane == 0) p.trace[(size_t)c * kTraceEntries + 75] = globaltimer_ns();
                const int rl = j / nparts, q = j - rl * nparts;
                const int chunk = ((cols + nparts - 1) / nparts + 7) & ~7;
                const int c0 = min(cols, q * chunk), nc = min(cols, c0 + chunk) - c0;
                const int row = sg.row0 + rl;
                const float rbias = (type == TILE_ROUTER && p.bias && q == 0) ? __ldg(p.bias + row) : 0.f;
                const uint32_t zs = smem_u32(zero4);
                const uint32_t wa = smem_u32(sl + sg.off[0] + (size_t)rl * 2 * cols + 2 * c0);
                float v0, v1 = 0.f;
                if (type == TILE_SHARED_GU) {
                  float o[2];
                  row_dot_t1<2, false>(wa, smem_u32(sl + sg.off[1] + (size_t)rl * 2 * cols + 2 * c0),
                                       smem_u32(xs) + 2u * c0, nc, zs, o);
                  v0 = o[0];
                  v1 = warp_sum(o[1]);
                } else {
                  float o[1];
                  row_dot_t1<1, false>(wa, 0u, smem_u32(xs) + 2u * c0, nc, zs, o);
                  v0 = o[0];
                }
                v0 = warp_sum(v0) + rbias;
                if (probe && lane == 0) p.trace[(size_t)c * kTraceEntries + 76] = globaltimer_after(v0 + v1);
                float* rp = rpart + ((size_t)slot * kSplitRows + rl) * kMaxParts * 2;
                int last = 0;
                if (lane == 0) {
                  rp[2 * q] = v0;
                  rp[2 * q + 1] = v1;
                  __threadfence_block();
                  last = atomicAdd(&rcnt[slot * kSplitRows + rl], 1) == nparts - 1 ? 1 : 0;
                  if (last) {
                    __threadfence_block();
                    const volatile float* vp = rp;
                    float a0 = 0.f, a1 = 0.f;
                    for (int k = 0; k < nparts; ++k) {
                      a0 += vp[2 * k];
                      a1 += vp[2 * k + 1];
                    }
                    rcnt[slot * kSplitRows + rl] = 0;
                    if (type == TILE_ROUTER) {
                      st_relaxed_gpu_b64(p.logits + row, epoch_word(epoch, a0));
                      if (TRACE)
                        atomicMax(reinterpret_cast<unsigned long long*>(p.trace + (size_t)c * kTraceEntries + 72),
                                  (unsigned long long)globaltimer_ns());
                    } else {
                      p.hs[row] = silu_mul(a0, a1);
                    }
                  }
                }
                if (probe) {
                  if (lane == 0) p.trace[(size_t)c * kTraceEntries + 77] = globaltimer_ns();
                  probed |= 4;
                }
                continue;
              }
              if (type == TILE_ROUTER || type == TILE_SHARED_GU) {
                // whole rows, one per work item
                const uint8_t* w0 = sl + sg.off[0] + (size_t)j * 2 * cols;
                const int row = sg.row0 + j;
                const float rbias = (type == TILE_ROUTER && p.bias) ? __ldg(p.bias + row) : 0.f;
                if (T == 1) {
                  const uint32_t zs = smem_u32(zero4);
                  float v0, v1 = 0.f;
                  if (type == TILE_SHARED_GU) {
                    float o[2];
                    row_dot_t1<2, false>(smem_u32(w0), smem_u32(sl + sg.off[1] + (size_t)j * 2 * cols), smem_u32(xs),
                                         H, zs, o);
                    v0 = o[0];
                    v1 = warp_sum(o[1]);
                  } else {
                    float o[1];
                    row_dot_t1<1, false>(smem_u32(w0), 0u, smem_u32(xs), H, zs, o);
                    v0 = o[0];
                  }
                  v0 = warp_sum(v0);
                  if (lane == 0) {
                    if (type == TILE_ROUTER) {
                      st_relaxed_gpu_b64(p.logits + row, epoch_word(epoch, v0 + rbias));
                      if (TRACE)
                        atomicMax(reinterpret_cast<unsigned long long*>(p.trace + (size_t)c * kTraceEntries + 72),
                                  (unsigned long long)globaltimer_ns());
                    } else {
                      p.hs[row] = silu_mul(v0, v1);
                    }
                  }
                  continue;
                }
#pragma unroll 1
                for (int t0 = 0; t0 < T; t0 += 4) {
                  const int nt = min(4, T - t0);
                  float acc[2][4];
                  bf16_dot4(w0, type == TILE_SHARED_GU ? sl + sg.off[1] + (size_t)j * 2 * cols : nullptr, H,
                            reinterpret_cast<const uint8_t*>(xs + (size_t)t0 * H), 2u * H, false, nt, acc);
#pragma unroll 1
                  for (int tt = 0; tt < nt; ++tt) {
                    const int t = t0 + tt;
                    float a0 = 0.f, a1 = 0.f;
#pragma unroll
                    for (int qq = 0; qq < 4; ++qq)
                      if (qq == tt) a0 = acc[0][qq], a1 = acc[1][qq];
                    a0 = warp_sum(a0);
                    if (type == TILE_SHARED_GU) a1 = warp_sum(a1);
                    if (lane == 0) {
                      if (type == TILE_ROUTER)
                        st_relaxed_gpu_b64(p.logits + (size_t)t * L.E + row, epoch_word(epoch, a0 + rbias));
                      else
                        p.hs[(size_t)t * I + row] = silu_mul(a0, a1);
                    }
                  }
                }
                continue;
              }
              // ---- one bf16 row of the shared expert's down projection ----
              const uint8_t* w0 = sl + sg.off[0] + (size_t)j * 2 * cols;
              const int row = sg.row0 + j;
              if (T == 1) {
                // one token: the chunked dot, no per-token branches
                float o[1];
                row_dot_t1<1, true>(smem_u32(w0), 0u, smem_u32(hs_s), I, smem_u32(zero4), o);
                const float v0 = warp_sum(o[0]);
                if (lane == 0) ys[row - r0] = v0;
                continue;
              }
#pragma unroll 1
              for (int t0 = 0; t0 < T; t0 += 4) {
                const int nt = min(4, T - t0);
                float acc[2][4];
                bf16_dot4(w0, nullptr, I, reinterpret_cast<const uint8_t*>(hs_s + (size_t)t0 * I), 4u * I, true, nt,
                          acc);
#pragma unroll 1
                for (int tt = 0; tt < nt; ++tt) {
                  float a0 = 0.f;
#pragma unroll
                  for (int q = 0; q < 4; ++q)
                    if (q == tt) a0 = acc[0][q];
                  a0 = warp_sum(a0);
                  if (lane == 0) ys[(t0 + tt) * nrows + row - r0] = a0;
                }
              }
            }
          }
        }
        item += nitems;
      }
      // this warp is done with the slot
      __syncwarp();
      const int post = d.post;
      if (lane == 0 && (post & F_ARRIVE_R)) mbar_arrive(&evt[EVT_R]);
      if (lane == 0 && (post & F_ARRIVE_E)) mbar_arrive(&evt[EVT_E]);
      if (TRACE && tid == 0 && (post & F_ARRIVE_R)) trace_mark<TRACE>(p, 1);
      if (TRACE && tid == 0 && (post & F_ARRIVE_S)) trace_mark<TRACE>(p, 2);
      if (TRACE && tid == 0 && (post & F_ARRIVE_E)) trace_mark<TRACE>(p, 3);
      const bool end = (post & F_END) != 0;
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[slot]);
      if (tid == 0 && ntile < 16) trace_mark<TRACE>(p, 17 + 2 * ntile);
      if (post & F_ARRIVE_S) {
        // S (after the slot is released): the last consumer warp past the
        // shared gate/up tiles arrives for the block, waits for every block
        // and stages the shared intermediate (warp-uniform, while the routing
        // is still being found)
        int last = 0;
        if (lane == 0) {
          __threadfence();
          last = atomicAdd(&flags[FLAG_SCNT], 1) == kConsumerWarps - 1 ? 1 : 0;
        }
        if (__shfl_sync(0xffffffffu, last, 0)) {
          if (lane == 0) {
            __threadfence();
            red_release_add(&ctr[1], 1u);
            trace_mark<TRACE>(p, 68);
          }
          __syncwarp();
          const bool need = L.has_shared && !L.spacked;  // the bf16 shared expert's intermediate
          const bool gw = ok && (!need || grid_wait_thread(&ctr[1], G, &ctr[5], p.err, p.timeout_ns));
          const bool gs = __all_sync(0xffffffffu, gw);
          if (lane == 0) {
            trace_mark<TRACE>(p, 70);
            flags[GO_S] = gs ? 1 : 0;
            if (gs && need) {
              fence_proxy_async_global();
              const uint32_t bytes = (uint32_t)(4ull * T * I);
              mbar_expect_tx(&go[GO_S], bytes);
              bulk_g2s(hs_s, p.hs, bytes, &go[GO_S]);
            }
            mbar_arrive(&go[GO_S]);
          }
        }
      }
      if (++slot == (uint32_t)nslots) {
        slot = 0;
        phase ^= 1u;
      }
      if (end) break;
    }
    if (tid == 0) trace_mark<TRACE>(p, 6);

    // ---- combine + residual, sum of squares ----
    consumer_sync();
    const bool routed = flags[FLAG_TOPK] != 0;
    if (ok && routed) {
#pragma unroll 1
      for (int q = tid; q < T * nrows; q += kConsumers) {
        const int t = q / nrows, j = q - t * nrows;
        float acc = 0.f;
#pragma unroll 1
        for (int k = 0; k < L.KP; ++k) {
          const int pair = t * L.KP + k;
          float yk = 0.f;
#pragma unroll 1
          for (int u = 0; u < gi.U; ++u) yk += ypart[(size_t)(pair * gi.U + u) * nrows + j];
          // pair K: the packed shared expert, scaled by its gate if any
          const float wk = k < K ? tk_w[pair] : (L.sgate ? sgt[t] : 1.f);
          acc = fmaf(wk, yk, acc);
        }
        float h = __bfloat162float(__ushort_as_bfloat16(res_s[q])) + acc;
        if (L.has_shared && !L.spacked) h += L.sgate ? sgt[t] * ys[q] : ys[q];
        hacc[q] = h;
        p.h_out[(size_t)t * H + r0 + j] = __bfloat16_as_ushort(__float2bfloat16_rn(h));
      }
      consumer_sync();
      // publish this block's sum of squares per token as an epoch word
      if (warp < T) {
        float s = 0.f;
#pragma unroll 1
        for (int j = lane; j < nrows; j += 32) s = fmaf(hacc[warp * nrows + j], hacc[warp * nrows + j], s);
        s = warp_sum(s);
        if (lane == 0) st_relaxed_gpu_b64(p.ss + (size_t)c * T + warp, epoch_word(epoch, s));
        if (TRACE && lane == 0 && warp == 0) p.trace[(size_t)c * kTraceEntries + 99] = globaltimer_ns();
      }
      // RMSNorm: block 0 polls all blocks' sums of squares (the words are
      // complete once they carry this launch's epoch), sums them in block
      // order and publishes the total per token; every other block polls that
      // one word, then all normalise their own rows of h with the same total
      bool got = true;
      if (warp < T && c != 0) {
        __shared__ uint32_t s_tot[kMaxTokensFused];
        got = warp_poll_words(p.sstot + warp, 1, epoch, s_tot + warp, &ctr[5], p.err, p.timeout_ns);
        __syncwarp();
        if (lane == 0) {
          inv[warp] = rsqrtf(__fdividef(__uint_as_float(s_tot[warp]), (float)H) + L.eps);
          if (!got) flags[FLAG_NOSS] = 1;  // the total never came
        }
      } else if (warp < T) {
        // lane l holds blocks l, l + 32, ...: every pass loads all the words
        // still missing at once, so a pass costs one round trip
        constexpr int kMaxPer = (kMaxGrid + 31) / 32;
        float v[kMaxPer];
        uint32_t need = 0;
#pragma unroll
        for (int i = 0; i < kMaxPer; ++i) {
          v[i] = 0.f;
          if (lane + 32 * i < G) need |= 1u << i;
        }
        uint64_t t0 = 0;
#pragma unroll 1
        for (uint32_t it = 0;; ++it) {
          if (TRACE && lane == 0 && warp == 0) {
            const uint64_t now = globaltimer_ns();
            if (it < 8) p.trace[(size_t)c * kTraceEntries + 120 + it] = now;
            p.trace[(size_t)c * kTraceEntries + 97] = it + 1;
          }
          uint64_t wd[kMaxPer];
#pragma unroll
          for (int i = 0; i < kMaxPer; ++i)
            wd[i] = (need >> i & 1u) ? ld_relaxed_gpu_b64(p.ss + (size_t)(lane + 32 * i) * T + warp) : 0ull;
          if (TRACE && lane == 0 && warp == 0)
            p.trace[(size_t)c * kTraceEntries + 98] = globaltimer_after((float)(wd[0] + wd[kMaxPer - 1]));
#pragma unroll
          for (int i = 0; i < kMaxPer; ++i)
            if ((need >> i & 1u) && (uint32_t)(wd[i] >> 32) == epoch) {
              need &= ~(1u << i);
              v[i] = __uint_as_float((uint32_t)wd[i]);
            }
          if (__all_sync(0xffffffffu, need == 0u)) break;
          if ((it & 15u) == 15u) {
            int stop = 0;
            if (lane == 0) {
              if (t0 == 0) t0 = globaltimer_ns();
              if (ld_relaxed_gpu(&ctr[5]) != 0u) {
                stop = 1;
              } else if (globaltimer_ns() - t0 > p.timeout_ns) {
                atomicCAS(p.err, 0u, 1u);
                atomicExch(&ctr[5], 1u);
                stop = 1;
              }
            }
            if (__shfl_sync(0xffffffffu, stop, 0)) {
              got = false;
              break;
            }
          }
        }
        // the sum in block order: lane partials over i, then across lanes
        // (a fixed order whatever the arrival order)
        float s = 0.f;
#pragma unroll
        for (int i = 0; i < kMaxPer; ++i) s += v[i];
        s = warp_sum(s);
        if (lane == 0) {
          if (got) st_relaxed_gpu_b64(p.sstot + warp, epoch_word(epoch, s));
          inv[warp] = rsqrtf(__fdividef(s, (float)H) + L.eps);
          if (!got) flags[FLAG_NOSS] = 1;  // some block's sum of squares never came
        }
      }
      consumer_sync();
      if (flags[FLAG_NOSS] == 0) {
#pragma unroll 1
        for (int q = tid; q < T * nrows; q += kConsumers) {
          const int t = q / nrows, j = q - t * nrows;
          const float g = __bfloat162float(__ushort_as_bfloat16(gam_s[j]));
          p.y_norm[(size_t)t * H + r0 + j] = __bfloat16_as_ushort(__float2bfloat16_rn(hacc[q] * inv[t] * g));
        }
      }
    }
  }

  // ---- exit: the block that arrives last on the final counter resets the
  // counters and records this launch's epoch for the next launch (every other
  // block is past its last use of them) ----
  __syncthreads();
  if (tid == 0) {
    if constexpr (TRACE)
      for (int k = 0; k < 8; ++k) p.trace[(size_t)c * kTraceEntries + 80 + k] = spin_s[k];
    trace_mark<TRACE>(p, 7);
    if (atomicAdd(&ctr[3], 1u) == (uint32_t)G - 1u) {
      // plain stores: the next launch reads them after this one ends
      volatile uint32_t* vc = reinterpret_cast<volatile uint32_t*>(ctr);
      for (int k = 0; k < 6; ++k) vc[k] = 0u;
      vc[6] = (uint32_t)flags[FLAG_EPOCH];
      vc[7] = 0u;
    }
  }
  if (tid == 0) trace_mark<TRACE>(p, 8);
}

// The kernel's dynamic shared-memory limit is raised per device to the
// largest size any launch asked for; the check and the set happen under one
// lock, so host threads launching different sizes cannot leave the cached
// value above the attribute.
template <int FMT, bool TRACE>
static cudaError_t launch_one(const DecodeParams& p, int grid, size_t smem, cudaStream_t st) {
  static size_t attr_set[64] = {};
  static std::mutex mu;
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64) {
    std::lock_guard<std::mutex> lk(mu);
    if (attr_set[dev] < smem) {
      const cudaError_t e = cudaFuncSetAttribute(moe_decode_kernel<FMT, TRACE>,
                                                 cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
      if (e != cudaSuccess) return e;
      attr_set[dev] = smem;
    }
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kDecodeThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, moe_decode_kernel<FMT, TRACE>, p);
}

cudaError_t launch_decode(const DecodeParams& p, int grid, size_t smem, cudaStream_t st) {
  if (p.trace)
    return p.L.bits == 4 ? launch_one<FMT_Q4, true>(p, grid, smem, st) : launch_one<FMT_Q2, true>(p, grid, smem, st);
  return p.L.bits == 4 ? launch_one<FMT_Q4, false>(p, grid, smem, st) : launch_one<FMT_Q2, false>(p, grid, smem, st);
}

// Ring geometry for a shape: the most slots (4, else 3, else 2) whose size
// (a multiple of 1 KB, at most 48 KB) holds the largest tile of every phase
// next to the rest of the shared-memory plan.  Returns the slot size and sets
// *nslots, or returns 0 if no ring fits.
uint32_t decode_slot_bytes(const Layout& L, int T, int nrows_max, int* nslots) {
  const size_t limit = 227 * 1024;
  const RoutedGeo gh = routed_geo(L.H, 8), gi = routed_geo(L.I, 4);
  const size_t per_group = 64ull * L.bits + 32;
  const size_t need[5] = {2ull * L.H + 16, 4ull * L.H + 32, 2ull * L.I + 16,
                          2ull * 2 * 8 * gh.W * per_group + 64, 2ull * 4 * gi.W * per_group + 64};
  for (int ns = kSlots; ns >= 2; --ns) {
    const size_t other = decode_smem_plan(T, L.KP, L.E, L.H, L.I, nrows_max, ns, 0, smem_opts(L)).total + 2048;  // + static shared memory and alignment
    if (other >= limit) return 0;
    size_t slot = (limit - other) / ns;
    slot = slot / 1024 * 1024;
    if (slot > (size_t)kMaxSlotBytes) slot = kMaxSlotBytes;
    bool fits = true;
    for (size_t n : need) fits = fits && n <= slot;
    if (fits) {
      *nslots = ns;
      return (uint32_t)slot;
    }
  }
  return 0;
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
