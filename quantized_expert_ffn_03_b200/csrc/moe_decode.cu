// moe_decode.cu -- the fused single-launch MoE layer for decode (T <= 8).
//
// One persistent cooperative launch, one block per SM.  Each block streams
// exactly the weight bytes it owns through a ring of shared-memory slots:
// a producer warp issues bulk copies (cp.async.bulk, completion counted on an
// mbarrier per slot) and 14 consumer warps compute from shared memory.  A
// sync warp does the block's grid-wide arrivals and waits and stages the
// activation vectors, so consumers never stall on a release fence, on
// polling global memory, or on block-wide barriers between tiles.
// The block's byte stream, in order:
//   router rows  -> [arrive R]  shared gate/up rows  -> [arrive S]
//   (producer: wait R, top-K, expert pointers)
//   routed gate/up rows of the chosen experts  -> [arrive E]
//   [wait S]  shared down rows of the block's output rows
//   [wait E]  routed down rows of the block's output rows
// then combine + residual, a grid-wide sum of squares, and RMSNorm of the
// block's rows.  The copies that follow a wait are already in flight while a
// block waits, so HBM stays busy across the waits.
//
// Consumer work unit: one weight row (or the gate/up pair of one row), done
// entirely by one warp over 1024-column chunks; rows are dealt round-robin to
// the consumer warps across tiles, and each warp releases a slot on its own.
//
// This is the single-kernel form of the pages' pipeline: router projection
// with the shared expert (CMD2), top-K, the K expert reads and the deferred
// expert forward with combine + residual + norm (CMD3)
// ("Flash-MoE: ラップトップでの397Bパラメータモデルの実行", section
// "パイプライン概要"; "Streaming experts: как запустить триллионную модель на
// MacBook", sections "Flash-MoE: чистый C, Metal и никакого Python" and
// "Оптимизации, которые сработали").
#include <cuda_bf16.h>

#include "moe_kernels.h"
#include "moe_phases.cuh"

namespace moe {

// 16 warps in all, 4 per SM sub-partition, so each thread may use up to 128
// registers: 14 consumer warps, the producer warp and the sync warp.
constexpr int kConsumerWarps = 14;
constexpr int kConsumers = kConsumerWarps * 32;  // 448
constexpr int kProducerWarp = kConsumerWarps;    // warp 14
constexpr int kSyncWarp = kConsumerWarps + 1;    // warp 15
constexpr int kDecodeThreads = kConsumers + 64;
static_assert(kDecodeThreads == kDecodeBlockThreads, "block size");
constexpr int kSlots = 4;
constexpr int kMaxSeg = 8;
constexpr int kMaxSlotBytes = 48 * 1024;
constexpr int kTraceEntries = 64;

enum TileType : int {
  TILE_ROUTER = 0,
  TILE_SHARED_GU,
  TILE_EXPERT_GU,
  TILE_SHARED_DOWN,
  TILE_EXPERT_DOWN,
  TILE_ARRIVE_R,
  TILE_ARRIVE_S,
  TILE_ARRIVE_E,
  TILE_WAIT_S,
  TILE_WAIT_E,
  TILE_END
};

struct Seg {
  int pair;  // (token, expert) pair of routed tiles
  int row0;  // first matrix row
  int nrows;
  uint32_t off[4];  // slot byte offset of each range's first valid byte
};

struct TileDesc {
  int type;
  int nseg;
  Seg seg[kMaxSeg];
};

// barriers consumers -> sync warp (evt) and sync warp -> consumers (go)
enum { EVT_R = 0, EVT_S, EVT_E, EVT_D, NEVT };
enum { GO_S = 0, GO_E, GO_D, NGO };

// ---- shared-memory plan ------------------------------------------------------
// xq: x in the quantised-row lane layout, permuted so that lane l's j-th
// 16-byte piece of 1024-column chunk ch sits at unit ((t*nch + ch)*4 + j)*32 + l;
// xc: (sum x, sum offset*x) of each lane's 32 columns.
struct DecodeSmem {
  size_t ring, bars, desc, xs, xq, xc, hs, he, tk_w, tk_i, eptr, ypart, ys, hacc, inv, flags, total;
};

__host__ __device__ inline size_t align_up(size_t n, size_t a) { return (n + a - 1) / a * a; }

__host__ __device__ inline DecodeSmem decode_smem_plan(int T, int K, int H, int I, int nrows,
                                                       uint32_t slot_bytes) {
  const int nch = (H + 1023) / 1024;
  DecodeSmem s;
  size_t pos = 0;
  s.ring = pos;
  pos = align_up(pos + (size_t)kSlots * slot_bytes, 128);
  s.bars = pos;  // full[kSlots], empty[kSlots], xbar, xcbar, evt[NEVT], go[NGO]
  pos = align_up(pos + 8 * (2 * kSlots + 2 + NEVT + NGO), 16);
  s.desc = pos;
  pos = align_up(pos + sizeof(TileDesc) * kSlots, 16);
  s.xs = pos;
  pos = align_up(pos + 2ull * T * H, 16);
  s.xq = pos;
  pos = align_up(pos + 16ull * T * nch * 128, 16);
  s.xc = pos;
  pos = align_up(pos + 8ull * T * nch * 32, 16);
  s.hs = pos;
  pos = align_up(pos + 4ull * T * I, 16);
  s.he = pos;
  pos = align_up(pos + 4ull * T * K * I, 16);
  s.tk_w = pos;
  pos = align_up(pos + sizeof(float) * T * K, 16);
  s.tk_i = pos;
  pos = align_up(pos + sizeof(int) * T * K, 16);
  s.eptr = pos;
  pos = align_up(pos + sizeof(void*) * T * K, 16);
  s.ypart = pos;
  pos = align_up(pos + sizeof(float) * T * K * nrows, 16);
  s.ys = pos;
  pos = align_up(pos + sizeof(float) * T * nrows, 16);
  s.hacc = pos;
  pos = align_up(pos + sizeof(float) * T * nrows, 16);
  s.inv = pos;
  pos = align_up(pos + sizeof(float) * T, 16);
  s.flags = pos;
  pos = align_up(pos + 16 * sizeof(int), 16);
  s.total = pos;
  return s;
}

size_t decode_smem_bytes(const Layout& L, int T, int nrows, uint32_t slot_bytes) {
  return decode_smem_plan(T, L.K, L.H, L.I, nrows, slot_bytes).total;
}

// ---- small helpers ----------------------------------------------------------------

__device__ __forceinline__ void consumer_sync() { named_sync(1, kConsumers); }

// Warp-wide bounded wait on an mbarrier phase: lane 0 polls, the warp
// synchronises on the result (other lanes see the data through __syncwarp).
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, uint64_t timeout_ns) {
  int ok = 1;
  if ((threadIdx.x & 31) == 0) ok = mbar_wait(bar, parity, timeout_ns) ? 1 : 0;
  ok = __shfl_sync(0xffffffffu, ok, 0);
  return ok != 0;
}

__device__ __forceinline__ void trace_mark(const DecodeParams& p, int k) {
  if (p.trace && k < kTraceEntries) p.trace[(size_t)blockIdx.x * kTraceEntries + k] = globaltimer_ns();
}

__device__ __forceinline__ void range_of(int n, int c, int G, int& a, int& b) {
  a = (int)((long long)n * c / G);
  b = (int)((long long)n * (c + 1) / G);
}

__device__ __forceinline__ int cap_rows(uint32_t slot_bytes, uint32_t slack, uint32_t per_row) {
  const int r = (int)((slot_bytes - slack) / per_row);
  return max(1, min(r, 1024));
}

// One grid wait by the calling thread only.
__device__ __forceinline__ bool grid_wait_thread(const uint32_t* ctr, uint32_t target, uint32_t* abort_flag,
                                                 uint32_t* err, uint64_t timeout_ns) {
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t it = 0;; ++it) {
    if (ld_acquire_gpu(ctr) >= target) return true;
    if (ld_relaxed_gpu(abort_flag) != 0u) return false;
    if ((it & 63u) == 63u && (globaltimer_ns() - t0 > timeout_ns || it > (1u << 28))) {
      atomicCAS(err, 0u, 1u);
      atomicExch(abort_flag, 1u);
      return false;
    }
  }
}

// ---- per-lane chunk loads and dots ----------------------------------------------------
// Chunk ch of a row covers columns [1024*ch, 1024*ch + 1024).
// bf16 rows: lane l owns columns 1024*ch + 256*j + 8*l + c (j < 4, c < 8), so
// each 16-byte read of a row (or of x) is contiguous across the warp.
// Quantised rows: lane l owns the 32 columns of group-half cidx = 32*ch + l.

__device__ __forceinline__ void x_strided_bf16(float (&x)[32], const uint16_t* v, int ch, int cols) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const int c0 = ch * 1024 + 256 * j + 8 * lane;
    if (c0 < cols) {
      unpack_bf16x8(*reinterpret_cast<const uint4*>(v + c0), x + 8 * j);
    } else {
#pragma unroll
      for (int c = 0; c < 8; ++c) x[8 * j + c] = 0.f;
    }
  }
}

__device__ __forceinline__ void x_strided_f32(float (&x)[32], const float* v, int ch, int cols) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const int c0 = ch * 1024 + 256 * j + 8 * lane;
    if (c0 < cols) {
      const float4 a = *reinterpret_cast<const float4*>(v + c0);
      const float4 b = *reinterpret_cast<const float4*>(v + c0 + 4);
      x[8 * j + 0] = a.x;
      x[8 * j + 1] = a.y;
      x[8 * j + 2] = a.z;
      x[8 * j + 3] = a.w;
      x[8 * j + 4] = b.x;
      x[8 * j + 5] = b.y;
      x[8 * j + 6] = b.z;
      x[8 * j + 7] = b.w;
    } else {
#pragma unroll
      for (int c = 0; c < 8; ++c) x[8 * j + c] = 0.f;
    }
  }
}

// bf16 row chunk dot (strided lane layout)
__device__ __forceinline__ float bf16_chunk(const uint8_t* row, int ch, int cols, const float (&x)[32]) {
  const int lane = threadIdx.x & 31;
  float2 a0 = make_float2(0.f, 0.f), a1 = make_float2(0.f, 0.f);
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const int c0 = ch * 1024 + 256 * j + 8 * lane;
    if (c0 < cols) {
      const uint4 q = *reinterpret_cast<const uint4*>(row + 2 * c0);
      const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        const float2 c = make_float2(__uint_as_float(w[m] << 16), __uint_as_float(w[m] & 0xffff0000u));
        const float2 xx = make_float2(x[8 * j + 2 * m], x[8 * j + 2 * m + 1]);
        if (m & 1)
          a1 = __ffma2_rn(c, xx, a1);
        else
          a0 = __ffma2_rn(c, xx, a0);
      }
    }
  }
  return (a0.x + a1.x) + (a0.y + a1.y);
}

// quantised row chunk dot (contiguous lane layout); lx holds the lane's 32
// activations and its two constants
template <int FMT>
__device__ __forceinline__ float q_chunk(const uint8_t* row, const uint8_t* srow, int cidx, bool active,
                                         const LaneX& lx) {
  if (!active) return 0.f;
  Frag<FMT> f;
  if constexpr (FMT == FMT_Q4)
    f.q = *reinterpret_cast<const uint4*>(row + cidx * 16);
  else
    f.q = *reinterpret_cast<const uint2*>(row + cidx * 8);
  f.s = *reinterpret_cast<const uint32_t*>(srow + (cidx >> 1) * 4);
  return frag_dot<FMT>(f, lx);
}

// x chunk for quantised rows from the permuted bf16 copy, constants from xc
__device__ __forceinline__ void xq_chunk(LaneX& lx, const uint4* xq, const float2* xc, int t, int nch, int ch) {
  const int lane = threadIdx.x & 31;
  const uint4* u = xq + (size_t)((t * nch + ch) * 4) * 32 + lane;
#pragma unroll
  for (int j = 0; j < 4; ++j) unpack_bf16x8(u[32 * j], lx.x + 8 * j);
  const float2 k = xc[(t * nch + ch) * 32 + lane];
  lx.xsum = k.x;
  lx.corr = k.y;
}

// ---- producer ----------------------------------------------------------------------
// One thread (lane 0 of the producer warp) builds each tile's descriptor in
// place in shared memory once the consumers have freed the slot, announces
// each copy's bytes on the slot's "full" barrier and issues it, and finally
// arrives on the barrier, which completes when every copy has landed.
struct Producer {
  uint8_t* ring;
  uint64_t* full;
  uint64_t* empty;
  TileDesc* descs;
  uint32_t slot_bytes;
  uint32_t slot, phase;
  uint64_t timeout_ns;
  uint32_t* err;
  uint32_t* abort_flag;
  uint64_t* trace;
  int ncommit;
  bool ok;
  TileDesc* d;
  uint32_t fill;
  uint64_t policy;  // L2 evict-first: weights are read once per launch

  __device__ __noinline__ bool begin(int type) {
    if (!ok) return false;
    if (!mbar_wait(&empty[slot], phase ^ 1u, timeout_ns)) {
      ok = false;
      atomicCAS(err, 0u, 1u);
      atomicExch(abort_flag, 1u);
      return false;
    }
    d = &descs[slot];
    d->type = type;
    d->nseg = 0;
    fill = 0;
    return true;
  }
  __device__ Seg& seg(int pair, int row0, int nrows) {
    Seg& s = d->seg[d->nseg++];
    s.pair = pair;
    s.row0 = row0;
    s.nrows = nrows;
    return s;
  }
  // Copy a byte range into the slot; returns the slot offset of its first
  // byte.  The copy is widened to 16-byte boundaries (the widened range stays
  // inside the same 256-byte aligned section).
  __device__ __noinline__ uint32_t range(const void* p, size_t bytes) {
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
  __device__ __noinline__ void commit() {
    if (trace && ncommit < 16) trace[48 + ncommit] = globaltimer_ns();
    ++ncommit;
    mbar_arrive(&full[slot]);
    if (++slot == kSlots) {
      slot = 0;
      phase ^= 1u;
    }
  }
  __device__ void marker(int type) {
    if (begin(type)) commit();
  }
};

template <int FMT>
__device__ void run_producer(const DecodeParams& p, Producer& pr, uint16_t* xs, uint64_t* xbar, float* tk_w,
                             int* tk_i, const uint8_t** eptr) {
  const Layout& L = p.L;
  const int T = p.T, K = L.K, H = L.H, I = L.I, E = L.E;
  const int G = gridDim.x, c = blockIdx.x;
  const int lane = threadIdx.x & 31;
  const bool leader = lane == 0;
  const int r0 = (int)((long long)H * c / G), r1 = (int)((long long)H * (c + 1) / G);

  if (leader) {
    // the token activations, once per block
    const uint32_t xb = (uint32_t)(2ull * T * H);
    mbar_expect_tx(xbar, xb);
    bulk_g2s(xs, p.x, xb, xbar);
    mbar_arrive(xbar);
    // router rows
    int a, b;
    range_of(E, c, G, a, b);
    const int rmax = cap_rows(pr.slot_bytes, 16, 2 * H);
#pragma unroll 1
    for (int e = a; e < b; e += rmax) {
      const int n = min(rmax, b - e);
      if (!pr.begin(TILE_ROUTER)) break;
      Seg& s = pr.seg(-1, e, n);
      s.off[0] = pr.range(p.wr + (size_t)e * H, (size_t)n * H * 2);
      pr.commit();
    }
    pr.marker(TILE_ARRIVE_R);
    // shared gate/up rows
    if (L.has_shared) {
      range_of(I, c, G, a, b);
      const int smax = cap_rows(pr.slot_bytes, 32, 4 * H);
#pragma unroll 1
      for (int i = a; i < b; i += smax) {
        const int n = min(smax, b - i);
        if (!pr.begin(TILE_SHARED_GU)) break;
        Seg& s = pr.seg(-1, i, n);
        s.off[0] = pr.range(p.sg + (size_t)i * H, (size_t)n * H * 2);
        s.off[1] = pr.range(p.su + (size_t)i * H, (size_t)n * H * 2);
        pr.commit();
      }
    }
    pr.marker(TILE_ARRIVE_S);
  }
  __syncwarp();

  // top-K, once the router logits of every block are written
  bool ok = true;
  if (leader) ok = grid_wait_thread(&p.ctr[0], G, &p.ctr[5], p.err, p.timeout_ns);
  ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
  if (ok) {
#pragma unroll 1
    for (int t = 0; t < T; ++t) warp_topk(p.logits + (size_t)t * E, E, K, tk_i + t * K, tk_w + t * K);
    __syncwarp();
#pragma unroll 1
    for (int j = lane; j < T * K; j += 32) {
      const int e = tk_i[j];
      const void* bp = (e >= 0 && e < E) ? p.expert_ptr[e] : nullptr;
      if (bp == nullptr || (reinterpret_cast<uintptr_t>(bp) & 255u)) {
        atomicCAS(p.err, 0u, 2u);
        atomicExch(&p.ctr[5], 1u);
        bp = nullptr;
      }
      eptr[j] = reinterpret_cast<const uint8_t*>(bp);
      if (c == 0) {
        if (p.idx_out) p.idx_out[j] = e;
        if (p.w_out) p.w_out[j] = tk_w[j];
      }
    }
    __syncwarp();
#pragma unroll 1
    for (int j = 0; j < T * K; ++j) ok = ok && eptr[j] != nullptr;
  }
  if (leader) {
    trace_mark(p, 9);
    const uint32_t cr_h = L.code_row_bytes[0], sr_h = L.scale_row_bytes[0];
    const uint32_t cr_i = L.code_row_bytes[2], sr_i = L.scale_row_bytes[2];
    if (ok) {
      // routed gate/up: this block's share of the T*K*I (pair, row) items
      int a, b;
      range_of(T * K * I, c, G, a, b);
      const int gmax = cap_rows(pr.slot_bytes, 64, 2 * (cr_h + sr_h));
#pragma unroll 1
      for (int q = a; q < b;) {
        const int pair = q / I, i = q - pair * I;
        const int n = min(gmax, min(b - q, I - i));
        const uint8_t* blob = eptr[pair];
        if (!pr.begin(TILE_EXPERT_GU)) break;
        Seg& s = pr.seg(pair, i, n);
        s.off[0] = pr.range(blob + L.off_codes[0] + (size_t)i * cr_h, (size_t)n * cr_h);
        s.off[1] = pr.range(blob + L.off_codes[1] + (size_t)i * cr_h, (size_t)n * cr_h);
        s.off[2] = pr.range(blob + L.off_scales[0] + (size_t)i * sr_h, (size_t)n * sr_h);
        s.off[3] = pr.range(blob + L.off_scales[1] + (size_t)i * sr_h, (size_t)n * sr_h);
        pr.commit();
        q += n;
      }
    }
    pr.marker(TILE_ARRIVE_E);
    pr.marker(TILE_WAIT_S);
    if (L.has_shared) {
      const int dmax = cap_rows(pr.slot_bytes, 16, 2 * I);
#pragma unroll 1
      for (int r = r0; r < r1; r += dmax) {
        const int n = min(dmax, r1 - r);
        if (!pr.begin(TILE_SHARED_DOWN)) break;
        Seg& s = pr.seg(-1, r, n);
        s.off[0] = pr.range(p.sd + (size_t)r * I, (size_t)n * I * 2);
        pr.commit();
      }
    }
    pr.marker(TILE_WAIT_E);
    if (ok) {
      // routed down rows [r0, r1) of every pair, several pairs per tile
      const uint32_t per_row = cr_i + sr_i;
      const int emax = cap_rows(pr.slot_bytes, 32, per_row);
      bool open = false;
#pragma unroll 1
      for (int pair = 0; pair < T * K && pr.ok; ++pair) {
#pragma unroll 1
        for (int r = r0; r < r1;) {
          const int n = min(emax, r1 - r);
          if (open && (pr.d->nseg == kMaxSeg || pr.fill + (uint32_t)n * per_row + 32 > pr.slot_bytes)) {
            pr.commit();
            open = false;
          }
          if (!open) {
            if (!pr.begin(TILE_EXPERT_DOWN)) break;
            open = true;
          }
          const uint8_t* blob = eptr[pair];
          Seg& s = pr.seg(pair, r, n);
          s.off[0] = pr.range(blob + L.off_codes[2] + (size_t)r * cr_i, (size_t)n * cr_i);
          s.off[1] = pr.range(blob + L.off_scales[2] + (size_t)r * sr_i, (size_t)n * sr_i);
          r += n;
        }
      }
      if (open) pr.commit();
    }
    pr.marker(TILE_END);
    trace_mark(p, 10);
  }
}

// ---- sync warp ----------------------------------------------------------------------
// Prepares the quantised-layout copy of x and its constants, then does the
// block's grid-wide arrivals (R, S, E, D) and waits (S, E, D).  After the S
// and E waits it stages the shared / routed intermediates into shared memory
// with bulk copies that complete the consumers' "go" barriers.
template <int FMT>
__device__ void run_sync(const DecodeParams& p, uint64_t* xbar, uint64_t* xcbar, uint64_t* evt, uint64_t* go,
                         int* flags, const uint16_t* xs, uint4* xq, float2* xc, float* hs_s, float* he_s) {
  const int lane = threadIdx.x & 31;
  const Layout& L = p.L;
  const int T = p.T, H = L.H, G = gridDim.x;
  const int nch = (H + 1023) / 1024;
  uint32_t* ctr = p.ctr;
  const uint64_t to = p.timeout_ns;
  bool ok = warp_wait(xbar, 0, to);
  if (ok) {
#pragma unroll 1
    for (int u = lane; u < T * nch * 32; u += 32) {
      const int t = u / (nch * 32), cidx = u - t * nch * 32;  // cidx = 32*ch + l
      const int ch = cidx >> 5, l = cidx & 31;
      LaneX lx;
      if (cidx * 32 < H) {
        const uint16_t* src = xs + (size_t)t * H + cidx * 32;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const uint4 v = *reinterpret_cast<const uint4*>(src + 8 * j);
          xq[(size_t)((t * nch + ch) * 4 + j) * 32 + l] = v;
          unpack_bf16x8(v, lx.x + 8 * j);
        }
      } else {
#pragma unroll
        for (int j = 0; j < 4; ++j) xq[(size_t)((t * nch + ch) * 4 + j) * 32 + l] = make_uint4(0, 0, 0, 0);
#pragma unroll
        for (int i = 0; i < 32; ++i) lx.x[i] = 0.f;
      }
      lane_constants<FMT>(lx);
      xc[u] = make_float2(lx.xsum, lx.corr);
    }
  }
  __syncwarp();
  if (lane == 0) {
    mbar_arrive(xcbar);
    // R, S, E: arrive once every consumer warp has passed the phase's marker
#pragma unroll 1
    for (int k = EVT_R; k <= EVT_E; ++k) {
      if (!mbar_wait(&evt[k], 0, to)) ok = false;
      red_release_add(&ctr[k], 1u);
    }
    // wait S, then E; stage the intermediates; release the consumers
#pragma unroll 1
    for (int k = 0; k < 2; ++k) {
      bool good = ok;
      if (good && (k == 1 || L.has_shared)) good = grid_wait_thread(&ctr[1 + k], G, &ctr[5], p.err, to);
      flags[GO_S + k] = good ? 1 : 0;
      uint64_t* bar = &go[GO_S + k];
      if (good && (k == 1 || L.has_shared)) {
        fence_proxy_async_global();
        const uint32_t bytes = k == 0 ? (uint32_t)(4ull * T * L.I) : (uint32_t)(4ull * T * L.K * L.I);
        mbar_expect_tx(bar, bytes);
        bulk_g2s(k == 0 ? hs_s : he_s, k == 0 ? p.hs : p.he, bytes, bar);
      }
      mbar_arrive(bar);
    }
    // D: sum of squares written -> arrive, wait, release the consumers
    if (!mbar_wait(&evt[EVT_D], 0, to)) ok = false;
    red_release_add(&ctr[3], 1u);
    const bool good = ok && grid_wait_thread(&ctr[3], G, &ctr[5], p.err, to);
    flags[GO_D] = good ? 1 : 0;
    mbar_arrive(&go[GO_D]);
  }
  __syncwarp();
}

template <int FMT>
__global__ void __launch_bounds__(kDecodeThreads, 1) moe_decode_kernel(const DecodeParams p) {
  extern __shared__ __align__(128) uint8_t smem[];
  const Layout& L = p.L;
  const int T = p.T, K = L.K, H = L.H, I = L.I;
  const int G = gridDim.x, c = blockIdx.x;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int r0 = (int)((long long)H * c / G), r1 = (int)((long long)H * (c + 1) / G);
  const int nrows = r1 - r0;
  const int nrows_max = (H + G - 1) / G;
  const int nch_h = (H + 1023) / 1024, nch_i = (I + 1023) / 1024;
  const DecodeSmem sp = decode_smem_plan(T, K, H, I, nrows_max, p.slot_bytes);
  uint8_t* ring = smem + sp.ring;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + sp.bars);
  uint64_t* empty = full + kSlots;
  uint64_t* xbar = empty + kSlots;
  uint64_t* xcbar = xbar + 1;
  uint64_t* evt = xcbar + 1;
  uint64_t* go = evt + NEVT;
  TileDesc* descs = reinterpret_cast<TileDesc*>(smem + sp.desc);
  uint16_t* xs = reinterpret_cast<uint16_t*>(smem + sp.xs);
  uint4* xq = reinterpret_cast<uint4*>(smem + sp.xq);
  float2* xc = reinterpret_cast<float2*>(smem + sp.xc);
  float* hs_s = reinterpret_cast<float*>(smem + sp.hs);
  float* he_s = reinterpret_cast<float*>(smem + sp.he);
  float* tk_w = reinterpret_cast<float*>(smem + sp.tk_w);
  int* tk_i = reinterpret_cast<int*>(smem + sp.tk_i);
  const uint8_t** eptr = reinterpret_cast<const uint8_t**>(smem + sp.eptr);
  float* ypart = reinterpret_cast<float*>(smem + sp.ypart);
  float* ys = reinterpret_cast<float*>(smem + sp.ys);
  float* hacc = reinterpret_cast<float*>(smem + sp.hacc);
  float* inv = reinterpret_cast<float*>(smem + sp.inv);
  int* flags = reinterpret_cast<int*>(smem + sp.flags);
  uint32_t* ctr = p.ctr;

  if (tid == 0) {
    for (int s = 0; s < kSlots; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kConsumerWarps);
    }
    mbar_init(xbar, 1);
    mbar_init(xcbar, 1);
    for (int k = 0; k < NEVT; ++k) mbar_init(&evt[k], k == EVT_D ? 1 : kConsumerWarps);
    for (int k = 0; k < NGO; ++k) mbar_init(&go[k], 1);
    mbar_fence_init();
    trace_mark(p, 0);
  }
  __syncthreads();

  if (warp == kProducerWarp) {
    Producer pr;
    pr.ring = ring;
    pr.full = full;
    pr.empty = empty;
    pr.descs = descs;
    pr.slot_bytes = p.slot_bytes;
    pr.slot = 0;
    pr.phase = 0;
    pr.timeout_ns = p.timeout_ns;
    pr.err = p.err;
    pr.abort_flag = &ctr[5];
    pr.trace = p.trace ? p.trace + (size_t)c * kTraceEntries : nullptr;
    pr.ncommit = 0;
    pr.ok = true;
    pr.d = descs;
    pr.fill = 0;
    pr.policy = l2_policy_evict_first();
    run_producer<FMT>(p, pr, xs, xbar, tk_w, tk_i, eptr);
  } else if (warp == kSyncWarp) {
    run_sync<FMT>(p, xbar, xcbar, evt, go, flags, xs, xq, xc, hs_s, he_s);
  } else {
    // ---------------- consumer warps ----------------
    // Every compute tile runs through one loop nest: segment -> this warp's
    // row items -> token -> matrix -> 1024-column chunk.  The tile kind only
    // selects the row format, the activation source and the epilogue, so the
    // dot-product code exists once and stays in the instruction cache.
    bool ok = true;
    bool have_x = false, have_xc = false;
    int item = 0;      // running count of row items over the compute tiles
    int held = -1;     // key of the activation chunk cached in lx
    bool probed = false;
    LaneX lx;
    uint32_t slot = 0, phase = 0;
    for (int ntile = 0;; ++ntile) {
      if (!warp_wait(&full[slot], phase, p.timeout_ns)) {
        if (lane == 0) {
          atomicCAS(p.err, 0u, 1u);
          atomicExch(&ctr[5], 1u);
        }
        ok = false;
        break;
      }
      if (tid == 0 && ntile < 16) trace_mark(p, 16 + 2 * ntile);
      const TileDesc& d = descs[slot];
      const int type = d.type;
      const uint8_t* sl = ring + (size_t)slot * p.slot_bytes;
      if (type == TILE_END) break;
      if (type >= TILE_ARRIVE_R) {
        if (type <= TILE_ARRIVE_E) {
          __syncwarp();  // the warp's stores of this phase precede its arrival
          if (lane == 0) mbar_arrive(&evt[type - TILE_ARRIVE_R]);
          if (tid == 0) trace_mark(p, 1 + type - TILE_ARRIVE_R);
        } else {
          const int k = type == TILE_WAIT_S ? GO_S : GO_E;
          ok = warp_wait(&go[k], 0, p.timeout_ns) && flags[k] != 0 && ok;
          if (tid == 0) trace_mark(p, type == TILE_WAIT_S ? 4 : 5);
        }
      } else {
        // ---- compute tile ----
        const bool routed = type == TILE_EXPERT_GU || type == TILE_EXPERT_DOWN;
        const bool down = type >= TILE_SHARED_DOWN;
        const int nm = (type == TILE_SHARED_GU || type == TILE_EXPERT_GU) ? 2 : 1;
        const int cols = down ? I : H;
        const int nch = down ? nch_i : nch_h;
        const int ntok = routed ? 1 : T;
        const uint32_t crow = routed ? L.code_row_bytes[down ? 2 : 0] : 2u * (uint32_t)cols;
        const uint32_t srow = routed ? L.scale_row_bytes[down ? 2 : 0] : 0u;
        // activation source: 0 x (bf16 rows), 1 x (quantised rows), 2 shared
        // intermediate (bf16 rows), 3 routed intermediate (quantised rows)
        const int xk = type == TILE_ROUTER || type == TILE_SHARED_GU ? 0
                       : type == TILE_EXPERT_GU                       ? 1
                       : type == TILE_SHARED_DOWN                     ? 2
                                                                      : 3;
        if (xk == 0 && !have_x) {
          ok = warp_wait(xbar, 0, p.timeout_ns) && ok;
          have_x = true;
        }
        if (xk == 1 && !have_xc) {
          ok = warp_wait(xcbar, 0, p.timeout_ns) && ok;
          have_xc = true;
        }
        const bool work = ok || !routed;  // routed tiles need the routing
#pragma unroll 1
        for (int si = 0; si < d.nseg; ++si) {
          const Seg& sg = d.seg[si];
          if (work && !(down && !ok)) {
#pragma unroll 1
            for (int j = (warp - item % kConsumerWarps + kConsumerWarps) % kConsumerWarps; j < sg.nrows;
                 j += kConsumerWarps) {
#pragma unroll 1
              for (int tt = 0; tt < ntok; ++tt) {
                const int t = routed ? sg.pair / K : tt;
                float a0 = 0.f, a1 = 0.f;
#pragma unroll 1
                for (int ch = 0; ch < nch; ++ch) {
                  const int cidx = ch * 32 + lane;
                  const bool act = cidx * 32 < cols;
                  const int key = ((xk * 64 + (xk == 3 ? sg.pair : t)) * 64 + ch);
                  const bool probe = tid == 0 && type == TILE_EXPERT_GU && !probed && ch == 0;
                  if (probe) trace_mark(p, 11);
                  if (key != held) {
                    if (xk == 0) {
                      x_strided_bf16(lx.x, xs + (size_t)t * H, ch, H);
                    } else if (xk == 1) {
                      xq_chunk(lx, xq, xc, t, nch_h, ch);
                    } else if (xk == 2) {
                      x_strided_f32(lx.x, hs_s + (size_t)t * I, ch, I);
                    } else {
                      if (act) {
                        const float4* hv = reinterpret_cast<const float4*>(he_s + (size_t)sg.pair * I + cidx * 32);
#pragma unroll
                        for (int q = 0; q < 8; ++q) {
                          const float4 v = hv[q];
                          lx.x[4 * q] = v.x;
                          lx.x[4 * q + 1] = v.y;
                          lx.x[4 * q + 2] = v.z;
                          lx.x[4 * q + 3] = v.w;
                        }
                      } else {
#pragma unroll
                        for (int q = 0; q < 32; ++q) lx.x[q] = 0.f;
                      }
                      lane_constants<FMT>(lx);
                    }
                    held = key;
                  }
                  if (probe) trace_mark(p, 12);
#pragma unroll 1
                  for (int m = 0; m < nm; ++m) {
                    const uint8_t* row = sl + sg.off[m] + (size_t)j * crow;
                    const float v = routed ? q_chunk<FMT>(row, sl + sg.off[nm + m] + (size_t)j * srow, cidx, act, lx)
                                           : bf16_chunk(row, ch, cols, lx.x);
                    if (m == 0)
                      a0 += v;
                    else
                      a1 += v;
                  }
                  if (probe) trace_mark(p, 13);
                }
                if (tid == 0 && type == TILE_EXPERT_GU && !probed) trace_mark(p, 14);
                a0 = warp_sum(a0);
                if (nm == 2) a1 = warp_sum(a1);
                if (lane == 0) {
                  const int row = sg.row0 + j;
                  if (type == TILE_ROUTER)
                    p.logits[(size_t)t * L.E + row] = a0 + (p.bias ? p.bias[row] : 0.f);
                  else if (type == TILE_SHARED_GU)
                    p.hs[(size_t)t * I + row] = silu_mul(a0, a1);
                  else if (type == TILE_EXPERT_GU)
                    p.he[(size_t)sg.pair * I + row] = silu_mul(a0, a1);
                  else if (type == TILE_SHARED_DOWN)
                    ys[t * nrows + row - r0] = a0;
                  else
                    ypart[sg.pair * nrows + row - r0] = a0;
                }
                if (tid == 0 && type == TILE_EXPERT_GU && !probed) {
                  trace_mark(p, 15);
                  probed = true;
                }
              }
            }
          }
          item += sg.nrows;
        }
      }
      // this warp is done with the slot
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[slot]);
      if (tid == 0 && ntile < 16) trace_mark(p, 17 + 2 * ntile);
      if (++slot == kSlots) {
        slot = 0;
        phase ^= 1u;
      }
    }
    if (tid == 0) trace_mark(p, 6);

    // ---- combine + residual, sum of squares ----
    consumer_sync();
    if (ok) {
#pragma unroll 1
      for (int q = tid; q < T * nrows; q += kConsumers) {
        const int t = q / nrows, j = q - t * nrows;
        float acc = 0.f;
#pragma unroll 1
        for (int k = 0; k < K; ++k) acc = fmaf(tk_w[t * K + k], ypart[(t * K + k) * nrows + j], acc);
        const float res = __bfloat162float(__ushort_as_bfloat16(p.res[(size_t)t * H + r0 + j]));
        float h = res + acc;
        if (L.has_shared) h += ys[t * nrows + j];
        hacc[t * nrows + j] = h;
        p.h_out[(size_t)t * H + r0 + j] = __bfloat16_as_ushort(__float2bfloat16_rn(h));
      }
      consumer_sync();
      if (warp < T) {
        float s = 0.f;
#pragma unroll 1
        for (int j = lane; j < nrows; j += 32) s = fmaf(hacc[warp * nrows + j], hacc[warp * nrows + j], s);
        s = warp_sum(s);
        if (lane == 0) p.ss[(size_t)c * T + warp] = s;
      }
    }
    consumer_sync();
    if (tid == 0) mbar_arrive(&evt[EVT_D]);
    ok = warp_wait(&go[GO_D], 0, p.timeout_ns) && flags[GO_D] != 0 && ok;
    if (tid == 0) trace_mark(p, 7);
    if (ok) {
      if (warp < T) {
        float s = 0.f;
#pragma unroll 1
        for (int b = lane; b < G; b += 32) s += __ldcg(p.ss + (size_t)b * T + warp);
        s = warp_sum(s);
        if (lane == 0) inv[warp] = 1.f / sqrtf(s / (float)H + L.eps);
      }
      consumer_sync();
#pragma unroll 1
      for (int q = tid; q < T * nrows; q += kConsumers) {
        const int t = q / nrows, j = q - t * nrows;
        const float gm = __bfloat162float(__ushort_as_bfloat16(p.gamma[r0 + j]));
        p.y_norm[(size_t)t * H + r0 + j] =
            __bfloat16_as_ushort(__float2bfloat16_rn(hacc[t * nrows + j] * inv[t] * gm));
      }
    }
  }

  // ---- exit: the last block out resets the counters for the next launch ----
  __syncthreads();
  if (tid == 0) {
    trace_mark(p, 8);
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
  static size_t attr_set[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && attr_set[dev] < smem) {
    cudaError_t e =
        cudaFuncSetAttribute(moe_decode_kernel<FMT>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    attr_set[dev] = smem;
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
  return cudaLaunchKernelEx(&cfg, moe_decode_kernel<FMT>, p);
}

cudaError_t launch_decode(const DecodeParams& p, int grid, size_t smem, cudaStream_t st) {
  return p.L.bits == 4 ? launch_one<FMT_Q4>(p, grid, smem, st) : launch_one<FMT_Q2>(p, grid, smem, st);
}

// Largest slot size (bytes, multiple of 1 KB, at most 48 KB) that fits the
// shared memory of one block together with the rest of the plan; 0 if the
// smallest tile of some phase would not fit.
uint32_t decode_slot_bytes(const Layout& L, int T, int nrows_max) {
  const size_t limit = 227 * 1024;
  const size_t other = decode_smem_plan(T, L.K, L.H, L.I, nrows_max, 0).total + 1024;
  if (other >= limit) return 0;
  size_t slot = (limit - other) / kSlots;
  slot = slot / 1024 * 1024;
  if (slot > (size_t)kMaxSlotBytes) slot = kMaxSlotBytes;
  const size_t need[5] = {2ull * L.H + 16, 4ull * L.H + 32,
                          2ull * (L.code_row_bytes[0] + L.scale_row_bytes[0]) + 64, 2ull * L.I + 16,
                          (size_t)L.code_row_bytes[2] + L.scale_row_bytes[2] + 32};
  for (size_t n : need)
    if (n > slot) return 0;
  return (uint32_t)slot;
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
