// moe_device.cuh -- device-side building blocks of libmoe (sm_100a).
//
// Row dot products over packed 4/2-bit group-affine weights and bf16 weights,
// warp/team reductions, bounded grid-wide waits and the router's top-K.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "moe_layout.h"

namespace moe {


enum Fmt { FMT_Q4 = 4, FMT_Q2 = 2, FMT_BF16 = 16 };

// ---------------------------------------------------------------------------
// Per-lane activation slice: 32 consecutive input columns in fp32 registers,
// plus the two per-lane constants of the factored dequant dot (below).
// ---------------------------------------------------------------------------
struct LaneX {
  float x[32];
  float xsum;  // sum of the 32 values (multiplies the group bias)
  float corr;  // sum of magic offsets times x (removed from the code sum)
};

// Dequant dot, factored per group.  For one group with scale s and bias beta:
//   sum_i (q_i*s + beta) x_i = s * sum_i q_i x_i + beta * sum_i x_i,
// the per-weight fma(q, s*x, beta*x) of the FMA kernel summed over the group
// ("Streaming experts: как запустить триллионную модель на MacBook",
// section "Оптимизации, которые сработали").  The code q is turned into a
// float without a conversion instruction: the word is rotated so that the
// code lands in the top mantissa bits (bits 15..22) and OR-ed with the
// exponent of 2^e, which gives exactly 2^e + q.  The known 2^e terms are
// summed once per lane into `corr` and subtracted after the loop.
//   4-bit: a rotation puts nibble 2p at bits 15..18 (256 + q) and nibble
//          2p+1 at bits 19..22 (16 + q).
//   2-bit: a rotation puts codes 4p..4p+3 at bits 15,17,19,21
//          (256 + q, 64 + q, 16 + q, 4 + q).
// The rotation for pair/quad p of a word is rotl(word, (15 - 8p) mod 32).
__device__ __forceinline__ uint32_t rotl(uint32_t v, int r) { return __funnelshift_l(v, v, r); }

__device__ __forceinline__ float magic(uint32_t r, uint32_t mask, uint32_t expo) {
  return __uint_as_float((r & mask) | expo);
}

template <int FMT>
__device__ __forceinline__ void lane_constants(LaneX& lx) {
  float s = 0.f, c = 0.f;
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    s += lx.x[i];
    float off;
    if (FMT == FMT_Q4) {
      off = (i & 1) ? 16.f : 256.f;
    } else if (FMT == FMT_Q2) {
      const int j = i & 3;
      off = j == 0 ? 256.f : j == 1 ? 64.f : j == 2 ? 16.f : 4.f;
    } else {
      off = 0.f;
    }
    c = fmaf(off, lx.x[i], c);
  }
  lx.xsum = s;
  lx.corr = c;
}

// Sum over 32 columns of (2^e + q_i) * x_i for one 4-bit fragment.  The two
// codes a rotation exposes multiply two adjacent activations, so each pair is
// one packed fp32 FMA (fma.rn.f32x2): lane x[2i] pairs with the 256+q code of
// its word position, x[2i+1] with the 16+q code.
__device__ __forceinline__ float2 f2(float a, float b) { return make_float2(a, b); }

__device__ __forceinline__ float codes_dot_q4(const uint4 q, const LaneX& lx) {
  const uint32_t w[4] = {q.x, q.y, q.z, q.w};
  float2 acc0 = f2(0.f, 0.f), acc1 = f2(0.f, 0.f);
#pragma unroll
  for (int j = 0; j < 4; ++j) {
#pragma unroll
    for (int p = 0; p < 4; ++p) {
      const uint32_t r = rotl(w[j], (15 - 8 * p) & 31);
      const float2 c = f2(magic(r, 0x00078000u, 0x43800000u), magic(r, 0x00780000u, 0x41800000u));
      const float2 xx = f2(lx.x[8 * j + 2 * p], lx.x[8 * j + 2 * p + 1]);
      if (p & 1)
        acc1 = __ffma2_rn(c, xx, acc1);
      else
        acc0 = __ffma2_rn(c, xx, acc0);
    }
  }
  return (acc0.x + acc1.x) + (acc0.y + acc1.y);
}

// Same for a 2-bit fragment (two words, 32 codes): codes 4p..4p+3 of a word
// sit at bits 15, 17, 19, 21 after one rotation (256+q, 64+q, 16+q, 4+q).
__device__ __forceinline__ float codes_dot_q2(const uint2 q, const LaneX& lx) {
  const uint32_t w[2] = {q.x, q.y};
  float2 acc0 = f2(0.f, 0.f), acc1 = f2(0.f, 0.f);
#pragma unroll
  for (int j = 0; j < 2; ++j) {
#pragma unroll
    for (int p = 0; p < 4; ++p) {
      const uint32_t r = rotl(w[j], (15 - 8 * p) & 31);
      const float* xx = lx.x + 16 * j + 4 * p;
      acc0 = __ffma2_rn(f2(magic(r, 0x00018000u, 0x43800000u), magic(r, 0x00060000u, 0x42800000u)),
                        f2(xx[0], xx[1]), acc0);
      acc1 = __ffma2_rn(f2(magic(r, 0x00180000u, 0x41800000u), magic(r, 0x00600000u, 0x40800000u)),
                        f2(xx[2], xx[3]), acc1);
    }
  }
  return (acc0.x + acc1.x) + (acc0.y + acc1.y);
}

__device__ __forceinline__ float bf16_dot(const uint4 (&q)[4], const LaneX& lx) {
  float2 acc0 = f2(0.f, 0.f), acc1 = f2(0.f, 0.f);
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const uint32_t w[4] = {q[j].x, q[j].y, q[j].z, q[j].w};
#pragma unroll
    for (int m = 0; m < 4; ++m) {
      const float2 c = f2(__uint_as_float(w[m] << 16), __uint_as_float(w[m] & 0xffff0000u));
      const float2 xx = f2(lx.x[8 * j + 2 * m], lx.x[8 * j + 2 * m + 1]);
      if (m & 1)
        acc1 = __ffma2_rn(c, xx, acc1);
      else
        acc0 = __ffma2_rn(c, xx, acc0);
    }
  }
  return (acc0.x + acc1.x) + (acc0.y + acc1.y);
}

// ---------------------------------------------------------------------------
// Per-lane fragment of one weight row: the lane's 32 columns.
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint4 ld_stream_v4(const void* p) {
  uint4 v;
  asm("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}
__device__ __forceinline__ uint2 ld_stream_v2(const void* p) {
  uint2 v;
  asm("ld.global.nc.L1::no_allocate.v2.u32 {%0,%1}, [%2];" : "=r"(v.x), "=r"(v.y) : "l"(p));
  return v;
}
__device__ __forceinline__ uint32_t ld_stream_u32(const void* p) {
  uint32_t v;
  asm("ld.global.nc.L1::no_allocate.u32 %0, [%1];" : "=r"(v) : "l"(p));
  return v;
}

template <int FMT>
struct Frag;
template <>
struct Frag<FMT_Q4> {
  uint4 q;
  uint32_t s;
};
template <>
struct Frag<FMT_Q2> {
  uint2 q;
  uint32_t s;
};
template <>
struct Frag<FMT_BF16> {
  uint4 q[4];
};

// Quantised row: codes_row / scales_row point at the row's first byte.
template <int FMT>
__device__ __forceinline__ void load_frag(Frag<FMT>& f, const uint8_t* codes_row,
                                          const uint8_t* scales_row, int chunk) {
  if constexpr (FMT == FMT_Q4) {
    f.q = ld_stream_v4(codes_row + chunk * 16);
    f.s = ld_stream_u32(scales_row + (chunk >> 1) * 4);
  } else if constexpr (FMT == FMT_Q2) {
    f.q = ld_stream_v2(codes_row + chunk * 8);
    f.s = ld_stream_u32(scales_row + (chunk >> 1) * 4);
  } else {
    const uint8_t* p = codes_row + chunk * 64;
#pragma unroll
    for (int j = 0; j < 4; ++j) f.q[j] = ld_stream_v4(p + 16 * j);
  }
}

template <int FMT>
__device__ __forceinline__ void zero_frag(Frag<FMT>& f) {
  if constexpr (FMT == FMT_BF16) {
#pragma unroll
    for (int j = 0; j < 4; ++j) f.q[j] = make_uint4(0, 0, 0, 0);
  } else if constexpr (FMT == FMT_Q4) {
    f.q = make_uint4(0, 0, 0, 0);
    f.s = 0;
  } else {
    f.q = make_uint2(0, 0);
    f.s = 0;
  }
}

// Partial dot of the lane's 32 columns with the lane's activations.
template <int FMT>
__device__ __forceinline__ float frag_dot(const Frag<FMT>& f, const LaneX& lx) {
  if constexpr (FMT == FMT_BF16) {
    return bf16_dot(f.q, lx);
  } else {
    float raw;
    if constexpr (FMT == FMT_Q4)
      raw = codes_dot_q4(f.q, lx);
    else
      raw = codes_dot_q2(f.q, lx);
    const float s = __uint_as_float(f.s << 16);
    const float beta = __uint_as_float(f.s & 0xffff0000u);
    return fmaf(s, raw - lx.corr, beta * lx.xsum);
  }
}

// ---------------------------------------------------------------------------
// Activation loads.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void unpack_bf16x8(const uint4 v, float* out) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int m = 0; m < 4; ++m) {
    out[2 * m] = __uint_as_float(w[m] << 16);
    out[2 * m + 1] = __uint_as_float(w[m] & 0xffff0000u);
  }
}

// bf16 activations (read-only for the whole kernel).
template <int FMT>
__device__ __forceinline__ void load_lane_x_bf16(LaneX& lx, const uint16_t* row, int chunk,
                                                 bool active) {
  if (active) {
    const uint4* p = reinterpret_cast<const uint4*>(row + chunk * 32);
#pragma unroll
    for (int j = 0; j < 4; ++j) unpack_bf16x8(__ldg(p + j), lx.x + 8 * j);
  } else {
#pragma unroll
    for (int i = 0; i < 32; ++i) lx.x[i] = 0.f;
  }
  lane_constants<FMT>(lx);
}

// fp32 activations written earlier in the same launch by other blocks: read
// through L2 only (ld.global.cg), never from a possibly stale L1 line.
template <int FMT>
__device__ __forceinline__ void load_lane_x_f32(LaneX& lx, const float* row, int chunk,
                                                bool active) {
  if (active) {
    const float4* p = reinterpret_cast<const float4*>(row + chunk * 32);
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const float4 v = __ldcg(p + j);
      lx.x[4 * j] = v.x;
      lx.x[4 * j + 1] = v.y;
      lx.x[4 * j + 2] = v.z;
      lx.x[4 * j + 3] = v.w;
    }
  } else {
#pragma unroll
    for (int i = 0; i < 32; ++i) lx.x[i] = 0.f;
  }
  lane_constants<FMT>(lx);
}

// ---------------------------------------------------------------------------
// Reductions and synchronisation.
// ---------------------------------------------------------------------------
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ void named_sync(int id, int nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ uint32_t ld_acquire_gpu(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ uint32_t ld_relaxed_gpu(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ void red_release_add(uint32_t* p, uint32_t v) {
  asm volatile("red.release.gpu.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// Block-wide "arrive" on a grid counter: all writes of this block made before
// the call become visible to any block that later observes the increment.
__device__ __forceinline__ void grid_arrive(uint32_t* ctr) {
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    red_release_add(ctr, 1u);
  }
}

// Block-wide bounded wait until *ctr >= target.  Gives up (returns false) if
// the launch's abort flag is raised or the time limit passes; in the latter
// case it records MOE device error 1 (timeout) in *err and raises the abort
// flag so that every other block stops waiting too.  Never traps.
__device__ __forceinline__ bool grid_wait(const uint32_t* ctr, uint32_t target, uint32_t* abort_flag,
                                          uint32_t* err, uint64_t timeout_ns, int* s_flag) {
  if (threadIdx.x == 0) {
    int ok = 1;
    const uint64_t t0 = globaltimer_ns();
    for (uint32_t it = 0;; ++it) {
      if (ld_acquire_gpu(ctr) >= target) break;
      if (ld_relaxed_gpu(abort_flag) != 0u) {
        ok = 0;
        break;
      }
      if ((it & 63u) == 63u) {
        if (globaltimer_ns() - t0 > timeout_ns || it > (1u << 28)) {
          atomicCAS(err, 0u, 1u);
          atomicExch(abort_flag, 1u);
          ok = 0;
          break;
        }
      }
      if (it > 256u) __nanosleep(32);
    }
    __threadfence();
    *s_flag = ok;
  }
  __syncthreads();
  return *s_flag != 0;
}

// ---------------------------------------------------------------------------
// Router top-K: one warp per token.  Order: larger logit first, ties to the
// lower expert index, NaN ranks as -inf.  Weights are the softmax over the K
// chosen logits (softmax over E renormalised over the K).
// ---------------------------------------------------------------------------
__device__ __forceinline__ float rank_key(float v) { return v != v ? -INFINITY : v; }

__device__ __forceinline__ bool ranks_before(float ka, int ia, float kb, int ib) {
  return ka > kb || (ka == kb && ia < ib);
}

// logits: [E] for this token (read through L2).  Writes idx[K], w[K] from
// lane 0..K-1 (any memory space).
static __device__ __noinline__ void warp_topk(const float* logits, int E, int K, int32_t* idx, float* w) {
  const int lane = threadIdx.x & 31;
  float prev_k = INFINITY;
  int prev_i = -1;
  float sel_k[kMaxK];
  int sel_i[kMaxK];
  const bool in_regs = E <= 1024;
  float vals[32];
  if (in_regs) {
#pragma unroll
    for (int m = 0; m < 32; ++m) {
      const int e = lane + 32 * m;
      vals[m] = e < E ? rank_key(__ldcg(logits + e)) : -INFINITY;
    }
  }
#pragma unroll 1
  for (int k = 0; k < K; ++k) {
    // best element of this lane that ranks strictly after the previous pick
    float bk = -INFINITY;
    int bi = 0x7fffffff;
    if (in_regs) {
#pragma unroll
      for (int m = 0; m < 32; ++m) {
        const int e = lane + 32 * m;
        if (e < E && ranks_before(prev_k, prev_i, vals[m], e) &&
            ranks_before(vals[m], e, bk, bi))
          bk = vals[m], bi = e;
      }
    } else {
      for (int e = lane; e < E; e += 32) {
        const float v = rank_key(__ldcg(logits + e));
        if (ranks_before(prev_k, prev_i, v, e) && ranks_before(v, e, bk, bi)) bk = v, bi = e;
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float ok = __shfl_xor_sync(0xffffffffu, bk, o);
      const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
      if (ranks_before(ok, oi, bk, bi)) bk = ok, bi = oi;
    }
    sel_k[k < kMaxK ? k : 0] = bk;
    sel_i[k < kMaxK ? k : 0] = bi;
    prev_k = bk;
    prev_i = bi;
  }
  // weights, computed redundantly by every lane; lane k writes entry k
  const float lmax = sel_k[0];
  float den = 0.f;
#pragma unroll 1
  for (int k = 0; k < K; ++k) den += expf(sel_k[k] - lmax);
#pragma unroll 1
  for (int k = 0; k < K; ++k) {
    if (lane == (k & 31)) {
      idx[k] = sel_i[k];
      w[k] = expf(sel_k[k] - lmax) / den;
    }
  }
}

__device__ __forceinline__ float silu_mul(float g, float u) { return g / (1.f + expf(-g)) * u; }

// L2 prefetch of a byte range through the bulk-copy engine (no shared
// memory).  The range is widened to 16-byte boundaries; callers keep it
// inside the allocation (all sections of a blob are 256-byte aligned).
__device__ __forceinline__ void l2_prefetch(const void* p, size_t bytes) {
  if (bytes == 0) return;
  uintptr_t a = reinterpret_cast<uintptr_t>(p) & ~uintptr_t(15);
  const uintptr_t end = (reinterpret_cast<uintptr_t>(p) + bytes + 15) & ~uintptr_t(15);
  while (a < end) {
    const uint32_t n = (uint32_t)((end - a) < 32768 ? (end - a) : 32768);
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(a), "r"(n) : "memory");
    a += n;
  }
}

// ---------------------------------------------------------------------------
// Shared-memory barriers (mbarrier) and bulk copies global -> shared.
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_fence_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
      " selp.u32 %0, 1, 0, p;\n}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// try_wait that lets the hardware suspend the thread for up to hint_ns while
// the phase is incomplete (it returns as soon as the phase completes), so a
// waiting warp issues almost no instructions.
__device__ __forceinline__ bool mbar_try_wait_sleep(uint64_t* bar, uint32_t parity, uint32_t hint_ns) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n"
      " selp.u32 %0, 1, 0, p;\n}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity), "r"(hint_ns)
      : "memory");
  return ok != 0;
}

// Bounded wait for phase `parity` of an mbarrier; false on timeout.
static __device__ __noinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, uint64_t timeout_ns) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t it = 0;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 1023u) == 1023u && globaltimer_ns() - t0 > timeout_ns) return false;
  }
}

// Orders this thread's earlier generic-proxy accesses (e.g. an acquire that
// observed other blocks' stores) before its later bulk copies from global.
__device__ __forceinline__ void fence_proxy_async_global() {
  asm volatile("fence.proxy.async.global;" ::: "memory");
}

// Adds `bytes` to the transaction count of the current phase (no arrival).
__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.expect_tx.relaxed.cta.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}

// Bulk copy of `bytes` (multiple of 16) from global `src` (16-byte aligned)
// to shared `dst` (16-byte aligned); completion is counted on `bar`.
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// L2 policy for data read once per launch: evict it before anything else, so
// the kernel's code and its small shared data stay in L2 across launches.
__device__ __forceinline__ uint64_t l2_policy_evict_first() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}

// bulk_g2s with an L2 cache-policy hint.
__device__ __forceinline__ void bulk_g2s_hint(void* dst, const void* src, uint32_t bytes, uint64_t* bar,
                                              uint64_t policy) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], "
      "%4;" ::"r"(smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar)), "l"(policy)
      : "memory");
}

}  // namespace moe
