// moe_device.cuh -- device-side building blocks of libmoe (sm_100a).
//
// bf16 unpacking, warp reductions, bounded grid-wide waits, the router's
// top-K, and the mbarrier / bulk-copy primitives of the streaming ring.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "moe_layout.h"

namespace moe {

enum Fmt { FMT_Q4 = 4, FMT_Q2 = 2 };

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
// The same, read only once `dep` has been computed (orders a trace stamp
// after the arithmetic that produced dep).
__device__ __forceinline__ uint64_t globaltimer_after(float dep) {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t) : "f"(dep) : "memory");
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

// 64-bit words that carry their own launch number: a value published as
// (epoch << 32 | value bits) with one relaxed store is complete once a
// reader sees the current epoch in it, without a separate flag or fence.
__device__ __forceinline__ void st_relaxed_gpu_b64(uint64_t* p, uint64_t v) {
  asm volatile("st.relaxed.gpu.global.b64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}
__device__ __forceinline__ uint64_t ld_relaxed_gpu_b64(const uint64_t* p) {
  uint64_t v;
  asm volatile("ld.relaxed.gpu.global.b64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ uint64_t epoch_word(uint32_t epoch, float v) {
  return ((uint64_t)epoch << 32) | __float_as_uint(v);
}

// Polls words[0..n) (n <= 128, four per lane, all loads of a pass in
// flight) until every one carries `epoch`; out[i] gets word i's low 32 bits
// (out may be shared memory; written by the lane that loaded the word).
// Warp-uniform.  Gives up, returning false, when *abort_flag is raised or the
// time limit passes (recording device error 1 and raising the flag).
__device__ __forceinline__ bool warp_poll_words(const uint64_t* words, int n, uint32_t epoch, uint32_t* out,
                                                uint32_t* abort_flag, uint32_t* err, uint64_t timeout_ns) {
  const int lane = threadIdx.x & 31;
  uint32_t need = 0;
#pragma unroll
  for (int i = 0; i < 4; ++i)
    if (lane + 32 * i < n) need |= 1u << i;
  uint64_t t0 = 0;
#pragma unroll 1
  for (uint32_t it = 0;; ++it) {
    uint64_t w[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) w[i] = (need >> i & 1u) ? ld_relaxed_gpu_b64(words + lane + 32 * i) : 0ull;
#pragma unroll
    for (int i = 0; i < 4; ++i)
      if ((need >> i & 1u) && (uint32_t)(w[i] >> 32) == epoch) {
        need &= ~(1u << i);
        out[lane + 32 * i] = (uint32_t)w[i];
      }
    if (__all_sync(0xffffffffu, need == 0u)) return true;
    if ((it & 31u) == 31u) {
      int stop = 0;
      if (lane == 0) {
        if (t0 == 0) t0 = globaltimer_ns();
        if (ld_relaxed_gpu(abort_flag) != 0u) {
          stop = 1;
        } else if (globaltimer_ns() - t0 > timeout_ns) {
          atomicCAS(err, 0u, 1u);
          atomicExch(abort_flag, 1u);
          stop = 1;
        }
      }
      if (__shfl_sync(0xffffffffu, stop, 0)) return false;
    }
  }
}

__device__ __forceinline__ void red_release_add(uint32_t* p, uint32_t v) {
  asm volatile("red.release.gpu.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// Fetch-and-add with acquire-release semantics at GPU scope: what this
// thread has observed is visible to whoever later observes the increment,
// and what the earlier increments released is visible to this thread.
__device__ __forceinline__ uint32_t atom_add_acq_rel_gpu(uint32_t* p, uint32_t v) {
  uint32_t old;
  asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
  return old;
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


// Top-K keys as one ordered 64-bit integer: the logit's bits mapped so that
// unsigned order is float order (after -0 -> +0 and NaN -> -inf), above the
// complemented expert index, so a larger key ranks first and equal logits
// rank by lower index.
__device__ __forceinline__ uint64_t topk_key(float v, int e) {
  v = rank_key(v);
  if (v == 0.f) v = 0.f;
  const uint32_t u = __float_as_uint(v);
  const uint32_t o = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
  return ((uint64_t)o << 32) | (uint32_t)~(uint32_t)e;
}
__device__ __forceinline__ float topk_key_value(uint64_t k) {
  const uint32_t o = (uint32_t)(k >> 32);
  return __uint_as_float((o & 0x80000000u) ? (o ^ 0x80000000u) : ~o);
}
__device__ __forceinline__ uint64_t warp_max_u64(uint64_t v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const uint64_t w = __shfl_xor_sync(0xffffffffu, v, o);
    v = w > v ? w : v;
  }
  return v;
}

// w[0..K) holds the chosen logits in rank order; replace them by the weights
// exp(l_k - l_max) / sum_j exp(l_j - l_max) over the K chosen logits (fast
// division: a few ulp).
__device__ __forceinline__ void topk_weights(int K, float* w) {
  const int lane = threadIdx.x & 31;
  __syncwarp();
  const float lmax = w[0];
  float den = 0.f;
#pragma unroll 1
  for (int k = 0; k < K; ++k) den += expf(w[k] - lmax);
  __syncwarp();
#pragma unroll 1
  for (int k = lane; k < K; k += 32) w[k] = __fdividef(expf(w[k] - lmax), den);
  __syncwarp();
}

// vals: [E] logits of one token, read with plain loads (memory written by an
// earlier launch, or staged by this warp).  Writes idx[K] and w[K] (any
// memory space; w holds the chosen logits before it receives the weights).
static __device__ __noinline__ void warp_topk(const float* vals, int E, int K, int32_t* idx, float* w) {
  const int lane = threadIdx.x & 31;
  uint64_t prev = ~0ull;
#pragma unroll 1
  for (int k = 0; k < K; ++k) {
    uint64_t best = 0;
#pragma unroll 4
    for (int e = lane; e < E; e += 32) {
      const uint64_t key = topk_key(vals[e], e);
      if (key < prev && key > best) best = key;
    }
    best = warp_max_u64(best);
    if (lane == 0) {
      idx[k] = (int)~(uint32_t)best;
      w[k] = topk_key_value(best);
    }
    prev = best;
  }
  topk_weights(K, w);
}

// The same for logits written earlier in this launch by other blocks
// (global memory, read through L2), read once with independent loads: for
// E <= 512 the keys stay in registers, otherwise they are staged into `keys`
// (E entries of shared memory) and each of the K rounds scans them.
static __device__ __noinline__ void warp_topk_keys(const float* logits, int E, int K, uint64_t* keys,
                                                   int32_t* idx, float* w) {
  const int lane = threadIdx.x & 31;
  if (E <= 512) {
    // Up to 16 keys per lane stay in registers.  Every real key is nonzero
    // (its high word is at least the order bits of -inf), so 0 means "none".
    // Each lane holds the best of its keys not yet taken; a round takes the
    // warp maximum (high words first, then the low words among the lanes
    // that hold that high word) and only the lane that held it rescans.
    // all 16 loads are issued before the first use (clamped, unconditional)
    float v[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = __ldcg(logits + min(lane + 32 * i, E - 1));
    // 32-bit ordered logits (the high word of topk_key; 0 for no expert);
    // each round: the largest not-yet-taken value (a tree over the lane's
    // 16, then a warp maximum), then among the lanes holding it the lowest
    // expert index (a warp minimum); the owner marks it taken.  No 64-bit
    // compares, no divergent rescan: a short dependent chain per round.
    uint32_t u[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const int e = lane + 32 * i;
      u[i] = e < E ? (uint32_t)(topk_key(v[i], e) >> 32) : 0u;
    }
    uint32_t taken = 0;
#pragma unroll 1
    for (int k = 0; k < K; ++k) {
      uint32_t m[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) m[i] = (taken >> i & 1u) ? 0u : u[i];
#pragma unroll
      for (int s2 = 8; s2 > 0; s2 >>= 1)
#pragma unroll
        for (int i = 0; i < s2; ++i) m[i] = max(m[i], m[i + s2]);
      const uint32_t hmax = __reduce_max_sync(0xffffffffu, m[0]);
      uint32_t eq = 0;
#pragma unroll
      for (int i = 0; i < 16; ++i) eq |= (uint32_t)(u[i] == hmax && !(taken >> i & 1u)) << i;
      const uint32_t mine = eq ? (uint32_t)(lane + 32 * (__ffs(eq) - 1)) : 0xffffffffu;
      const uint32_t best = __reduce_min_sync(0xffffffffu, mine);
      if ((int)(best & 31u) == lane) taken |= 1u << (best >> 5);
      if (lane == 0) {
        idx[k] = (int)best;
        w[k] = topk_key_value((uint64_t)hmax << 32);
      }
    }
  } else {
    // 16 independent loads per lane in flight per 512 logits, staged in
    // shared memory; each of the K rounds scans them
#pragma unroll 1
    for (int e0 = 0; e0 < E; e0 += 512) {
      float v[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const int e = e0 + lane + 32 * i;
        v[i] = e < E ? __ldcg(logits + e) : 0.f;
      }
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const int e = e0 + lane + 32 * i;
        if (e < E) keys[e] = topk_key(v[i], e);
      }
    }
    __syncwarp();
    uint64_t prev = ~0ull;
#pragma unroll 1
    for (int k = 0; k < K; ++k) {
      uint64_t best = 0;
#pragma unroll 4
      for (int e = lane; e < E; e += 32) {
        const uint64_t key = keys[e];
        best = (key < prev && key > best) ? key : best;
      }
      best = warp_max_u64(best);
      if (lane == 0) {
        idx[k] = (int)~(uint32_t)best;
        w[k] = topk_key_value(best);
      }
      prev = best;
    }
  }
  topk_weights(K, w);
}

// The same for logits that other blocks of this launch publish as epoch
// words (epoch_word): every lane polls its words (one load each, all in
// flight) until each carries `epoch`, then the K rounds run as above.
// epoch == 0 accepts any word (a dry run over whatever the buffer holds).
// Gives up, returning false, when *abort_flag is raised or the time limit
// passes (recording MOE device error 1 and raising the flag).  E <= 512:
// keys in registers; larger E: staged in `keys` (E entries of shared memory).
static __device__ __noinline__ bool warp_topk_poll(const uint64_t* words, uint32_t epoch, int E, int K,
                                                   uint64_t* keys, int32_t* idx, float* w, uint32_t* abort_flag,
                                                   uint32_t* err, uint64_t timeout_ns, uint32_t* polls,
                                                   uint64_t* tr = nullptr) {
  const int lane = threadIdx.x & 31;
  uint64_t t0 = 0;
  uint32_t nit = 0;
  bool ok = true;
  // poll words [e0, e0 + 512) into v[]: lane's i-th word is e0 + lane + 32 i
  // (tr, traced launches: start time of the last pass and the number of passes)
  auto poll = [&](int e0, float (&v)[16]) -> bool {
    uint32_t need = 0, have = 0;
#pragma unroll
    for (int i = 0; i < 16; ++i)
      if (e0 + lane + 32 * i < E) need |= 1u << i;
    for (uint32_t it = 0;; ++it) {
      if (tr && lane == 0) {
        const uint64_t now = globaltimer_ns();
        tr[0] = now;
        if (it < 8) tr[15 + it] = now;  // start of each of the first 8 passes
      }
      uint64_t wv[16];
#pragma unroll
      for (int i = 0; i < 16; ++i)
        wv[i] = ((need & ~have) >> i & 1u) ? ld_relaxed_gpu_b64(words + e0 + lane + 32 * i) : 0ull;
#pragma unroll
      for (int i = 0; i < 16; ++i)
        if (((need & ~have) >> i & 1u) && (epoch == 0u || (uint32_t)(wv[i] >> 32) == epoch)) {
          have |= 1u << i;
          v[i] = __uint_as_float((uint32_t)wv[i]);
        }
      ++nit;
      if (tr && lane == 0) tr[23] = globaltimer_after(wv[0] + wv[15]);  // this pass's loads returned
      if (__all_sync(0xffffffffu, have == need)) {
        if (tr && lane == 0) tr[1] = globaltimer_ns();  // every word present: the top-K starts
        return true;
      }
      if ((it & 31u) == 31u) {
        int stop = 0;
        if (lane == 0) {
          if (t0 == 0) t0 = globaltimer_ns();
          if (ld_relaxed_gpu(abort_flag) != 0u) {
            stop = 1;
          } else if (globaltimer_ns() - t0 > timeout_ns) {
            atomicCAS(err, 0u, 1u);
            atomicExch(abort_flag, 1u);
            stop = 1;
          }
        }
        if (__shfl_sync(0xffffffffu, stop, 0)) return false;
      }
    }
  };
  if (E <= 512) {
    float v[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = 0.f;
    ok = poll(0, v);
    if (polls && lane == 0) atomicAdd(polls, nit);
    if (!ok) return false;
    uint64_t kr[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const int e = lane + 32 * i;
      kr[i] = e < E ? topk_key(v[i], e) : 0ull;
    }
    uint64_t mine = 0;
#pragma unroll
    for (int i = 0; i < 16; ++i) mine = kr[i] > mine ? kr[i] : mine;
#pragma unroll 1
    for (int k = 0; k < K; ++k) {
      const uint32_t hi = (uint32_t)(mine >> 32);
      const uint32_t hmax = __reduce_max_sync(0xffffffffu, hi);
      const uint32_t lmax = __reduce_max_sync(0xffffffffu, hi == hmax ? (uint32_t)mine : 0u);
      const uint64_t best = ((uint64_t)hmax << 32) | lmax;
      if (lane == 0) {
        idx[k] = (int)~lmax;
        w[k] = topk_key_value(best);
      }
      if (mine == best) {
        uint64_t m = 0;
#pragma unroll
        for (int i = 0; i < 16; ++i) m = (kr[i] < best && kr[i] > m) ? kr[i] : m;
        mine = m;
      }
    }
  } else {
#pragma unroll 1
    for (int e0 = 0; e0 < E && ok; e0 += 512) {
      float v[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) v[i] = 0.f;
      ok = poll(e0, v);
      if (ok) {
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const int e = e0 + lane + 32 * i;
          if (e < E) keys[e] = topk_key(v[i], e);
        }
      }
    }
    if (polls && lane == 0) atomicAdd(polls, nit);
    if (!ok) return false;
    __syncwarp();
    uint64_t prev = ~0ull;
#pragma unroll 1
    for (int k = 0; k < K; ++k) {
      uint64_t best = 0;
#pragma unroll 4
      for (int e = lane; e < E; e += 32) {
        const uint64_t key = keys[e];
        best = (key < prev && key > best) ? key : best;
      }
      best = warp_max_u64(best);
      if (lane == 0) {
        idx[k] = (int)~(uint32_t)best;
        w[k] = topk_key_value(best);
      }
      prev = best;
    }
  }
  topk_weights(K, w);
  return true;
}

// SiLU(g) * u with a fast division (relative error of a few ulp).
__device__ __forceinline__ float silu_mul(float g, float u) { return __fdividef(g, 1.f + expf(-g)) * u; }

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

// Bounded wait for phase `parity` of an mbarrier; false on timeout.  If
// `spins` is not null, the number of polls is added to it (shared memory).
static __device__ __noinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, uint64_t timeout_ns,
                                              uint32_t* spins = nullptr) {
  bool ok = true;
  uint32_t it = 0;
  if (!mbar_try_wait(bar, parity)) {
    const uint64_t t0 = globaltimer_ns();
    for (;; ++it) {
      // the hardware may suspend the waiting thread (up to 1 us) until the
      // phase completes: waiting warps then issue almost nothing and leave
      // the load/store pipe to the warps that work
      if (mbar_try_wait_sleep(bar, parity, 1000u)) break;
      if ((it & 15u) == 15u && globaltimer_ns() - t0 > timeout_ns) {
        ok = false;
        break;
      }
    }
  }
  if (spins) atomicAdd(spins, it + 1);
  return ok;
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
