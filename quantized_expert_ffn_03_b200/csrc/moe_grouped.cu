// moe_grouped.cu -- the batched layer (many tokens per call): the same MoE
// layer as the fused decode kernel, organised as grouped GEMMs on the
// tcgen05 tensor cores once several tokens share an expert.
//
// The pages run one token at a time ("Flash-MoE: ラップトップでの397Bパラメー
// タモデルの実行", section "パイプライン概要"); for a batch, the router's
// choices group the (token, expert) pairs by expert, so that each chosen
// expert's packed weights are read once per 128 of its tokens and multiplied
// as a matrix:
//   1. x -> fp16 copy (the routed experts' B operand);
//   2. router logits = x . Wr^T + bias (bf16 GEMM), top-K and weights;
//   3. grouping: the T*K pairs sorted by expert into slots, chunks of up to
//      128 slots of one expert;
//   4. routed gate/up GEMM per chunk and 128-row tile of I: the weights are
//      dequantised (w = q*scale + bias, "Streaming experts: как запустить
//      триллионную модель на MacBook", section "Оптимизации, которые
//      сработали") into fp16 tiles, the chunk's tokens' x rows are the other
//      operand, fp32 accumulators in tensor memory; SiLU(gate)*up -> fp16;
//   5. routed down GEMM per chunk and 128-row tile of H -> fp32 per slot;
//   6. shared expert gate/up and down (bf16 GEMMs; the intermediate enters
//      the down GEMM as bf16 hi + lo parts);
//   7. combine + residual + RMSNorm per token.
//
// One GEMM kernel serves steps 2 and 4-6: a persistent CTA per SM walks
// tiles of 128 output rows x up to 128 columns (tokens or slots).  Four
// producer warps stage the operands into shared memory (cp.async copies;
// packed weights are dequantised by the threads, one weight row per thread),
// one thread issues the tcgen05.mma instructions, and the producer warps
// read the accumulators back from tensor memory for the epilogue.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "moe_device.cuh"
#include "moe_grouped.h"
#include "moe_kernels.h"
#include "moe_tc.cuh"

namespace moe {

namespace {

// 4 owner warps (producers and epilogue), the MMA warp (warp 4), 4 helper
// warps (producers only): each of the tile's 128 rows has an owner thread
// and a helper thread, which split its copies and dequantisation (the
// dequantisation of the codes, not the MMA or the bytes, sets the time of
// the packed GEMMs at a few tokens per expert)
constexpr int kGThreads = 288;
constexpr int kProducers = 256;
constexpr int kMmaWarp = 4;
constexpr int kTileM = 128;      // output rows per tile (the MMA's M)
constexpr int kTileN = 128;      // columns (tokens / slots) per tile at most
constexpr int kKB = 64;          // reduction columns per k-block (one quantisation group)
constexpr int kTmemCols = 256;   // two accumulators of kTileN columns
constexpr uint32_t kATile = kTileM * 128;  // bytes of one 128 x 64 16-bit tile
constexpr uint32_t kBTile = kTileN * 128;

// Shared-memory plan of the GEMM kernel: SA operand stages (NA A tiles and a
// B tile each), SC code stages of packed weights (NA x 128 rows x (32 code
// bytes + 4 scale bytes)), mbarriers.
struct GemmSmem {
  int SA, SC, LB, LC;
  uint32_t stage, a0, b0, code0, code_stage, bars, total;
};

__host__ __device__ inline GemmSmem gemm_smem(int na, bool packed) {
  GemmSmem s;
  s.SA = packed ? 3 : 4;
  s.SC = packed ? 8 : 0;
  s.LB = s.SA - 1;
  s.LC = packed ? s.SC - 1 : s.LB;
  s.stage = na * kATile + kBTile;
  s.a0 = 0;
  s.b0 = na * kATile;
  s.code0 = s.SA * s.stage;
  s.code_stage = packed ? na * kTileM * 36u : 0u;
  s.bars = s.code0 + s.SC * s.code_stage;
  s.bars = (s.bars + 15u) & ~15u;
  s.total = s.bars + 8u * (2 * s.SA + 2) + 16u;
  return s;
}

__device__ __forceinline__ uint32_t smem_addr(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }

__device__ __forceinline__ void bar_init(uint32_t a, uint32_t n) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(a), "r"(n) : "memory");
}
__device__ __forceinline__ void bar_arrive(uint32_t a) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(a) : "memory");
}
__device__ __forceinline__ bool bar_try(uint32_t a, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}"
      : "=r"(ok)
      : "r"(a), "r"(parity)
      : "memory");
  return ok != 0;
}

}  // namespace

namespace {

// Bounded wait on an mbarrier phase by every lane of the calling warp (or a
// single thread); false when the launch was aborted or the wait timed out
// (then the error word and the abort flag are set).
__device__ bool gwait(uint32_t bar, uint32_t parity, const GemmParams& p, uint64_t& t0) {
  if (bar_try(bar, parity)) return true;
  if (t0 == 0) t0 = globaltimer_ns();
  for (uint32_t it = 0;; ++it) {
    if (bar_try(bar, parity)) return true;
    if ((it & 255u) == 255u) {
      if (ld_relaxed_gpu(p.abort_flag) != 0u) return false;
      if (globaltimer_ns() - t0 > p.timeout_ns) {
        atomicCAS(p.err, 0u, 1u);
        atomicExch(p.abort_flag, 1u);
        return false;
      }
    }
  }
}

// fp16 pair (lo, hi) -> packed 32 bits
__device__ __forceinline__ uint32_t h2u(__half2 h) { return *reinterpret_cast<uint32_t*>(&h); }
__device__ __forceinline__ __half2 u2h(uint32_t u) { return *reinterpret_cast<__half2*>(&u); }

// Dequantise one 64-weight row segment (this thread's row of the tile) into
// the swizzled fp16 A tile.  codes: the row's 32 (4-bit) or 16 (2-bit) code
// bytes in the packed lane order (lane slot t = 0..3 of the row's 8-row
// block); sw: its scale word.  w = q*scale + bias is formed by one fp16 fma
// of exact operands, i.e. the exact weight rounded once to fp16.
template <int BITS>
__device__ __forceinline__ void dequant_row(uint32_t code_saddr, uint32_t sw, uint32_t a_row_saddr, uint32_t row) {
  const float sf = __uint_as_float(sw << 16), bf = __uint_as_float(sw & 0xffff0000u);
  const __half2 s2 = __float2half2_rn(sf), b2 = __float2half2_rn(bf);
  const __half2 k1024 = __float2half2_rn(1024.f);
  uint32_t w[8];
  if constexpr (BITS == 4) {
    uint4 v0, v1;
    asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(v0.x), "=r"(v0.y), "=r"(v0.z), "=r"(v0.w) : "r"(code_saddr));
    asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(v1.x), "=r"(v1.y), "=r"(v1.z), "=r"(v1.w) : "r"(code_saddr + 16));
    // lane slot t: words 2t (steps 0, 1) and 2t + 1 (steps 2, 3)
    w[0] = v0.x, w[1] = v0.y, w[2] = v0.z, w[3] = v0.w, w[4] = v1.x, w[5] = v1.y, w[6] = v1.z, w[7] = v1.w;
  } else {
    uint4 v0;
    asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(v0.x), "=r"(v0.y), "=r"(v0.z), "=r"(v0.w) : "r"(code_saddr));
    w[0] = v0.x, w[1] = v0.y, w[2] = v0.z, w[3] = v0.w;
  }
#pragma unroll
  for (int c = 0; c < 8; ++c) {  // 16-byte chunk c = columns 8c .. 8c + 7
    const int s = c >> 1, half = c & 1;
    uint32_t out[4];
#pragma unroll
    for (int t = 0; t < 4; ++t) {  // columns 16s + 8half + 2t, +1
      uint32_t q2;
      if constexpr (BITS == 4)
        q2 = (w[2 * t + (s >> 1)] >> (4 * (2 * (s & 1) + half))) & 0x000F000Fu;
      else
        q2 = (w[t] >> (4 * s + 2 * half)) & 0x00030003u;
      const __half2 q = __hsub2(u2h(q2 | 0x64006400u), k1024);
      out[t] = h2u(__hfma2(q, s2, b2));
    }
    const uint32_t dst = a_row_saddr + (uint32_t)(((c ^ (row & 7u)) << 4));
    asm volatile("st.shared.v4.u32 [%0], {%1,%2,%3,%4};" ::"r"(dst), "r"(out[0]), "r"(out[1]), "r"(out[2]),
                 "r"(out[3])
                 : "memory");
  }
}

// SwiGLU with a fast division (a few ulp)
__device__ __forceinline__ float silu_mul_f(float g, float u) { return __fdividef(g, 1.f + __expf(-g)) * u; }

}  // namespace

// AK: 0 dense bf16 A, 4 / 2 packed A of that many bits.  NA: A matrices (2 =
// gate and up, each with its own accumulator).  EPI: 0 fp32 store (+ bias),
// 1 SwiGLU -> fp16, 2 SwiGLU -> bf16 hi and lo.
template <int AK, int NA, int EPI>
__global__ void __launch_bounds__(kGThreads, 1) grouped_gemm_kernel(const GemmParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // the swizzled tiles need 1024-byte alignment
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  constexpr bool kPacked = AK != 0;
  const GemmSmem L = gemm_smem(NA, kPacked);
  const uint32_t sbase = smem_addr(smem);
  const uint32_t full0 = sbase + L.bars, empty0 = full0 + 8u * L.SA, accfull = empty0 + 8u * L.SA;
  const uint32_t fin = accfull + 8u;
  volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(smem + L.bars + 8u * (2 * L.SA + 2));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  if (tid == 0) {
    for (int s = 0; s < L.SA; ++s) {
      bar_init(full0 + 8u * s, kProducers);
      bar_init(empty0 + 8u * s, 1);
    }
    bar_init(accfull, 1);
    bar_init(fin, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == kMmaWarp) {
    tc::tmem_alloc(smem_addr((const void*)tmem_slot), kTmemCols);
    tc::tmem_relinquish();
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = *tmem_slot;

  const int MT = (p.M + kTileM - 1) / kTileM;
  const int KB1 = p.K / kKB;
  const int KB = p.b2 ? 2 * KB1 : KB1;
  const int nchunks = p.ch_e ? *p.n_chunks_dev : (p.n_cols + kTileN - 1) / kTileN;
  const int ntiles = nchunks * MT;
  const int G = p.K / 64;
  uint64_t t0 = 0;
  bool ok = true;
  uint32_t kb_global = 0;  // k-blocks consumed by this CTA so far (stage / phase counter)
  uint32_t tile_iter = 0;

  if (warp != kMmaWarp) {
    // ================= producers (and, for the owners, the epilogue) =================
    // this thread's A row (and, for an owner, its TMEM lane: warp w reaches
    // lanes 32 (w % 4) ..); half 0 = owner, 1 = helper.  With two A
    // matrices half h copies and dequantises matrix h; with one, the
    // k-blocks g (counted over the CTA's tiles, which also picks their code
    // slot, an even number of them) of parity h, so a helper that runs
    // ahead into the next tile never writes a slot its owner still reads.
    // Each half copies half of every k-block's B rows.
    const uint32_t row = 32u * (uint32_t)(warp & 3) + (uint32_t)lane;
    const int half = warp > kMmaWarp ? 1 : 0;
    auto mine = [&](int a, uint32_t g) { return NA == 2 ? a == half : (int)(g & 1u) == half; };
#pragma unroll 1
    for (int tile = blockIdx.x; tile < ntiles && ok; tile += gridDim.x, ++tile_iter) {
      const int chunk = tile / MT, mt = tile - chunk * MT;
      const int m0 = mt * kTileM;
      int e = 0, c0, n;
      if (p.ch_e) {
        e = p.ch_e[chunk];
        c0 = p.ch_c0[chunk];
        n = p.ch_n[chunk];
      } else {
        c0 = chunk * kTileN;
        n = min(kTileN, p.n_cols - c0);
      }
      const bool row_ok = m0 + (int)row < p.M;
      const uint8_t* blob = kPacked ? static_cast<const uint8_t*>(p.expert_ptr[e]) : nullptr;
      // this thread's B rows: chunk id = row + 128 q -> tile row 16 q + row / 8, chunk row % 8
      const int bc = (int)(row & 7u);
      int brow_src[kTileN / 32];  // the B rows of this half: q = half * kTileN / 32 + qq
#pragma unroll
      for (int qq = 0; qq < kTileN / 32; ++qq) {
        const int r = 16 * (half * (kTileN / 32) + qq) + (int)(row >> 3);
        brow_src[qq] = r < n ? (p.b_rows ? p.b_rows[c0 + r] : c0 + r) : -1;
      }
      const uint32_t gbase = kb_global;
      // issue the copies of k-block kb (B and dense A) into its stage
      auto issue_ab = [&](int kb) {
        const uint32_t g = gbase + (uint32_t)kb;
        const uint32_t s = g % (uint32_t)L.SA;
        if (g >= (uint32_t)L.SA && ok) ok = gwait(empty0 + 8u * s, ((g / L.SA) & 1u) ^ 1u, p, t0);
        const uint32_t st = sbase + s * L.stage;
        const int kbb = kb % KB1;
        const uint16_t* bsrc = (kb >= KB1) ? p.b2 : p.b;
#pragma unroll
        for (int qq = 0; qq < kTileN / 32; ++qq) {
          const int q = half * (kTileN / 32) + qq;
          const int r = 16 * q + (int)(row >> 3);
          const uint32_t dst = st + L.b0 + tc::sw128((uint32_t)r, (uint32_t)bc);
          const int src_row = brow_src[qq];
          const uint16_t* src = bsrc + (size_t)(src_row < 0 ? 0 : src_row) * p.K + kbb * kKB + 8 * bc;
          tc::cp16(dst, src, src_row < 0 ? 0u : 16u);
        }
        if constexpr (!kPacked) {
#pragma unroll
          for (int a = 0; a < NA; ++a) {
            if (!mine(a, gbase + (uint32_t)kb)) continue;
            const uint16_t* arow = p.a_dense[a] + (size_t)(row_ok ? m0 + (int)row : 0) * p.K + kbb * kKB;
#pragma unroll
            for (int c = 0; c < 8; ++c)
              tc::cp16(st + L.a0 + a * kATile + tc::sw128(row, (uint32_t)c), arow + 8 * c, row_ok ? 16u : 0u);
          }
        }
      };
      // packed A: the row's codes and scale word of k-block kb into code stage
      auto issue_codes = [&](int kb) {
        if constexpr (kPacked) {
          const uint32_t cs = sbase + L.code0 + ((gbase + (uint32_t)kb) % (uint32_t)L.SC) * L.code_stage;
          if (row_ok) {
            const int grow = m0 + (int)row;
            const size_t blk = (size_t)(grow >> 3) * G + (kb % KB1);
            const int CB = AK == 4 ? 32 : 16;  // code bytes of one row in one group
#pragma unroll
            for (int a = 0; a < NA; ++a) {
              if (!mine(a, gbase + (uint32_t)kb)) continue;
              const uint8_t* cp = blob + p.off_codes[a] + blk * (size_t)(8 * CB) + (size_t)(grow & 7) * CB;
              const uint32_t dst = cs + (uint32_t)a * kTileM * 36u + row * 32u;
              tc::cp16(dst, cp, 16u);
              if (CB == 32) tc::cp16(dst + 16u, cp + 16, 16u);
              tc::cp4(cs + (uint32_t)a * kTileM * 36u + kTileM * 32u + row * 4u,
                      blob + p.off_scales[a] + (blk * 8 + (grow & 7)) * 4);
            }
          }
        }
      };
      // prologue: group u holds codes(u) (u < LC) and B / dense A of k-block u (u < LB)
#pragma unroll 1
      for (int u = 0; u < L.LC; ++u) {
        if (u < KB) issue_codes(u);
        if (u < L.LB && u < KB) issue_ab(u);
        tc::cp_commit();
      }
#pragma unroll 1
      for (int kb = 0; kb < KB && ok; ++kb) {
        if (kb + L.LC < KB) issue_codes(kb + L.LC);
        if (kb + L.LB < KB) issue_ab(kb + L.LB);
        tc::cp_commit();
        // groups up to (LC + kb - LB) are complete: codes(kb), B(kb), A(kb)
        if constexpr (kPacked)
          tc::cp_wait<2>();
        else
          tc::cp_wait<3>();
        const uint32_t g = gbase + (uint32_t)kb;
        const uint32_t s = g % (uint32_t)L.SA;
        const uint32_t st = sbase + s * L.stage;
        if constexpr (kPacked) {
          const uint32_t cs = sbase + L.code0 + (g % (uint32_t)L.SC) * L.code_stage;
#pragma unroll
          for (int a = 0; a < NA; ++a) {
            if (!mine(a, gbase + (uint32_t)kb)) continue;
            const uint32_t arow = st + L.a0 + a * kATile + row * 128u;
            if (row_ok) {
              uint32_t sw;
              asm volatile("ld.shared.u32 %0, [%1];" : "=r"(sw) : "r"(cs + (uint32_t)a * kTileM * 36u + kTileM * 32u + row * 4u));
              dequant_row<AK>(cs + (uint32_t)a * kTileM * 36u + row * 32u, sw, arow, row);
            } else {
#pragma unroll
              for (int c = 0; c < 8; ++c)
                asm volatile("st.shared.v4.u32 [%0], {%1,%1,%1,%1};" ::"r"(arow + (uint32_t)(c << 4)), "r"(0u)
                             : "memory");
            }
          }
        }
        tc::fence_proxy_async_smem();
        bar_arrive(full0 + 8u * s);
      }
      tc::cp_wait<0>();
      kb_global += (uint32_t)KB;
      if (!ok) break;
      if (half) continue;  // helpers: on to the next tile's copies
      // ---- epilogue: wait for the tile's accumulators ----
      ok = gwait(accfull, tile_iter & 1u, p, t0);
      if (!ok) break;
      tc::fence_after_sync();
      const uint32_t lane_base = tmem + ((uint32_t)(warp * 32) << 16);
      const int feat = m0 + (int)row;
#pragma unroll 1
      for (int j = 0; j < (n + 15) / 16; ++j) {
        uint32_t v0[16], v1[16];
        tc::ld_32x32b_x16(lane_base + (uint32_t)(16 * j), v0);
        if constexpr (NA == 2) tc::ld_32x32b_x16(lane_base + (uint32_t)(kTileN + 16 * j), v1);
        tc::wait_ld();
        if (feat < p.M) {
#pragma unroll
          for (int q = 0; q < 16; ++q) {
            const int c = 16 * j + q;
            if (c < n) {
              const size_t o = (size_t)(c0 + c) * p.M + feat;
              if constexpr (EPI == 0) {
                float v = __uint_as_float(v0[q]);
                if (p.bias) v += p.bias[feat];
                static_cast<float*>(p.out)[o] = v;
              } else {
                const float h = silu_mul_f(__uint_as_float(v0[q]), __uint_as_float(v1[q]));
                if constexpr (EPI == 1) {
                  static_cast<__half*>(p.out)[o] = __float2half_rn(h);
                } else {
                  const __nv_bfloat16 hi = __float2bfloat16_rn(h);
                  static_cast<__nv_bfloat16*>(p.out)[o] = hi;
                  static_cast<__nv_bfloat16*>(p.out2)[o] = __float2bfloat16_rn(h - __bfloat162float(hi));
                }
              }
            }
          }
        }
      }
      tc::fence_before_sync();
    }
  } else if (lane == 0) {
    // ================= MMA issuer (one thread) =================
#pragma unroll 1
    for (int tile = blockIdx.x; tile < ntiles && ok; tile += gridDim.x, ++tile_iter) {
      const int chunk = tile / MT;
      const int n = p.ch_e ? p.ch_n[chunk] : min(kTileN, p.n_cols - chunk * kTileN);
      const int N = (n + 15) & ~15;
      const uint32_t idesc = tc::idesc_f16(kTileM, N, AK == 0);
#pragma unroll 1
      for (int kb = 0; kb < KB && ok; ++kb) {
        const uint32_t g = kb_global + (uint32_t)kb;
        const uint32_t s = g % (uint32_t)L.SA;
        ok = gwait(full0 + 8u * s, (g / L.SA) & 1u, p, t0);
        if (!ok) break;
        tc::fence_after_sync();
        const uint32_t st = sbase + s * L.stage;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const uint64_t bd = tc::smem_desc_sw128(st + L.b0 + 32u * k);
#pragma unroll
          for (int a = 0; a < NA; ++a) {
            const uint64_t ad = tc::smem_desc_sw128(st + L.a0 + a * kATile + 32u * k);
            tc::mma_f16_ss(tmem + (uint32_t)(a * kTileN), ad, bd, idesc, (kb > 0 || k > 0) ? 1u : 0u);
          }
        }
        tc::commit(empty0 + 8u * s);  // the stage is free once these MMAs are done
      }
      kb_global += (uint32_t)KB;
      if (ok) tc::commit(accfull);
    }
    // every MMA issued has completed before the accumulators are released
    tc::commit(fin);
    uint64_t tf = 0;
    gwait(fin, 0, p, tf);
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  if (warp == kMmaWarp) {
    __syncwarp();
    tc::tmem_dealloc(tmem, kTmemCols);
  }
}

size_t grouped_gemm_smem_bytes(int na, bool packed) { return gemm_smem(na, packed).total + 1024; }

template <int AK, int NA, int EPI>
static cudaError_t launch_gemm_t(const GemmParams& p, int grid, cudaStream_t st) {
  const size_t smem = grouped_gemm_smem_bytes(NA, AK != 0);
  static int set_dev[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && !set_dev[dev]) {
    cudaError_t e = cudaFuncSetAttribute(grouped_gemm_kernel<AK, NA, EPI>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    set_dev[dev] = 1;
  }
  grouped_gemm_kernel<AK, NA, EPI><<<grid, kGThreads, smem, st>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_grouped_gemm(int ak, int na, int epi, const GemmParams& p, int grid, cudaStream_t st) {
  if (ak == 4 && na == 2 && epi == 1) return launch_gemm_t<4, 2, 1>(p, grid, st);
  if (ak == 2 && na == 2 && epi == 1) return launch_gemm_t<2, 2, 1>(p, grid, st);
  if (ak == 4 && na == 1 && epi == 0) return launch_gemm_t<4, 1, 0>(p, grid, st);
  if (ak == 2 && na == 1 && epi == 0) return launch_gemm_t<2, 1, 0>(p, grid, st);
  if (ak == 0 && na == 2 && epi == 2) return launch_gemm_t<0, 2, 2>(p, grid, st);
  if (ak == 0 && na == 1 && epi == 0) return launch_gemm_t<0, 1, 0>(p, grid, st);
  return cudaErrorInvalidValue;
}

// ---- small kernels of the batched path ------------------------------------------------

// x (bf16) -> fp16, 8 values per thread.
// It also clears the launch sequence's abort flag (stream-ordered before the
// GEMMs of the call).
__global__ void to_half_kernel(const uint16_t* __restrict__ x, __half* __restrict__ xh, size_t n8,
                               uint32_t* abort_flag) {
  if (blockIdx.x == 0 && threadIdx.x == 0) *abort_flag = 0u;
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n8; i += (size_t)gridDim.x * blockDim.x) {
    const uint4 v = reinterpret_cast<const uint4*>(x)[i];
    float f[8];
    unpack_bf16x8(v, f);
    uint4 o;
    o.x = h2u(__floats2half2_rn(f[0], f[1]));
    o.y = h2u(__floats2half2_rn(f[2], f[3]));
    o.z = h2u(__floats2half2_rn(f[4], f[5]));
    o.w = h2u(__floats2half2_rn(f[6], f[7]));
    reinterpret_cast<uint4*>(xh)[i] = o;
  }
}

// The T*K (token, expert) pairs sorted by expert: per expert its count and
// first slot, per slot its token, per pair its slot, and the chunk list
// (expert, first slot, count <= 128).  One block; counts and offsets in
// shared memory (E <= 2048).  Slots of one expert follow the order in which
// the pairs claim them; each slot's results do not depend on that order.
__global__ void __launch_bounds__(1024) group_kernel(const int32_t* __restrict__ idx, int TK, int E,
                                                     int* __restrict__ slot_token, int* __restrict__ pair_slot,
                                                     int K, int* __restrict__ ch_e, int* __restrict__ ch_c0,
                                                     int* __restrict__ ch_n, int* __restrict__ n_chunks,
                                                     const void* const* __restrict__ expert_ptr,
                                                     uint32_t* __restrict__ err) {
  __shared__ int cnt[2048], off[2048], fill[2048], choff[2048];
  __shared__ int wsum[32], wsum2[32];
  const int tid = threadIdx.x;
  for (int e = tid; e < E; e += blockDim.x) cnt[e] = 0, fill[e] = 0;
  __syncthreads();
  for (int q = tid; q < TK; q += blockDim.x) {
    const int e = idx[q];
    if (e >= 0 && e < E)
      atomicAdd(&cnt[e], 1);
    else
      atomicCAS(err, 0u, 2u);
  }
  __syncthreads();
  // every chosen expert's blob must be a non-null, 256-byte aligned pointer
  // (checked before any GEMM reads it; a bad one is MOE device error 2 and
  // the layer's GEMMs then get no chunks)
  __shared__ int bad;
  if (tid == 0) bad = 0;
  __syncthreads();
  for (int e = tid; e < E; e += blockDim.x) {
    if (cnt[e] == 0) continue;
    const uintptr_t a = reinterpret_cast<uintptr_t>(expert_ptr[e]);
    if (a == 0 || (a & 255u)) {
      atomicCAS(err, 0u, 2u);
      bad = 1;
    }
  }
  __syncthreads();
  // exclusive scans of the counts and of the chunk counts: each thread owns a
  // run of experts, warp scans combine the runs
  const int per = (E + blockDim.x - 1) / blockDim.x;
  const int e0 = tid * per, e1 = min(E, e0 + per);
  int s = 0, sc = 0;
  for (int e = e0; e < e1; ++e) s += cnt[e], sc += (cnt[e] + kTileN - 1) / kTileN;
  int incl = s, inclc = sc;
  const int lane = tid & 31, w = tid >> 5;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int a = __shfl_up_sync(0xffffffffu, incl, o), b = __shfl_up_sync(0xffffffffu, inclc, o);
    if (lane >= o) incl += a, inclc += b;
  }
  if (lane == 31) wsum[w] = incl, wsum2[w] = inclc;
  __syncthreads();
  if (w == 0) {
    int v = lane < (int)(blockDim.x >> 5) ? wsum[lane] : 0, v2 = lane < (int)(blockDim.x >> 5) ? wsum2[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int a = __shfl_up_sync(0xffffffffu, v, o), b = __shfl_up_sync(0xffffffffu, v2, o);
      if (lane >= o) v += a, v2 += b;
    }
    wsum[lane] = v;
    wsum2[lane] = v2;
  }
  __syncthreads();
  int run = incl - s + (w > 0 ? wsum[w - 1] : 0), runc = inclc - sc + (w > 0 ? wsum2[w - 1] : 0);
  for (int e = e0; e < e1; ++e) {
    off[e] = run;
    choff[e] = runc;
    run += cnt[e];
    runc += (cnt[e] + kTileN - 1) / kTileN;
  }
  __syncthreads();
  for (int q = tid; q < TK; q += blockDim.x) {
    const int e = idx[q];
    if (e < 0 || e >= E) continue;
    const int sl = off[e] + atomicAdd(&fill[e], 1);
    slot_token[sl] = q / K;
    pair_slot[q] = sl;
  }
  for (int e = tid; e < E; e += blockDim.x) {
    const int c = cnt[e];
    for (int j = 0; j * kTileN < c; ++j) {
      ch_e[choff[e] + j] = e;
      ch_c0[choff[e] + j] = off[e] + j * kTileN;
      ch_n[choff[e] + j] = min(kTileN, c - j * kTileN);
    }
  }
  if (tid == blockDim.x - 1) *n_chunks = bad ? 0 : runc;
}

// Combine + residual + RMSNorm, one block per token:
//   h = residual + sum_k w[t][k] * Y[slot(t, k)] + Ys[t];  y = h / sqrt(mean(h^2) + eps) * gamma.
// The second pass recomputes h in the same order (its inputs are in L2).
__device__ __forceinline__ float combine_h(const float* __restrict__ Y, const float* __restrict__ Ys,
                                           const int* __restrict__ pair_slot, const float* __restrict__ w,
                                           const uint16_t* __restrict__ res, int t, int c, int H, int K,
                                           float sg) {
  float h = __uint_as_float((uint32_t)res[(size_t)t * H + c] << 16);
  float acc = 0.f;
  for (int k = 0; k < K; ++k) acc = fmaf(w[t * K + k], Y[(size_t)pair_slot[t * K + k] * H + c], acc);
  h += acc;
  if (Ys) h += sg * Ys[(size_t)t * H + c];
  return h;
}

__global__ void __launch_bounds__(256) combine_kernel(const float* __restrict__ Y, const float* __restrict__ Ys,
                                                      const int* __restrict__ pair_slot, const float* __restrict__ w,
                                                      const uint16_t* __restrict__ res,
                                                      const uint16_t* __restrict__ gamma, int H, int K, float eps,
                                                      const uint16_t* __restrict__ x,
                                                      const uint16_t* __restrict__ sgate,
                                                      uint16_t* __restrict__ h_out, uint16_t* __restrict__ y_norm) {
  const int t = blockIdx.x;
  __shared__ float red[8];
  __shared__ float inv_s, sg_s;
  // the shared output gate sigmoid(x . g) of this token, when given
  float sg = 1.f;
  if (sgate) {
    float d = 0.f;
    for (int c = threadIdx.x; c < H; c += blockDim.x)
      d = fmaf(__uint_as_float((uint32_t)x[(size_t)t * H + c] << 16), __uint_as_float((uint32_t)sgate[c] << 16), d);
    d = warp_sum(d);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = d;
    __syncthreads();
    if (threadIdx.x == 0) {
      float z = 0.f;
      for (int i = 0; i < (int)(blockDim.x >> 5); ++i) z += red[i];
      sg_s = 1.f / (1.f + expf(-z));
    }
    __syncthreads();
    sg = sg_s;
  }
  float ss = 0.f;
  for (int c = threadIdx.x; c < H; c += blockDim.x) {
    const float h = combine_h(Y, Ys, pair_slot, w, res, t, c, H, K, sg);
    ss = fmaf(h, h, ss);
    h_out[(size_t)t * H + c] = __bfloat16_as_ushort(__float2bfloat16_rn(h));
  }
  ss = warp_sum(ss);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = ss;
  __syncthreads();
  if (threadIdx.x == 0) {
    float a = 0.f;
    for (int i = 0; i < (int)(blockDim.x >> 5); ++i) a += red[i];
    inv_s = rsqrtf(__fdividef(a, (float)H) + eps);
  }
  __syncthreads();
  const float inv = inv_s;
  for (int c = threadIdx.x; c < H; c += blockDim.x) {
    const float h = combine_h(Y, Ys, pair_slot, w, res, t, c, H, K, sg);
    const float g = __uint_as_float((uint32_t)gamma[c] << 16);
    y_norm[(size_t)t * H + c] = __bfloat16_as_ushort(__float2bfloat16_rn(h * inv * g));
  }
}

// RMSNorm of the residual stream before the layer, one block per token:
// x = bf16(h / sqrt(mean(h^2) + eps) * gamma_pre), h read as bf16 16 bytes
// at a time (H a multiple of 8).
__global__ void __launch_bounds__(256) prenorm_kernel(const uint16_t* __restrict__ h,
                                                      const uint16_t* __restrict__ gamma, int H, float eps,
                                                      uint16_t* __restrict__ x) {
  const int t = blockIdx.x;
  __shared__ float red[8];
  __shared__ float inv_s;
  const uint4* hr = reinterpret_cast<const uint4*>(h + (size_t)t * H);
  float ss = 0.f;
  for (int q = threadIdx.x; q < H / 8; q += blockDim.x) {
    float v[8];
    unpack_bf16x8(__ldg(hr + q), v);
    float sq = 0.f;
#pragma unroll
    for (int i = 0; i < 8; ++i) sq = fmaf(v[i], v[i], sq);
    ss += sq;
  }
  ss = warp_sum(ss);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = ss;
  __syncthreads();
  if (threadIdx.x == 0) {
    float a = 0.f;
    for (int i = 0; i < (int)(blockDim.x >> 5); ++i) a += red[i];
    inv_s = __fdiv_rn(1.f, __fsqrt_rn(__fdiv_rn(a, (float)H) + eps));
  }
  __syncthreads();
  const float inv = inv_s;
  uint4* xr = reinterpret_cast<uint4*>(x + (size_t)t * H);
  for (int q = threadIdx.x; q < H / 8; q += blockDim.x) {
    float v[8], g[8];
    unpack_bf16x8(__ldg(hr + q), v);
    unpack_bf16x8(__ldg(reinterpret_cast<const uint4*>(gamma) + q), g);
    uint32_t o[4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
      o[i] = (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(__fmul_rn(__fmul_rn(v[2 * i], inv), g[2 * i]))) |
             ((uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(__fmul_rn(__fmul_rn(v[2 * i + 1], inv), g[2 * i + 1])))
              << 16);
    xr[q] = make_uint4(o[0], o[1], o[2], o[3]);
  }
}

cudaError_t launch_prenorm(const uint16_t* h, const uint16_t* gamma, int T, int H, float eps, uint16_t* x,
                           cudaStream_t st) {
  if (T <= 0) return cudaSuccess;
  prenorm_kernel<<<T, 256, 0, st>>>(h, gamma, H, eps, x);
  return cudaGetLastError();
}

__global__ void set_ptr_kernel(const void** dst, const void* v) { *dst = v; }

// Writes one pointer value into device memory (stream-ordered, and usable
// under stream capture, unlike a copy from a host variable).
cudaError_t launch_set_ptr(const void** dst, const void* v, cudaStream_t st) {
  set_ptr_kernel<<<1, 1, 0, st>>>(dst, v);
  return cudaGetLastError();
}

cudaError_t launch_to_half(const uint16_t* x, void* xh, size_t n, uint32_t* abort_flag, cudaStream_t st) {
  const size_t n8 = n / 8;
  const int grid = (int)((n8 + 255) / 256 < 1184 ? (n8 + 255) / 256 : 1184);
  to_half_kernel<<<grid > 0 ? grid : 1, 256, 0, st>>>(x, static_cast<__half*>(xh), n8, abort_flag);
  return cudaGetLastError();
}

cudaError_t launch_group(const int32_t* idx, int TK, int E, int K, int* slot_token, int* pair_slot, int* ch_e,
                         int* ch_c0, int* ch_n, int* n_chunks, const void* const* expert_ptr, uint32_t* err,
                         cudaStream_t st) {
  group_kernel<<<1, 1024, 0, st>>>(idx, TK, E, slot_token, pair_slot, K, ch_e, ch_c0, ch_n, n_chunks, expert_ptr,
                                   err);
  return cudaGetLastError();
}

cudaError_t launch_combine(const float* Y, const float* Ys, const int* pair_slot, const float* w, const uint16_t* res,
                           const uint16_t* gamma, int T, int H, int K, float eps, const uint16_t* x,
                           const uint16_t* sgate, uint16_t* h_out, uint16_t* y_norm, cudaStream_t st) {
  combine_kernel<<<T, 256, 0, st>>>(Y, Ys, pair_slot, w, res, gamma, H, K, eps, x, sgate, h_out, y_norm);
  return cudaGetLastError();
}

}  // namespace moe
