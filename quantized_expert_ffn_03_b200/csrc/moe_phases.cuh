// moe_phases.cuh -- the GEMV phases of the MoE layer, written once and used by
// the fused decode kernel and the stand-alone router kernels.
//
// Work layout: a "team" of tw warps covers one weight row; lane l of warp w
// of the team owns input columns [32*(32w+l), +32).  Rows are handed out in
// chunks of R consecutive rows; a block owns a contiguous range of chunks and
// its teams take chunk b+team, b+team+nteams, ...  Partial sums are reduced
// with warp shuffles, then across the team's warps through shared memory.
#pragma once

#include "moe_device.cuh"

namespace moe {

struct TeamGeo {
  int tw;      // warps per team
  int nteams;  // teams per block
  int team, wt, chunk;
  bool active;  // this lane owns real columns
};

__device__ __forceinline__ TeamGeo team_geo(int tw, int cols) {
  TeamGeo g;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  g.tw = tw;
  g.nteams = kWarps / tw;
  g.team = warp / tw;
  g.wt = warp % tw;
  g.chunk = g.wt * 32 + lane;
  g.active = g.chunk < cols / 32;
  return g;
}

// Reduce R*NM lane partials over the team.  On return, every lane of the
// team's first warp (wt == 0) holds the row sums in out.  `it` alternates the
// two halves of the shared buffer `red` (2 * kWarps * R * NM floats) so a
// single barrier per chunk suffices.
template <int R, int NM>
__device__ __forceinline__ void team_reduce(float (&v)[R][NM], const TeamGeo& g, float* red, int it) {
#pragma unroll
  for (int r = 0; r < R; ++r)
#pragma unroll
    for (int m = 0; m < NM; ++m) v[r][m] = warp_sum(v[r][m]);
  if (g.tw > 1) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    float* base = red + (size_t)(it & 1) * kWarps * R * NM;
    if (lane == 0) {
#pragma unroll
      for (int r = 0; r < R; ++r)
#pragma unroll
        for (int m = 0; m < NM; ++m) base[warp * R * NM + r * NM + m] = v[r][m];
    }
    named_sync(1 + g.team, g.tw * 32);
    if (g.wt == 0) {
#pragma unroll
      for (int r = 0; r < R; ++r)
#pragma unroll
        for (int m = 0; m < NM; ++m) {
          float a = 0.f;
          for (int w = 0; w < g.tw; ++w) a += base[(g.team * g.tw + w) * R * NM + r * NM + m];
          v[r][m] = a;
        }
    }
  }
}

// Dot products of R x NM rows with the lane activations, reduced over the
// team.  crow/srow: per row, the start of its codes and scales (scales unused
// for bf16).
template <int FMT, int R, int NM>
__device__ __forceinline__ void team_rows_dot(const uint8_t* const (&crow)[R][NM],
                                              const uint8_t* const (&srow)[R][NM],
                                              const bool (&valid)[R], const LaneX& lx,
                                              const TeamGeo& g, float* red, int it,
                                              float (&out)[R][NM]) {
  Frag<FMT> f[R][NM];
#pragma unroll
  for (int r = 0; r < R; ++r)
#pragma unroll
    for (int m = 0; m < NM; ++m) {
      if (valid[r] && g.active)
        load_frag<FMT>(f[r][m], crow[r][m], srow[r][m], g.chunk);
      else
        zero_frag<FMT>(f[r][m]);
    }
#pragma unroll
  for (int r = 0; r < R; ++r)
#pragma unroll
    for (int m = 0; m < NM; ++m) out[r][m] = frag_dot<FMT>(f[r][m], lx);
  team_reduce<R, NM>(out, g, red, it);
}

template <int R, int NM>
__device__ __forceinline__ float pick(const float (&v)[R][NM], int r, int m) {
  float o = 0.f;
#pragma unroll
  for (int i = 0; i < R; ++i)
    if (i == r) o = v[i][m];
  return o;
}

__device__ __forceinline__ void chunk_range(int nch, int& cb, int& ce) {
  cb = (int)((long long)nch * blockIdx.x / gridDim.x);
  ce = (int)((long long)nch * (blockIdx.x + 1) / gridDim.x);
}

// ---- router: logits[t][e] = x_t . Wr[e] + bias[e] ----------------------------
template <int R>
__device__ void phase_router(const uint16_t* wr, const float* bias, const uint16_t* x, int T,
                             int H, int E, int tw, float* logits, float* red) {
  const TeamGeo g = team_geo(tw, H);
  const int nch = (E + R - 1) / R;
  int cb, ce;
  chunk_range(nch, cb, ce);
  int it = 0;
  LaneX lx;
  for (int t = 0; t < T; ++t) {
    if (cb + g.team >= ce) break;
    load_lane_x_bf16<FMT_BF16>(lx, x + (size_t)t * H, g.chunk, g.active);
    for (int ch = cb + g.team; ch < ce; ch += g.nteams, ++it) {
      const uint8_t* crow[R][1];
      bool valid[R];
#pragma unroll
      for (int r = 0; r < R; ++r) {
        const int e = ch * R + r;
        valid[r] = e < E;
        crow[r][0] = reinterpret_cast<const uint8_t*>(wr + (size_t)(valid[r] ? e : 0) * H);
      }
      float out[R][1];
      team_rows_dot<FMT_BF16, R, 1>(crow, crow, valid, lx, g, red, it, out);
      const int lane = threadIdx.x & 31;
      if (g.wt == 0 && lane < R) {
        const int e = ch * R + lane;
        if (e < E) logits[(size_t)t * E + e] = pick<R, 1>(out, lane, 0) + (bias ? bias[e] : 0.f);
      }
    }
  }
}

// ---- shared expert gate/up: hs[t][i] = silu(Wg[i] x_t) * (Wu[i] x_t) ----------
template <int R>
__device__ void phase_shared_gateup(const uint16_t* sg, const uint16_t* su, const uint16_t* x,
                                    int T, int H, int I, int tw, float* hs, float* red) {
  const TeamGeo g = team_geo(tw, H);
  const int nch = I / R;
  int cb, ce;
  chunk_range(nch, cb, ce);
  int it = 0;
  LaneX lx;
  for (int t = 0; t < T; ++t) {
    if (cb + g.team >= ce) break;
    load_lane_x_bf16<FMT_BF16>(lx, x + (size_t)t * H, g.chunk, g.active);
    for (int ch = cb + g.team; ch < ce; ch += g.nteams, ++it) {
      const uint8_t* crow[R][2];
      bool valid[R];
#pragma unroll
      for (int r = 0; r < R; ++r) {
        const int i = ch * R + r;
        valid[r] = true;
        crow[r][0] = reinterpret_cast<const uint8_t*>(sg + (size_t)i * H);
        crow[r][1] = reinterpret_cast<const uint8_t*>(su + (size_t)i * H);
      }
      float out[R][2];
      team_rows_dot<FMT_BF16, R, 2>(crow, crow, valid, lx, g, red, it, out);
      const int lane = threadIdx.x & 31;
      if (g.wt == 0 && lane < R)
        hs[(size_t)t * I + ch * R + lane] = silu_mul(pick<R, 2>(out, lane, 0), pick<R, 2>(out, lane, 1));
    }
  }
}

// ---- routed experts gate/up: he[t][k][i] = silu(Wg_e[i] x_t) * (Wu_e[i] x_t) ---
// eptr: [T*K] blob pointers of the chosen experts (shared memory).
template <int FMT, int R>
__device__ void phase_expert_gateup(const uint8_t* const* eptr, const Layout& L, const uint16_t* x,
                                    int T, int tw, float* he, float* red) {
  const TeamGeo g = team_geo(tw, L.H);
  const int cpp = L.I / R;  // chunks per (token, expert) pair
  const int nch = T * L.K * cpp;
  int cb, ce;
  chunk_range(nch, cb, ce);
  int it = 0, cur_t = -1;
  LaneX lx;
  for (int ch = cb + g.team; ch < ce; ch += g.nteams, ++it) {
    const int pair = ch / cpp;
    const int i0 = (ch - pair * cpp) * R;
    const int t = pair / L.K;
    if (t != cur_t) {
      load_lane_x_bf16<FMT>(lx, x + (size_t)t * L.H, g.chunk, g.active);
      cur_t = t;
    }
    const uint8_t* blob = eptr[pair];
    const uint8_t* crow[R][2];
    const uint8_t* srow[R][2];
    bool valid[R];
#pragma unroll
    for (int r = 0; r < R; ++r) {
      valid[r] = true;
#pragma unroll
      for (int m = 0; m < 2; ++m) {
        crow[r][m] = blob + L.off_codes[m] + (size_t)(i0 + r) * L.code_row_bytes[m];
        srow[r][m] = blob + L.off_scales[m] + (size_t)(i0 + r) * L.scale_row_bytes[m];
      }
    }
    float out[R][2];
    team_rows_dot<FMT, R, 2>(crow, srow, valid, lx, g, red, it, out);
    const int lane = threadIdx.x & 31;
    if (g.wt == 0 && lane < R)
      he[(size_t)pair * L.I + i0 + lane] = silu_mul(pick<R, 2>(out, lane, 0), pick<R, 2>(out, lane, 1));
  }
}

// ---- shared expert down, rows [r0, r1) of this block: ys[t][j] ---------------
template <int R>
__device__ void phase_shared_down(const uint16_t* sd, const float* hs, int T, int H, int I, int tw,
                                  int r0, int r1, float* ys, float* red) {
  const TeamGeo g = team_geo(tw, I);
  const int nrows = r1 - r0;
  const int cpt = (nrows + R - 1) / R;
  int it = 0;
  LaneX lx;
  for (int t = 0; t < T; ++t) {
    if (g.team >= cpt) break;
    load_lane_x_f32<FMT_BF16>(lx, hs + (size_t)t * I, g.chunk, g.active);
    for (int ch = g.team; ch < cpt; ch += g.nteams, ++it) {
      const uint8_t* crow[R][1];
      bool valid[R];
#pragma unroll
      for (int r = 0; r < R; ++r) {
        const int j = ch * R + r;
        valid[r] = j < nrows;
        crow[r][0] = reinterpret_cast<const uint8_t*>(sd + (size_t)(r0 + (valid[r] ? j : 0)) * I);
      }
      float out[R][1];
      team_rows_dot<FMT_BF16, R, 1>(crow, crow, valid, lx, g, red, it, out);
      const int lane = threadIdx.x & 31;
      if (g.wt == 0 && lane < R && ch * R + lane < nrows)
        ys[t * nrows + ch * R + lane] = pick<R, 1>(out, lane, 0);
    }
  }
}

// ---- routed experts down, rows [r0, r1): ypart[pair][j] ------------------------
template <int FMT, int R>
__device__ void phase_expert_down(const uint8_t* const* eptr, const Layout& L, const float* he,
                                  int T, int tw, int r0, int r1, float* ypart, float* red) {
  const TeamGeo g = team_geo(tw, L.I);
  const int nrows = r1 - r0;
  const int cpp = (nrows + R - 1) / R;
  const int nch = T * L.K * cpp;
  int it = 0, cur_pair = -1;
  LaneX lx;
  for (int ch = g.team; ch < nch; ch += g.nteams, ++it) {
    const int pair = ch / cpp;
    const int j0 = (ch - pair * cpp) * R;
    if (pair != cur_pair) {
      load_lane_x_f32<FMT>(lx, he + (size_t)pair * L.I, g.chunk, g.active);
      cur_pair = pair;
    }
    const uint8_t* blob = eptr[pair];
    const uint8_t* crow[R][1];
    const uint8_t* srow[R][1];
    bool valid[R];
#pragma unroll
    for (int r = 0; r < R; ++r) {
      const int j = j0 + r;
      valid[r] = j < nrows;
      const int row = r0 + (valid[r] ? j : 0);
      crow[r][0] = blob + L.off_codes[2] + (size_t)row * L.code_row_bytes[2];
      srow[r][0] = blob + L.off_scales[2] + (size_t)row * L.scale_row_bytes[2];
    }
    float out[R][1];
    team_rows_dot<FMT, R, 1>(crow, srow, valid, lx, g, red, it, out);
    const int lane = threadIdx.x & 31;
    if (g.wt == 0 && lane < R && j0 + lane < nrows)
      ypart[pair * nrows + j0 + lane] = pick<R, 1>(out, lane, 0);
  }
}

}  // namespace moe
