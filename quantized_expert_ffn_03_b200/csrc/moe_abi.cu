// moe_abi.cu -- the extern "C" entry points of libmoe: argument checks,
// workspace carving and kernel launches.  See include/moe.h for the contract.
#include <cuda_runtime.h>

#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>

#include "../../include/moe.h"
#include "moe_grouped.h"
#include "moe_kernels.h"

namespace moe {
// The kernel's view of a device-resolved streaming cache (moe_stream.cu).
moe_status stream_view(moe_stream_cache* c, int layer, int E, uint64_t blob_bytes, StreamView* v);

void pack_host(const Layout& L, const float* wg, const float* wu, const float* wd, int e_begin,
               int e_count, uint8_t* out);
}

using namespace moe;

namespace {

thread_local std::string g_err;

moe_status fail(moe_status s, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_err = buf;
  return s;
}

moe_status bad_shape(const moe_config* cfg) {
  if (!cfg) return fail(MOE_ERR_INVALID_ARG, "cfg is NULL");
  return fail(MOE_ERR_UNSUPPORTED,
              "unsupported shape: bits=%d (2 or 4), group=%d (64), hidden=%d and inter=%d "
              "(positive multiples of 64)",
              cfg->bits, cfg->group, cfg->hidden, cfg->inter);
}

moe_status ok() {
  g_err.clear();
  return MOE_OK;
}

#define CUDA_TRY(call)                                                                       \
  do {                                                                                       \
    cudaError_t e_ = (call);                                                                 \
    if (e_ != cudaSuccess)                                                                   \
      return fail(MOE_ERR_CUDA, "%s failed: %s", #call, cudaGetErrorString(e_));             \
  } while (0)

constexpr uint64_t kTimeoutNs = 2000000000ull;  // 2 s per bounded wait

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// The optional forms of the shared expert that a weight set selects.
void weight_opts(const moe_layer_weights* wts, Layout* L) {
  L->sgate = (wts && L->has_shared && wts->shared_out_gate) ? 1 : 0;
  L->spacked = (wts && L->has_shared && wts->shared_packed) ? 1 : 0;
  L->KP = L->K + L->spacked;
}

moe_status check_cfg(const moe_config* cfg, Layout* L) {
  if (!cfg) return fail(MOE_ERR_INVALID_ARG, "cfg is NULL");
  if (cfg->n_experts <= 0 || cfg->top_k <= 0)
    return fail(MOE_ERR_INVALID_ARG, "n_experts and top_k must be positive");
  if (!make_layout(cfg->hidden, cfg->inter, cfg->n_experts, cfg->top_k, cfg->bits, cfg->group,
                   cfg->has_shared, cfg->eps, L))
    return fail(MOE_ERR_UNSUPPORTED,
                "unsupported shape: bits=%d (2 or 4), group=%d (64), hidden=%d and inter=%d "
                "(positive multiples of 64)",
                cfg->bits, cfg->group, cfg->hidden, cfg->inter);
  if (cfg->top_k > cfg->n_experts) return fail(MOE_ERR_UNSUPPORTED, "top_k > n_experts");
  if (cfg->top_k > kMaxK) return fail(MOE_ERR_UNSUPPORTED, "top_k > %d", kMaxK);
  if (cfg->hidden > 16384 || cfg->inter > 16384)
    return fail(MOE_ERR_UNSUPPORTED, "hidden and inter must be <= 16384");
  if (cfg->n_experts > 65536) return fail(MOE_ERR_UNSUPPORTED, "n_experts must be <= 65536");
  return MOE_OK;
}

struct DeviceInfo {
  int sms = 0;
};

moe_status device_info(DeviceInfo* out) {
  static std::mutex mu;
  static DeviceInfo cache[64];
  int dev = 0;
  CUDA_TRY(cudaGetDevice(&dev));
  if (dev < 0 || dev >= 64) return fail(MOE_ERR_UNSUPPORTED, "device index %d", dev);
  std::lock_guard<std::mutex> lk(mu);
  if (cache[dev].sms == 0) {
    int sms = 0;
    CUDA_TRY(cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev));
    cache[dev].sms = sms;
  }
  *out = cache[dev];
  return MOE_OK;
}

struct WsPlan {
  size_t logits, hs, hf, hx, ss, route, sstot, total;
};

// Tokens per launch of the fused kernel: at most kMaxTokensFused, and at
// most 64 (token, expert) pairs.  Larger T runs in chunks of this size.
int chunk_tokens(const Layout& L) {
  const int c = 64 / L.K;
  return c < kMaxTokensFused ? (c > 0 ? c : 1) : kMaxTokensFused;
}

// Tokens one launch takes on a grid of `grid` blocks: the largest
// T <= max_tokens whose shared-memory plan fits (0 if not even one token).
int tokens_per_launch(const Layout& L, int grid, int max_tokens) {
  for (int t = max_tokens; t >= 1; --t) {
    int ns = 0;
    if (decode_slot_bytes(L, t, decode_rows_max(L.H, grid), &ns) > 0) return t;
  }
  return 0;
}

// The fused kernel publishes its router logits and sums of squares as 64-bit
// words tagged with the launch's epoch.  Their region follows the 256-byte
// header in every plan (fused and batched), so no other data of either path
// is ever written where a later launch looks for its epoch words.
// Words: the router logits [C][E], the blocks' sums of squares
// [kMaxGrid][C], the routing block 0 publishes [C][K][2] (index, weight) and
// the total sums of squares it publishes [C].
size_t epoch_region_bytes(const Layout& L) {
  const size_t C = (size_t)chunk_tokens(L);
  return round_up_256(sizeof(uint64_t) * C * L.E) + round_up_256(sizeof(uint64_t) * C * kMaxGrid) +
         round_up_256(sizeof(uint64_t) * C * L.K * 2) + round_up_256(sizeof(uint64_t) * C);
}

WsPlan ws_plan(const Layout& L, int T) {
  WsPlan w;
  const size_t C = (size_t)chunk_tokens(L);
  size_t pos = 256;
  w.logits = pos;
  w.ss = round_up_256(pos + sizeof(uint64_t) * C * L.E);
  w.route = round_up_256(w.ss + sizeof(uint64_t) * C * kMaxGrid);
  w.sstot = round_up_256(w.route + sizeof(uint64_t) * C * L.K * 2);
  pos = 256 + epoch_region_bytes(L);
  w.hs = pos;
  pos = round_up_256(pos + sizeof(float) * (size_t)T * L.I);
  // the routed intermediate of K pairs per token, one more when a shared
  // expert exists (the workspace size does not depend on its form)
  const size_t kp = (size_t)L.K + (L.has_shared ? 1 : 0);
  w.hf = pos;
  pos = round_up_256(pos + 4ull * (size_t)T * kp * L.I);
  w.hx = pos;
  pos = round_up_256(pos + sizeof(float) * (size_t)T * kp * (L.I / 16));
  w.total = pos;
  return w;
}

// Workspace of the batched path for T tokens: the 256-byte header (error
// word, abort flag), then x as fp16, router logits, routing, the grouping
// (slot -> token, pair -> slot, chunk lists), the routed intermediate (fp16
// [slot][I]), the routed outputs (fp32 [slot][H]), the shared intermediate
// (bf16 hi and lo [T][I]) and the shared output (fp32 [T][H]).
struct BatchPlan {
  size_t xh, logits, idx, w, slot_token, pair_slot, ch_e, ch_c0, ch_n, nch, sptr, hr, y, hs_hi, hs_lo, ys, total;
  int max_chunks;
};

constexpr int kBatchedMaxExperts = 2048;

BatchPlan batch_plan(const Layout& L, int T) {
  BatchPlan b;
  const size_t TK = (size_t)T * L.K;
  b.max_chunks = (int)(TK / 128 + (size_t)L.E + 1);
  size_t pos = 256 + epoch_region_bytes(L);
  auto take = [&](size_t bytes) {
    const size_t at = pos;
    pos = round_up_256(pos + bytes);
    return at;
  };
  b.xh = take(2ull * T * L.H);
  b.logits = take(4ull * T * L.E);
  b.idx = take(4 * TK);
  b.w = take(4 * TK);
  b.slot_token = take(4 * TK);
  b.pair_slot = take(4 * TK);
  b.ch_e = take(4ull * b.max_chunks);
  b.ch_c0 = take(4ull * b.max_chunks);
  b.ch_n = take(4ull * b.max_chunks);
  b.nch = take(16);
  b.sptr = take(16);  // a one-entry pointer table: the packed shared expert
  b.hr = take(2 * TK * L.I);
  b.y = take(4 * TK * L.H);
  b.hs_hi = take(2ull * T * L.I);
  b.hs_lo = take(2ull * T * L.I);
  b.ys = take(4ull * T * L.H);
  b.total = pos;
  return b;
}

// Tokens from which moe_layer_forward takes the batched path instead of the
// fused decode kernel on chunks of tokens.
constexpr int kBatchedMinTokens = 32;

bool batched_ok(const Layout& L) { return L.E <= kBatchedMaxExperts; }

}  // namespace

extern "C" {

const char* moe_last_error(void) { return g_err.c_str(); }

size_t moe_packed_expert_bytes(const moe_config* cfg) {
  Layout L;
  if (!cfg || !make_layout(cfg->hidden, cfg->inter, 1, 1, cfg->bits, cfg->group, 0, 0.f, &L)) return 0;
  return (size_t)L.blob_bytes;
}

moe_status moe_packed_layout(const moe_config* cfg, size_t offsets[6]) {
  Layout L;
  if (!offsets) return fail(MOE_ERR_INVALID_ARG, "offsets is NULL");
  if (!cfg || !make_layout(cfg->hidden, cfg->inter, 1, 1, cfg->bits, cfg->group, 0, 0.f, &L))
    return bad_shape(cfg);
  for (int m = 0; m < 3; ++m) {
    offsets[m] = L.off_codes[m];
    offsets[3 + m] = L.off_scales[m];
  }
  return ok();
}

moe_status moe_pack_experts(const moe_config* cfg, const float* w_gate, const float* w_up,
                            const float* w_down, int e_begin, int e_count, void* out,
                            size_t out_bytes) {
  Layout L;
  if (!cfg || !make_layout(cfg->hidden, cfg->inter, 1, 1, cfg->bits, cfg->group, 0, 0.f, &L))
    return bad_shape(cfg);
  if (e_begin < 0 || e_count < 0) return fail(MOE_ERR_INVALID_ARG, "negative expert range");
  if (e_count == 0) return ok();
  if (!w_gate || !w_up || !w_down || !out) return fail(MOE_ERR_INVALID_ARG, "NULL pointer");
  if (out_bytes < (size_t)L.blob_bytes * e_count)
    return fail(MOE_ERR_INVALID_ARG, "out_bytes %zu < %zu", out_bytes, (size_t)L.blob_bytes * e_count);
  pack_host(L, w_gate, w_up, w_down, e_begin, e_count, static_cast<uint8_t*>(out));
  return ok();
}

moe_status moe_pack_experts_device(const moe_config* cfg, const float* w_gate,
                                   const float* w_up, const float* w_down, int e_count,
                                   void* out, size_t out_bytes, cudaStream_t stream) {
  Layout L;
  if (!cfg || !make_layout(cfg->hidden, cfg->inter, 1, 1, cfg->bits, cfg->group, 0, 0.f, &L))
    return bad_shape(cfg);
  if (e_count < 0) return fail(MOE_ERR_INVALID_ARG, "negative expert count");
  if (e_count == 0) return ok();
  if (!w_gate || !w_up || !w_down || !out) return fail(MOE_ERR_INVALID_ARG, "NULL pointer");
  if (!aligned(w_gate, 16) || !aligned(w_up, 16) || !aligned(w_down, 16) || !aligned(out, 16))
    return fail(MOE_ERR_INVALID_ARG, "device packer pointers must be 16-byte aligned");
  if (out_bytes < (size_t)L.blob_bytes * e_count)
    return fail(MOE_ERR_INVALID_ARG, "out_bytes %zu < %zu", out_bytes, (size_t)L.blob_bytes * e_count);
  CUDA_TRY(launch_pack(L, w_gate, w_up, w_down, e_count, static_cast<uint8_t*>(out), stream));
  return ok();
}

size_t moe_router_workspace_bytes(const moe_config* cfg, int T) {
  if (!cfg || T < 0 || cfg->n_experts <= 0) return 0;
  return (size_t)round_up_256(sizeof(float) * (size_t)T * cfg->n_experts);
}

moe_status moe_topk_from_logits(const moe_config* cfg, const float* logits, int T, int32_t* idx,
                                float* w, cudaStream_t stream) {
  if (!cfg) return fail(MOE_ERR_INVALID_ARG, "cfg is NULL");
  if (cfg->n_experts <= 0 || cfg->top_k <= 0 || T < 0) return fail(MOE_ERR_INVALID_ARG, "bad sizes");
  if (cfg->top_k > cfg->n_experts || cfg->top_k > kMaxK) return fail(MOE_ERR_UNSUPPORTED, "top_k");
  if (T == 0) return ok();
  if (!logits || !idx || !w) return fail(MOE_ERR_INVALID_ARG, "NULL pointer");
  CUDA_TRY(launch_topk(logits, T, cfg->n_experts, cfg->top_k, idx, w, stream));
  return ok();
}

moe_status moe_router_topk(const moe_config* cfg, const void* x_bf16, const void* wr_bf16,
                           const float* bias, int T, int32_t* idx, float* w, float* logits_out,
                           void* workspace, size_t ws_bytes, cudaStream_t stream) {
  Layout L;
  moe_status s = check_cfg(cfg, &L);
  if (s != MOE_OK) return s;
  if (T < 0) return fail(MOE_ERR_INVALID_ARG, "T < 0");
  if (T == 0) return ok();
  if (!x_bf16 || !wr_bf16 || !idx || !w) return fail(MOE_ERR_INVALID_ARG, "NULL pointer");
  if (!aligned(x_bf16, 16) || !aligned(wr_bf16, 16))
    return fail(MOE_ERR_INVALID_ARG, "x and router weights must be 16-byte aligned");
  float* logits = logits_out;
  if (!logits) {
    if (!workspace || ws_bytes < moe_router_workspace_bytes(cfg, T))
      return fail(MOE_ERR_WORKSPACE, "router workspace too small (need %zu)",
                  moe_router_workspace_bytes(cfg, T));
    logits = static_cast<float*>(workspace);
  }
  DeviceInfo di;
  if ((s = device_info(&di)) != MOE_OK) return s;
  int grid = (L.E + 15) / 16;
  if (grid > 4 * di.sms) grid = 4 * di.sms;
  CUDA_TRY(launch_router_logits(static_cast<const uint16_t*>(x_bf16), static_cast<const uint16_t*>(wr_bf16),
                                bias, T, L.H, L.E, grid, logits, stream));
  CUDA_TRY(launch_topk(logits, T, L.E, L.K, idx, w, stream));
  return ok();
}

size_t moe_layer_workspace_bytes(const moe_config* cfg, int T) {
  Layout L;
  if (!cfg || T < 0 || cfg->n_experts <= 0 || cfg->top_k <= 0) return 0;
  if (!make_layout(cfg->hidden, cfg->inter, cfg->n_experts, cfg->top_k, cfg->bits, cfg->group,
                   cfg->has_shared, cfg->eps, &L))
    return 0;
  const size_t fused = ws_plan(L, T < chunk_tokens(L) ? T : chunk_tokens(L)).total;
  if (T >= kBatchedMinTokens && batched_ok(L)) {
    const size_t b = batch_plan(L, T).total;
    return b > fused ? b : fused;
  }
  return fused;
}

size_t moe_layer_batched_workspace_bytes(const moe_config* cfg, int T) {
  Layout L;
  if (!cfg || T < 0 || cfg->n_experts <= 0 || cfg->top_k <= 0) return 0;
  if (!make_layout(cfg->hidden, cfg->inter, cfg->n_experts, cfg->top_k, cfg->bits, cfg->group,
                   cfg->has_shared, cfg->eps, &L) || !batched_ok(L))
    return 0;
  return batch_plan(L, T).total;
}

moe_status moe_workspace_init(void* workspace, size_t ws_bytes, cudaStream_t stream) {
  if (!workspace || ws_bytes < 256) return fail(MOE_ERR_WORKSPACE, "workspace missing or < 256 bytes");
  CUDA_TRY(cudaMemsetAsync(workspace, 0, ws_bytes, stream));
  return ok();
}

}  // extern "C"

static moe_status layer_forward_chunk(const moe_config* cfg, const moe_layer_weights* wts,
                                      const void* x_bf16, const void* residual_bf16, int T,
                                      void* h_out_bf16, void* y_norm_bf16, int32_t* idx_out,
                                      float* w_out, void* workspace, size_t ws_bytes,
                                      void* trace, size_t trace_entries, cudaStream_t stream,
                                      const int32_t* idx_in, const float* w_in, const void* gamma_pre = nullptr,
                                      void* x_out = nullptr, const StreamView* sv = nullptr) {
  Layout L;
  moe_status s = check_cfg(cfg, &L);
  if (s != MOE_OK) return s;
  L.prenorm = gamma_pre ? 1 : 0;
  weight_opts(wts, &L);
  if (T > chunk_tokens(L)) return fail(MOE_ERR_UNSUPPORTED, "T=%d: at most %d tokens per launch", T, chunk_tokens(L));
  if (!aligned(gamma_pre, 16) || !aligned(x_out, 16) || (L.sgate && !aligned(wts->shared_out_gate, 16)))
    return fail(MOE_ERR_INVALID_ARG, "bf16 arrays must be 16-byte aligned");
  const bool given = idx_in != nullptr;  // routing given: the router weights are not read
  if (given && !w_in) return fail(MOE_ERR_INVALID_ARG, "NULL routing weights");
  if (!wts || (!wts->expert_ptr && !sv) || (!given && !wts->router_w) || !wts->gamma || !x_bf16 ||
      !residual_bf16 || !h_out_bf16 || !y_norm_bf16)
    return fail(MOE_ERR_INVALID_ARG, "NULL pointer");
  if (L.has_shared && !L.spacked && (!wts->shared_gate || !wts->shared_up || !wts->shared_down))
    return fail(MOE_ERR_INVALID_ARG, "has_shared=1 but a shared-expert pointer is NULL");
  if (L.spacked && !aligned(wts->shared_packed, 256))
    return fail(MOE_ERR_INVALID_ARG, "the packed shared expert must be 256-byte aligned");
  const void* a16[] = {x_bf16, residual_bf16, h_out_bf16, y_norm_bf16, given ? nullptr : wts->router_w,
                       wts->gamma};
  for (const void* p : a16)
    if (!aligned(p, 16)) return fail(MOE_ERR_INVALID_ARG, "bf16 arrays must be 16-byte aligned");
  if (L.has_shared && !L.spacked && (!aligned(wts->shared_gate, 16) || !aligned(wts->shared_up, 16) ||
                                     !aligned(wts->shared_down, 16)))
    return fail(MOE_ERR_INVALID_ARG, "shared-expert weights must be 16-byte aligned");
  const WsPlan wp = ws_plan(L, T);
  if (!workspace || ws_bytes < wp.total || !aligned(workspace, 256))
    return fail(MOE_ERR_WORKSPACE, "workspace must be 256-byte aligned and >= %zu bytes", wp.total);
  DeviceInfo di;
  if ((s = device_info(&di)) != MOE_OK) return s;
  const int grid = di.sms < kMaxGrid ? di.sms : kMaxGrid;
  const int nrows_max = decode_rows_max(L.H, grid);
  int nslots = 0;
  const uint32_t slot_bytes = decode_slot_bytes(L, T, nrows_max, &nslots);
  if (slot_bytes == 0)
    return fail(MOE_ERR_UNSUPPORTED, "shape does not fit the fused kernel's shared memory (H=%d, I=%d, T=%d)",
                L.H, L.I, T);
  const size_t smem = decode_smem_bytes(L, T, nrows_max, nslots, slot_bytes);

  uint8_t* ws = static_cast<uint8_t*>(workspace);
  DecodeParams p = {};
  p.L = L;
  p.T = T;
  p.expert_ptr = sv ? nullptr : wts->expert_ptr;
  p.streamed = sv ? 1 : 0;
  if (sv) p.sv = *sv;
  p.wr = static_cast<const uint16_t*>(wts->router_w);
  p.bias = wts->router_bias;
  p.sg = static_cast<const uint16_t*>(wts->shared_gate);
  p.su = static_cast<const uint16_t*>(wts->shared_up);
  p.sd = static_cast<const uint16_t*>(wts->shared_down);
  p.gamma = static_cast<const uint16_t*>(wts->gamma);
  p.gamma_pre = static_cast<const uint16_t*>(gamma_pre);
  p.x_out = static_cast<uint16_t*>(x_out);
  p.sgate = L.sgate ? static_cast<const uint16_t*>(wts->shared_out_gate) : nullptr;
  p.spacked = L.spacked ? static_cast<const uint8_t*>(wts->shared_packed) : nullptr;
  p.x = static_cast<const uint16_t*>(x_bf16);
  p.res = static_cast<const uint16_t*>(residual_bf16);
  p.h_out = static_cast<uint16_t*>(h_out_bf16);
  p.y_norm = static_cast<uint16_t*>(y_norm_bf16);
  p.idx_out = idx_out;
  p.w_out = w_out;
  p.idx_in = idx_in;
  p.w_in = w_in;
  p.ctr = reinterpret_cast<uint32_t*>(ws);
  p.err = reinterpret_cast<uint32_t*>(ws + 64);
  p.logits = reinterpret_cast<uint64_t*>(ws + wp.logits);
  p.hs = reinterpret_cast<float*>(ws + wp.hs);
  p.hf = ws + wp.hf;
  p.hx = reinterpret_cast<float*>(ws + wp.hx);
  p.ss = reinterpret_cast<uint64_t*>(ws + wp.ss);
  p.route = reinterpret_cast<uint64_t*>(ws + wp.route);
  p.sstot = reinterpret_cast<uint64_t*>(ws + wp.sstot);
  if (trace && trace_entries < (size_t)grid * 128)
    return fail(MOE_ERR_INVALID_ARG, "trace needs %d entries", grid * 128);
  p.timeout_ns = kTimeoutNs;
  p.slot_bytes = slot_bytes;
  p.nslots = nslots;
  p.trace = static_cast<uint64_t*>(trace);
  CUDA_TRY(launch_decode(p, grid, smem, stream));
  return ok();
}

// The batched path (moe_grouped.cu): router GEMM, top-K, grouping by
// expert, grouped GEMMs for the routed experts, GEMMs for the shared expert,
// combine + residual + RMSNorm.
static moe_status layer_forward_batched(const moe_config* cfg, const moe_layer_weights* wts, const void* x_bf16,
                                        const void* residual_bf16, int T, void* h_out_bf16, void* y_norm_bf16,
                                        int32_t* idx_out, float* w_out, void* workspace, size_t ws_bytes,
                                        cudaStream_t stream) {
  Layout L;
  moe_status s = check_cfg(cfg, &L);
  if (s != MOE_OK) return s;
  if (T < 0) return fail(MOE_ERR_INVALID_ARG, "T < 0");
  if (T == 0) return ok();
  if (!batched_ok(L)) return fail(MOE_ERR_UNSUPPORTED, "the batched path takes at most %d experts", kBatchedMaxExperts);
  if (!wts || !wts->expert_ptr || !wts->router_w || !wts->gamma || !x_bf16 || !residual_bf16 || !h_out_bf16 ||
      !y_norm_bf16)
    return fail(MOE_ERR_INVALID_ARG, "NULL pointer");
  weight_opts(wts, &L);
  const bool bf16_shared = L.has_shared && !L.spacked;
  if (bf16_shared && (!wts->shared_gate || !wts->shared_up || !wts->shared_down))
    return fail(MOE_ERR_INVALID_ARG, "has_shared=1 but a shared-expert pointer is NULL");
  if (L.spacked && !aligned(wts->shared_packed, 256))
    return fail(MOE_ERR_INVALID_ARG, "the packed shared expert must be 256-byte aligned");
  const void* a16[] = {x_bf16, residual_bf16, h_out_bf16, y_norm_bf16, wts->router_w, wts->gamma,
                       bf16_shared ? wts->shared_gate : nullptr, bf16_shared ? wts->shared_up : nullptr,
                       bf16_shared ? wts->shared_down : nullptr, L.sgate ? wts->shared_out_gate : nullptr};
  for (const void* q : a16)
    if (!aligned(q, 16)) return fail(MOE_ERR_INVALID_ARG, "bf16 arrays must be 16-byte aligned");
  const BatchPlan bp = batch_plan(L, T);
  if (!workspace || ws_bytes < bp.total || !aligned(workspace, 256))
    return fail(MOE_ERR_WORKSPACE, "workspace must be 256-byte aligned and >= %zu bytes", bp.total);
  DeviceInfo di;
  if ((s = device_info(&di)) != MOE_OK) return s;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  uint32_t* err = reinterpret_cast<uint32_t*>(ws + 64);
  uint32_t* abort_flag = reinterpret_cast<uint32_t*>(ws) + 5;
  const int TK = T * L.K;
  const uint16_t* x = static_cast<const uint16_t*>(x_bf16);
  int32_t* idx = idx_out ? idx_out : reinterpret_cast<int32_t*>(ws + bp.idx);
  float* w = w_out ? w_out : reinterpret_cast<float*>(ws + bp.w);
  float* logits = reinterpret_cast<float*>(ws + bp.logits);
  int* slot_token = reinterpret_cast<int*>(ws + bp.slot_token);
  int* pair_slot = reinterpret_cast<int*>(ws + bp.pair_slot);
  int* ch_e = reinterpret_cast<int*>(ws + bp.ch_e);
  int* ch_c0 = reinterpret_cast<int*>(ws + bp.ch_c0);
  int* ch_n = reinterpret_cast<int*>(ws + bp.ch_n);
  int* nch = reinterpret_cast<int*>(ws + bp.nch);
  const int grid = di.sms;
  auto tiles = [](int cols, int M) { return ((cols + 127) / 128) * ((M + 127) / 128); };

  CUDA_TRY(launch_to_half(x, ws + bp.xh, (size_t)T * L.H, abort_flag, stream));
  // router logits (bf16 GEMM, bias in the epilogue), top-K
  GemmParams g = {};
  g.err = err;
  g.abort_flag = abort_flag;
  g.timeout_ns = kTimeoutNs;
  {
    GemmParams r = g;
    r.M = L.E;
    r.K = L.H;
    r.a_dense[0] = static_cast<const uint16_t*>(wts->router_w);
    r.b = x;
    r.n_cols = T;
    r.out = logits;
    r.bias = wts->router_bias;
    const int gr = tiles(T, L.E) < grid ? tiles(T, L.E) : grid;
    CUDA_TRY(launch_grouped_gemm(0, 1, 0, r, gr, stream));
  }
  CUDA_TRY(launch_topk(logits, T, L.E, L.K, idx, w, stream));
  CUDA_TRY(launch_group(idx, TK, L.E, L.K, slot_token, pair_slot, ch_e, ch_c0, ch_n, nch, wts->expert_ptr, err,
                        stream));
  // routed gate/up: dequantised weights x the chunk's tokens (fp16), SwiGLU -> hr
  {
    GemmParams r = g;
    r.M = L.I;
    r.K = L.H;
    r.bits = L.bits;
    r.expert_ptr = wts->expert_ptr;
    r.off_codes[0] = L.off_codes[0];
    r.off_codes[1] = L.off_codes[1];
    r.off_scales[0] = L.off_scales[0];
    r.off_scales[1] = L.off_scales[1];
    r.b = reinterpret_cast<const uint16_t*>(ws + bp.xh);
    r.b_rows = slot_token;
    r.ch_e = ch_e;
    r.ch_c0 = ch_c0;
    r.ch_n = ch_n;
    r.n_chunks_dev = nch;
    r.out = ws + bp.hr;
    CUDA_TRY(launch_grouped_gemm(L.bits, 2, 1, r, grid, stream));
  }
  // routed down: hr (per slot) -> y (fp32 per slot)
  {
    GemmParams r = g;
    r.M = L.H;
    r.K = L.I;
    r.bits = L.bits;
    r.expert_ptr = wts->expert_ptr;
    r.off_codes[0] = L.off_codes[2];
    r.off_scales[0] = L.off_scales[2];
    r.b = reinterpret_cast<const uint16_t*>(ws + bp.hr);
    r.ch_e = ch_e;
    r.ch_c0 = ch_c0;
    r.ch_n = ch_n;
    r.n_chunks_dev = nch;
    r.out = ws + bp.y;
    CUDA_TRY(launch_grouped_gemm(L.bits, 1, 0, r, grid, stream));
  }
  const float* ys = nullptr;
  if (L.spacked) {
    // the packed shared expert on every token: the same dequant GEMMs over
    // dense chunks of the T tokens, with a one-entry pointer table
    CUDA_TRY(launch_set_ptr(reinterpret_cast<const void**>(ws + bp.sptr), wts->shared_packed, stream));
    GemmParams r = g;
    r.M = L.I;
    r.K = L.H;
    r.bits = L.bits;
    r.expert_ptr = reinterpret_cast<const void* const*>(ws + bp.sptr);
    r.off_codes[0] = L.off_codes[0];
    r.off_codes[1] = L.off_codes[1];
    r.off_scales[0] = L.off_scales[0];
    r.off_scales[1] = L.off_scales[1];
    r.b = reinterpret_cast<const uint16_t*>(ws + bp.xh);
    r.n_cols = T;
    r.out = ws + bp.hs_hi;  // fp16 [T][I]
    const int gr = tiles(T, L.I) < grid ? tiles(T, L.I) : grid;
    CUDA_TRY(launch_grouped_gemm(L.bits, 2, 1, r, gr, stream));
    GemmParams d = g;
    d.M = L.H;
    d.K = L.I;
    d.bits = L.bits;
    d.expert_ptr = reinterpret_cast<const void* const*>(ws + bp.sptr);
    d.off_codes[0] = L.off_codes[2];
    d.off_scales[0] = L.off_scales[2];
    d.b = reinterpret_cast<const uint16_t*>(ws + bp.hs_hi);
    d.n_cols = T;
    d.out = ws + bp.ys;
    const int gd = tiles(T, L.H) < grid ? tiles(T, L.H) : grid;
    CUDA_TRY(launch_grouped_gemm(L.bits, 1, 0, d, gd, stream));
    ys = reinterpret_cast<const float*>(ws + bp.ys);
  } else if (L.has_shared) {
    GemmParams r = g;
    r.M = L.I;
    r.K = L.H;
    r.a_dense[0] = static_cast<const uint16_t*>(wts->shared_gate);
    r.a_dense[1] = static_cast<const uint16_t*>(wts->shared_up);
    r.b = x;
    r.n_cols = T;
    r.out = ws + bp.hs_hi;
    r.out2 = ws + bp.hs_lo;
    const int gr = tiles(T, L.I) < grid ? tiles(T, L.I) : grid;
    CUDA_TRY(launch_grouped_gemm(0, 2, 2, r, gr, stream));
    GemmParams d = g;
    d.M = L.H;
    d.K = L.I;
    d.a_dense[0] = static_cast<const uint16_t*>(wts->shared_down);
    d.b = reinterpret_cast<const uint16_t*>(ws + bp.hs_hi);
    d.b2 = reinterpret_cast<const uint16_t*>(ws + bp.hs_lo);
    d.n_cols = T;
    d.out = ws + bp.ys;
    const int gd = tiles(T, L.H) < grid ? tiles(T, L.H) : grid;
    CUDA_TRY(launch_grouped_gemm(0, 1, 0, d, gd, stream));
    ys = reinterpret_cast<const float*>(ws + bp.ys);
  }
  const bool sgate = L.sgate != 0;
  CUDA_TRY(launch_combine(reinterpret_cast<const float*>(ws + bp.y), ys, pair_slot, w,
                          static_cast<const uint16_t*>(residual_bf16), static_cast<const uint16_t*>(wts->gamma), T,
                          L.H, L.K, L.eps, static_cast<const uint16_t*>(x_bf16),
                          sgate ? static_cast<const uint16_t*>(wts->shared_out_gate) : nullptr,
                          static_cast<uint16_t*>(h_out_bf16), static_cast<uint16_t*>(y_norm_bf16), stream));
  return ok();
}

// Any T: the fused kernel on successive chunks of as many tokens as one
// launch takes on this device (tokens_per_launch), one after another
// on the stream (each token's result depends on that
// token only; each chunk reads the experts its tokens chose).
static moe_status layer_forward_impl(const moe_config* cfg, const moe_layer_weights* wts,
                                     const void* x_bf16, const void* residual_bf16, int T,
                                     void* h_out_bf16, void* y_norm_bf16, int32_t* idx_out,
                                     float* w_out, void* workspace, size_t ws_bytes,
                                     void* trace, size_t trace_entries, cudaStream_t stream,
                                     const int32_t* idx_in = nullptr, const float* w_in = nullptr,
                                     const StreamView* sv = nullptr) {
  Layout L;
  moe_status s = check_cfg(cfg, &L);
  if (s != MOE_OK) return s;
  if (T < 0) return fail(MOE_ERR_INVALID_ARG, "T < 0");
  if (T == 0) return ok();
  // argument checks before any device query
  if (trace && T > chunk_tokens(L))
    return fail(MOE_ERR_UNSUPPORTED, "a traced call takes at most %d tokens", chunk_tokens(L));
  const bool given = idx_in != nullptr;
  if (given && !w_in) return fail(MOE_ERR_INVALID_ARG, "NULL routing weights");
  if (!wts || (!wts->expert_ptr && !sv) || (!given && !wts->router_w) || !wts->gamma || !x_bf16 ||
      !residual_bf16 || !h_out_bf16 || !y_norm_bf16)
    return fail(MOE_ERR_INVALID_ARG, "NULL pointer");
  weight_opts(wts, &L);
  DeviceInfo di;
  if ((s = device_info(&di)) != MOE_OK) return s;
  const int C = tokens_per_launch(L, di.sms < kMaxGrid ? di.sms : kMaxGrid, chunk_tokens(L));
  if (C == 0)
    return fail(MOE_ERR_UNSUPPORTED, "shape does not fit the fused kernel's shared memory (H=%d, I=%d)", L.H, L.I);
  if (T <= C)
    return layer_forward_chunk(cfg, wts, x_bf16, residual_bf16, T, h_out_bf16, y_norm_bf16, idx_out, w_out,
                               workspace, ws_bytes, trace, trace_entries, stream, idx_in, w_in, nullptr, nullptr,
                               sv);
  if (trace) return fail(MOE_ERR_UNSUPPORTED, "a traced call takes at most %d tokens", C);
  const size_t row = 2ull * (size_t)L.H;
  for (int t0 = 0; t0 < T; t0 += C) {
    const int n = T - t0 < C ? T - t0 : C;
    const size_t o = (size_t)t0 * row, ok_ = (size_t)t0 * L.K;
    s = layer_forward_chunk(cfg, wts, static_cast<const uint8_t*>(x_bf16) + o,
                            static_cast<const uint8_t*>(residual_bf16) + o, n, static_cast<uint8_t*>(h_out_bf16) + o,
                            static_cast<uint8_t*>(y_norm_bf16) + o, idx_out ? idx_out + ok_ : nullptr,
                            w_out ? w_out + ok_ : nullptr, workspace, ws_bytes, nullptr, 0, stream,
                            idx_in ? idx_in + ok_ : nullptr, w_in ? w_in + ok_ : nullptr, nullptr, nullptr, sv);
    if (s != MOE_OK) return s;
  }
  return ok();
}

namespace moe {
// For the library's other translation units: record an error message, the
// workspace of the fused kernel's path, and run that path on a given
// workspace.
moe_status abi_fail(moe_status s, const char* msg) { return fail(s, "%s", msg); }
size_t fused_workspace_bytes(const moe_config* cfg, int T) {
  Layout L;
  if (!cfg || T < 0 || cfg->n_experts <= 0 || cfg->top_k <= 0) return 0;
  if (!make_layout(cfg->hidden, cfg->inter, cfg->n_experts, cfg->top_k, cfg->bits, cfg->group,
                   cfg->has_shared, cfg->eps, &L))
    return 0;
  return ws_plan(L, T < chunk_tokens(L) ? T : chunk_tokens(L)).total;
}
moe_status layer_forward_on(const moe_config* cfg, const moe_layer_weights* wts, const void* x_bf16,
                            const void* residual_bf16, int T, void* h_out_bf16, void* y_norm_bf16,
                            int32_t* idx_out, float* w_out, void* workspace, size_t ws_bytes,
                            cudaStream_t stream) {
  return layer_forward_impl(cfg, wts, x_bf16, residual_bf16, T, h_out_bf16, y_norm_bf16, idx_out, w_out,
                            workspace, ws_bytes, nullptr, 0, stream);
}
}  // namespace moe

extern "C" {

int moe_layer_tokens_per_launch(const moe_config* cfg) {
  Layout L;
  if (!cfg || cfg->n_experts <= 0 || cfg->top_k <= 0 || cfg->top_k > cfg->n_experts ||
      !make_layout(cfg->hidden, cfg->inter, cfg->n_experts, cfg->top_k, cfg->bits, cfg->group, cfg->has_shared,
                   cfg->eps, &L))
    return 0;
  DeviceInfo di;
  if (device_info(&di) != MOE_OK) return 0;
  return tokens_per_launch(L, di.sms < kMaxGrid ? di.sms : kMaxGrid, chunk_tokens(L));
}

moe_status moe_layer_forward_routed(const moe_config* cfg, const moe_layer_weights* wts,
                                    const void* x_bf16, const void* residual_bf16, int T,
                                    const int32_t* idx, const float* w, void* h_out_bf16,
                                    void* y_norm_bf16, void* workspace, size_t ws_bytes,
                                    cudaStream_t stream) {
  if (T > 0 && (!idx || !w)) return fail(MOE_ERR_INVALID_ARG, "NULL routing");
  return layer_forward_impl(cfg, wts, x_bf16, residual_bf16, T, h_out_bf16, y_norm_bf16, nullptr, nullptr,
                            workspace, ws_bytes, nullptr, 0, stream, idx, w);
}

moe_status moe_layer_forward_streamed(const moe_config* cfg, const moe_layer_weights* wts, const void* x_bf16,
                                      const void* residual_bf16, int T, void* h_out_bf16, void* y_norm_bf16,
                                      int32_t* idx_out, float* w_out, moe_stream_cache* cache, int layer,
                                      void* workspace, size_t ws_bytes, cudaStream_t stream) {
  Layout L;
  moe_status s = check_cfg(cfg, &L);
  if (s != MOE_OK) return s;
  if (T < 0) return fail(MOE_ERR_INVALID_ARG, "T < 0");
  if (!cache) return fail(MOE_ERR_INVALID_ARG, "cache is NULL");
  if (L.E > kStreamMaxExperts) return fail(MOE_ERR_UNSUPPORTED, "a streamed call takes at most %d experts", kStreamMaxExperts);
  StreamView v;
  if ((s = stream_view(cache, layer, L.E, L.blob_bytes, &v)) != MOE_OK) return s;
  if (v.S > kStreamMaxSlots || v.S > 64 * L.E)
    return fail(MOE_ERR_UNSUPPORTED, "a streamed call takes at most %d slots (and 64 per expert of a layer)",
                kStreamMaxSlots);
  if (T == 0) return ok();
  return layer_forward_impl(cfg, wts, x_bf16, residual_bf16, T, h_out_bf16, y_norm_bf16, idx_out, w_out,
                            workspace, ws_bytes, nullptr, 0, stream, nullptr, nullptr, &v);
}

moe_status moe_layer_forward(const moe_config* cfg, const moe_layer_weights* wts,
                             const void* x_bf16, const void* residual_bf16, int T,
                             void* h_out_bf16, void* y_norm_bf16, int32_t* idx_out, float* w_out,
                             void* workspace, size_t ws_bytes, cudaStream_t stream) {
  Layout L;
  if (cfg && T >= kBatchedMinTokens && check_cfg(cfg, &L) == MOE_OK && batched_ok(L))
    return layer_forward_batched(cfg, wts, x_bf16, residual_bf16, T, h_out_bf16, y_norm_bf16, idx_out, w_out,
                                 workspace, ws_bytes, stream);
  return layer_forward_impl(cfg, wts, x_bf16, residual_bf16, T, h_out_bf16, y_norm_bf16, idx_out, w_out,
                            workspace, ws_bytes, nullptr, 0, stream);
}

moe_status moe_layer_forward_batched(const moe_config* cfg, const moe_layer_weights* wts,
                                     const void* x_bf16, const void* residual_bf16, int T,
                                     void* h_out_bf16, void* y_norm_bf16, int32_t* idx_out, float* w_out,
                                     void* workspace, size_t ws_bytes, cudaStream_t stream) {
  return layer_forward_batched(cfg, wts, x_bf16, residual_bf16, T, h_out_bf16, y_norm_bf16, idx_out, w_out,
                               workspace, ws_bytes, stream);
}

moe_status moe_layer_forward_chunked(const moe_config* cfg, const moe_layer_weights* wts,
                                     const void* x_bf16, const void* residual_bf16, int T,
                                     void* h_out_bf16, void* y_norm_bf16, int32_t* idx_out, float* w_out,
                                     void* workspace, size_t ws_bytes, cudaStream_t stream) {
  return layer_forward_impl(cfg, wts, x_bf16, residual_bf16, T, h_out_bf16, y_norm_bf16, idx_out, w_out,
                            workspace, ws_bytes, nullptr, 0, stream);
}

moe_status moe_layer_forward_prenorm(const moe_config* cfg, const moe_layer_weights* wts,
                                     const void* gamma_pre_bf16, const void* h_in_bf16, int T,
                                     void* h_out_bf16, void* y_norm_bf16, int32_t* idx_out, float* w_out,
                                     void* x_out_bf16, void* workspace, size_t ws_bytes, cudaStream_t stream) {
  Layout L;
  moe_status s = check_cfg(cfg, &L);
  if (s != MOE_OK) return s;
  if (T < 0) return fail(MOE_ERR_INVALID_ARG, "T < 0");
  if (T == 0) return ok();
  if (!gamma_pre_bf16 || !h_in_bf16 || !x_out_bf16) return fail(MOE_ERR_INVALID_ARG, "NULL pointer");
  if (!aligned(gamma_pre_bf16, 16) || !aligned(h_in_bf16, 16) || !aligned(x_out_bf16, 16))
    return fail(MOE_ERR_INVALID_ARG, "bf16 arrays must be 16-byte aligned");
  if (x_out_bf16 == h_in_bf16 || x_out_bf16 == h_out_bf16 || h_out_bf16 == h_in_bf16)
    return fail(MOE_ERR_INVALID_ARG, "h_in, h_out and x_out must be distinct buffers");
  L.prenorm = 1;
  weight_opts(wts, &L);
  if (!(T >= kBatchedMinTokens && batched_ok(L))) {
    DeviceInfo di;
    if ((s = device_info(&di)) != MOE_OK) return s;
    const int C = tokens_per_launch(L, di.sms < kMaxGrid ? di.sms : kMaxGrid, chunk_tokens(L));
    if (C > 0 && T <= C)
      return layer_forward_chunk(cfg, wts, h_in_bf16, h_in_bf16, T, h_out_bf16, y_norm_bf16, idx_out, w_out,
                                 workspace, ws_bytes, nullptr, 0, stream, nullptr, nullptr, gamma_pre_bf16,
                                 x_out_bf16);
  }
  // more tokens than one fused launch takes: the normalisation as a kernel
  // of its own, then the layer on its output
  CUDA_TRY(launch_prenorm(static_cast<const uint16_t*>(h_in_bf16), static_cast<const uint16_t*>(gamma_pre_bf16), T,
                          L.H, L.eps, static_cast<uint16_t*>(x_out_bf16), stream));
  return moe_layer_forward(cfg, wts, x_out_bf16, h_in_bf16, T, h_out_bf16, y_norm_bf16, idx_out, w_out, workspace,
                           ws_bytes, stream);
}

int moe_layer_trace_blocks(void) {
  DeviceInfo di;
  if (device_info(&di) != MOE_OK) return -1;
  return di.sms < kMaxGrid ? di.sms : kMaxGrid;
}

moe_status moe_layer_forward_traced(const moe_config* cfg, const moe_layer_weights* wts,
                                    const void* x_bf16, const void* residual_bf16, int T,
                                    void* h_out_bf16, void* y_norm_bf16, void* workspace,
                                    size_t ws_bytes, uint64_t* trace, size_t trace_entries,
                                    cudaStream_t stream) {
  if (!trace) return fail(MOE_ERR_INVALID_ARG, "trace is NULL");
  return layer_forward_impl(cfg, wts, x_bf16, residual_bf16, T, h_out_bf16, y_norm_bf16, nullptr, nullptr,
                            workspace, ws_bytes, trace, trace_entries, stream);
}

size_t moe_layer_host_workspace_bytes(const moe_config* cfg, int T) {
  const size_t base = moe_layer_workspace_bytes(cfg, T);
  if (base == 0) return 0;
  const size_t act = (size_t)round_up_256(2ull * (size_t)T * cfg->hidden);
  return base + 4 * act;
}

// Host-buffer forms: x and residual are copied into staging areas of the
// workspace (one copy when they arrive packed in one host buffer), the layer
// runs, h_out and y_norm are copied back.
static moe_status host_path(const moe_config* cfg, const moe_layer_weights* wts, const void* x_host,
                            const void* res_host, const void* xr_host, int T, void* h_host, void* y_host,
                            void* hy_host, void* workspace, size_t ws_bytes, cudaStream_t stream) {
  if (!cfg) return fail(MOE_ERR_INVALID_ARG, "cfg is NULL");
  if (T < 0) return fail(MOE_ERR_INVALID_ARG, "T < 0");
  if (T == 0) return ok();
  if ((!xr_host && (!x_host || !res_host)) || (!hy_host && (!h_host || !y_host)))
    return fail(MOE_ERR_INVALID_ARG, "NULL host pointer");
  const size_t base = moe_layer_workspace_bytes(cfg, T);
  const size_t need = moe_layer_host_workspace_bytes(cfg, T);
  if (base == 0) return bad_shape(cfg);
  if (!workspace || ws_bytes < need)
    return fail(MOE_ERR_WORKSPACE, "host-path workspace must be >= %zu bytes", need);
  const size_t bytes = 2ull * (size_t)T * cfg->hidden;
  const size_t act = (size_t)round_up_256(bytes);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  uint8_t* dx = ws + base;
  uint8_t* dr = ws + base + act;
  uint8_t* dh = ws + base + 2 * act;
  uint8_t* dy = ws + base + 3 * act;
  if (xr_host) {
    // staging areas are adjacent exactly when a token block is a multiple of 256 bytes
    if (act == bytes) {
      CUDA_TRY(cudaMemcpyAsync(dx, xr_host, 2 * bytes, cudaMemcpyHostToDevice, stream));
    } else {
      CUDA_TRY(cudaMemcpyAsync(dx, xr_host, bytes, cudaMemcpyHostToDevice, stream));
      CUDA_TRY(cudaMemcpyAsync(dr, static_cast<const uint8_t*>(xr_host) + bytes, bytes, cudaMemcpyHostToDevice,
                               stream));
    }
  } else {
    CUDA_TRY(cudaMemcpyAsync(dx, x_host, bytes, cudaMemcpyHostToDevice, stream));
    CUDA_TRY(cudaMemcpyAsync(dr, res_host, bytes, cudaMemcpyHostToDevice, stream));
  }
  moe_status s = moe_layer_forward(cfg, wts, dx, dr, T, dh, dy, nullptr, nullptr, workspace, base, stream);
  if (s != MOE_OK) return s;
  if (hy_host) {
    if (act == bytes) {
      CUDA_TRY(cudaMemcpyAsync(hy_host, dh, 2 * bytes, cudaMemcpyDeviceToHost, stream));
    } else {
      CUDA_TRY(cudaMemcpyAsync(hy_host, dh, bytes, cudaMemcpyDeviceToHost, stream));
      CUDA_TRY(cudaMemcpyAsync(static_cast<uint8_t*>(hy_host) + bytes, dy, bytes, cudaMemcpyDeviceToHost, stream));
    }
  } else {
    CUDA_TRY(cudaMemcpyAsync(h_host, dh, bytes, cudaMemcpyDeviceToHost, stream));
    CUDA_TRY(cudaMemcpyAsync(y_host, dy, bytes, cudaMemcpyDeviceToHost, stream));
  }
  return ok();
}

moe_status moe_layer_forward_host_async(const moe_config* cfg, const moe_layer_weights* wts,
                                        const void* x_bf16_host, const void* residual_bf16_host, int T,
                                        void* h_out_bf16_host, void* y_norm_bf16_host, void* workspace,
                                        size_t ws_bytes, cudaStream_t stream) {
  return host_path(cfg, wts, x_bf16_host, residual_bf16_host, nullptr, T, h_out_bf16_host, y_norm_bf16_host, nullptr,
                   workspace, ws_bytes, stream);
}

moe_status moe_layer_forward_host_packed(const moe_config* cfg, const moe_layer_weights* wts,
                                         const void* xr_bf16_host, int T, void* hy_bf16_host, void* workspace,
                                         size_t ws_bytes, cudaStream_t stream) {
  return host_path(cfg, wts, nullptr, nullptr, xr_bf16_host, T, nullptr, nullptr, hy_bf16_host, workspace, ws_bytes,
                   stream);
}

moe_status moe_layer_forward_host(const moe_config* cfg, const moe_layer_weights* wts,
                                  const void* x_bf16_host, const void* residual_bf16_host, int T,
                                  void* h_out_bf16_host, void* y_norm_bf16_host, void* workspace,
                                  size_t ws_bytes, cudaStream_t stream) {
  moe_status s = moe_layer_forward_host_async(cfg, wts, x_bf16_host, residual_bf16_host, T, h_out_bf16_host,
                                              y_norm_bf16_host, workspace, ws_bytes, stream);
  if (s != MOE_OK || T == 0) return s;
  CUDA_TRY(cudaStreamSynchronize(stream));
  return ok();
}

moe_status moe_device_error(void* workspace, uint32_t* detail, cudaStream_t stream) {
  if (!workspace) return fail(MOE_ERR_INVALID_ARG, "workspace is NULL");
  uint32_t code = 0;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  CUDA_TRY(cudaMemcpyAsync(&code, ws + 64, 4, cudaMemcpyDeviceToHost, stream));
  CUDA_TRY(cudaStreamSynchronize(stream));
  if (code != 0) {
    CUDA_TRY(cudaMemsetAsync(ws + 64, 0, 4, stream));
    CUDA_TRY(cudaStreamSynchronize(stream));
  }
  if (detail) *detail = code;
  if (code == 0) return ok();
  if (code == 1) return fail(MOE_ERR_TIMEOUT, "a bounded device-side wait expired");
  return fail(MOE_ERR_DEVICE, "device-side check failed (code %u: bad or misaligned expert pointer)", code);
}

moe_status moe_selftest_bounded_wait(void* workspace, size_t ws_bytes, uint64_t timeout_ns,
                                     cudaStream_t stream) {
  if (!workspace || ws_bytes < 256) return fail(MOE_ERR_WORKSPACE, "workspace missing or < 256 bytes");
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  CUDA_TRY(launch_barrier_timeout_probe(reinterpret_cast<uint32_t*>(ws), reinterpret_cast<uint32_t*>(ws + 64),
                                        timeout_ns, stream));
  return ok();
}

}  // extern "C"
