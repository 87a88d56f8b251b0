// moe_stream.cu -- the expert-streaming tier: every expert of every layer in
// pinned host memory, a cache of device slots in front of it, and the
// pointer table that the routed layer reads.
//
// The pages stream the K chosen experts of each layer from SSD with parallel
// pread and leave caching to the OS page cache ("Flash-MoE:
// ラップトップでの397Bパラメータモデルの実行", sections "パイプライン概要" and
// "試行錯誤と最適化").  On a B200 the store is host memory and the link is
// the host-to-device copy engine, so the cache is explicit: n_slots blobs of
// device memory, least recently used replacement (StreamPolicy), one CUDA
// event per slot marking its copy done ("ready") and one marking the last
// kernel that read it done ("used").
//
// Ordering rules (all on the GPU; the one host wait is noted below):
//   - a copy into a slot waits for the slot's "used" event and for any copy
//     into it still in flight ("ready"), then records "ready";
//   - a resolve makes the compute stream wait for "ready" of every slot it
//     hands out; those slots are held (never chosen as victims) until the
//     next resolve, which records their "used" event on its compute stream,
//     i.e. after the layer kernel the caller enqueued in between;
//   - the pointer table is copied from a pinned staging buffer of a ring of
//     kStage; a buffer is reused only after the event of its last copy, which
//     the host waits for (cudaEventSynchronize) when kStage resolves are still
//     in flight on the GPU.  A resolve can therefore block the host thread,
//     and must not be called while its stream is being captured into a
//     CUDA graph.
//
// Failures: a copy that cannot be enqueued (MOE_ERR_IO) leaves its slot
// empty, and a resolve that fails releases the slots it took, so the next
// call starts from a consistent cache.  Tests drive these paths with
// moe_stream_inject_fault (a host-side countdown that makes a chosen copy,
// or the next create's slot allocation, report failure without touching
// the GPU).
#include <cuda_runtime.h>

#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <vector>

#include "../../include/moe.h"
#include "moe_stream_policy.h"

namespace moe {
moe_status abi_fail(moe_status s, const char* msg);
}

namespace {

constexpr int kStage = 8;  // pointer-table staging buffers

moe_status failf(moe_status s, const char* fmt, ...) __attribute__((format(printf, 2, 3)));
moe_status failf(moe_status s, const char* fmt, ...) {
  char msg[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(msg, sizeof(msg), fmt, ap);
  va_end(ap);
  return moe::abi_fail(s, msg);
}

}  // namespace

struct moe_stream_cache {
  int L = 0, E = 0, S = 0;
  size_t blob = 0;
  int device = 0;
  const uint8_t* host = nullptr;
  uint8_t* slots = nullptr;
  moe::StreamPolicy pol;
  std::vector<cudaEvent_t> ready, used;
  const void** stage[kStage] = {};
  cudaEvent_t stage_ev[kStage] = {};
  bool stage_used[kStage] = {};
  int stage_next = 0;
  uint64_t bytes_h2d = 0;
  int fault_copy = -1;  // injected: copies left before one fails (-1: none)
  std::mutex mu;
};

namespace {
int g_fault_alloc = 0;  // injected: the next create's slot allocation fails
std::mutex g_fault_mu;
}  // namespace

namespace {

void destroy_parts(moe_stream_cache* c) {
  for (cudaEvent_t e : c->ready)
    if (e) cudaEventDestroy(e);
  for (cudaEvent_t e : c->used)
    if (e) cudaEventDestroy(e);
  for (int i = 0; i < kStage; ++i) {
    if (c->stage_ev[i]) cudaEventDestroy(c->stage_ev[i]);
    if (c->stage[i]) cudaFreeHost(c->stage[i]);
  }
  if (c->slots) cudaFree(c->slots);
}

// Enqueue the copy of (layer, e) into slot s on stream st (see the ordering
// rules at the top of the file); the policy has already assigned the slot.
moe_status fill_slot(moe_stream_cache* c, int s, int layer, int e, cudaStream_t st) {
  cudaError_t err = cudaStreamWaitEvent(st, c->used[s], 0);
  if (err == cudaSuccess) err = cudaStreamWaitEvent(st, c->ready[s], 0);
  if (err != cudaSuccess) return failf(MOE_ERR_CUDA, "CUDA error: %s", cudaGetErrorString(err));
  const uint8_t* src = c->host + ((size_t)layer * c->E + e) * c->blob;
  if (c->fault_copy >= 0 && c->fault_copy-- == 0) {
    c->pol.evict(s);
    return failf(MOE_ERR_IO, "copy of expert %d of layer %d from the host store failed: injected fault", e, layer);
  }
  err = cudaMemcpyAsync(c->slots + (size_t)s * c->blob, src, c->blob, cudaMemcpyHostToDevice, st);
  if (err != cudaSuccess) {
    c->pol.evict(s);
    return failf(MOE_ERR_IO, "copy of expert %d of layer %d from the host store failed: %s", e, layer,
                 cudaGetErrorString(err));
  }
  err = cudaEventRecord(c->ready[s], st);
  if (err != cudaSuccess) return failf(MOE_ERR_CUDA, "CUDA error: %s", cudaGetErrorString(err));
  c->bytes_h2d += c->blob;
  return MOE_OK;
}

moe_status check_ids(const moe_stream_cache* c, int layer, const int32_t* ids, int n) {
  if (layer < 0 || layer >= c->L) return failf(MOE_ERR_INVALID_ARG, "layer %d outside [0, %d)", layer, c->L);
  if (n < 0 || (n > 0 && !ids)) return failf(MOE_ERR_INVALID_ARG, "bad expert id list");
  for (int i = 0; i < n; ++i)
    if (ids[i] < 0 || ids[i] >= c->E) return failf(MOE_ERR_INVALID_ARG, "expert id %d outside [0, %d)", ids[i], c->E);
  return MOE_OK;
}

struct DeviceGuard {
  int prev = -1;
  explicit DeviceGuard(int dev) {
    if (cudaGetDevice(&prev) == cudaSuccess && prev != dev) cudaSetDevice(dev);
  }
  ~DeviceGuard() {
    int cur = -1;
    if (prev >= 0 && cudaGetDevice(&cur) == cudaSuccess && cur != prev) cudaSetDevice(prev);
  }
};

}  // namespace

extern "C" {

moe_status moe_stream_create(const moe_config* cfg, int n_layers, const void* host_pinned_experts,
                             size_t store_bytes, int n_slots, moe_stream_cache** out) {
  if (!out) return failf(MOE_ERR_INVALID_ARG, "out is NULL");
  *out = nullptr;
  if (!cfg) return failf(MOE_ERR_INVALID_ARG, "cfg is NULL");
  const size_t blob = moe_packed_expert_bytes(cfg);
  if (blob == 0 || cfg->n_experts <= 0) return failf(MOE_ERR_UNSUPPORTED, "unsupported shape");
  if (n_layers < 1 || n_slots < 1) return failf(MOE_ERR_INVALID_ARG, "n_layers and n_slots must be >= 1");
  if (!host_pinned_experts) return failf(MOE_ERR_INVALID_ARG, "host store is NULL");
  const size_t need = blob * (size_t)cfg->n_experts * (size_t)n_layers;
  if (store_bytes < need)
    return failf(MOE_ERR_INVALID_ARG, "the host store holds %zu bytes; %d layers of %d experts need %zu", store_bytes,
                 n_layers, cfg->n_experts, need);
  // both ends of the store must be page-locked memory
  cudaPointerAttributes attr, attr_end;
  const uint8_t* last_byte = static_cast<const uint8_t*>(host_pinned_experts) + need - 1;
  if (cudaPointerGetAttributes(&attr, host_pinned_experts) != cudaSuccess || attr.type != cudaMemoryTypeHost ||
      cudaPointerGetAttributes(&attr_end, last_byte) != cudaSuccess || attr_end.type != cudaMemoryTypeHost) {
    cudaGetLastError();
    return failf(MOE_ERR_INVALID_ARG, "the host store must be page-locked (cudaHostAlloc or cudaHostRegister)");
  }
  moe_stream_cache* c = new moe_stream_cache;
  c->L = n_layers;
  c->E = cfg->n_experts;
  c->S = n_slots;
  c->blob = blob;
  c->host = static_cast<const uint8_t*>(host_pinned_experts);
  cudaGetDevice(&c->device);
  c->pol.init(n_layers, cfg->n_experts, n_slots);
  bool alloc_fault = false;
  {
    std::lock_guard<std::mutex> lk(g_fault_mu);
    alloc_fault = g_fault_alloc != 0;
    g_fault_alloc = 0;
  }
  if (alloc_fault || cudaMalloc(&c->slots, blob * (size_t)n_slots) != cudaSuccess) {
    cudaGetLastError();
    c->slots = nullptr;
    destroy_parts(c);
    delete c;
    return failf(MOE_ERR_OOM, "%d slots of %zu bytes do not fit in device memory", n_slots, blob);
  }
  c->ready.assign(n_slots, nullptr);
  c->used.assign(n_slots, nullptr);
  bool okk = true;
  for (int s = 0; s < n_slots && okk; ++s)
    okk = cudaEventCreateWithFlags(&c->ready[s], cudaEventDisableTiming) == cudaSuccess &&
          cudaEventCreateWithFlags(&c->used[s], cudaEventDisableTiming) == cudaSuccess;
  for (int i = 0; i < kStage && okk; ++i)
    okk = cudaHostAlloc(reinterpret_cast<void**>(&c->stage[i]), sizeof(void*) * (size_t)c->E,
                        cudaHostAllocDefault) == cudaSuccess &&
          cudaEventCreateWithFlags(&c->stage_ev[i], cudaEventDisableTiming) == cudaSuccess;
  if (!okk) {
    cudaGetLastError();
    destroy_parts(c);
    delete c;
    return failf(MOE_ERR_OOM, "could not create the cache's events or staging buffers");
  }
  *out = c;
  return MOE_OK;
}

moe_status moe_stream_prefetch(moe_stream_cache* c, int layer, const int32_t* ids, int n, cudaStream_t copy_stream) {
  if (!c) return failf(MOE_ERR_INVALID_ARG, "cache is NULL");
  std::lock_guard<std::mutex> lk(c->mu);
  moe_status s = check_ids(c, layer, ids, n);
  if (s != MOE_OK) return s;
  DeviceGuard dg(c->device);
  for (int i = 0; i < n; ++i) {
    const int v = c->pol.prefetch(layer, ids[i]);
    if (v >= 0 && (s = fill_slot(c, v, layer, ids[i], copy_stream)) != MOE_OK) {
      --c->pol.prefetches;  // not issued
      return s;
    }
  }
  return MOE_OK;
}

moe_status moe_stream_resolve(moe_stream_cache* c, int layer, const int32_t* idx, int n, const void** expert_ptr_dev,
                              cudaStream_t st) {
  if (!c) return failf(MOE_ERR_INVALID_ARG, "cache is NULL");
  if (!expert_ptr_dev) return failf(MOE_ERR_INVALID_ARG, "expert_ptr_dev is NULL");
  std::lock_guard<std::mutex> lk(c->mu);
  moe_status s = check_ids(c, layer, idx, n);
  if (s != MOE_OK) return s;
  DeviceGuard dg(c->device);
  cudaError_t err = cudaSuccess;
  // the slots of the previous resolve were read by the kernels enqueued on
  // this stream since: mark that point, and let them go
  for (int h : c->pol.release())
    if ((err = cudaEventRecord(c->used[h], st)) != cudaSuccess)
      return failf(MOE_ERR_CUDA, "CUDA error: %s", cudaGetErrorString(err));
  // staging buffer for the pointer table
  const int sb = c->stage_next;
  c->stage_next = (sb + 1) % kStage;
  if (c->stage_used[sb] && (err = cudaEventSynchronize(c->stage_ev[sb])) != cudaSuccess)
    return failf(MOE_ERR_CUDA, "CUDA error: %s", cudaGetErrorString(err));
  const void** tab = c->stage[sb];
  std::memset(tab, 0, sizeof(void*) * (size_t)c->E);
  for (int i = 0; i < n; ++i) {
    const int e = idx[i];
    if (tab[e]) continue;  // already resolved in this call
    bool fill = false;
    const int slot = c->pol.resolve(layer, e, &fill);
    if (slot < 0)
      return failf(MOE_ERR_OOM, "the cache's %d slots cannot hold the distinct experts of one call", c->S);
    if (fill) {
      if ((s = fill_slot(c, slot, layer, e, st)) != MOE_OK) {
        --c->pol.misses;  // not issued
        c->pol.release();  // no layer will read this call's slots
        return s;
      }
    } else if ((err = cudaStreamWaitEvent(st, c->ready[slot], 0)) != cudaSuccess) {
      c->pol.release();
      return failf(MOE_ERR_CUDA, "CUDA error: %s", cudaGetErrorString(err));
    }
    tab[e] = c->slots + (size_t)slot * c->blob;
  }
  if ((err = cudaMemcpyAsync(expert_ptr_dev, tab, sizeof(void*) * (size_t)c->E, cudaMemcpyHostToDevice, st)) !=
          cudaSuccess ||
      (err = cudaEventRecord(c->stage_ev[sb], st)) != cudaSuccess)
    return failf(MOE_ERR_CUDA, "CUDA error: %s", cudaGetErrorString(err));
  c->stage_used[sb] = true;
  return MOE_OK;
}

moe_status moe_stream_inject_fault(moe_stream_cache* c, int what, int countdown) {
  if (what == MOE_FAULT_NONE) {
    if (c) {
      std::lock_guard<std::mutex> lk(c->mu);
      c->fault_copy = -1;
    }
    std::lock_guard<std::mutex> lk(g_fault_mu);
    g_fault_alloc = 0;
    return MOE_OK;
  }
  if (what == MOE_FAULT_COPY) {
    if (!c || countdown < 0) return failf(MOE_ERR_INVALID_ARG, "a copy fault needs a cache and a countdown >= 0");
    std::lock_guard<std::mutex> lk(c->mu);
    c->fault_copy = countdown;
    return MOE_OK;
  }
  if (what == MOE_FAULT_ALLOC) {
    std::lock_guard<std::mutex> lk(g_fault_mu);
    g_fault_alloc = 1;
    return MOE_OK;
  }
  return failf(MOE_ERR_INVALID_ARG, "unknown fault %d", what);
}

moe_status moe_stream_stats(const moe_stream_cache* c, moe_stream_counters* out) {
  if (!c || !out) return failf(MOE_ERR_INVALID_ARG, "NULL pointer");
  std::lock_guard<std::mutex> lk(const_cast<moe_stream_cache*>(c)->mu);
  const moe::StreamPolicy& p = c->pol;
  out->hits = p.hits;
  out->misses = p.misses;
  out->prefetches = p.prefetches;
  out->prefetch_hits = p.prefetch_hits;
  out->prefetch_dropped = p.prefetch_dropped;
  out->bytes_h2d = c->bytes_h2d;
  return MOE_OK;
}

void moe_stream_destroy(moe_stream_cache* c) {
  if (!c) return;
  {
    DeviceGuard dg(c->device);
    cudaDeviceSynchronize();
    destroy_parts(c);
  }
  delete c;
}

}  // extern "C"
