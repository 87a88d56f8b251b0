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
// Device-resolved caches (moe_stream_resolve_device) keep the same policy on
// the GPU instead: a slot table [layer][expert] -> slot, the key and the last
// use of every slot, and counters, all in device memory, updated by one
// single-block kernel per call; the misses are then copied by a grid of
// blocks reading the mapped host store.  The routing never leaves the device
// and no host thread waits.
//
// Failures: a copy that cannot be enqueued (MOE_ERR_IO) leaves its slot
// empty, and a resolve that fails releases the slots it took, so the next
// call starts from a consistent cache.  Tests drive these paths with
// moe_stream_inject_fault (a host-side countdown that makes a chosen copy,
// or the next create's slot allocation, report failure without touching
// the GPU).
#include <cuda_runtime.h>

#include <fcntl.h>
#include <sys/stat.h>
#include <unistd.h>

#include <algorithm>
#include <cerrno>
#include <chrono>
#include <condition_variable>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <deque>
#include <functional>
#include <mutex>
#include <thread>
#include <utility>
#include <vector>

#include "../../include/moe.h"
#include "moe_kernels.h"
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

namespace {

// A fixed pool of host threads that run the reads of one call in parallel
// (the pages read the K chosen experts of a layer with parallel pread).
struct IoPool {
  std::vector<std::thread> th;
  std::mutex m;
  std::condition_variable cv, done;
  std::deque<std::function<void()>> q;
  int pending = 0;
  bool stop = false;

  void start(int n) {
    for (int i = 0; i < n; ++i)
      th.emplace_back([this] {
        for (;;) {
          std::function<void()> job;
          {
            std::unique_lock<std::mutex> lk(m);
            cv.wait(lk, [this] { return stop || !q.empty(); });
            if (stop && q.empty()) return;
            job = std::move(q.front());
            q.pop_front();
          }
          job();
          std::lock_guard<std::mutex> lk(m);
          if (--pending == 0) done.notify_all();
        }
      });
  }
  // runs the jobs on the pool and returns when all of them have finished
  void run(std::vector<std::function<void()>>& jobs) {
    if (jobs.empty()) return;
    {
      std::lock_guard<std::mutex> lk(m);
      for (auto& j : jobs) q.push_back(std::move(j));
      pending += (int)jobs.size();
    }
    cv.notify_all();
    std::unique_lock<std::mutex> lk(m);
    done.wait(lk, [this] { return pending == 0; });
  }
  void shutdown() {
    {
      std::lock_guard<std::mutex> lk(m);
      stop = true;
    }
    cv.notify_all();
    for (auto& t : th) t.join();
    th.clear();
  }
};

// Reads `bytes` at `off` of fd into dst, retrying short reads; false on error.
bool read_full(int fd, uint8_t* dst, size_t bytes, off_t off) {
  size_t got = 0;
  while (got < bytes) {
    const ssize_t r = pread(fd, dst + got, bytes - got, off + (off_t)got);
    if (r < 0 && errno == EINTR) continue;
    if (r <= 0) return false;
    got += (size_t)r;
  }
  return true;
}

constexpr int kFileStage = 16;  // pinned staging buffers of a file-backed store

}  // namespace

namespace moe {
namespace {
constexpr int kMaxResolveIds = 64;  // ids of one device-resolved call
struct DevTables {
  int32_t* slot_of = nullptr;  // [L * E] -> slot, or -1
  int32_t* key = nullptr;      // [S] -> layer * E + expert, or -1
  uint64_t* tick = nullptr;    // [S] last use
  uint64_t* ctr = nullptr;     // [DC_N]
  int32_t* jobs = nullptr;     // [2 * kMaxResolveIds]: slot, then key, of each fill
  int32_t* njobs = nullptr;    // [1]
};
}  // namespace
}  // namespace moe

struct moe_stream_cache {
  int L = 0, E = 0, S = 0;
  int mode = 0;                        // 0 unused, 1 host-resolved, 2 device-resolved
  int sms = 0;                         // the device's SM count (fill grid)
  moe::DevTables dt;                   // device-resolved state (pinned stores only)
  const uint8_t* host_dev = nullptr;   // the store as the device addresses it
  uint64_t dev_seen_ns = 0, dev_seen_bytes = 0, dev_seen_fills = 0;  // copy timing already reported
  size_t blob = 0;
  int device = 0;
  const uint8_t* host = nullptr;  // pinned host store, or null for a file store
  // file store: the file, pinned staging buffers (each reused once the copy
  // that last read it is done), the read pool, and read statistics
  int fd = -1;
  uint8_t* fstage[kFileStage] = {};
  cudaEvent_t fstage_ev[kFileStage] = {};
  bool fstage_used[kFileStage] = {};
  int fstage_next = 0;
  IoPool io;
  uint64_t reads = 0, read_ns = 0, read_bytes = 0;
  uint8_t* slots = nullptr;
  moe::StreamPolicy pol;
  std::vector<cudaEvent_t> ready, used;
  const void** stage[kStage] = {};
  cudaEvent_t stage_ev[kStage] = {};
  bool stage_used[kStage] = {};
  int stage_next = 0;
  uint64_t bytes_h2d = 0;
  int fault_copy = -1;  // injected: copies left before one fails (-1: none)
  // optional copy timing: an event pair around each copy, relative to `ref`
  bool timing = false;
  bool ref_recorded = false;
  cudaEvent_t ref = nullptr;
  std::vector<std::pair<cudaEvent_t, cudaEvent_t>> timed;
  std::vector<cudaEvent_t> spare;
  uint64_t timed_bytes = 0;
  std::mutex mu;
};

namespace {
int g_fault_alloc = 0;  // injected: the next create's slot allocation fails
std::mutex g_fault_mu;
}  // namespace

namespace {

cudaEvent_t take_event(moe_stream_cache* c) {
  if (!c->spare.empty()) {
    cudaEvent_t e = c->spare.back();
    c->spare.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  if (cudaEventCreate(&e) != cudaSuccess) {
    cudaGetLastError();
    return nullptr;
  }
  return e;
}

void destroy_parts(moe_stream_cache* c) {
  c->io.shutdown();
  for (int i = 0; i < kFileStage; ++i) {
    if (c->fstage_ev[i]) cudaEventDestroy(c->fstage_ev[i]);
    if (c->fstage[i]) cudaFreeHost(c->fstage[i]);
  }
  if (c->fd >= 0) close(c->fd);
  for (auto& pr : c->timed) {
    cudaEventDestroy(pr.first);
    cudaEventDestroy(pr.second);
  }
  for (cudaEvent_t e : c->spare) cudaEventDestroy(e);
  if (c->ref) cudaEventDestroy(c->ref);
  for (cudaEvent_t e : c->ready)
    if (e) cudaEventDestroy(e);
  for (cudaEvent_t e : c->used)
    if (e) cudaEventDestroy(e);
  for (int i = 0; i < kStage; ++i) {
    if (c->stage_ev[i]) cudaEventDestroy(c->stage_ev[i]);
    if (c->stage[i]) cudaFreeHost(c->stage[i]);
  }
  if (c->slots) cudaFree(c->slots);
  void* dts[] = {c->dt.slot_of, c->dt.key, c->dt.tick, c->dt.ctr, c->dt.jobs, c->dt.njobs};
  for (void* q : dts)
    if (q) cudaFree(q);
}

// Enqueue the copy of (layer, e) into slot s on stream st (see the ordering
// rules at the top of the file); the policy has already assigned the slot.
moe_status fill_slot(moe_stream_cache* c, int s, int layer, int e, cudaStream_t st, const uint8_t* src_stage = nullptr) {
  cudaError_t err = cudaStreamWaitEvent(st, c->used[s], 0);
  if (err == cudaSuccess) err = cudaStreamWaitEvent(st, c->ready[s], 0);
  if (err != cudaSuccess) return failf(MOE_ERR_CUDA, "CUDA error: %s", cudaGetErrorString(err));
  const uint8_t* src = src_stage ? src_stage : c->host + ((size_t)layer * c->E + e) * c->blob;
  if (c->fault_copy >= 0 && c->fault_copy-- == 0) {
    c->pol.evict(s);
    return failf(MOE_ERR_IO, "copy of expert %d of layer %d from the host store failed: injected fault", e, layer);
  }
  cudaEvent_t tb = nullptr, te = nullptr;
  if (c->timing) {
    if (!c->ref_recorded && cudaEventRecord(c->ref, st) == cudaSuccess) c->ref_recorded = true;
    tb = take_event(c);
    te = take_event(c);
    if (tb && te && c->ref_recorded) {
      cudaEventRecord(tb, st);
    } else {
      if (tb) c->spare.push_back(tb);
      if (te) c->spare.push_back(te);
      tb = te = nullptr;
    }
  }
  err = cudaMemcpyAsync(c->slots + (size_t)s * c->blob, src, c->blob, cudaMemcpyHostToDevice, st);
  if (tb) {
    cudaEventRecord(te, st);
    c->timed.emplace_back(tb, te);
    c->timed_bytes += c->blob;
  }
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

struct Fill {
  int slot, layer, e;
};

// Issues the fills of one call.  A pinned store is copied from directly.  A
// file store first reads every blob of the call into its own pinned staging
// buffer, in parallel on the read pool, then enqueues the copies; a staging
// buffer is reused once the copy that last read it has completed (the host
// waits for that).  On failure, the slots of the fills not issued are left
// empty and *issued says how many fills were enqueued.
moe_status do_fills(moe_stream_cache* c, const std::vector<Fill>& fills, cudaStream_t st, int* issued) {
  *issued = 0;
  if (c->fd < 0) {
    for (const Fill& f : fills) {
      const moe_status s = fill_slot(c, f.slot, f.layer, f.e, st);
      if (s != MOE_OK) {
        for (size_t k = *issued + 1; k < fills.size(); ++k) c->pol.evict(fills[k].slot);
        return s;
      }
      ++*issued;
    }
    return MOE_OK;
  }
  for (size_t b0 = 0; b0 < fills.size(); b0 += kFileStage) {
    const size_t nb = std::min(fills.size() - b0, (size_t)kFileStage);
    std::vector<int> sb(nb);
    for (size_t k = 0; k < nb; ++k) {
      const int i = c->fstage_next;
      c->fstage_next = (i + 1) % kFileStage;
      if (c->fstage_used[i]) {
        const cudaError_t err = cudaEventSynchronize(c->fstage_ev[i]);
        if (err != cudaSuccess) return failf(MOE_ERR_CUDA, "CUDA error: %s", cudaGetErrorString(err));
      }
      sb[k] = i;
    }
    std::vector<char> okv(nb, 0);
    std::vector<std::function<void()>> jobs;
    const uint64_t t0 = (uint64_t)std::chrono::duration_cast<std::chrono::nanoseconds>(
                            std::chrono::steady_clock::now().time_since_epoch()).count();
    for (size_t k = 0; k < nb; ++k) {
      const Fill f = fills[b0 + k];
      uint8_t* dst = c->fstage[sb[k]];
      const off_t off = (off_t)(((size_t)f.layer * c->E + f.e) * c->blob);
      const int fd = c->fd;
      const size_t bytes = c->blob;
      char* okp = &okv[k];
      jobs.push_back([fd, dst, bytes, off, okp] { *okp = read_full(fd, dst, bytes, off) ? 1 : 0; });
    }
    c->io.run(jobs);
    const uint64_t t1 = (uint64_t)std::chrono::duration_cast<std::chrono::nanoseconds>(
                            std::chrono::steady_clock::now().time_since_epoch()).count();
    c->reads += nb;
    c->read_bytes += nb * c->blob;
    c->read_ns += t1 - t0;
    for (size_t k = 0; k < nb; ++k) {
      const Fill& f = fills[b0 + k];
      moe_status s = MOE_OK;
      if (!okv[k]) {
        c->pol.evict(f.slot);
        s = failf(MOE_ERR_IO, "read of expert %d of layer %d from the store file failed", f.e, f.layer);
      } else {
        s = fill_slot(c, f.slot, f.layer, f.e, st, c->fstage[sb[k]]);
      }
      if (s == MOE_OK) {
        const cudaError_t err = cudaEventRecord(c->fstage_ev[sb[k]], st);
        if (err != cudaSuccess) s = failf(MOE_ERR_CUDA, "CUDA error: %s", cudaGetErrorString(err));
        c->fstage_used[sb[k]] = true;
      }
      if (s != MOE_OK) {
        for (size_t j = b0 + k + 1; j < fills.size(); ++j) c->pol.evict(fills[j].slot);
        return s;
      }
      ++*issued;
    }
  }
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

// The part of creating a cache common to both stores: the policy, the slots
// (the library's one device allocation), the per-slot events and the pinned
// staging ring of the pointer table.  Takes ownership of c.
moe_status finish_create(moe_stream_cache* c, const moe_config* cfg, int n_layers, int n_slots,
                         moe_stream_cache** out) {
  const size_t blob = moe_packed_expert_bytes(cfg);
  c->L = n_layers;
  c->E = cfg->n_experts;
  c->S = n_slots;
  c->blob = blob;
  cudaGetDevice(&c->device);
  c->pol.init(n_layers, cfg->n_experts, n_slots);
  cudaDeviceGetAttribute(&c->sms, cudaDevAttrMultiProcessorCount, c->device);
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
  if (c->host) {
    // the device-resolved state: the tables start empty (all -1), the
    // counters at zero; and the store's device address, if it is mapped
    moe::DevTables& t = c->dt;
    const size_t le = (size_t)n_layers * cfg->n_experts;
    okk = cudaMalloc(&t.slot_of, 4 * le) == cudaSuccess && cudaMalloc(&t.key, 4ull * n_slots) == cudaSuccess &&
          cudaMalloc(&t.tick, 8ull * n_slots) == cudaSuccess && cudaMalloc(&t.ctr, 8ull * moe::DC_N) == cudaSuccess &&
          cudaMalloc(&t.jobs, 8ull * moe::kMaxResolveIds) == cudaSuccess &&
          cudaMalloc(&t.njobs, 16) == cudaSuccess && cudaMemset(t.slot_of, 0xff, 4 * le) == cudaSuccess &&
          cudaMemset(t.key, 0xff, 4ull * n_slots) == cudaSuccess &&
          cudaMemset(t.tick, 0, 8ull * n_slots) == cudaSuccess && cudaMemset(t.njobs, 0, 16) == cudaSuccess;
    if (okk) {
      uint64_t c0[moe::DC_N] = {};
      c0[moe::DC_FILL_T0] = ~0ull;  // a running minimum
      okk = cudaMemcpy(t.ctr, c0, sizeof(c0), cudaMemcpyHostToDevice) == cudaSuccess &&
            cudaDeviceSynchronize() == cudaSuccess;
    }
    if (!okk) {
      cudaGetLastError();
      destroy_parts(c);
      delete c;
      return failf(MOE_ERR_OOM, "could not allocate the cache's device tables");
    }
    void* hd = nullptr;
    if (cudaHostGetDevicePointer(&hd, const_cast<uint8_t*>(c->host), 0) == cudaSuccess)
      c->host_dev = static_cast<const uint8_t*>(hd);
    else
      cudaGetLastError();  // not mapped: the device-resolved calls are unavailable
  }
  *out = c;
  return MOE_OK;
}

// ---- device-resolved calls -----------------------------------------------------------

// One block: the distinct ids of the call, in order, each looked up in the
// slot table; a miss takes an empty slot (lowest index) or else the least
// recently used slot not taken by this call (the same choice as
// StreamPolicy), found by a block-wide reduction.  Table pointers are
// written only when every id found a slot.
__global__ void __launch_bounds__(1024) stream_resolve_kernel(moe::DevTables t, int E, int S, int layer,
                                                              const int32_t* __restrict__ idx, int n,
                                                              const void** __restrict__ eptr, uint8_t* slots,
                                                              size_t blob) {
  extern __shared__ uint32_t held[];  // [(S + 31) / 32] bits: slots taken by this call
  __shared__ int s_ids[moe::kMaxResolveIds], s_slot[moe::kMaxResolveIds], s_look[moe::kMaxResolveIds];
  __shared__ unsigned long long s_tick[moe::kMaxResolveIds];
  __shared__ int s_jobslot[moe::kMaxResolveIds];  // slots this call's misses took
  __shared__ int s_cur, s_abort, s_nj;
  __shared__ unsigned long long s_red[32], s_clock;
  __shared__ int s_redi[32];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nw = blockDim.x >> 5;
  const int nwords = (S + 31) / 32;
  uint64_t* ctr = t.ctr;
  for (int i = tid; i < nwords; i += blockDim.x) held[i] = 0u;
  // every id's table entry in one round trip (thread i looks up id i)
  if (tid < n) {
    const int e = idx[tid];
    s_ids[tid] = e;
    s_look[tid] = (e >= 0 && e < E) ? t.slot_of[(size_t)layer * E + e] : -2;  // -2: invalid id
    s_tick[tid] = 0ull;
  }
  if (tid == 0) {
    s_abort = 0;
    s_nj = 0;
    s_clock = ctr[moe::DC_CLOCK];
  }
  __syncthreads();
#pragma unroll 1
  for (int i = 0; i < n; ++i) {
    if (tid == 0) {
      const int e = s_ids[i];
      int sl = s_look[i];
      // an id seen earlier in this call may have been mapped by a miss since,
      // and a slot looked up before the loop may have been taken by one
      if (sl != -2) {
        for (int j = 0; j < s_nj; ++j)
          if (s_jobslot[j] == sl) sl = -1;
        for (int q = 0; q < i; ++q)
          if (s_ids[q] == e) sl = s_slot[q];
      }
      if (sl >= 0 && !(held[sl >> 5] >> (sl & 31) & 1u)) {
        held[sl >> 5] |= 1u << (sl & 31);
        s_tick[i] = ++s_clock;  // written to the table after the loop
        ++ctr[moe::DC_HITS];
      }
      s_slot[i] = sl;
      s_cur = sl;
    }
    __syncthreads();
    if (s_cur != -1) continue;  // a hit, a repeat or an invalid id (uniform)
    // a miss: the lowest empty slot not taken, else the least recently used
    int be = 0x7fffffff;
    unsigned long long bl = ~0ull;
    for (int j = tid; j < S; j += blockDim.x) {
      if (held[j >> 5] >> (j & 31) & 1u) continue;
      if (t.key[j] < 0) {
        be = min(be, j);
      } else {
        const unsigned long long k = ((unsigned long long)t.tick[j] << 24) | (unsigned long long)j;
        bl = k < bl ? k : bl;
      }
    }
    for (int o = 16; o > 0; o >>= 1) {
      be = min(be, __shfl_xor_sync(0xffffffffu, be, o));
      const unsigned long long ob = __shfl_xor_sync(0xffffffffu, bl, o);
      bl = ob < bl ? ob : bl;
    }
    if (lane == 0) {
      s_redi[warp] = be;
      s_red[warp] = bl;
    }
    __syncthreads();
    if (tid == 0) {
      int b = 0x7fffffff;
      unsigned long long l = ~0ull;
      for (int w = 0; w < nw; ++w) {
        b = min(b, s_redi[w]);
        l = s_red[w] < l ? s_red[w] : l;
      }
      const int v = b != 0x7fffffff ? b : (l != ~0ull ? (int)(l & 0xffffffull) : -1);
      if (v < 0) {
        s_abort = 1;
        if (ctr[moe::DC_ERROR] == 0) ctr[moe::DC_ERROR] = MOE_ERR_OOM;
      } else {
        const int e = s_ids[i];
        const int32_t kv = t.key[v];
        if (kv >= 0) t.slot_of[kv] = -1;
        t.key[v] = layer * E + e;
        t.slot_of[(size_t)layer * E + e] = v;
        held[v >> 5] |= 1u << (v & 31);
        t.tick[v] = ++s_clock;
        ++ctr[moe::DC_MISSES];
        t.jobs[s_nj] = v;
        t.jobs[moe::kMaxResolveIds + s_nj] = layer * E + e;
        s_jobslot[s_nj] = v;
        ++s_nj;
        s_slot[i] = v;
      }
    }
    __syncthreads();
    if (s_abort) break;
  }
  if (tid == 0) {
    if (s_abort) {
      // undo this call's assignments: their slots were never filled (the
      // experts they held before are gone, as on the host)
      for (int j = 0; j < s_nj; ++j) {
        t.slot_of[t.jobs[moe::kMaxResolveIds + j]] = -1;
        t.key[t.jobs[j]] = -1;
      }
      ctr[moe::DC_MISSES] -= (uint64_t)s_nj;
    }
    *t.njobs = s_abort ? 0 : s_nj;
    ctr[moe::DC_CLOCK] = s_clock;
  }
  __syncthreads();
  // the hits' new last-use ticks and the pointer table, one id per thread
  if (!s_abort && tid < n) {
    const int e = s_ids[tid];
    const int sl = s_slot[tid];
    if (s_tick[tid] != 0ull) t.tick[sl] = s_tick[tid];
    if (sl >= 0) eptr[e] = slots + (size_t)sl * blob;
  }
}

// Copies the fills of the last resolve from the mapped host store into their
// slots, 16 bytes per load, four loads in flight per thread; returns at once
// when nothing missed.  The last block to finish adds the bytes and the
// span of the copy (device timestamps) to the counters.
__global__ void __launch_bounds__(256) stream_fill_kernel(moe::DevTables t, const uint8_t* __restrict__ host,
                                                          uint8_t* slots, size_t blob) {
  const int nj = *t.njobs;
  if (nj == 0) return;
  uint64_t* ctr = t.ctr;
  __shared__ int s_last;
  if (threadIdx.x == 0) {
    uint64_t now;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(now));
    atomicMin(reinterpret_cast<unsigned long long*>(&ctr[moe::DC_FILL_T0]), (unsigned long long)now);
  }
  const size_t per = blob / 16;
  const size_t total = (size_t)nj * per;
  const size_t stride = (size_t)gridDim.x * blockDim.x;
  for (size_t u0 = (size_t)blockIdx.x * blockDim.x + threadIdx.x; u0 < total; u0 += 4 * stride) {
    uint4 v[4];
    size_t dst[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const size_t u = u0 + (size_t)k * stride;
      if (u < total) {
        const size_t j = u / per, off = u - j * per;
        const size_t src = (size_t)t.jobs[moe::kMaxResolveIds + j] * blob + 16 * off;
        v[k] = *reinterpret_cast<const uint4*>(host + src);
        dst[k] = (size_t)t.jobs[j] * blob + 16 * off;
      } else {
        dst[k] = ~size_t(0);
      }
    }
#pragma unroll
    for (int k = 0; k < 4; ++k)
      if (dst[k] != ~size_t(0)) *reinterpret_cast<uint4*>(slots + dst[k]) = v[k];
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    uint64_t now;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(now));
    atomicMax(reinterpret_cast<unsigned long long*>(&ctr[moe::DC_FILL_T1]), (unsigned long long)now);
    __threadfence();
    s_last = atomicAdd(reinterpret_cast<unsigned long long*>(&ctr[moe::DC_FILL_DONE]), 1ull) ==
             (unsigned long long)gridDim.x - 1ull;
  }
  __syncthreads();
  if (s_last && threadIdx.x == 0) {
    __threadfence();
    volatile uint64_t* vc = ctr;
    vc[moe::DC_FILL_NS] += vc[moe::DC_FILL_T1] - vc[moe::DC_FILL_T0];
    vc[moe::DC_BYTES] += (uint64_t)nj * blob;
    vc[moe::DC_FILLS] += 1;
    vc[moe::DC_FILL_T0] = ~0ull;
    vc[moe::DC_FILL_T1] = 0;
    vc[moe::DC_FILL_DONE] = 0;
  }
}

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
  c->host = static_cast<const uint8_t*>(host_pinned_experts);
  return finish_create(c, cfg, n_layers, n_slots, out);
}

moe_status moe_stream_create_file(const moe_config* cfg, int n_layers, const char* path, int direct_io, int n_slots,
                                  int n_read_threads, moe_stream_cache** out) {
  if (!out) return failf(MOE_ERR_INVALID_ARG, "out is NULL");
  *out = nullptr;
  if (!cfg) return failf(MOE_ERR_INVALID_ARG, "cfg is NULL");
  const size_t blob = moe_packed_expert_bytes(cfg);
  if (blob == 0 || cfg->n_experts <= 0) return failf(MOE_ERR_UNSUPPORTED, "unsupported shape");
  if (n_layers < 1 || n_slots < 1 || n_read_threads < 1 || n_read_threads > 64)
    return failf(MOE_ERR_INVALID_ARG, "n_layers and n_slots must be >= 1, n_read_threads in [1, 64]");
  if (!path) return failf(MOE_ERR_INVALID_ARG, "path is NULL");
  if (direct_io && blob % 4096)
    return failf(MOE_ERR_UNSUPPORTED, "direct reads need blobs of a multiple of 4096 bytes (this shape: %zu)", blob);
  const int fd = open(path, O_RDONLY | (direct_io ? O_DIRECT : 0));
  if (fd < 0) return failf(MOE_ERR_IO, "cannot open the store file %s: %s", path, strerror(errno));
  struct stat sb;
  const size_t need = blob * (size_t)cfg->n_experts * (size_t)n_layers;
  if (fstat(fd, &sb) != 0 || (size_t)sb.st_size < need) {
    close(fd);
    return failf(MOE_ERR_INVALID_ARG, "the store file holds %lld bytes; %d layers of %d experts need %zu",
                 (long long)sb.st_size, n_layers, cfg->n_experts, need);
  }
  moe_stream_cache* c = new moe_stream_cache;
  c->fd = fd;
  bool okk = true;
  for (int i = 0; i < kFileStage && okk; ++i)
    okk = cudaHostAlloc(reinterpret_cast<void**>(&c->fstage[i]), blob, cudaHostAllocDefault) == cudaSuccess &&
          cudaEventCreateWithFlags(&c->fstage_ev[i], cudaEventDisableTiming) == cudaSuccess;
  if (!okk) {
    cudaGetLastError();
    destroy_parts(c);
    delete c;
    return failf(MOE_ERR_OOM, "could not allocate the store file's pinned staging buffers");
  }
  c->io.start(n_read_threads);
  return finish_create(c, cfg, n_layers, n_slots, out);
}

moe_status moe_stream_file_stats(const moe_stream_cache* c, uint64_t* reads, uint64_t* read_bytes,
                                 double* read_ms) {
  if (!c) return failf(MOE_ERR_INVALID_ARG, "cache is NULL");
  std::lock_guard<std::mutex> lk(const_cast<moe_stream_cache*>(c)->mu);
  if (reads) *reads = c->reads;
  if (read_bytes) *read_bytes = c->read_bytes;
  if (read_ms) *read_ms = (double)c->read_ns * 1e-6;
  return MOE_OK;
}

moe_status moe_stream_prefetch(moe_stream_cache* c, int layer, const int32_t* ids, int n, cudaStream_t copy_stream) {
  if (!c) return failf(MOE_ERR_INVALID_ARG, "cache is NULL");
  std::lock_guard<std::mutex> lk(c->mu);
  if (c->mode == 2) return failf(MOE_ERR_INVALID_ARG, "this cache is resolved on the device");
  c->mode = 1;
  moe_status s = check_ids(c, layer, ids, n);
  if (s != MOE_OK) return s;
  DeviceGuard dg(c->device);
  std::vector<Fill> fills;
  for (int i = 0; i < n; ++i) {
    const int v = c->pol.prefetch(layer, ids[i]);
    if (v >= 0) fills.push_back(Fill{v, layer, ids[i]});
  }
  int issued = 0;
  s = do_fills(c, fills, copy_stream, &issued);
  if (s != MOE_OK) c->pol.prefetches -= (uint64_t)(fills.size() - issued);  // not issued
  return s;
}

moe_status moe_stream_resolve(moe_stream_cache* c, int layer, const int32_t* idx, int n, const void** expert_ptr_dev,
                              cudaStream_t st) {
  if (!c) return failf(MOE_ERR_INVALID_ARG, "cache is NULL");
  if (!expert_ptr_dev) return failf(MOE_ERR_INVALID_ARG, "expert_ptr_dev is NULL");
  std::lock_guard<std::mutex> lk(c->mu);
  if (c->mode == 2) return failf(MOE_ERR_INVALID_ARG, "this cache is resolved on the device");
  c->mode = 1;
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
  std::vector<Fill> fills;
  for (int i = 0; i < n; ++i) {
    const int e = idx[i];
    if (tab[e]) continue;  // already resolved in this call
    bool fill = false;
    const int slot = c->pol.resolve(layer, e, &fill);
    if (slot < 0) {
      for (const Fill& f : fills) c->pol.evict(f.slot);
      c->pol.misses -= fills.size();
      c->pol.release();
      return failf(MOE_ERR_OOM, "the cache's %d slots cannot hold the distinct experts of one call", c->S);
    }
    if (fill) {
      fills.push_back(Fill{slot, layer, e});
    } else if ((err = cudaStreamWaitEvent(st, c->ready[slot], 0)) != cudaSuccess) {
      for (const Fill& f : fills) c->pol.evict(f.slot);
      c->pol.misses -= fills.size();
      c->pol.release();
      return failf(MOE_ERR_CUDA, "CUDA error: %s", cudaGetErrorString(err));
    }
    tab[e] = c->slots + (size_t)slot * c->blob;
  }
  int issued = 0;
  if ((s = do_fills(c, fills, st, &issued)) != MOE_OK) {
    c->pol.misses -= (uint64_t)(fills.size() - issued);  // not issued
    c->pol.release();  // no layer will read this call's slots
    return s;
  }
  if ((err = cudaMemcpyAsync(expert_ptr_dev, tab, sizeof(void*) * (size_t)c->E, cudaMemcpyHostToDevice, st)) !=
          cudaSuccess ||
      (err = cudaEventRecord(c->stage_ev[sb], st)) != cudaSuccess)
    return failf(MOE_ERR_CUDA, "CUDA error: %s", cudaGetErrorString(err));
  c->stage_used[sb] = true;
  return MOE_OK;
}

moe_status moe_stream_resolve_device(moe_stream_cache* c, int layer, const int32_t* idx_dev, int n,
                                     const void** expert_ptr_dev, cudaStream_t st) {
  if (!c) return failf(MOE_ERR_INVALID_ARG, "cache is NULL");
  if (!expert_ptr_dev || (n > 0 && !idx_dev)) return failf(MOE_ERR_INVALID_ARG, "NULL pointer");
  if (n < 0 || n > moe::kMaxResolveIds)
    return failf(MOE_ERR_INVALID_ARG, "n = %d: a device resolve takes 0..%d ids", n, moe::kMaxResolveIds);
  if (layer < 0 || layer >= c->L) return failf(MOE_ERR_INVALID_ARG, "layer %d outside [0, %d)", layer, c->L);
  std::lock_guard<std::mutex> lk(c->mu);
  if (!c->host || !c->host_dev)
    return failf(MOE_ERR_UNSUPPORTED, "device resolves need a pinned host store the device can map");
  if (c->mode == 1) return failf(MOE_ERR_INVALID_ARG, "this cache is resolved on the host");
  c->mode = 2;
  if (n == 0) return MOE_OK;
  DeviceGuard dg(c->device);
  const size_t held = 4ull * ((size_t)(c->S + 31) / 32);
  if (held > 48 * 1024) return failf(MOE_ERR_UNSUPPORTED, "more than %d slots", 48 * 1024 * 8);
  stream_resolve_kernel<<<1, 1024, held, st>>>(c->dt, c->E, c->S, layer, idx_dev, n, expert_ptr_dev, c->slots,
                                               c->blob);
  cudaError_t err = cudaGetLastError();
  if (err == cudaSuccess) {
    const int grid = c->sms > 0 ? 4 * c->sms : 256;
    stream_fill_kernel<<<grid, 256, 0, st>>>(c->dt, c->host_dev, c->slots, c->blob);
    err = cudaGetLastError();
  }
  if (err != cudaSuccess) return failf(MOE_ERR_CUDA, "CUDA error: %s", cudaGetErrorString(err));
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

moe_status moe_stream_enable_copy_timing(moe_stream_cache* c, int on) {
  if (!c) return failf(MOE_ERR_INVALID_ARG, "cache is NULL");
  std::lock_guard<std::mutex> lk(c->mu);
  DeviceGuard dg(c->device);
  if (on && !c->ref && cudaEventCreate(&c->ref) != cudaSuccess) {
    cudaGetLastError();
    return failf(MOE_ERR_OOM, "could not create a timing event");
  }
  c->timing = on != 0;
  return MOE_OK;
}

moe_status moe_stream_copy_timing(moe_stream_cache* c, moe_stream_copy_times* out) {
  if (!c || !out) return failf(MOE_ERR_INVALID_ARG, "NULL pointer");
  std::lock_guard<std::mutex> lk(c->mu);
  DeviceGuard dg(c->device);
  if (c->mode == 2) {
    // the fill kernels' own spans and bytes since the last call
    uint64_t v[moe::DC_N];
    const cudaError_t err = cudaDeviceSynchronize();
    if (err != cudaSuccess || cudaMemcpy(v, c->dt.ctr, sizeof(v), cudaMemcpyDeviceToHost) != cudaSuccess)
      return failf(MOE_ERR_CUDA, "CUDA error: %s", cudaGetErrorString(cudaGetLastError()));
    out->busy_ms = (double)(v[moe::DC_FILL_NS] - c->dev_seen_ns) * 1e-6;
    out->copy_ms = out->busy_ms;
    out->copies = v[moe::DC_FILLS] - c->dev_seen_fills;
    out->bytes = v[moe::DC_BYTES] - c->dev_seen_bytes;
    c->dev_seen_ns = v[moe::DC_FILL_NS];
    c->dev_seen_fills = v[moe::DC_FILLS];
    c->dev_seen_bytes = v[moe::DC_BYTES];
    return MOE_OK;
  }
  std::vector<std::pair<double, double>> iv;
  double sum = 0.0;
  for (auto& pr : c->timed) {
    float a = 0.f, b = 0.f;
    cudaError_t err = cudaEventSynchronize(pr.second);
    if (err == cudaSuccess) err = cudaEventElapsedTime(&a, c->ref, pr.first);
    if (err == cudaSuccess) err = cudaEventElapsedTime(&b, c->ref, pr.second);
    if (err != cudaSuccess) return failf(MOE_ERR_CUDA, "CUDA error: %s", cudaGetErrorString(err));
    iv.emplace_back(a, b);
    sum += b - a;
  }
  std::sort(iv.begin(), iv.end());
  double busy = 0.0, cur_a = 0.0, cur_b = -1.0;
  for (auto& x : iv) {
    if (x.first > cur_b) {
      if (cur_b > cur_a) busy += cur_b - cur_a;
      cur_a = x.first;
      cur_b = x.second;
    } else if (x.second > cur_b) {
      cur_b = x.second;
    }
  }
  if (cur_b > cur_a) busy += cur_b - cur_a;
  out->busy_ms = busy;
  out->copy_ms = sum;
  out->copies = c->timed.size();
  out->bytes = c->timed_bytes;
  for (auto& pr : c->timed) {
    c->spare.push_back(pr.first);
    c->spare.push_back(pr.second);
  }
  c->timed.clear();
  c->timed_bytes = 0;
  return MOE_OK;
}

moe_status moe_stream_stats(const moe_stream_cache* c, moe_stream_counters* out) {
  if (!c || !out) return failf(MOE_ERR_INVALID_ARG, "NULL pointer");
  std::lock_guard<std::mutex> lk(const_cast<moe_stream_cache*>(c)->mu);
  out->device_error = 0;
  if (c->mode == 2) {
    uint64_t v[moe::DC_N];
    DeviceGuard dg(c->device);
    if (cudaDeviceSynchronize() != cudaSuccess ||
        cudaMemcpy(v, c->dt.ctr, sizeof(v), cudaMemcpyDeviceToHost) != cudaSuccess)
      return failf(MOE_ERR_CUDA, "CUDA error: %s", cudaGetErrorString(cudaGetLastError()));
    out->hits = v[moe::DC_HITS];
    out->misses = v[moe::DC_MISSES];
    out->prefetches = out->prefetch_hits = out->prefetch_dropped = 0;
    out->bytes_h2d = v[moe::DC_BYTES];
    out->device_error = v[moe::DC_ERROR];
    return MOE_OK;
  }
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

namespace moe {

// The fused kernel's view of a device-resolved cache for one streamed layer
// call (moe_layer_forward_streamed): the cache must hold a pinned store the
// device maps, serve the device-resolved protocol (an unused cache becomes
// device-resolved), live on the current device and hold blobs of
// `blob_bytes` for `E` experts per layer.
moe_status stream_view(moe_stream_cache* c, int layer, int E, uint64_t blob_bytes, StreamView* v) {
  if (!c || !v) return failf(MOE_ERR_INVALID_ARG, "cache is NULL");
  if (layer < 0 || layer >= c->L) return failf(MOE_ERR_INVALID_ARG, "layer %d outside [0, %d)", layer, c->L);
  std::lock_guard<std::mutex> lk(c->mu);
  if (!c->host || !c->host_dev || !c->dt.slot_of)
    return failf(MOE_ERR_UNSUPPORTED, "streamed layer calls need a pinned host store the device can map");
  if (c->mode == 1) return failf(MOE_ERR_INVALID_ARG, "this cache is resolved on the host");
  if (c->E != E || c->blob != blob_bytes)
    return failf(MOE_ERR_INVALID_ARG, "the cache holds %d experts of %zu bytes per layer, the layer %d of %llu",
                 c->E, c->blob, E, (unsigned long long)blob_bytes);
  int dev = -1;
  cudaGetDevice(&dev);
  if (dev != c->device) return failf(MOE_ERR_INVALID_ARG, "the cache lives on device %d, not %d", c->device, dev);
  c->mode = 2;
  v->slot_of = c->dt.slot_of;
  v->key = c->dt.key;
  v->tick = c->dt.tick;
  v->dctr = c->dt.ctr;
  v->host = c->host_dev;
  v->slots = c->slots;
  v->S = c->S;
  v->layer = layer;
  return MOE_OK;
}

}  // namespace moe
