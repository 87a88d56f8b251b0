// moe_stream_policy.h -- the decisions of the expert-streaming cache (host
// only, no CUDA): which (layer, expert) each device slot holds, the slot
// table [layer][expert] -> slot or -1, least-recently-used replacement, the
// slots held by the step in flight, and the hit / miss counters.  The
// streaming runtime (moe_stream.cu) issues the copies and events that these
// decisions call for; a host test drives this class directly.
#pragma once

#include <stdint.h>

#include <vector>

namespace moe {

struct StreamPolicy {
  int L = 0, E = 0, S = 0;
  std::vector<int32_t> table;  // [L][E] -> slot, or -1
  std::vector<int32_t> key;    // [S] -> layer * E + expert, or -1 (empty)
  std::vector<uint64_t> last;  // [S] tick of the last use
  std::vector<uint8_t> held;   // [S] handed out by the resolve call in flight
  std::vector<uint8_t> fresh;  // [S] filled by a prefetch, not yet resolved
  std::vector<int> held_list;  // the held slots, in the order they were handed out
  uint64_t tick = 0;
  uint64_t hits = 0, misses = 0, prefetches = 0, prefetch_hits = 0, prefetch_dropped = 0;

  void init(int n_layers, int n_experts, int n_slots) {
    L = n_layers;
    E = n_experts;
    S = n_slots;
    table.assign((size_t)L * E, -1);
    key.assign(S, -1);
    last.assign(S, 0);
    held.assign(S, 0);
    fresh.assign(S, 0);
    held_list.clear();
    tick = 0;
    hits = misses = prefetches = prefetch_hits = prefetch_dropped = 0;
  }
  int lookup(int layer, int e) const { return table[(size_t)layer * E + e]; }
  void touch(int s) { last[s] = ++tick; }
  // The slot to fill next: an empty slot if any (lowest index), else the
  // least recently used slot not held; -1 if every slot is held.
  int victim() const {
    int best = -1;
    for (int s = 0; s < S; ++s) {
      if (held[s]) continue;
      if (key[s] < 0) return s;
      if (best < 0 || last[s] < last[best]) best = s;
    }
    return best;
  }
  // Slot s now holds (layer, e).
  void assign(int s, int layer, int e) {
    if (key[s] >= 0) table[key[s]] = -1;
    key[s] = layer * E + e;
    table[(size_t)layer * E + e] = s;
    fresh[s] = 0;
  }
  // Slot s holds nothing valid any more (its fill could not be issued).
  void evict(int s) {
    if (key[s] >= 0) table[key[s]] = -1;
    key[s] = -1;
    fresh[s] = 0;
  }
  // Prefetch of (layer, e): the slot to fill, or -1 (already resident, which
  // counts as a use, or no slot free of the step in flight: dropped).
  int prefetch(int layer, int e) {
    int s = lookup(layer, e);
    if (s >= 0) {
      touch(s);
      return -1;
    }
    s = victim();
    if (s < 0) {
      ++prefetch_dropped;
      return -1;
    }
    assign(s, layer, e);
    fresh[s] = 1;
    touch(s);
    ++prefetches;
    return s;
  }
  // Start of a resolve call: the previous call's slots are no longer held.
  // Returns them (their last reader is the kernel enqueued since).
  std::vector<int> release() {
    std::vector<int> r;
    r.swap(held_list);
    for (int s : r) held[s] = 0;
    return r;
  }
  // Resolve (layer, e) in the current call: returns its slot and sets *fill
  // when the slot must be filled first (a miss); -1 if every slot is held.
  // An id already resolved in this call returns its slot again, uncounted.
  int resolve(int layer, int e, bool* fill) {
    *fill = false;
    int s = lookup(layer, e);
    if (s >= 0) {
      if (held[s]) return s;
      ++hits;
      if (fresh[s]) ++prefetch_hits;
      fresh[s] = 0;
    } else {
      s = victim();
      if (s < 0) return -1;
      assign(s, layer, e);
      ++misses;
      *fill = true;
    }
    held[s] = 1;
    held_list.push_back(s);
    touch(s);
    return s;
  }
};

}  // namespace moe
