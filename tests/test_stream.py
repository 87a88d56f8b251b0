"""The expert-streaming tier (moe_stream_*) and the routed layer call
(moe_layer_forward_routed).

- CPU: the cache's decisions (moe_stream_policy.h, compiled with g++ into a
  small driver) against RefCache, a separate model of the documented policy
  written here: an empty slot first, else the least recently used slot that
  the resolve call in flight does not hold; prefetch only fills free slots.
- CPU: argument checks of moe_stream_create that need no device.
- GPU: the routed call given the fused kernel's own routing reproduces
  moe_layer_forward bit for bit, and matches the oracle given the same
  routing; a multi-layer run through the cache (with evictions and
  prefetches on a side stream) reproduces the resident routed call bit for
  bit, and its counters equal RefCache's (invariant: streaming changes where
  the bytes come from, not the arithmetic).
"""
import os
import subprocess
from dataclasses import replace

import numpy as np
import pytest

import oracle as O
import synth as S
from layer_setup import (DeviceLayer, assert_outputs_close, from_dev_bits, mcfg, ocfg, oracle_forward,
                         to_dev_bits)

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "quantized_expert_ffn_03_b200", "csrc")


@pytest.fixture(scope="module")
def M():
    import quantized_expert_ffn_03_b200 as M
    return M


class RefCache:
    """Model of the cache policy: slots keyed by (layer, expert); a fill
    takes the lowest-numbered empty slot, else the least recently used slot
    not held by the resolve call in flight; every lookup or fill is a use."""

    def __init__(self, n_slots):
        self.n = n_slots
        self.key = [None] * n_slots
        self.age = [0] * n_slots
        self.held = set()
        self.fresh = set()
        self.clock = 0
        self.c = dict(hits=0, misses=0, prefetches=0, prefetch_hits=0, prefetch_dropped=0)

    def _use(self, s):
        self.clock += 1
        self.age[s] = self.clock

    def _find(self, k):
        return self.key.index(k) if k in self.key else None

    def _free_slot(self):
        free = [s for s in range(self.n) if s not in self.held]
        if not free:
            return None
        empty = [s for s in free if self.key[s] is None]
        return empty[0] if empty else min(free, key=lambda s: (self.age[s], s))

    def prefetch(self, layer, ids):
        for e in ids:
            s = self._find((layer, e))
            if s is not None:
                self._use(s)
                continue
            s = self._free_slot()
            if s is None:
                self.c["prefetch_dropped"] += 1
                continue
            self.key[s] = (layer, e)
            self.fresh.add(s)
            self._use(s)
            self.c["prefetches"] += 1

    def resolve(self, layer, ids):
        self.held = set()
        got = {}
        for e in ids:
            if e in got:
                continue
            s = self._find((layer, e))
            if s is not None:
                self.c["hits"] += 1
                if s in self.fresh:
                    self.c["prefetch_hits"] += 1
            else:
                s = self._free_slot()
                assert s is not None
                self.key[s] = (layer, e)
                self.c["misses"] += 1
            self.fresh.discard(s)
            self.held.add(s)
            self._use(s)
            got[e] = s
        return got


DRIVER = r"""
#include <cstdio>
#include <vector>
#include "moe_stream_policy.h"
int main(int argc, char** argv) {
  int L, E, S;
  if (scanf("%d %d %d", &L, &E, &S) != 3) return 2;
  moe::StreamPolicy p;
  p.init(L, E, S);
  char op[4];
  while (scanf("%3s", op) == 1) {
    int layer, n;
    if (scanf("%d %d", &layer, &n) != 2) return 2;
    std::vector<int> ids(n);
    for (int i = 0; i < n; ++i)
      if (scanf("%d", &ids[i]) != 1) return 2;
    if (op[0] == 'P') {
      for (int e : ids) p.prefetch(layer, e);
    } else {
      p.release();
      std::vector<int> seen;
      printf("R");
      for (int e : ids) {
        bool dup = false;
        for (int q : seen) dup = dup || q == e;
        if (dup) continue;
        seen.push_back(e);
        bool fill = false;
        printf(" %d:%d", e, p.resolve(layer, e, &fill));
      }
      printf("\n");
    }
  }
  printf("C %llu %llu %llu %llu %llu\n", (unsigned long long)p.hits, (unsigned long long)p.misses,
         (unsigned long long)p.prefetches, (unsigned long long)p.prefetch_hits,
         (unsigned long long)p.prefetch_dropped);
  return 0;
}
"""


def test_cache_policy_matches_reference_model(tmp_path):
    src = tmp_path / "driver.cpp"
    exe = tmp_path / "driver"
    src.write_text(DRIVER)
    subprocess.check_call(["g++", "-std=c++17", "-O1", "-I", CSRC, str(src), "-o", str(exe)])
    g = np.random.default_rng(7)
    L, E, NS = 3, 10, 4
    ops = []
    for _ in range(400):
        kind = "R" if g.random() < 0.6 else "P"
        n = int(g.integers(1, 4))
        ops.append((kind, int(g.integers(0, L)), [int(v) for v in g.integers(0, E, n)]))
    text = "%d %d %d\n" % (L, E, NS) + "".join("%s %d %d %s\n" % (k, l, len(ids), " ".join(map(str, ids)))
                                             for k, l, ids in ops)
    out = subprocess.run([str(exe)], input=text, capture_output=True, text=True, check=True).stdout.split("\n")
    ref = RefCache(NS)
    lines = iter(out)
    n_resolves = 0
    for kind, layer, ids in ops:
        if kind == "P":
            ref.prefetch(layer, ids)
            continue
        got = ref.resolve(layer, ids)
        want = "R" + "".join(" %d:%d" % (e, s) for e, s in got.items())
        assert next(lines) == want, (kind, layer, ids)
        n_resolves += 1
    counters = next(lines).split()
    assert counters[0] == "C"
    c = ref.c
    assert [int(v) for v in counters[1:]] == [c["hits"], c["misses"], c["prefetches"], c["prefetch_hits"],
                                              c["prefetch_dropped"]]
    assert n_resolves > 200 and c["misses"] > 0 and c["prefetch_hits"] > 0 and c["hits"] > 0


def test_stream_create_rejects_bad_arguments(M):
    cfg = M.config(256, 128, 16, 2, bits=4)
    store = np.zeros(16 * M.moe_packed_expert_bytes(cfg), np.uint8)
    cases = [(cfg, 1, None, 4, M.STATUS_BY_NAME["MOE_ERR_INVALID_ARG"]),
             (cfg, 0, store, 4, M.STATUS_BY_NAME["MOE_ERR_INVALID_ARG"]),
             (cfg, 1, store, 0, M.STATUS_BY_NAME["MOE_ERR_INVALID_ARG"]),
             (M.config(256, 128, 16, 2, bits=3), 1, store, 4, M.STATUS_BY_NAME["MOE_ERR_UNSUPPORTED"]),
             (cfg, 1, store, 4, M.STATUS_BY_NAME["MOE_ERR_INVALID_ARG"])]  # pageable store
    for c, nl, st, ns, want in cases:
        with pytest.raises(M.MoeError) as ei:
            M.moe_stream_create(c, nl, st, ns)
        assert ei.value.status == want, (nl, ns, str(ei.value))


# ---------------------------------------------------------------------------- GPU

def _dev(a):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


@pytest.mark.gpu
@pytest.mark.parametrize("shape", [replace(S.TINY, tokens=4), replace(S.QWEN_4BIT, tokens=1)],
                         ids=["tiny_T4", "h4096_T1"])
def test_routed_forward_matches_fused_and_oracle(M, shape):
    import torch
    s = shape
    x, res = S.activations(s, step=5)
    dense = S.dense_weights(s)
    _, idx_o, w_o = O.router(ocfg(s), x, dense["wr"], dense["bias"])
    dl = DeviceLayer(s, expert_ids=idx_o.ravel().tolist() if s.n_experts > 64 else None, dense=dense)
    h_f, y_f, idx_f, w_f = dl.forward(x, res)
    xd, rd = to_dev_bits(x), to_dev_bits(res)
    # given the fused kernel's own routing: the same bits
    h, y = torch.empty_like(xd), torch.empty_like(xd)
    M.moe_layer_forward_routed(dl.cfg, dl.wts, xd, rd, _dev(idx_f), _dev(w_f), h, y, dl.ws)
    torch.cuda.synchronize()
    assert M.moe_device_error(dl.ws)[0] == 0
    assert np.array_equal(from_dev_bits(h), h_f) and np.array_equal(from_dev_bits(y), y_f)
    # given the oracle's routing (fp64 weights rounded to fp32): the oracle's outputs
    w32 = w_o.astype(np.float32)
    M.moe_layer_forward_routed(dl.cfg, dl.wts, xd, rd, _dev(idx_o.astype(np.int32)), _dev(w32), h, y, dl.ws)
    torch.cuda.synchronize()
    assert M.moe_device_error(dl.ws)[0] == 0
    _, _, h_ref, y_ref = oracle_forward(s, dl.oracle_blobs(), dense, x, res, idx_in=idx_o, w_in=w32)
    assert_outputs_close(from_dev_bits(h), h_ref, "h_out")
    assert_outputs_close(from_dev_bits(y), y_ref, "y_norm")


@pytest.mark.gpu
def test_routed_forward_reports_a_missing_expert(M):
    import torch
    s = replace(S.TINY, tokens=2)
    dl = DeviceLayer(s)
    x, res = S.activations(s, step=1)
    table = torch.zeros_like(dl.expert_ptr)  # every pointer NULL
    wts = M.layer_weights(table, None, None, dl.sg, dl.su, dl.sd, dl.gamma)
    xd, rd = to_dev_bits(x), to_dev_bits(res)
    h, y = torch.empty_like(xd), torch.empty_like(xd)
    idx = _dev(np.array([[0, 1], [2, 3]], np.int32))
    w = _dev(np.full((2, 2), 0.5, np.float32))
    M.moe_layer_forward_routed(dl.cfg, wts, xd, rd, idx, w, h, y, dl.ws)
    st, detail = M.moe_device_error(dl.ws)
    assert st == M.STATUS_BY_NAME["MOE_ERR_DEVICE"], (st, detail)


class _Layers:
    """n_layers layers of one shape: per layer its own router, shared expert
    and experts (replica = layer), resident on the device, and the pinned host
    store [layer][expert] of the packed experts."""

    def __init__(self, M, s, n_layers, device_pack=False, **layer_kw):
        import torch
        self.M, self.s, self.L = M, s, n_layers
        self.cfg = mcfg(s)
        nb = M.moe_packed_expert_bytes(self.cfg)
        self.nb = nb
        E = s.n_experts
        self.store = torch.empty((n_layers * E, nb), dtype=torch.uint8).pin_memory()
        self.layers = []
        for l in range(n_layers):
            if device_pack:
                blobs = torch.empty((E, nb), dtype=torch.uint8, device="cuda")
                for e0 in range(0, E, 8):
                    wg, wu, wd = S.torch_expert_weights(s, e0, 8, l, "cuda")
                    M.moe_pack_experts_device(self.cfg, wg, wu, wd, blobs[e0:e0 + 8])
                torch.cuda.synchronize()
                dl = self._resident(l, blobs)
            else:
                dl = DeviceLayer(s, replica=l, **layer_kw)
                blobs = dl.pool[:E]
            self.store[l * E:(l + 1) * E].copy_(blobs.cpu())
            self.layers.append(dl)

    def _resident(self, l, blobs):
        """A DeviceLayer-like object over device-packed blobs."""
        import torch
        M, s = self.M, self.s
        dl = DeviceLayer.__new__(DeviceLayer)
        dl.s, dl.M, dl.cfg = s, M, self.cfg
        dl.pool = blobs
        dl.expert_ptr = torch.tensor([blobs.data_ptr() + self.nb * e for e in range(s.n_experts)],
                                     dtype=torch.int64, device="cuda")
        d = S.dense_weights(s, l)
        dl.dense = d
        dl.wr, dl.bias = to_dev_bits(d["wr"]), torch.from_numpy(d["bias"]).cuda()
        dl.sg, dl.su, dl.sd = to_dev_bits(d["shared_gate"]), to_dev_bits(d["shared_up"]), to_dev_bits(d["shared_down"])
        dl.gamma = to_dev_bits(d["gamma"])
        dl.wts = M.layer_weights(dl.expert_ptr, dl.wr, dl.bias, dl.sg, dl.su, dl.sd, dl.gamma)
        dl.ws = torch.zeros(M.moe_layer_workspace_bytes(self.cfg, 8), dtype=torch.uint8, device="cuda")
        M.moe_workspace_init(dl.ws)
        return dl


def _run_streaming(M, lay, n_slots, steps):
    import torch
    s, L, E = lay.s, lay.L, lay.s.n_experts
    cache = M.moe_stream_create(lay.cfg, L, lay.store, n_slots)
    ref = RefCache(n_slots)
    side = torch.cuda.Stream()
    table = torch.zeros(E, dtype=torch.int64, device="cuda")
    ws = torch.zeros(M.moe_layer_workspace_bytes(lay.cfg, 8), dtype=torch.uint8, device="cuda")
    M.moe_workspace_init(ws)
    try:
        for step in range(steps):
            for l in range(L):
                dl = lay.layers[l]
                x, res = S.activations(s, step=step, replica=l)
                _, idx, w = dl.router(x)
                xd, rd = to_dev_bits(x), to_dev_bits(res)
                idd, wd = _dev(idx), _dev(w)
                h1, y1 = torch.empty_like(xd), torch.empty_like(xd)
                M.moe_layer_forward_routed(lay.cfg, dl.wts, xd, rd, idd, wd, h1, y1, dl.ws)
                M.moe_stream_resolve(cache, l, idx.ravel(), table)
                ref.resolve(l, idx.ravel().tolist())
                wts = M.layer_weights(table, None, None, dl.sg, dl.su, dl.sd, dl.gamma)
                h2, y2 = torch.empty_like(xd), torch.empty_like(xd)
                M.moe_layer_forward_routed(lay.cfg, wts, xd, rd, idd, wd, h2, y2, ws)
                if l + 1 < L:  # predicted experts of the next layer: its router on this input
                    _, pred, _ = lay.layers[l + 1].router(x)
                    M.moe_stream_prefetch(cache, l + 1, pred.ravel(), copy_stream=side)
                    ref.prefetch(l + 1, pred.ravel().tolist())
                torch.cuda.synchronize()
                assert M.moe_device_error(ws)[0] == 0
                assert np.array_equal(from_dev_bits(h1), from_dev_bits(h2)), (step, l)
                assert np.array_equal(from_dev_bits(y1), from_dev_bits(y2)), (step, l)
        st = M.moe_stream_stats(cache)
        for k in ("hits", "misses", "prefetches", "prefetch_hits", "prefetch_dropped"):
            assert st[k] == ref.c[k], (k, st, ref.c)
        assert st["bytes_h2d"] == (st["misses"] + st["prefetches"]) * lay.nb
        return st
    finally:
        torch.cuda.synchronize()
        M.moe_stream_destroy(cache)


@pytest.mark.gpu
def test_streaming_matches_resident_tiny(M):
    lay = _Layers(M, replace(S.TINY, tokens=2), n_layers=3)
    st = _run_streaming(M, lay, n_slots=5, steps=4)
    assert st["misses"] > 0 and st["hits"] > 0 and st["prefetches"] > 0


@pytest.mark.gpu
def test_streaming_matches_resident_h4096(M):
    s = replace(S.QWEN_4BIT, name="h4096_e64_k4_i1024_4bit", n_experts=64, tokens=1)
    lay = _Layers(M, s, n_layers=2, device_pack=True)
    st = _run_streaming(M, lay, n_slots=10, steps=4)
    assert st["misses"] > 0


@pytest.mark.gpu
def test_streaming_overlapped_matches_resident(M):
    """Layers, resolves and prefetches enqueued back to back with one
    synchronisation at the very end, so the side-stream prefetch of layer
    l+1 may evict a slot that layer l-1's kernel is still reading: its copy
    must wait for that kernel (the slot's "used" event).  Fewer slots than the
    distinct experts of two layers force such evictions.  Every layer's
    outputs must equal, bit for bit, the resident routed call's."""
    import torch
    s = replace(S.TINY, tokens=2)
    L, steps, n_slots = 4, 6, 5
    lay = _Layers(M, s, n_layers=L)
    E = s.n_experts
    # routing, inputs and resident reference outputs first (these synchronise)
    plan = []
    for step in range(steps):
        for l in range(L):
            dl = lay.layers[l]
            x, res = S.activations(s, step=step, replica=l)
            _, idx, w = dl.router(x)
            pred = lay.layers[l + 1].router(x)[1] if l + 1 < L else None
            xd, rd, idd, wd = to_dev_bits(x), to_dev_bits(res), _dev(idx), _dev(w)
            h1, y1 = torch.empty_like(xd), torch.empty_like(xd)
            M.moe_layer_forward_routed(lay.cfg, dl.wts, xd, rd, idd, wd, h1, y1, dl.ws)
            plan.append((l, idx, pred, xd, rd, idd, wd, h1, y1))
    torch.cuda.synchronize()
    cache = M.moe_stream_create(lay.cfg, L, lay.store, n_slots)
    side = torch.cuda.Stream()
    table = torch.zeros(E, dtype=torch.int64, device="cuda")
    ws = torch.zeros(M.moe_layer_workspace_bytes(lay.cfg, 8), dtype=torch.uint8, device="cuda")
    M.moe_workspace_init(ws)
    outs = []
    try:
        torch.cuda.synchronize()
        for l, idx, pred, xd, rd, idd, wd, _, _ in plan:
            dl = lay.layers[l]
            M.moe_stream_resolve(cache, l, idx.ravel(), table)
            wts = M.layer_weights(table, None, None, dl.sg, dl.su, dl.sd, dl.gamma)
            h2, y2 = torch.empty_like(xd), torch.empty_like(xd)
            M.moe_layer_forward_routed(lay.cfg, wts, xd, rd, idd, wd, h2, y2, ws)
            outs.append((h2, y2))
            if pred is not None:
                M.moe_stream_prefetch(cache, l + 1, pred.ravel(), copy_stream=side)
        torch.cuda.synchronize()
        assert M.moe_device_error(ws)[0] == 0
        st = M.moe_stream_stats(cache)
        assert st["misses"] > 0 and st["prefetches"] > 0
        for i, ((h2, y2), p) in enumerate(zip(outs, plan)):
            assert np.array_equal(from_dev_bits(h2), from_dev_bits(p[7])), i
            assert np.array_equal(from_dev_bits(y2), from_dev_bits(p[8])), i
    finally:
        torch.cuda.synchronize()
        M.moe_stream_destroy(cache)


# ---- resolved on the device ---------------------------------------------------------------

def _run_device_resolved(M, lay, n_slots, steps, tokens):
    """Every layer's router, moe_stream_resolve_device and the routed call
    enqueued back to back on one stream with one synchronisation at the end
    (the routing never reaches the host); outputs must equal the resident
    routed call's bit for bit, and the device counters RefCache's (fed the
    same routing afterwards)."""
    import torch
    s, L, E = lay.s, lay.L, lay.s.n_experts
    plan = []
    for step in range(steps):
        for l in range(L):
            dl = lay.layers[l]
            x, res = S.activations(s, step=step, tokens=tokens, replica=l)
            xd, rd = to_dev_bits(x), to_dev_bits(res)
            idd = torch.empty((tokens, s.top_k), dtype=torch.int32, device="cuda")
            wd = torch.empty((tokens, s.top_k), dtype=torch.float32, device="cuda")
            lg = torch.empty((tokens, s.n_experts), dtype=torch.float32, device="cuda")
            M.moe_router_topk(dl.cfg, xd, dl.wr, dl.bias, idd, wd, logits_out=lg)
            h1, y1 = torch.empty_like(xd), torch.empty_like(xd)
            M.moe_layer_forward_routed(lay.cfg, dl.wts, xd, rd, idd, wd, h1, y1, dl.ws)
            plan.append((l, xd, rd, idd, wd, h1, y1))
    torch.cuda.synchronize()
    cache = M.moe_stream_create(lay.cfg, L, lay.store, n_slots)
    table = torch.zeros(E, dtype=torch.int64, device="cuda")
    ws = torch.zeros(M.moe_layer_workspace_bytes(lay.cfg, 8), dtype=torch.uint8, device="cuda")
    M.moe_workspace_init(ws)
    outs = []
    try:
        for l, xd, rd, idd, wd, _, _ in plan:
            dl = lay.layers[l]
            M.moe_stream_resolve_device(cache, l, idd, table)
            wts = M.layer_weights(table, None, None, dl.sg, dl.su, dl.sd, dl.gamma)
            h2, y2 = torch.empty_like(xd), torch.empty_like(xd)
            M.moe_layer_forward_routed(lay.cfg, wts, xd, rd, idd, wd, h2, y2, ws)
            outs.append((h2, y2))
        torch.cuda.synchronize()
        assert M.moe_device_error(ws)[0] == 0
        for i, ((h2, y2), p) in enumerate(zip(outs, plan)):
            assert np.array_equal(from_dev_bits(h2), from_dev_bits(p[5])), i
            assert np.array_equal(from_dev_bits(y2), from_dev_bits(p[6])), i
        ref = RefCache(n_slots)
        for l, _, _, idd, _, _, _ in plan:
            ref.resolve(l, idd.cpu().numpy().ravel().tolist())
        st = M.moe_stream_stats(cache)
        assert st["device_error"] == 0
        for k in ("hits", "misses"):
            assert st[k] == ref.c[k], (k, st, ref.c)
        assert st["bytes_h2d"] == st["misses"] * lay.nb
        ct = M.moe_stream_copy_timing(cache)
        assert ct["bytes"] == st["bytes_h2d"] and (ct["busy_ms"] > 0) == (st["misses"] > 0)
        # the cache stays bound to device resolves
        with pytest.raises(M.MoeError):
            M.moe_stream_resolve(cache, 0, np.array([0], np.int32), table)
        return st
    finally:
        torch.cuda.synchronize()
        M.moe_stream_destroy(cache)


@pytest.mark.gpu
@pytest.mark.parametrize("tokens", [1, 3])
def test_device_resolved_streaming_matches_resident_tiny(M, tokens):
    lay = _Layers(M, replace(S.TINY, tokens=2), n_layers=3)
    # enough slots that later tokens find some experts resident, too few for
    # all 3 layers' experts (evictions)
    st = _run_device_resolved(M, lay, n_slots=7 if tokens == 1 else 20, steps=5, tokens=tokens)
    assert st["misses"] > 0 and st["hits"] > 0


@pytest.mark.gpu
def test_device_resolved_streaming_h4096(M):
    s = replace(S.QWEN_4BIT, name="h4096_e64_k4_i1024_4bit", n_experts=64, tokens=1)
    lay = _Layers(M, s, n_layers=2, device_pack=True)
    st = _run_device_resolved(M, lay, n_slots=10, steps=4, tokens=1)
    assert st["misses"] > 0


@pytest.mark.gpu
def test_device_resolve_reports_too_few_slots(M):
    """More distinct ids in one call than slots: the kernel leaves
    MOE_ERR_OOM in the device counters and writes no pointer; nothing faults."""
    import torch
    s = replace(S.TINY, tokens=2)
    lay = _Layers(M, s, n_layers=1)
    cache = M.moe_stream_create(lay.cfg, 1, lay.store, 2)
    table = torch.zeros(s.n_experts, dtype=torch.int64, device="cuda")
    try:
        M.moe_stream_resolve_device(cache, 0, _dev(np.array([1, 2, 3], np.int32)), table)
        st = M.moe_stream_stats(cache)
        assert st["device_error"] == M.STATUS_BY_NAME["MOE_ERR_OOM"]
        assert not table.cpu().numpy().any()
    finally:
        torch.cuda.synchronize()
        M.moe_stream_destroy(cache)


# ---- streamed layer calls (lookup, fill and layer in one launch) --------------------

def _run_streamed(M, lay, n_slots, steps, tokens):
    """moe_layer_forward_streamed for every layer of every step, back to back
    on one stream with one synchronisation at the end: outputs and routing
    must equal the resident fused call's bit for bit (the same kernel routes
    both; only where the expert bytes come from differs), and the device
    counters RefCache's fed the same routing."""
    import torch
    s, L, E = lay.s, lay.L, lay.s.n_experts
    plan = []
    for step in range(steps):
        for l in range(L):
            dl = lay.layers[l]
            x, res = S.activations(s, step=step, tokens=tokens, replica=l)
            xd, rd = to_dev_bits(x), to_dev_bits(res)
            h1, y1 = torch.empty_like(xd), torch.empty_like(xd)
            i1 = torch.empty((tokens, s.top_k), dtype=torch.int32, device="cuda")
            w1 = torch.empty((tokens, s.top_k), dtype=torch.float32, device="cuda")
            M.moe_layer_forward(lay.cfg, dl.wts, xd, rd, h1, y1, i1, w1, dl.ws)
            plan.append((l, xd, rd, h1, y1, i1, w1))
    torch.cuda.synchronize()
    cache = M.moe_stream_create(lay.cfg, L, lay.store, n_slots)
    ws = torch.zeros(M.moe_layer_workspace_bytes(lay.cfg, 8), dtype=torch.uint8, device="cuda")
    M.moe_workspace_init(ws)
    outs = []
    try:
        for l, xd, rd, _, _, _, _ in plan:
            dl = lay.layers[l]
            spacked, sgate = getattr(dl, "spacked", None), getattr(dl, "sgate", None)
            bf = spacked is None  # the shared expert's form as in the resident layer
            wts = M.layer_weights(None, dl.wr, dl.bias, dl.sg if bf else None, dl.su if bf else None,
                                  dl.sd if bf else None, dl.gamma, shared_out_gate=sgate, shared_packed=spacked)
            h2, y2 = torch.empty_like(xd), torch.empty_like(xd)
            i2 = torch.empty((tokens, s.top_k), dtype=torch.int32, device="cuda")
            w2 = torch.empty((tokens, s.top_k), dtype=torch.float32, device="cuda")
            M.moe_layer_forward_streamed(lay.cfg, wts, xd, rd, h2, y2, cache, l, ws, idx_out=i2, w_out=w2)
            outs.append((h2, y2, i2, w2))
        torch.cuda.synchronize()
        assert M.moe_device_error(ws)[0] == 0
        for i, ((h2, y2, i2, w2), p) in enumerate(zip(outs, plan)):
            assert np.array_equal(i2.cpu().numpy(), p[5].cpu().numpy()), i
            assert np.array_equal(w2.cpu().numpy(), p[6].cpu().numpy()), i
            assert np.array_equal(from_dev_bits(h2), from_dev_bits(p[3])), i
            assert np.array_equal(from_dev_bits(y2), from_dev_bits(p[4])), i
        # one resolve per launch: tokens beyond one launch's limit run in
        # successive launches, each looking up its own experts
        chunk = M.moe_layer_tokens_per_launch(lay.cfg)
        ref = RefCache(n_slots)
        for (l, *_), (_, _, i2, _) in zip(plan, outs):
            ids = i2.cpu().numpy()
            for t0 in range(0, ids.shape[0], chunk):
                ref.resolve(l, ids[t0:t0 + chunk].ravel().tolist())
        st = M.moe_stream_stats(cache)
        assert st["device_error"] == 0
        for k in ("hits", "misses"):
            assert st[k] == ref.c[k], (k, st, ref.c)
        assert st["bytes_h2d"] == st["misses"] * lay.nb
        # the same cache also serves the separate device resolve
        table = torch.zeros(E, dtype=torch.int64, device="cuda")
        M.moe_stream_resolve_device(cache, 0, outs[0][2], table)
        torch.cuda.synchronize()
        assert M.moe_stream_stats(cache)["device_error"] == 0
        return st
    finally:
        torch.cuda.synchronize()
        M.moe_stream_destroy(cache)


@pytest.mark.gpu
@pytest.mark.parametrize("tokens", [1, 3])
def test_streamed_layer_matches_resident_tiny(M, tokens):
    lay = _Layers(M, replace(S.TINY, tokens=2), n_layers=3)
    st = _run_streamed(M, lay, n_slots=7 if tokens == 1 else 20, steps=5, tokens=tokens)
    assert st["misses"] > 0 and st["hits"] > 0


@pytest.mark.gpu
@pytest.mark.parametrize("form", ["2bit", "more_tokens_than_one_launch", "packed_shared_gated"])
def test_streamed_layer_forms(M, form):
    """The streamed call with 2-bit experts; with more tokens than one
    launch takes (successive launches, each resolving its own experts); and
    with the shared expert packed like the routed ones (its pair is not
    looked up in the cache) behind a sigmoid gate."""
    if form == "2bit":
        lay = _Layers(M, replace(S.TINY, bits=2, tokens=2), n_layers=2)
        st = _run_streamed(M, lay, n_slots=7, steps=4, tokens=2)
    elif form == "more_tokens_than_one_launch":
        lay = _Layers(M, replace(S.TINY, tokens=12), n_layers=2, max_tokens=12)
        assert M.moe_layer_tokens_per_launch(lay.cfg) < 12
        st = _run_streamed(M, lay, n_slots=24, steps=3, tokens=12)
    else:
        s = replace(S.TINY, tokens=2)
        g = S.rng(s.seed, 0, "shared_out_gate", s.hidden).standard_normal(s.hidden).astype(np.float32)
        lay = _Layers(M, s, n_layers=2, shared_packed=True, shared_out_gate=S.f32_to_bf16_bits(g * np.float32(0.1)))
        st = _run_streamed(M, lay, n_slots=7, steps=4, tokens=2)
    assert st["misses"] > 0


@pytest.mark.gpu
def test_streamed_layer_h4096(M):
    s = replace(S.QWEN_4BIT, name="h4096_e64_k4_i1024_4bit", n_experts=64, tokens=1)
    lay = _Layers(M, s, n_layers=2, device_pack=True)
    st = _run_streamed(M, lay, n_slots=10, steps=4, tokens=1)
    assert st["misses"] > 0


@pytest.mark.gpu
def test_streamed_layer_reports_too_few_slots(M):
    """More distinct experts in one launch than slots: MOE_ERR_OOM in the
    cache's counters, a bad expert pointer in the layer's error word, the
    call's assignments undone; nothing faults or waits out."""
    import torch
    s = replace(S.TINY, tokens=3)
    lay = _Layers(M, s, n_layers=1)
    cache = M.moe_stream_create(lay.cfg, 1, lay.store, 1)
    dl = lay.layers[0]
    ws = torch.zeros(M.moe_layer_workspace_bytes(lay.cfg, 8), dtype=torch.uint8, device="cuda")
    M.moe_workspace_init(ws)
    try:
        x, res = S.activations(s, step=0, tokens=3, replica=0)
        xd, rd = to_dev_bits(x), to_dev_bits(res)
        h, y = torch.empty_like(xd), torch.empty_like(xd)
        i2 = torch.empty((3, s.top_k), dtype=torch.int32, device="cuda")
        wts = M.layer_weights(None, dl.wr, dl.bias, dl.sg, dl.su, dl.sd, dl.gamma)
        M.moe_layer_forward_streamed(lay.cfg, wts, xd, rd, h, y, cache, 0, ws, idx_out=i2)
        torch.cuda.synchronize()
        assert len(set(i2.cpu().numpy().ravel().tolist())) > 1
        st = M.moe_stream_stats(cache)
        assert st["device_error"] == M.STATUS_BY_NAME["MOE_ERR_OOM"]
        assert st["misses"] == 0
        assert M.moe_device_error(ws)[0] == M.STATUS_BY_NAME["MOE_ERR_DEVICE"]
    finally:
        torch.cuda.synchronize()
        M.moe_stream_destroy(cache)


# ---- failures injected on the host (no GPU fault) ------------------------------------

@pytest.mark.gpu
def test_stream_create_rejects_a_short_store_and_an_injected_alloc_failure(M):
    import torch
    s = replace(S.TINY, tokens=2)
    cfg = mcfg(s)
    nb = M.moe_packed_expert_bytes(cfg)
    store = torch.zeros((2 * s.n_experts, nb), dtype=torch.uint8).pin_memory()
    with pytest.raises(M.MoeError) as ei:  # 2 layers' blobs, 3 layers claimed
        M.moe_stream_create(cfg, 3, store, 4)
    assert ei.value.status == M.STATUS_BY_NAME["MOE_ERR_INVALID_ARG"] and "holds" in str(ei.value)
    with pytest.raises(M.MoeError) as ei:  # a byte count below the blobs' size
        M.moe_stream_create(cfg, 2, store, 4, store_bytes=2 * s.n_experts * nb - 1)
    assert ei.value.status == M.STATUS_BY_NAME["MOE_ERR_INVALID_ARG"]
    M.moe_stream_inject_fault(None, M.MOE_FAULT_ALLOC)
    with pytest.raises(M.MoeError) as ei:
        M.moe_stream_create(cfg, 2, store, 4)
    assert ei.value.status == M.STATUS_BY_NAME["MOE_ERR_OOM"]
    cache = M.moe_stream_create(cfg, 2, store, 4)  # one-shot: the next create works
    M.moe_stream_destroy(cache)


@pytest.mark.gpu
def test_stream_copy_failure_is_reported_and_the_cache_recovers(M):
    """A failing host-to-device copy (injected on the host) makes resolve and
    prefetch return MOE_ERR_IO with a message; the cache keeps no slot for the
    expert whose copy failed, and the next calls produce the resident routed
    call's outputs bit for bit."""
    import torch
    s = replace(S.TINY, tokens=2)
    lay = _Layers(M, s, n_layers=2)
    E = s.n_experts
    cache = M.moe_stream_create(lay.cfg, 2, lay.store, 6)
    table = torch.zeros(E, dtype=torch.int64, device="cuda")
    ws = torch.zeros(M.moe_layer_workspace_bytes(lay.cfg, 8), dtype=torch.uint8, device="cuda")
    M.moe_workspace_init(ws)
    try:
        dl = lay.layers[0]
        x, res = S.activations(s, step=7)
        _, idx, w = dl.router(x)
        distinct = len(set(idx.ravel().tolist()))
        assert distinct >= 2
        # the second miss of this resolve fails
        M.moe_stream_inject_fault(cache, M.MOE_FAULT_COPY, 1)
        with pytest.raises(M.MoeError) as ei:
            M.moe_stream_resolve(cache, 0, idx.ravel(), table)
        assert ei.value.status == M.STATUS_BY_NAME["MOE_ERR_IO"] and "injected" in str(ei.value)
        st = M.moe_stream_stats(cache)
        assert st["misses"] == 1 and st["hits"] == 0
        # a prefetch whose first copy fails
        M.moe_stream_inject_fault(cache, M.MOE_FAULT_COPY, 0)
        with pytest.raises(M.MoeError) as ei:
            M.moe_stream_prefetch(cache, 1, [0, 1])
        assert ei.value.status == M.STATUS_BY_NAME["MOE_ERR_IO"]
        assert M.moe_stream_stats(cache)["prefetches"] == 0
        # recovery: resolve again and run the layer
        M.moe_stream_resolve(cache, 0, idx.ravel(), table)
        st = M.moe_stream_stats(cache)
        assert st["misses"] + st["hits"] == 1 + distinct
        xd, rd, idd, wd = to_dev_bits(x), to_dev_bits(res), _dev(idx), _dev(w)
        wts = M.layer_weights(table, None, None, dl.sg, dl.su, dl.sd, dl.gamma)
        h2, y2 = torch.empty_like(xd), torch.empty_like(xd)
        M.moe_layer_forward_routed(lay.cfg, wts, xd, rd, idd, wd, h2, y2, ws)
        h1, y1 = torch.empty_like(xd), torch.empty_like(xd)
        M.moe_layer_forward_routed(lay.cfg, dl.wts, xd, rd, idd, wd, h1, y1, dl.ws)
        torch.cuda.synchronize()
        assert M.moe_device_error(ws)[0] == 0
        assert np.array_equal(from_dev_bits(h1), from_dev_bits(h2))
        assert np.array_equal(from_dev_bits(y1), from_dev_bits(y2))
    finally:
        M.moe_stream_inject_fault(cache, M.MOE_FAULT_NONE)
        torch.cuda.synchronize()
        M.moe_stream_destroy(cache)


# ---- file-backed store (the pages' SSD tier) -------------------------------------------

@pytest.mark.gpu
@pytest.mark.parametrize("direct", [False, True], ids=["page_cache", "direct_io"])
def test_file_store_matches_resident(M, tmp_path, direct):
    """The same multi-layer run with the cache's store in a file (parallel
    pread into pinned staging, then the copy to the slot): every layer's
    outputs equal the resident routed call's bit for bit, and the reads
    counted equal the misses plus the prefetches."""
    import torch
    if direct:
        s = replace(S.QWEN_4BIT, name="h4096_e16_k4_i1024_4bit", n_experts=16, tokens=1)  # 4096-byte blobs
    else:
        s = replace(S.TINY, tokens=2)
    lay = _Layers(M, s, n_layers=2, device_pack=direct)
    path = tmp_path / "experts.bin"
    lay.store.numpy().tofile(str(path))
    try:
        cache = M.moe_stream_create_file(lay.cfg, 2, str(path), 6, direct_io=direct, n_read_threads=4)
    except M.MoeError as e:
        if direct and e.status == M.STATUS_BY_NAME["MOE_ERR_IO"]:
            pytest.skip("O_DIRECT is not available on this file system: %s" % e)
        raise
    E = s.n_experts
    table = torch.zeros(E, dtype=torch.int64, device="cuda")
    ws = torch.zeros(M.moe_layer_workspace_bytes(lay.cfg, 8), dtype=torch.uint8, device="cuda")
    M.moe_workspace_init(ws)
    side = torch.cuda.Stream()
    try:
        for step in range(3):
            for l in range(2):
                dl = lay.layers[l]
                x, res = S.activations(s, step=step, replica=l)
                _, idx, w = dl.router(x)
                xd, rd, idd, wd = to_dev_bits(x), to_dev_bits(res), _dev(idx), _dev(w)
                h1, y1 = torch.empty_like(xd), torch.empty_like(xd)
                M.moe_layer_forward_routed(lay.cfg, dl.wts, xd, rd, idd, wd, h1, y1, dl.ws)
                M.moe_stream_resolve(cache, l, idx.ravel(), table)
                wts = M.layer_weights(table, None, None, dl.sg, dl.su, dl.sd, dl.gamma)
                h2, y2 = torch.empty_like(xd), torch.empty_like(xd)
                M.moe_layer_forward_routed(lay.cfg, wts, xd, rd, idd, wd, h2, y2, ws)
                if l == 0:
                    _, pred, _ = lay.layers[1].router(x)
                    M.moe_stream_prefetch(cache, 1, pred.ravel(), copy_stream=side)
                torch.cuda.synchronize()
                assert M.moe_device_error(ws)[0] == 0
                assert np.array_equal(from_dev_bits(h1), from_dev_bits(h2)), (step, l)
                assert np.array_equal(from_dev_bits(y1), from_dev_bits(y2)), (step, l)
        st = M.moe_stream_stats(cache)
        fs = M.moe_stream_file_stats(cache)
        assert fs["reads"] == st["misses"] + st["prefetches"] and fs["reads"] > 0
        assert fs["read_bytes"] == fs["reads"] * lay.nb
    finally:
        torch.cuda.synchronize()
        M.moe_stream_destroy(cache)


@pytest.mark.gpu
def test_file_store_rejects_a_short_or_missing_file(M, tmp_path):
    s = replace(S.TINY, tokens=2)
    cfg = mcfg(s)
    nb = M.moe_packed_expert_bytes(cfg)
    path = tmp_path / "short.bin"
    np.zeros(2 * s.n_experts * nb - 1, np.uint8).tofile(str(path))
    with pytest.raises(M.MoeError) as ei:
        M.moe_stream_create_file(cfg, 2, str(path), 4)
    assert ei.value.status == M.STATUS_BY_NAME["MOE_ERR_INVALID_ARG"] and "file holds" in str(ei.value)
    with pytest.raises(M.MoeError) as ei:
        M.moe_stream_create_file(cfg, 1, str(tmp_path / "missing.bin"), 4)
    assert ei.value.status == M.STATUS_BY_NAME["MOE_ERR_IO"]
