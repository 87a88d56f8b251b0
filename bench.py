#!/usr/bin/env python
"""Benchmark: MoE-layer tokens/s and achieved HBM GB/s (4-bit experts, K=4, batch 1).

Workload: one MoE layer shaped like the Qwen3.5-397B layer the pages run
(hidden 4096, 512 experts, top-4, expert intermediate 1024, 4-bit group-64
experts with bf16 scale/bias, a bf16 shared expert of the same size), one
token per step, router bias Zipf(1.1)-skewed.  All inputs are seeded
synthetic data.  A step is one call of moe_layer_forward (router, top-K,
routed experts, shared expert, combine, residual, RMSNorm) on one token.

L2 guard: R=8 independent replicas of the layer (3.6 GB of experts each,
29 GB in all) are used round-robin, so no step finds its weights in the
126 MB L2 from an earlier step.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--bits 4|2] [--impl ours|reference]

For N > 1 run under torch.distributed.run: every rank runs its own replica
of the workload (replicas only: the layer has no exchange step), the timed
region is bracketed by barriers, and the time is the max over ranks.
"""
import argparse
import hashlib
import json
import os
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import synth as S  # noqa: E402

METRIC = "MoE-layer tokens/s and achieved HBM GB/s (4-bit experts, K=4, batch 1)"
FALLBACK_HBM_GBS = 6650.0
KERNEL_SOURCES = ["moe_decode.cu", "moe_device.cuh", "moe_layout.h", "moe_kernels.h"]


def decode_dtype(bits):
    """Arithmetic of the fused decode kernel: gate/up on the integer tensor
    cores (codes times x as two int8 limbs), the rest bf16 with fp32 sums."""
    return (f"u{bits} x i8 -> i32 ({bits}-bit gate/up, x as two int8 limbs), "
            "bf16 -> f32 (router, shared, down)")


def parse_args(argv=None):
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=2000)
    p.add_argument("--warmup", type=int, default=50)
    p.add_argument("--bits", type=int, default=4, choices=(4, 2))
    p.add_argument("--impl", default="ours", choices=("ours", "reference"))
    p.add_argument("--replicas", type=int, default=8)
    p.add_argument("--e2e-steps", type=int, default=300)
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-graph", action="store_true")
    p.add_argument("--trace", action="store_true",
                   help="also print per-phase timestamps of a few traced layer calls")
    p.add_argument("--streaming", action="store_true",
                   help="measure the expert-streaming tier instead (its own JSON line)")
    p.add_argument("--stream-layers", type=int, default=4)
    p.add_argument("--stream-slots", type=int, default=512)
    p.add_argument("--stream-steps", type=int, default=64)
    p.add_argument("--stream-warmup", type=int, default=32)
    p.add_argument("--store", default="pinned", choices=("pinned", "file"),
                   help="streaming store: pinned host memory, or a file read with parallel pread")
    p.add_argument("--direct-io", action="store_true", help="file store: O_DIRECT reads (bypass the page cache)")
    p.add_argument("--store-path", default="/tmp/moe_expert_store.bin")
    p.add_argument("--stream-resolve", default="fused", choices=("fused", "device", "host"),
                   help="streaming: each layer as one launch that routes, looks its experts up in the cache and "
                        "copies the misses (fused), the router, a resolve kernel and the routed layer as "
                        "separate launches (device), or the routing resolved on the host (host)")
    p.add_argument("--predictor", default="next_router", choices=("next_router", "temporal", "none"),
                   help="streaming prefetch: the next layer's router on this layer's input, the experts the "
                        "next layer chose for the previous token, or no prefetch")
    p.add_argument("--batched", default="",
                   help="comma-separated token counts: measure batches of T tokens per step instead")
    return p.parse_args(argv)


def workload(bits):
    return S.QWEN_4BIT if bits == 4 else S.QWEN_2BIT


def algorithmic_bytes(s, T=1):
    """Bytes one launch must move at least: the K chosen experts' packed blobs,
    the bf16 shared expert, the bf16 router, bias, gamma, activations in and
    out."""
    import quantized_expert_ffn_03_b200 as M
    cfg = M.config(s.hidden, s.inter, s.n_experts, s.top_k, bits=s.bits)
    experts = T * s.top_k * M.moe_packed_expert_bytes(cfg)  # distinct experts per token
    shared = 3 * s.hidden * s.inter * 2 if s.has_shared else 0
    router = s.n_experts * s.hidden * 2 + s.n_experts * 4
    small = s.hidden * 2 + 4 * T * s.hidden * 2 + 2 * T * s.top_k * 4
    return experts + shared + router + small


def kernel_source_hash():
    h = hashlib.sha256()
    for f in KERNEL_SOURCES:
        with open(os.path.join(ROOT, "quantized_expert_ffn_03_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def measured_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def profiled_traffic(bits):
    """dram bytes per launch from a committed ncu summary, if it was taken on
    the kernel as it is now."""
    path = os.path.join(ROOT, "profiles", "moe_decode_kernel_traffic.json")
    try:
        with open(path) as f:
            d = json.load(f)
        ent = d.get("%dbit" % bits)
        if ent and ent.get("src_sha") == kernel_source_hash():
            return float(ent["dram_bytes_per_launch"])
    except Exception:
        pass
    return None


# ---- distributed plumbing (replicas only) -------------------------------------------

def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    return ws, int(os.environ.get("RANK", "0")), int(os.environ.get("LOCAL_RANK", "0"))


def aggregate(elapsed_ms, units, group_backend_device=None):
    """Max of elapsed over ranks and sum of units over ranks (all ranks call)."""
    import torch
    import torch.distributed as dist
    if not dist.is_available() or not dist.is_initialized():
        return elapsed_ms, units
    dev = group_backend_device or "cpu"
    t = torch.tensor([elapsed_ms], dtype=torch.float64, device=dev)
    u = torch.tensor([units], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    dist.all_reduce(u, op=dist.ReduceOp.SUM)
    return float(t.item()), float(u.item())


def barrier():
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized():
        dist.barrier()


# ---- clocks -------------------------------------------------------------------------------

class ClockSampler:
    """Samples SM clock and throttle reasons through NVML while running."""

    REASONS = {
        "hw_slowdown": 0x8, "hw_thermal_slowdown": 0x40, "sw_thermal_slowdown": 0x20,
        "sw_power_cap": 0x4, "hw_power_brake_slowdown": 0x80,
    }

    def __init__(self, device_index, period_s=0.005):
        self.dev, self.period = device_index, period_s
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self._stop = threading.Event()
        self._t = None
        self.ok = False

    def __enter__(self):
        try:
            import pynvml
            pynvml.nvmlInit()
            h = pynvml.nvmlDeviceGetHandleByIndex(self.dev)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)
            self.ok = True

            def run():
                while not self._stop.is_set():
                    try:
                        self.samples.append(pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM))
                        r = pynvml.nvmlDeviceGetCurrentClocksEventReasons(h)
                        for k, bit in self.REASONS.items():
                            if r & bit:
                                self.reasons.add(k)
                    except Exception:
                        pass
                    time.sleep(self.period)

            self._t = threading.Thread(target=run, daemon=True)
            self._t.start()
        except Exception:
            self.ok = False
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self._t is not None:
            self._t.join()

    def summary(self):
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                    "samples": len(self.samples)}
        return {"sm_mhz": float(np.median(self.samples)), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


# ---- CPU oracle timing ------------------------------------------------------------------

def oracle_token_rate(s, n_tokens, seconds_cap=None, threads=1):
    """Time the plain C oracle on n_tokens tokens of the workload; expert
    generation and quantisation are done first, untimed.  threads > 1 runs
    that many tokens at a time on host threads (the oracle call releases the
    interpreter lock; each token is computed exactly as single-threaded)."""
    import oracle as O
    oc = O.cfg(s.hidden, s.inter, s.n_experts, s.top_k, bits=s.bits, eps=s.eps, has_shared=s.has_shared)
    d = S.dense_weights(s, 0)
    toks = [S.activations(s, step=k) for k in range(n_tokens)]
    need = set()
    for x, _ in toks:
        _, idx, _ = O.router(oc, x, d["wr"], d["bias"])
        need |= set(idx.ravel().tolist())
    blobs = {e: O.quantize_expert(oc, *S.expert_weights(s, e)) for e in sorted(need)}
    first = blobs[min(blobs)]
    lst = [blobs.get(e, first) for e in range(s.n_experts)]

    def one(tok):
        x, res = tok
        O.layer_forward(oc, lst, d["wr"], d["bias"], d["shared_gate"], d["shared_up"], d["shared_down"],
                        d["gamma"], x, res)

    done, t0 = 0, time.perf_counter()
    if threads <= 1:
        for tok in toks:
            one(tok)
            done += 1
            if seconds_cap is not None and time.perf_counter() - t0 > seconds_cap:
                break
    else:
        from concurrent.futures import ThreadPoolExecutor
        with ThreadPoolExecutor(max_workers=threads) as ex:
            for k in range(0, len(toks), threads):
                list(ex.map(one, toks[k:k + threads]))
                done += len(toks[k:k + threads])
                if seconds_cap is not None and time.perf_counter() - t0 > seconds_cap:
                    break
    dt = time.perf_counter() - t0
    return done / dt, done, dt


def host_cores():
    try:
        return len(os.sched_getaffinity(0))
    except Exception:
        return os.cpu_count() or 1


def run_reference(args):
    ws, rank, _ = dist_env()
    if rank != 0:
        return 0
    s = workload(args.bits)
    # each step is one token through the oracle; the run is capped so that the
    # whole --steps/--warmup invocation ends within a few minutes
    # warm-up tokens (at most 3, at least 1), which also size the timed run
    nw = max(1, min(args.warmup, 3))
    rate1, _, t1 = oracle_token_rate(s, nw)
    n = max(1, min(args.steps, int(150.0 / max(t1 / nw, 1e-3))))
    rate, done, dt = oracle_token_rate(s, n, seconds_cap=150.0)
    line = {
        "impl": "reference", "metric": METRIC, "value": rate, "unit": "tokens/s", "n_gpus": args.gpus,
        "steps": done, "warmup": nw, "ms_per_step": 1e3 * dt / done, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": s.name, "hidden": s.hidden, "inter": s.inter, "n_experts": s.n_experts,
                   "top_k": s.top_k, "bits": s.bits, "tokens_per_step": 1},
        "cpu_baseline": {"value": rate, "unit": "tokens/s", "cores": 1, "kind": "oracle",
                         "sample": "%d tokens of the workload through the single-threaded C oracle "
                                   "(fp64, dequantise-then-dot), experts generated and quantised "
                                   "before timing" % done},
        "e2e": {"value": rate, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ---- GPU run ----------------------------------------------------------------------------

def build_replica(M, s, replica, T, chunk=32):
    import torch
    cfg = M.config(s.hidden, s.inter, s.n_experts, s.top_k, bits=s.bits, eps=s.eps, has_shared=s.has_shared)
    nb = M.moe_packed_expert_bytes(cfg)
    pool = torch.empty(s.n_experts * nb, dtype=torch.uint8, device="cuda")
    for e0 in range(0, s.n_experts, chunk):
        n = min(chunk, s.n_experts - e0)
        wg, wu, wd = S.torch_expert_weights(s, e0, n, replica, "cuda")
        M.moe_pack_experts_device(cfg, wg, wu, wd, pool[e0 * nb:(e0 + n) * nb])
        del wg, wu, wd
    ptrs = (torch.arange(s.n_experts, dtype=torch.int64, device="cuda") * nb + pool.data_ptr()).contiguous()
    d = S.dense_weights(s, replica)
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).cuda()
    r = dict(pool=pool, ptrs=ptrs, wr=dev(d["wr"]), bias=torch.from_numpy(d["bias"]).cuda(),
             sg=dev(d["shared_gate"]), su=dev(d["shared_up"]), sd=dev(d["shared_down"]), gamma=dev(d["gamma"]))
    r["wts"] = M.layer_weights(r["ptrs"], r["wr"], r["bias"], r["sg"], r["su"], r["sd"], r["gamma"])
    r["ws"] = torch.zeros(M.moe_layer_host_workspace_bytes(cfg, T), dtype=torch.uint8, device="cuda")
    M.moe_workspace_init(r["ws"])
    r["cfg"] = cfg
    return r


TRACE_NAMES = ["start", "router_done", "shared_gu_done", "expert_gu_done", "wait_S_done", "wait_E_done",
               "tiles_done", "arrived_D", "exit", "producer_topk", "producer_last_copy"]


SPIN_NAMES = ["consumer_slot", "consumer_phase", "consumer_x", "producer_slot", "producer_routing",
              "sync_arrivals", "sync_grid", "sync_x"]


def print_trace(M, reps, cfg, xs, rs, h_out, y_out, stream, P, R, calls=16):
    """Per-phase timestamps (median over blocks, then over calls), relative
    to the earliest block start of each call; printed to stderr."""
    import torch
    nb = M.moe_layer_trace_blocks()
    tr = torch.zeros((calls, nb, 128), dtype=torch.int64, device="cuda")
    with torch.cuda.stream(stream):
        for i in range(calls):
            r = reps[i % R]
            M.moe_layer_forward_traced(cfg, r["wts"], xs[i % P], rs[i % P], h_out[0], y_out[0], tr[i],
                                       r["ws"], stream=stream)
        torch.cuda.synchronize()
    t = tr.cpu().numpy().astype(np.float64)
    rel = t - t[:, :, 0:1].min(axis=1, keepdims=True)
    out = {}
    for k, name in enumerate(TRACE_NAMES):
        v = rel[:, :, k]
        out[name] = {"median_us": float(np.median(np.median(v, axis=1)) / 1e3),
                     "max_us": float(np.median(v.max(axis=1)) / 1e3)}
    print("trace " + json.dumps(out), file=sys.stderr, flush=True)
    # per-tile view of block 0 of the last call: (ready, released) per tile
    # and the producer's publish times, in us after that block's start
    b0 = t[-1, 0]
    tiles = [(round((b0[16 + 2 * n] - b0[0]) / 1e3, 2), round((b0[17 + 2 * n] - b0[0]) / 1e3, 2))
             for n in range(16) if b0[16 + 2 * n] > 0]
    pub = [round((b0[48 + n] - b0[0]) / 1e3, 2) for n in range(16) if b0[48 + n] > 0]
    print("trace_block0 tiles=%s publish=%s" % (tiles, pub), file=sys.stderr, flush=True)
    probe = [round((b0[k] - b0[0]) / 1e3, 3) for k in range(11, 15)]
    print("trace_block0 first routed units (gate/up start, end, down start, end): %s" % probe,
          file=sys.stderr, flush=True)
    # marks a launch did not write hold stale values (negative or absurd times): skipped
    sync = {}
    for k in list(range(64, 74)) + list(range(100, 104)):
        v = float(np.median(rel[:, :, k])) / 1e3
        if 0.0 <= v < 1e5:
            sync[k] = round(v, 3)
    units = [(round((b0[104 + 2 * n] - b0[0]) / 1e3, 2), round((b0[105 + 2 * n] - b0[104 + 2 * n]) / 1e3, 2))
             for n in range(8) if b0[104 + 2 * n] > 0]
    print("trace_block0 warp0 routed units (start, duration): %s" % units, file=sys.stderr, flush=True)
    print("trace sync warp (median us): %s" % json.dumps(sync), file=sys.stderr, flush=True)
    # router logits: each block's last logit write; block 0's poll passes
    lw = rel[:, :, 72]
    starts = [round(float(np.median(rel[:, 0, 88 + k])) / 1e3, 3) for k in range(8)
              if np.all(t[:, 0, 88 + k] > 0)]
    print("trace logits: last write median %.3f max %.3f us; block 0's poll passes start at %s us" %
          (np.median(np.median(lw, axis=1)) / 1e3, np.median(lw.max(axis=1)) / 1e3, starts),
          file=sys.stderr, flush=True)
    lead = [float(np.median(rel[:, 0, k])) / 1e3 for k in (73, 96, 74, 78, 79)]
    others = rel[:, 1:, 78]
    print("trace routing: block 0 last poll pass starts %.3f, its loads returned %.3f, all words seen %.3f, "
          "top-K done %.3f, published %.3f us; other blocks have it: median %.3f max %.3f us" %
          (tuple(lead) + (float(np.median(np.median(others, axis=1))) / 1e3,
                          float(np.median(others.max(axis=1))) / 1e3)), file=sys.stderr, flush=True)
    it = [float(np.median(rel[:, :, k])) / 1e3 for k in (75, 76, 77)]
    print("trace warp 0 first shared gate/up row part: start %.3f, dot done %.3f, exchange done %.3f us" % tuple(it),
          file=sys.stderr, flush=True)
    sp = int(min(8, np.median(t[:, :, 97])))
    ss_starts = [round(float(np.median(rel[:, :, 120 + k])) / 1e3, 3) for k in range(sp)]
    print("trace RMSNorm sums: published median %.3f max %.3f us; poll pass starts (median us) %s; "
          "last pass loads returned at %.3f us" %
          (float(np.median(np.median(rel[:, :, 99], axis=1))) / 1e3, float(np.median(rel[:, :, 99].max(axis=1))) / 1e3,
           ss_starts, float(np.median(rel[:, :, 98])) / 1e3), file=sys.stderr, flush=True)
    polls = {SPIN_NAMES[k]: float(np.median(t[:, :, 80 + k])) for k in range(8)}
    print("trace polls per block (median): %s" % json.dumps(polls), file=sys.stderr, flush=True)


def run_ours(args):
    import torch
    import quantized_expert_ffn_03_b200 as M

    world, rank, local = dist_env()
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    else:
        torch.cuda.set_device(0)
    dev_index = torch.cuda.current_device()
    s = workload(args.bits)
    T = 1
    R = max(1, args.replicas)
    reps = [build_replica(M, s, rr + 17 * rank, T) for rr in range(R)]
    torch.cuda.synchronize()

    # token pool: fresh N(0,1) bf16 activations per step
    P = min(args.steps + args.warmup, 4096)
    gen = torch.Generator(device="cuda")
    gen.manual_seed(1234 + rank)
    xs = torch.randn((P, T, s.hidden), generator=gen, device="cuda").to(torch.bfloat16).view(torch.int16)
    rs = torch.randn((P, T, s.hidden), generator=gen, device="cuda").to(torch.bfloat16).view(torch.int16)
    h_out = torch.empty((R, T, s.hidden), dtype=torch.int16, device="cuda")
    y_out = torch.empty((R, T, s.hidden), dtype=torch.int16, device="cuda")
    cfg = reps[0]["cfg"]

    def step(i):
        r = reps[i % R]
        k = i % P
        M.moe_layer_forward(cfg, r["wts"], xs[k], rs[k], h_out[i % R], y_out[i % R], workspace=r["ws"])

    stream = torch.cuda.Stream()
    used_graph = False
    with torch.cuda.stream(stream):
        for i in range(args.warmup):
            step(i)
        torch.cuda.synchronize()
        graph = None
        if not args.no_graph:
            try:
                graph = torch.cuda.CUDAGraph()
                with torch.cuda.graph(graph, stream=stream):
                    for i in range(args.steps):
                        step(args.warmup + i)
                graph.replay()  # untimed: uploads the graph
                torch.cuda.synchronize()
                used_graph = True
            except Exception as e:  # capture not possible: time direct launches
                print("graph capture failed (%s); timing direct launches" % e, file=sys.stderr)
                graph = None
                torch.cuda.synchronize()
        st, detail = M.moe_device_error(reps[0]["ws"])
        assert st == 0, (st, detail)

        start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        barrier()
        torch.cuda.synchronize()
        with ClockSampler(dev_index) as clk:
            start.record(stream)
            if graph is not None:
                graph.replay()
            else:
                for i in range(args.steps):
                    step(args.warmup + i)
            stop.record(stream)
            torch.cuda.synchronize()
        barrier()
        local_ms = start.elapsed_time(stop)
        for r in reps:
            st, detail = M.moe_device_error(r["ws"])
            assert st == 0, ("device error after timed run", st, detail)

        # L2-assisted (single replica, warm) figure, for context
        warm = None
        if graph is not None:
            g1 = torch.cuda.CUDAGraph()
            n1 = min(args.steps, 500)
            with torch.cuda.graph(g1, stream=stream):
                for i in range(n1):
                    M.moe_layer_forward(cfg, reps[0]["wts"], xs[i % P], rs[i % P], h_out[0], y_out[0],
                                        workspace=reps[0]["ws"])
            g1.replay()
            torch.cuda.synchronize()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            g1.replay()
            e1.record(stream)
            torch.cuda.synchronize()
            warm = e0.elapsed_time(e1) / n1
            del g1

    if args.trace and rank == 0:
        print_trace(M, reps, cfg, xs, rs, h_out, y_out, stream, P, R)

    elapsed_ms, units = aggregate(local_ms, float(args.steps * T), "cuda" if world > 1 else None)
    ms_per_step = elapsed_ms / args.steps
    value = units / (elapsed_ms / 1e3)

    # end to end through the host-buffer entry points: every step copies its
    # inputs from pinned host memory and its outputs back (x|residual and
    # h_out|y_norm adjacent, one copy each way).  Pipelined: the asynchronous
    # call for every step, alternating between two streams with a workspace
    # each, so one step's copies overlap the other's kernel; one
    # synchronisation at the end (each step's host buffers serve one call).
    # Blocking: moe_layer_forward_host, which synchronises every step.
    ne = min(args.e2e_steps, P)
    inp = torch.stack([xs[:ne], rs[:ne]], dim=1).cpu().pin_memory()  # [ne][2][T][H]
    out = torch.empty_like(inp).pin_memory()
    for i in range(5):
        M.moe_layer_forward_host(cfg, reps[i % R]["wts"], inp[i, 0], inp[i, 1], out[i, 0], out[i, 1],
                                 reps[i % R]["ws"], stream=stream)
    torch.cuda.synchronize()
    barrier()
    e2e_streams = [stream, torch.cuda.Stream()]
    e2e_ws = [torch.zeros_like(reps[0]["ws"]) for _ in range(2)]
    for wsb in e2e_ws:
        M.moe_workspace_init(wsb)
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    for i in range(ne):
        M.moe_layer_forward_host_packed(cfg, reps[i % R]["wts"], inp[i], out[i], e2e_ws[i % 2],
                                        stream=e2e_streams[i % 2])
    for st in e2e_streams:
        st.synchronize()
    e2e_ms = (time.perf_counter() - t0) * 1e3
    e2e_err = max(M.moe_device_error(wsb)[0] for wsb in e2e_ws)
    out_pipe = out.clone()
    barrier()
    t0 = time.perf_counter()
    for i in range(ne):
        r = reps[i % R]
        M.moe_layer_forward_host(cfg, r["wts"], inp[i, 0], inp[i, 1], out[i, 0], out[i, 1], r["ws"], stream=stream)
    e2e_sync_ms = (time.perf_counter() - t0) * 1e3
    e2e_same = bool(torch.equal(out, out_pipe))  # the kernel is deterministic: both loops agree bit for bit
    barrier()
    e2e_ms, e2e_units = aggregate(e2e_ms, float(ne * T), "cuda" if world > 1 else None)
    e2e_sync_ms, _ = aggregate(e2e_sync_ms, float(ne * T), "cuda" if world > 1 else None)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        nc = min(host_cores(), 32)
        rate, done, dt = oracle_token_rate(s, nc, seconds_cap=30.0, threads=nc)
        rate1, done1, dt1 = oracle_token_rate(s, 4, seconds_cap=10.0)
        cpu = {"value": rate, "unit": "tokens/s", "cores": nc, "kind": "oracle",
               "sample": "%d tokens of this workload through the C oracle (fp64 dequantise-then-dot), "
                         "%d tokens at a time on %d host threads, %.1f s; experts generated and "
                         "quantised before timing" % (done, nc, nc, dt),
               "single_thread": {"value": rate1, "unit": "tokens/s", "cores": 1,
                                 "sample": "%d tokens, %.1f s" % (done1, dt1)}}

    peak, peak_src = measured_peaks()
    abytes = algorithmic_bytes(s, T)
    achieved = abytes / (ms_per_step * 1e-3) / 1e9
    line = {
        "metric": METRIC if args.bits == 4 else METRIC.replace("4-bit", "2-bit"), "value": value,
        "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None,
        "dtype": decode_dtype(args.bits),
        "data": "synthetic",
        "config": {"workload": s.name, "hidden": s.hidden, "inter": s.inter, "n_experts": s.n_experts,
                   "top_k": s.top_k, "bits": s.bits, "group": s.group, "tokens_per_step": T,
                   "shared_expert": "bf16", "router_bias": "zipf1.1", "replicas": R,
                   "l2": "inputs larger than L2: %d replicas round-robin, %.1f GB of experts" %
                         (R, R * s.n_experts * M.moe_packed_expert_bytes(cfg) / 1e9),
                   "cuda_graph": used_graph, "parallelism": "replicas" if world > 1 else "single"},
        "hbm_gbs": achieved,
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak, "traffic": profiled_traffic(args.bits),
                     "peak_source": peak_src, "algorithmic_bytes_per_launch": abytes,
                     "kernel": "moe_decode_kernel"},
        "e2e": {"value": e2e_units / (e2e_ms / 1e3), "unit": "tokens/s",
                "h2d_bytes_per_step": 2 * T * s.hidden * 2, "d2h_bytes_per_step": 2 * T * s.hidden * 2,
                "api": "moe_layer_forward_host_packed per step (x|residual in, h_out|y_norm out, one copy "
                       "each way), steps alternating over two streams with a workspace each, one "
                       "synchronisation at the end",
                "device_error": e2e_err, "outputs_equal_blocking": e2e_same,
                "blocking_value": e2e_units / (e2e_sync_ms / 1e3),
                "blocking_api": "moe_layer_forward_host (synchronises every step)"},
        "gpu_launches": args.steps,
        "clocks": clk.summary(),
        "l2_warm_tokens_per_s": (T / (warm * 1e-3)) if warm else None,
    }
    if cpu is not None:
        line["cpu_baseline"] = cpu
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()
    return 0


def run_streaming(args):
    """The expert-streaming tier on one GPU: L layers of the workload shape,
    every expert in one pinned host store ([layer][expert] blobs), n_slots
    device slots.  A step is one token through the L layers; per layer: the
    layer's router and the next layer's router on the same input (the
    prediction), one device-to-host read of both top-K results,
    moe_stream_resolve, moe_layer_forward_routed, and moe_stream_prefetch of
    the predicted experts on a side stream.  The layer output (y_norm, h_out)
    is the next layer's (x, residual).  The link figure is the bytes copied
    over the time the copies kept the host-to-device link busy (the union of
    their event-timed intervals), against a 1 GiB pinned copy on the same
    box.  After timing, a few more tokens are checked: every layer's outputs
    must equal, bit for bit, the routed call on the same experts copied
    straight from the store.  --stream-resolve device keeps the routing on
    the GPU: per layer the router, moe_stream_resolve_device (a resolve and a
    fill kernel) and the routed layer; --stream-resolve fused runs each layer
    as one moe_layer_forward_streamed launch (routing, cache lookup, copy of
    the misses by the layer's own blocks, the layer).  Both are captured as a
    CUDA graph per token and have no prediction."""
    import torch
    import quantized_expert_ffn_03_b200 as M

    torch.cuda.set_device(0)
    s = workload(args.bits)
    E, K = s.n_experts, s.top_k
    cfg = M.config(s.hidden, s.inter, E, K, bits=s.bits, eps=s.eps, has_shared=s.has_shared)
    nb = M.moe_packed_expert_bytes(cfg)
    L_req, NS = args.stream_layers, args.stream_slots
    try:
        import psutil
        avail = psutil.virtual_memory().available
    except Exception:
        avail = None
    L = L_req
    if avail is not None:
        L = max(1, min(L_req, int(0.7 * avail) // (E * nb)))
    store = torch.empty((L * E, nb), dtype=torch.uint8, pin_memory=True)
    chunk = 32
    buf = torch.empty((chunk, nb), dtype=torch.uint8, device="cuda")
    for l in range(L):
        for e0 in range(0, E, chunk):
            wg, wu, wd = S.torch_expert_weights(s, e0, chunk, 100 + l, "cuda")
            M.moe_pack_experts_device(cfg, wg, wu, wd, buf)
            del wg, wu, wd
            store[l * E + e0:l * E + e0 + chunk].copy_(buf)
    del buf
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).cuda()
    dense = []
    for l in range(L):
        d = S.dense_weights(s, 100 + l)
        dense.append(dict(wr=dev(d["wr"]), bias=torch.from_numpy(d["bias"]).cuda(), sg=dev(d["shared_gate"]),
                          su=dev(d["shared_up"]), sd=dev(d["shared_down"]), gamma=dev(d["gamma"])))
    table = torch.zeros(E, dtype=torch.int64, device="cuda")
    wts = [M.layer_weights(table, None, None, d["sg"], d["su"], d["sd"], d["gamma"]) for d in dense]
    ws = torch.zeros(M.moe_layer_workspace_bytes(cfg, 1), dtype=torch.uint8, device="cuda")
    M.moe_workspace_init(ws)
    idx_d = torch.empty((2, 1, K), dtype=torch.int32, device="cuda")
    w_d = torch.empty((2, 1, K), dtype=torch.float32, device="cuda")
    lg = torch.empty((2, 1, E), dtype=torch.float32, device="cuda")
    idx_h = torch.empty((2, K), dtype=torch.int32).pin_memory()
    comp = torch.cuda.current_stream()
    side = torch.cuda.Stream()

    # pinned host -> device copy peak (1 GiB, one cudaMemcpyAsync)
    big = torch.empty(1 << 30, dtype=torch.uint8).pin_memory()
    bigd = torch.empty(1 << 30, dtype=torch.uint8, device="cuda")
    bigd.copy_(big, non_blocking=True)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(3):
        bigd.copy_(big, non_blocking=True)
    e1.record()
    torch.cuda.synchronize()
    h2d_peak = 3 * (1 << 30) / (e0.elapsed_time(e1) * 1e-3) / 1e9
    del big, bigd

    if args.store == "file":
        t_w = time.perf_counter()
        store.numpy().tofile(args.store_path)
        write_s = time.perf_counter() - t_w
        cache = M.moe_stream_create_file(cfg, L, args.store_path, NS, direct_io=args.direct_io,
                                         n_read_threads=2 * K)
    else:
        write_s = None
        cache = M.moe_stream_create(cfg, L, store, NS)
    gen = torch.Generator(device="cuda")
    gen.manual_seed(4321)
    h = torch.empty((1, s.hidden), dtype=torch.int16, device="cuda")
    y = torch.empty_like(h)

    fused = args.stream_resolve == "fused"
    on_device = args.stream_resolve in ("device", "fused")
    if on_device and args.store == "file":
        raise SystemExit("--stream-resolve %s needs the pinned store" % args.stream_resolve)
    # fused: each layer's weights with its router (the expert table is the cache)
    wts_f = [M.layer_weights(None, d["wr"], d["bias"], d["sg"], d["su"], d["sd"], d["gamma"]) for d in dense]
    # device-resolved: no prediction (the routing never reaches the host)
    pred = "none" if on_device else args.predictor
    last_idx = [None] * L  # experts each layer chose for the previous token (temporal predictor)

    def token(record=None):
        x = torch.randn((1, s.hidden), generator=gen, device="cuda").to(torch.bfloat16).view(torch.int16)
        res = torch.randn((1, s.hidden), generator=gen, device="cuda").to(torch.bfloat16).view(torch.int16)
        for l in range(L):
            d = dense[l]
            if fused:
                # one launch: route, look the experts up, copy the misses, the layer
                M.moe_layer_forward_streamed(cfg, wts_f[l], x, res, h, y, cache, l, ws, idx_out=idx_d[0],
                                             w_out=w_d[0])
                if record is not None:
                    record.append((l, x.clone(), res.clone(), idx_d[0].clone(), w_d[0].clone(), h.clone(),
                                   y.clone()))
                x, res = y.clone(), h.clone()
                continue
            if on_device:
                # router, device resolve (+ fill of the misses), routed layer: back to back
                M.moe_router_topk(cfg, x, d["wr"], d["bias"], idx_d[0], w_d[0], logits_out=lg[0])
                M.moe_stream_resolve_device(cache, l, idx_d[0], table)
                M.moe_layer_forward_routed(cfg, wts[l], x, res, idx_d[0], w_d[0], h, y, ws)
                if record is not None:
                    record.append((l, x.clone(), res.clone(), idx_d[0].clone(), w_d[0].clone(), h.clone(),
                                   y.clone()))
                x, res = y.clone(), h.clone()
                continue
            M.moe_router_topk(cfg, x, d["wr"], d["bias"], idx_d[0], w_d[0], logits_out=lg[0])
            if pred == "next_router" and l + 1 < L:
                dn = dense[l + 1]
                M.moe_router_topk(cfg, x, dn["wr"], dn["bias"], idx_d[1], w_d[1], logits_out=lg[1])
            idx_h.copy_(idx_d.view(2, K), non_blocking=True)
            comp.synchronize()
            M.moe_stream_resolve(cache, l, idx_h[0].numpy(), table)
            M.moe_layer_forward_routed(cfg, wts[l], x, res, idx_d[0], w_d[0], h, y, ws)
            if record is not None:
                record.append((l, x.clone(), res.clone(), idx_d[0].clone(), w_d[0].clone(), h.clone(), y.clone()))
            if l + 1 < L:
                if pred == "next_router":
                    M.moe_stream_prefetch(cache, l + 1, idx_h[1].numpy(), copy_stream=side)
                elif pred == "temporal" and last_idx[l + 1] is not None:
                    M.moe_stream_prefetch(cache, l + 1, last_idx[l + 1], copy_stream=side)
            last_idx[l] = idx_h[0].numpy().copy()
            x, res = y.clone(), h.clone()

    # device-resolved: one token through the L layers captured as a CUDA
    # graph (router, resolve, fill, routed layer per layer; layer outputs in
    # ping-pong buffers), replayed per token after copying the token's
    # inputs into its input buffers
    graph = None
    use_graph = on_device and not args.no_graph
    if use_graph:
        npool = args.stream_steps + 4
        pool_x = torch.randn((npool, 1, s.hidden), generator=gen, device="cuda").to(torch.bfloat16).view(torch.int16)
        pool_r = torch.randn((npool, 1, s.hidden), generator=gen, device="cuda").to(torch.bfloat16).view(torch.int16)
        xin, rin = torch.empty_like(h), torch.empty_like(h)
        hb = [torch.empty_like(h) for _ in range(2)]
        yb = [torch.empty_like(h) for _ in range(2)]

        def token_body():
            xx, rr = xin, rin
            for l in range(L):
                d = dense[l]
                if fused:
                    M.moe_layer_forward_streamed(cfg, wts_f[l], xx, rr, hb[l % 2], yb[l % 2], cache, l, ws)
                else:
                    M.moe_router_topk(cfg, xx, d["wr"], d["bias"], idx_d[0], w_d[0], logits_out=lg[0])
                    M.moe_stream_resolve_device(cache, l, idx_d[0], table)
                    M.moe_layer_forward_routed(cfg, wts[l], xx, rr, idx_d[0], w_d[0], hb[l % 2], yb[l % 2], ws)
                xx, rr = yb[l % 2], hb[l % 2]

    checked, mismatches = 0, 0
    try:
        for i in range(args.stream_warmup):
            token()
        torch.cuda.synchronize()
        if use_graph:
            cap = torch.cuda.Stream()
            with torch.cuda.stream(cap):
                graph = torch.cuda.CUDAGraph()
                with torch.cuda.graph(graph, stream=cap):
                    token_body()
            torch.cuda.synchronize()
        st0 = M.moe_stream_stats(cache)
        fs0 = M.moe_stream_file_stats(cache) if args.store == "file" else None
        M.moe_stream_copy_timing(cache)  # (enables nothing yet: clears)
        M.moe_stream_enable_copy_timing(cache, True)
        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        wall0 = time.perf_counter()
        t0.record()
        for i in range(args.stream_steps):
            if graph is not None:
                xin.copy_(pool_x[i], non_blocking=True)
                rin.copy_(pool_r[i], non_blocking=True)
                graph.replay()
            else:
                token()
        t1.record()
        torch.cuda.synchronize()
        wall = time.perf_counter() - wall0
        ms = t0.elapsed_time(t1)
        st1 = M.moe_stream_stats(cache)
        fs1 = M.moe_stream_file_stats(cache) if args.store == "file" else None
        ct = M.moe_stream_copy_timing(cache)
        M.moe_stream_enable_copy_timing(cache, False)
        err = M.moe_device_error(ws)[0]
        # check: two more tokens recorded, then each layer recomputed with its
        # experts copied straight from the host store
        rec = []
        for i in range(2):
            token(rec)
        torch.cuda.synchronize()
        tab2 = torch.zeros(E, dtype=torch.int64, device="cuda")
        ws2 = torch.zeros_like(ws)
        M.moe_workspace_init(ws2)
        blobs = torch.empty((K, nb), dtype=torch.uint8, device="cuda")
        for l, x, res, idd, wdd, hh, yy in rec:
            ids = idd.cpu().numpy().ravel()
            for j, e in enumerate(ids):
                blobs[j].copy_(store[l * E + int(e)])
            ptrs = tab2.cpu().numpy()
            for j, e in enumerate(ids):
                ptrs[int(e)] = blobs[j].data_ptr()
            tab2.copy_(torch.from_numpy(ptrs))
            w2 = M.layer_weights(tab2, None, None, dense[l]["sg"], dense[l]["su"], dense[l]["sd"], dense[l]["gamma"])
            h2, y2 = torch.empty_like(hh), torch.empty_like(yy)
            M.moe_layer_forward_routed(cfg, w2, x, res, idd, wdd, h2, y2, ws2)
            torch.cuda.synchronize()
            checked += 1
            if not (torch.equal(h2, hh) and torch.equal(y2, yy)):
                mismatches += 1
        err = err or M.moe_device_error(ws2)[0]
    finally:
        torch.cuda.synchronize()
        M.moe_stream_destroy(cache)
    dst = {k: st1[k] - st0[k] for k in st1}
    looked = dst["hits"] + dst["misses"]
    secs = ms * 1e-3
    link = (ct["bytes"] / (ct["busy_ms"] * 1e-3) / 1e9) if ct["busy_ms"] > 0 else None
    line = {
        "metric": "streaming tier: tokens/s through %d layers, experts in pinned host memory" % L,
        "value": args.stream_steps / secs, "unit": "tokens/s", "impl": "ours", "mode": "streaming",
        "n_gpus": 1, "steps": args.stream_steps, "warmup": args.stream_warmup,
        "ms_per_step": ms / args.stream_steps, "higher_is_better": True, "dtype": decode_dtype(s.bits), "data": "synthetic",
        "config": {"workload": "%s_x%d_layers" % (s.name, L), "layers": L, "layers_requested": L_req,
                   "predictor": pred, "resolve": args.stream_resolve,
                   "copier": ("every block of the layer kernel over mapped host memory" if fused else
                              "fill kernel over mapped host memory" if on_device else "cudaMemcpyAsync"),
                   "launches_per_layer": 1 if fused else (5 if on_device else 3 + 2 * (pred == "next_router")),
                   "host_available_gb": (avail / 1e9) if avail else None, "slots": NS,
                   "slot_bytes": nb, "host_store_gb": L * E * nb / 1e9, "device_cache_gb": NS * nb / 1e9,
                   "tokens_per_step": 1, "router_bias": "zipf1.1, a different permutation per layer"},
        "hit_rate": dst["hits"] / looked if looked else None,
        "misses_per_token": dst["misses"] / args.stream_steps,
        "prefetches_per_token": dst["prefetches"] / args.stream_steps,
        "prefetch_hits_per_token": dst["prefetch_hits"] / args.stream_steps,
        "predictor": pred,
        "prefetch_unused_per_token": (dst["prefetches"] - dst["prefetch_hits"]) / args.stream_steps,
        "prefetch_precision": (dst["prefetch_hits"] / dst["prefetches"]) if dst["prefetches"] else None,
        "h2d_gb_per_token": dst["bytes_h2d"] / args.stream_steps / 1e9,
        "h2d_gbs_average": dst["bytes_h2d"] / secs / 1e9,
        "link": {"gbs_while_copying": link, "peak_gbs": h2d_peak,
                 "frac": (link / h2d_peak) if link else None, "busy_ms": ct["busy_ms"],
                 "copy_ms_sum": ct["copy_ms"], "copies": ct["copies"], "bytes": ct["bytes"],
                 "busy_share_of_step": ct["busy_ms"] / ms if ms > 0 else None},
        "ms_per_layer": ms / args.stream_steps / L,
        "cuda_graph": graph is not None,
        "wall_ms_per_step": wall * 1e3 / args.stream_steps,
        "checked_layers": checked, "mismatched_layers": mismatches,
        "device_error": err, "cache_device_error": st1.get("device_error", 0),
    }
    if args.store == "file":
        reads = fs1["reads"] - fs0["reads"]
        rms = fs1["read_ms"] - fs0["read_ms"]
        rbytes = fs1["read_bytes"] - fs0["read_bytes"]
        line["config"].update({"store": "file", "direct_io": bool(args.direct_io), "read_threads": 2 * K,
                               "store_write_s": write_s})
        line["file_reads"] = {"reads_per_token": reads / args.stream_steps, "read_ms_per_token": rms / args.stream_steps,
                              "read_ms_per_layer": rms / args.stream_steps / L,
                              "read_gbs_while_reading": (rbytes / (rms * 1e-3) / 1e9) if rms > 0 else None}
        try:
            os.remove(args.store_path)
        except OSError:
            pass
    print(json.dumps(line), flush=True)
    return 0 if (err == 0 and mismatches == 0 and st1.get("device_error", 0) == 0) else 1


def run_batched(args):
    """Batches of T tokens per step, under uniform and Zipf(1.1) routing, each
    through both forms of the layer: the batched path (grouped dequant GEMMs
    on the tensor cores, moe_layer_forward_batched) and the fused decode
    kernel on chunks of moe_layer_tokens_per_launch tokens
    (moe_layer_forward_chunked).  One JSON line per (routing, T, path), then
    one line with the measured crossover (the smallest T from which the
    batched path is faster).  Replicas round-robin as in the decode
    measurement; the steps of each measurement are captured in a CUDA graph."""
    import dataclasses
    import torch
    import quantized_expert_ffn_03_b200 as M

    torch.cuda.set_device(0)
    base = workload(args.bits)
    R = max(1, min(args.replicas, 4))
    Ts = [int(v) for v in args.batched.split(",") if v]
    gen = torch.Generator(device="cuda")
    gen.manual_seed(99)
    rc = 0
    results = {}
    for routing in ("uniform", "zipf"):
        s = dataclasses.replace(base, routing=routing)
        reps = [build_replica(M, s, rr, 1) for rr in range(R)]
        cfg = reps[0]["cfg"]
        nb = max(M.moe_layer_batched_workspace_bytes(cfg, max(Ts)), M.moe_layer_workspace_bytes(cfg, 8))
        ws = torch.zeros(nb, dtype=torch.uint8, device="cuda")
        M.moe_workspace_init(ws)
        stream = torch.cuda.Stream()
        for T in Ts:
            x = torch.randn((T, s.hidden), generator=gen, device="cuda").to(torch.bfloat16).view(torch.int16)
            r = torch.randn((T, s.hidden), generator=gen, device="cuda").to(torch.bfloat16).view(torch.int16)
            h, y = torch.empty_like(x), torch.empty_like(x)
            idx = torch.empty((T, s.top_k), dtype=torch.int32, device="cuda")
            w = torch.empty((T, s.top_k), dtype=torch.float32, device="cuda")
            for path in ("batched", "chunked"):
                fn = M.moe_layer_forward_batched if path == "batched" else M.moe_layer_forward_chunked
                launches = -(-T // max(1, M.moe_layer_tokens_per_launch(cfg)))
                steps = max(2, min(20, 2048 // T)) if path == "batched" else max(2, min(20, 256 // launches))
                with torch.cuda.stream(stream):
                    for i in range(3):
                        fn(cfg, reps[i % R]["wts"], x, r, h, y, idx, w, workspace=ws, stream=stream)
                    torch.cuda.synchronize()
                    g = torch.cuda.CUDAGraph()
                    with torch.cuda.graph(g, stream=stream):
                        for i in range(steps):
                            fn(cfg, reps[i % R]["wts"], x, r, h, y, idx, w, workspace=ws, stream=stream)
                    g.replay()
                    torch.cuda.synchronize()
                    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                    e0.record(stream)
                    g.replay()
                    e1.record(stream)
                    torch.cuda.synchronize()
                    del g
                ms = e0.elapsed_time(e1) / steps
                err = M.moe_device_error(ws)[0]
                rc = rc or (1 if err else 0)
                ic = idx.cpu().numpy()
                counts = np.bincount(ic.ravel(), minlength=s.n_experts)
                results[(routing, T, path)] = ms
                line = {"metric": "batched MoE-layer tokens/s (T tokens per step)", "value": T / (ms * 1e-3),
                        "unit": "tokens/s", "impl": "ours", "mode": "batched", "path": path, "n_gpus": 1,
                        "steps": steps, "warmup": 3, "ms_per_step": ms, "higher_is_better": True,
                        "dtype": ("f16 x f16 -> f32 (routed), bf16 (shared, router)" if path == "batched"
                                  else decode_dtype(s.bits)),
                        "data": "synthetic",
                        "config": {"workload": "%s_T%d_%s" % (s.name, T, routing), "tokens_per_step": T,
                                   "routing": routing, "replicas": R, "cuda_graph": True},
                        "experts_used": int((counts > 0).sum()), "max_tokens_per_expert": int(counts.max()),
                        "expert_bytes_per_step": int((counts > 0).sum()) * M.moe_packed_expert_bytes(cfg),
                        "launches_per_step": (8 if path == "batched" else launches), "device_error": err}
                print(json.dumps(line), flush=True)
    for routing in ("uniform", "zipf"):
        cross = None
        for T in Ts:
            if results[(routing, T, "batched")] < results[(routing, T, "chunked")]:
                cross = T
                break
        print(json.dumps({"metric": "GEMV/GEMM crossover (smallest measured T where the batched path is faster)",
                          "mode": "batched", "routing": routing, "crossover_tokens": cross, "measured_T": Ts}),
              flush=True)
    return rc


def main(argv=None):
    args = parse_args(argv)
    if args.impl == "reference":
        return run_reference(args)
    if args.streaming:
        return run_streaming(args)
    if args.batched:
        return run_batched(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
