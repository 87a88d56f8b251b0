"""Python binding of libmoe: the streaming-experts MoE layer on B200.

Argument marshalling only.  Every computation of the layer runs in the CUDA
library (``libmoe.so``, built by ``python quantized_expert_ffn_03_b200/build.py``);
if the library is missing, importing this package raises ImportError.
Device arguments are torch CUDA tensors (bf16 tensors may be torch.bfloat16
or 16-bit integer views); host arguments of the host packer are numpy arrays.
Entry points keep the names of the C ABI in include/moe.h.
"""
import ctypes as C
import os

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmoe.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        "libmoe.so is not built (%s); run `python quantized_expert_ffn_03_b200/build.py`" % LIB_PATH)

_lib = C.CDLL(LIB_PATH)

MOE_OK = 0
MOE_ERR_WORKSPACE = 3
MOE_ERR_DEVICE = 8
NOALLOC_SCRATCH_BYTES = 4 << 20  # MOE_NOALLOC_SCRATCH_BYTES of moe.h
STATUS = {0: "MOE_OK", 1: "MOE_ERR_INVALID_ARG", 2: "MOE_ERR_UNSUPPORTED", 3: "MOE_ERR_WORKSPACE",
          4: "MOE_ERR_CUDA", 5: "MOE_ERR_OOM", 6: "MOE_ERR_TIMEOUT", 7: "MOE_ERR_IO",
          8: "MOE_ERR_DEVICE"}
STATUS_BY_NAME = {v: k for k, v in STATUS.items()}


class MoeError(RuntimeError):
    def __init__(self, status, msg):
        super().__init__("%s: %s" % (STATUS.get(status, status), msg))
        self.status = status


class MoeConfig(C.Structure):
    _fields_ = [("hidden", C.c_int), ("inter", C.c_int), ("n_experts", C.c_int),
                ("top_k", C.c_int), ("bits", C.c_int), ("group", C.c_int),
                ("eps", C.c_float), ("has_shared", C.c_int)]


class MoeLayerWeights(C.Structure):
    _fields_ = [("expert_ptr", C.c_void_p), ("router_w", C.c_void_p), ("router_bias", C.c_void_p),
                ("shared_gate", C.c_void_p), ("shared_up", C.c_void_p), ("shared_down", C.c_void_p),
                ("gamma", C.c_void_p), ("shared_out_gate", C.c_void_p), ("shared_packed", C.c_void_p)]


EXPORTS = {
    "moe_last_error": (C.c_char_p, []),
    "moe_packed_expert_bytes": (C.c_size_t, [C.c_void_p]),
    "moe_packed_layout": (C.c_int, [C.c_void_p, C.c_void_p]),
    "moe_pack_experts": (C.c_int, [C.c_void_p, C.c_void_p, C.c_void_p, C.c_void_p, C.c_int, C.c_int,
                                   C.c_void_p, C.c_size_t]),
    "moe_pack_experts_device": (C.c_int, [C.c_void_p, C.c_void_p, C.c_void_p, C.c_void_p, C.c_int,
                                          C.c_void_p, C.c_size_t, C.c_void_p]),
    "moe_router_workspace_bytes": (C.c_size_t, [C.c_void_p, C.c_int]),
    "moe_router_topk": (C.c_int, [C.c_void_p, C.c_void_p, C.c_void_p, C.c_void_p, C.c_int, C.c_void_p,
                                  C.c_void_p, C.c_void_p, C.c_void_p, C.c_size_t, C.c_void_p]),
    "moe_topk_from_logits": (C.c_int, [C.c_void_p, C.c_void_p, C.c_int, C.c_void_p, C.c_void_p,
                                       C.c_void_p]),
    "moe_layer_workspace_bytes": (C.c_size_t, [C.c_void_p, C.c_int]),
    "moe_workspace_init": (C.c_int, [C.c_void_p, C.c_size_t, C.c_void_p]),
    "moe_layer_forward": (C.c_int, [C.c_void_p, C.c_void_p, C.c_void_p, C.c_void_p, C.c_int,
                                    C.c_void_p, C.c_void_p, C.c_void_p, C.c_void_p, C.c_void_p,
                                    C.c_size_t, C.c_void_p]),
    "moe_layer_host_workspace_bytes": (C.c_size_t, [C.c_void_p, C.c_int]),
    "moe_layer_forward_host": (C.c_int, [C.c_void_p, C.c_void_p, C.c_void_p, C.c_void_p, C.c_int,
                                         C.c_void_p, C.c_void_p, C.c_void_p, C.c_size_t, C.c_void_p]),
    "moe_layer_forward_host_async": (C.c_int, [C.c_void_p, C.c_void_p, C.c_void_p, C.c_void_p, C.c_int,
                                               C.c_void_p, C.c_void_p, C.c_void_p, C.c_size_t, C.c_void_p]),
    "moe_layer_forward_host_packed": (C.c_int, [C.c_void_p, C.c_void_p, C.c_void_p, C.c_int, C.c_void_p,
                                                C.c_void_p, C.c_size_t, C.c_void_p]),
    "moe_layer_trace_blocks": (C.c_int, []),
    "moe_layer_forward_traced": (C.c_int, [C.c_void_p, C.c_void_p, C.c_void_p, C.c_void_p, C.c_int,
                                           C.c_void_p, C.c_void_p, C.c_void_p, C.c_size_t, C.c_void_p,
                                           C.c_size_t, C.c_void_p]),
    "moe_layer_forward_noalloc": (C.c_int, [C.c_void_p, C.c_void_p, C.c_void_p, C.c_void_p, C.c_int,
                                            C.c_void_p, C.c_void_p, C.c_void_p, C.c_void_p, C.c_void_p]),
    "moe_layer_tokens_per_launch": (C.c_int, [C.c_void_p]),
    "moe_layer_batched_workspace_bytes": (C.c_size_t, [C.c_void_p, C.c_int]),
    "moe_layer_forward_batched": (C.c_int, [C.c_void_p, C.c_void_p, C.c_void_p, C.c_void_p, C.c_int,
                                            C.c_void_p, C.c_void_p, C.c_void_p, C.c_void_p, C.c_void_p,
                                            C.c_size_t, C.c_void_p]),
    "moe_layer_forward_chunked": (C.c_int, [C.c_void_p, C.c_void_p, C.c_void_p, C.c_void_p, C.c_int,
                                            C.c_void_p, C.c_void_p, C.c_void_p, C.c_void_p, C.c_void_p,
                                            C.c_size_t, C.c_void_p]),
    "moe_layer_forward_prenorm": (C.c_int, [C.c_void_p, C.c_void_p, C.c_void_p, C.c_void_p, C.c_int,
                                            C.c_void_p, C.c_void_p, C.c_void_p, C.c_void_p, C.c_void_p,
                                            C.c_void_p, C.c_size_t, C.c_void_p]),
    "moe_layer_forward_routed": (C.c_int, [C.c_void_p, C.c_void_p, C.c_void_p, C.c_void_p, C.c_int,
                                           C.c_void_p, C.c_void_p, C.c_void_p, C.c_void_p, C.c_void_p,
                                           C.c_size_t, C.c_void_p]),
    "moe_stream_create": (C.c_int, [C.c_void_p, C.c_int, C.c_void_p, C.c_size_t, C.c_int, C.c_void_p]),
    "moe_stream_inject_fault": (C.c_int, [C.c_void_p, C.c_int, C.c_int]),
    "moe_stream_create_file": (C.c_int, [C.c_void_p, C.c_int, C.c_char_p, C.c_int, C.c_int, C.c_int,
                                         C.c_void_p]),
    "moe_stream_file_stats": (C.c_int, [C.c_void_p, C.c_void_p, C.c_void_p, C.c_void_p]),
    "moe_stream_enable_copy_timing": (C.c_int, [C.c_void_p, C.c_int]),
    "moe_stream_copy_timing": (C.c_int, [C.c_void_p, C.c_void_p]),
    "moe_stream_prefetch": (C.c_int, [C.c_void_p, C.c_int, C.c_void_p, C.c_int, C.c_void_p]),
    "moe_stream_resolve": (C.c_int, [C.c_void_p, C.c_int, C.c_void_p, C.c_int, C.c_void_p, C.c_void_p]),
    "moe_stream_stats": (C.c_int, [C.c_void_p, C.c_void_p]),
    "moe_stream_resolve_device": (C.c_int, [C.c_void_p, C.c_int, C.c_void_p, C.c_int, C.c_void_p, C.c_void_p]),
    "moe_layer_forward_streamed": (C.c_int, [C.c_void_p, C.c_void_p, C.c_void_p, C.c_void_p, C.c_int,
                                             C.c_void_p, C.c_void_p, C.c_void_p, C.c_void_p, C.c_void_p,
                                             C.c_int, C.c_void_p, C.c_size_t, C.c_void_p]),
    "moe_stream_destroy": (None, [C.c_void_p]),
    "moe_device_error": (C.c_int, [C.c_void_p, C.c_void_p, C.c_void_p]),
    "moe_noalloc_device_error": (C.c_int, [C.c_void_p, C.c_void_p]),
    "moe_selftest_bounded_wait": (C.c_int, [C.c_void_p, C.c_size_t, C.c_uint64, C.c_void_p]),
}

for _name, (_res, _args) in EXPORTS.items():
    _f = getattr(_lib, _name)
    _f.restype = _res
    _f.argtypes = _args


def lib():
    return _lib


def last_error():
    return _lib.moe_last_error().decode()


def _check(status):
    if status != MOE_OK:
        raise MoeError(status, last_error())


def config(hidden, inter, n_experts, top_k, bits=4, group=64, eps=1e-6, has_shared=1):
    return MoeConfig(hidden, inter, n_experts, top_k, bits, group, eps, has_shared)


def _ptr(t):
    """Device or host address of a torch tensor / numpy array / int / None."""
    if t is None:
        return None
    if isinstance(t, int):
        return t
    if isinstance(t, np.ndarray):
        return t.ctypes.data
    return t.data_ptr()


def _nbytes(t):
    """Byte size of a torch tensor / numpy array (0 for None)."""
    if t is None:
        return 0
    if isinstance(t, np.ndarray):
        return t.nbytes
    if isinstance(t, int):
        raise TypeError("a raw address needs an explicit byte count")
    return t.numel() * t.element_size()


def _stream(stream):
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


# ---- packed format -------------------------------------------------------------

def moe_packed_expert_bytes(cfg):
    return _lib.moe_packed_expert_bytes(C.byref(cfg))


def moe_packed_layout(cfg):
    off = (C.c_size_t * 6)()
    _check(_lib.moe_packed_layout(C.byref(cfg), off))
    return [int(v) for v in off]


def moe_pack_experts(cfg, w_gate, w_up, w_down, e_begin=0, e_count=None):
    """Host packer.  w_gate/w_up: float32 [n][I][H], w_down: float32 [n][H][I]
    (numpy).  Returns uint8 [e_count][bytes]."""
    wg = np.ascontiguousarray(w_gate, dtype=np.float32)
    wu = np.ascontiguousarray(w_up, dtype=np.float32)
    wd = np.ascontiguousarray(w_down, dtype=np.float32)
    if wg.ndim == 2:
        wg, wu, wd = wg[None], wu[None], wd[None]
    if e_count is None:
        e_count = wg.shape[0] - e_begin
    nb = moe_packed_expert_bytes(cfg)
    out = np.zeros((e_count, nb), dtype=np.uint8)
    _check(_lib.moe_pack_experts(C.byref(cfg), _ptr(wg), _ptr(wu), _ptr(wd), e_begin, e_count,
                                 _ptr(out), out.nbytes))
    return out


def moe_pack_experts_device(cfg, w_gate, w_up, w_down, out, stream=None):
    """Device packer: torch float32 CUDA tensors [n][I][H], [n][I][H], [n][H][I];
    out: torch uint8 CUDA tensor of n * moe_packed_expert_bytes bytes."""
    n = w_gate.shape[0]
    _check(_lib.moe_pack_experts_device(C.byref(cfg), _ptr(w_gate), _ptr(w_up), _ptr(w_down), n,
                                        _ptr(out), out.numel() * out.element_size(), _stream(stream)))
    return out


# ---- router ----------------------------------------------------------------------

def moe_router_workspace_bytes(cfg, T):
    return _lib.moe_router_workspace_bytes(C.byref(cfg), T)


def moe_router_topk(cfg, x, wr, bias, idx, w, logits_out=None, workspace=None, stream=None):
    T = x.shape[0]
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(_lib.moe_router_topk(C.byref(cfg), _ptr(x), _ptr(wr), _ptr(bias), T, _ptr(idx), _ptr(w),
                                _ptr(logits_out), _ptr(workspace), ws_bytes, _stream(stream)))


def moe_topk_from_logits(cfg, logits, idx, w, stream=None):
    _check(_lib.moe_topk_from_logits(C.byref(cfg), _ptr(logits), logits.shape[0], _ptr(idx), _ptr(w),
                                     _stream(stream)))


# ---- layer -----------------------------------------------------------------------

def moe_layer_workspace_bytes(cfg, T):
    return _lib.moe_layer_workspace_bytes(C.byref(cfg), T)


def moe_layer_host_workspace_bytes(cfg, T):
    return _lib.moe_layer_host_workspace_bytes(C.byref(cfg), T)


def moe_workspace_init(workspace, stream=None):
    _check(_lib.moe_workspace_init(_ptr(workspace), workspace.numel() * workspace.element_size(),
                                   _stream(stream)))


def layer_weights(expert_ptr, router_w, router_bias, shared_gate, shared_up, shared_down, gamma,
                  shared_out_gate=None, shared_packed=None):
    """expert_ptr: int64 CUDA tensor [E] of blob addresses; the rest CUDA tensors or None
    (shared_packed: a uint8 CUDA tensor holding one packed blob)."""
    return MoeLayerWeights(_ptr(expert_ptr), _ptr(router_w), _ptr(router_bias), _ptr(shared_gate),
                           _ptr(shared_up), _ptr(shared_down), _ptr(gamma), _ptr(shared_out_gate),
                           _ptr(shared_packed))


def moe_layer_forward(cfg, wts, x, residual, h_out, y_norm, idx_out=None, w_out=None,
                      workspace=None, stream=None):
    T = x.shape[0]
    _check(_lib.moe_layer_forward(C.byref(cfg), C.byref(wts), _ptr(x), _ptr(residual), T, _ptr(h_out),
                                  _ptr(y_norm), _ptr(idx_out), _ptr(w_out), _ptr(workspace),
                                  workspace.numel() * workspace.element_size(), _stream(stream)))


def moe_layer_tokens_per_launch(cfg):
    return _lib.moe_layer_tokens_per_launch(C.byref(cfg))


def moe_layer_batched_workspace_bytes(cfg, T):
    return _lib.moe_layer_batched_workspace_bytes(C.byref(cfg), int(T))


def moe_layer_forward_batched(cfg, wts, x, residual, h_out, y_norm, idx_out=None, w_out=None,
                              workspace=None, stream=None):
    """The layer through the grouped tensor-core GEMMs (see moe.h)."""
    T = x.shape[0]
    _check(_lib.moe_layer_forward_batched(C.byref(cfg), C.byref(wts), _ptr(x), _ptr(residual), T, _ptr(h_out),
                                          _ptr(y_norm), _ptr(idx_out), _ptr(w_out), _ptr(workspace),
                                          workspace.numel() * workspace.element_size(), _stream(stream)))


def moe_layer_forward_chunked(cfg, wts, x, residual, h_out, y_norm, idx_out=None, w_out=None,
                              workspace=None, stream=None):
    """The layer through the fused decode kernel on chunks of tokens (see moe.h)."""
    T = x.shape[0]
    _check(_lib.moe_layer_forward_chunked(C.byref(cfg), C.byref(wts), _ptr(x), _ptr(residual), T, _ptr(h_out),
                                          _ptr(y_norm), _ptr(idx_out), _ptr(w_out), _ptr(workspace),
                                          workspace.numel() * workspace.element_size(), _stream(stream)))


def moe_layer_forward_prenorm(cfg, wts, gamma_pre, h_in, h_out, y_norm, x_out, idx_out=None, w_out=None,
                              workspace=None, stream=None):
    """The layer with the RMSNorm before it, on the residual stream h_in (see moe.h)."""
    T = h_in.shape[0]
    _check(_lib.moe_layer_forward_prenorm(C.byref(cfg), C.byref(wts), _ptr(gamma_pre), _ptr(h_in), T,
                                          _ptr(h_out), _ptr(y_norm), _ptr(idx_out), _ptr(w_out), _ptr(x_out),
                                          _ptr(workspace), workspace.numel() * workspace.element_size(),
                                          _stream(stream)))


def moe_layer_forward_routed(cfg, wts, x, residual, idx, w, h_out, y_norm, workspace, stream=None):
    """The layer with the routing given: idx int32 [T][K], w float32 [T][K] (CUDA)."""
    T = x.shape[0]
    _check(_lib.moe_layer_forward_routed(C.byref(cfg), C.byref(wts), _ptr(x), _ptr(residual), T, _ptr(idx),
                                         _ptr(w), _ptr(h_out), _ptr(y_norm), _ptr(workspace),
                                         workspace.numel() * workspace.element_size(), _stream(stream)))


def moe_layer_forward_noalloc(cfg, wts, x, residual, h_out, y_norm, idx_out=None, w_out=None, stream=None):
    """moe_layer_forward on the library's built-in scratch (no workspace)."""
    T = x.shape[0]
    _check(_lib.moe_layer_forward_noalloc(C.byref(cfg), C.byref(wts), _ptr(x), _ptr(residual), T, _ptr(h_out),
                                          _ptr(y_norm), _ptr(idx_out), _ptr(w_out), _stream(stream)))


def moe_layer_trace_blocks():
    return _lib.moe_layer_trace_blocks()


def moe_layer_forward_traced(cfg, wts, x, residual, h_out, y_norm, trace, workspace, stream=None):
    """trace: int64 CUDA tensor of moe_layer_trace_blocks()*128 entries."""
    T = x.shape[0]
    _check(_lib.moe_layer_forward_traced(C.byref(cfg), C.byref(wts), _ptr(x), _ptr(residual), T,
                                         _ptr(h_out), _ptr(y_norm), _ptr(workspace),
                                         workspace.numel() * workspace.element_size(), _ptr(trace),
                                         trace.numel(), _stream(stream)))


def moe_layer_forward_host(cfg, wts, x, residual, h_out, y_norm, workspace, stream=None):
    """x, residual, h_out, y_norm: host arrays/tensors (pinned for async copies)."""
    T = x.shape[0]
    _check(_lib.moe_layer_forward_host(C.byref(cfg), C.byref(wts), _ptr(x), _ptr(residual), T,
                                       _ptr(h_out), _ptr(y_norm), _ptr(workspace),
                                       workspace.numel() * workspace.element_size(), _stream(stream)))


def moe_layer_forward_host_async(cfg, wts, x, residual, h_out, y_norm, workspace, stream=None):
    """moe_layer_forward_host without the final synchronisation (see moe.h)."""
    T = x.shape[0]
    _check(_lib.moe_layer_forward_host_async(C.byref(cfg), C.byref(wts), _ptr(x), _ptr(residual), T,
                                             _ptr(h_out), _ptr(y_norm), _ptr(workspace),
                                             workspace.numel() * workspace.element_size(), _stream(stream)))


def moe_layer_forward_host_packed(cfg, wts, xr, hy, workspace, stream=None):
    """xr: pinned host [2][T][H] (x, residual); hy: pinned host [2][T][H]
    (h_out, y_norm), filled once the stream reaches the end of the call."""
    T = xr.shape[1]
    _check(_lib.moe_layer_forward_host_packed(C.byref(cfg), C.byref(wts), _ptr(xr), T, _ptr(hy), _ptr(workspace),
                                              workspace.numel() * workspace.element_size(), _stream(stream)))


# ---- expert-streaming tier -------------------------------------------------------

class MoeStreamCounters(C.Structure):
    _fields_ = [("hits", C.c_uint64), ("misses", C.c_uint64), ("prefetches", C.c_uint64),
                ("prefetch_hits", C.c_uint64), ("prefetch_dropped", C.c_uint64), ("bytes_h2d", C.c_uint64),
                ("device_error", C.c_uint64)]


def moe_stream_create(cfg, n_layers, host_store, n_slots, store_bytes=None):
    """host_store: pinned host tensor (or address) of n_layers*E packed blobs;
    store_bytes defaults to the tensor's size.  Returns the cache handle (an
    int)."""
    if store_bytes is None:
        store_bytes = _nbytes(host_store)
    h = C.c_void_p(0)
    _check(_lib.moe_stream_create(C.byref(cfg), int(n_layers), _ptr(host_store), int(store_bytes), int(n_slots),
                                  C.byref(h)))
    return h.value


def moe_stream_create_file(cfg, n_layers, path, n_slots, direct_io=False, n_read_threads=4):
    """A cache whose store is a file of n_layers*E packed blobs (see moe.h).
    Returns the cache handle (an int)."""
    h = C.c_void_p(0)
    _check(_lib.moe_stream_create_file(C.byref(cfg), int(n_layers), os.fsencode(path), 1 if direct_io else 0,
                                       int(n_slots), int(n_read_threads), C.byref(h)))
    return h.value


def moe_stream_file_stats(cache):
    reads, nbytes, ms = C.c_uint64(0), C.c_uint64(0), C.c_double(0.0)
    _check(_lib.moe_stream_file_stats(cache, C.byref(reads), C.byref(nbytes), C.byref(ms)))
    return {"reads": int(reads.value), "read_bytes": int(nbytes.value), "read_ms": float(ms.value)}


MOE_FAULT_NONE, MOE_FAULT_COPY, MOE_FAULT_ALLOC = 0, 1, 2


def moe_stream_inject_fault(cache, what, countdown=0):
    _check(_lib.moe_stream_inject_fault(cache, int(what), int(countdown)))


def _ids(ids):
    a = np.ascontiguousarray(np.asarray(ids, dtype=np.int32).reshape(-1))
    return a, a.size


def moe_stream_prefetch(cache, layer, expert_ids, copy_stream=None):
    a, n = _ids(expert_ids)
    _check(_lib.moe_stream_prefetch(cache, int(layer), a.ctypes.data, n, _stream(copy_stream)))


def moe_stream_resolve(cache, layer, idx, expert_ptr, stream=None):
    """idx: host ids (numpy / list); expert_ptr: int64 CUDA tensor [E] (written)."""
    a, n = _ids(idx)
    _check(_lib.moe_stream_resolve(cache, int(layer), a.ctypes.data, n, _ptr(expert_ptr), _stream(stream)))


def moe_stream_resolve_device(cache, layer, idx, expert_ptr, stream=None):
    """idx: int32 CUDA tensor of expert ids (any shape, at most 64); expert_ptr:
    int64 CUDA tensor [E] (written on the device).  Nothing is read back."""
    _check(_lib.moe_stream_resolve_device(cache, int(layer), _ptr(idx), int(idx.numel()), _ptr(expert_ptr),
                                          _stream(stream)))


def moe_layer_forward_streamed(cfg, wts, x, residual, h_out, y_norm, cache, layer, workspace, idx_out=None,
                               w_out=None, stream=None):
    """One streamed layer in one launch: the routed experts come from the
    device-resolved cache `cache` (layer `layer`); wts' expert_ptr is ignored."""
    T = x.shape[0]
    _check(_lib.moe_layer_forward_streamed(C.byref(cfg), C.byref(wts), _ptr(x), _ptr(residual), T, _ptr(h_out),
                                           _ptr(y_norm), _ptr(idx_out), _ptr(w_out), cache, int(layer),
                                           _ptr(workspace), workspace.numel() * workspace.element_size(),
                                           _stream(stream)))


def moe_stream_stats(cache):
    out = MoeStreamCounters()
    _check(_lib.moe_stream_stats(cache, C.byref(out)))
    return {f: int(getattr(out, f)) for f, _ in MoeStreamCounters._fields_}


class MoeStreamCopyTimes(C.Structure):
    _fields_ = [("busy_ms", C.c_double), ("copy_ms", C.c_double), ("copies", C.c_uint64), ("bytes", C.c_uint64)]


def moe_stream_enable_copy_timing(cache, on=True):
    _check(_lib.moe_stream_enable_copy_timing(cache, 1 if on else 0))


def moe_stream_copy_timing(cache):
    out = MoeStreamCopyTimes()
    _check(_lib.moe_stream_copy_timing(cache, C.byref(out)))
    return {f: (float(getattr(out, f)) if f.endswith("_ms") else int(getattr(out, f)))
            for f, _ in MoeStreamCopyTimes._fields_}


def moe_stream_destroy(cache):
    _lib.moe_stream_destroy(cache)


def moe_device_error(workspace, stream=None):
    """Returns (status, detail) and clears the workspace's error word."""
    detail = C.c_uint32(0)
    st = _lib.moe_device_error(_ptr(workspace), C.byref(detail), _stream(stream))
    return st, detail.value


def moe_noalloc_device_error(stream=None):
    """Returns (status, detail) of the last moe_layer_forward_noalloc call on
    the current device and clears it."""
    detail = C.c_uint32(0)
    st = _lib.moe_noalloc_device_error(C.byref(detail), _stream(stream))
    return st, detail.value


def moe_selftest_bounded_wait(workspace, timeout_ns, stream=None):
    _check(_lib.moe_selftest_bounded_wait(_ptr(workspace), workspace.numel() * workspace.element_size(),
                                          int(timeout_ns), _stream(stream)))
