"""numpy wrapper over the C oracle (test infrastructure only).

Arrays: bf16 tensors travel as numpy uint16 bit patterns, float weights as
float32, results of the oracle as float64.
"""
import ctypes as C
import os

import numpy as np

from .build import build

_lib = None


class OrcCfg(C.Structure):
    _fields_ = [("hidden", C.c_int), ("inter", C.c_int), ("n_experts", C.c_int),
                ("top_k", C.c_int), ("bits", C.c_int), ("group", C.c_int),
                ("eps", C.c_float), ("has_shared", C.c_int)]


def use_library(path):
    """Point the wrapper at another build of the oracle (planted-mistake
    builds in the pin tests); returns the previous handle."""
    global _lib
    prev = _lib
    _lib = None
    lib(path)
    return prev


def restore_library(handle):
    global _lib
    _lib = handle


def lib(path=None):
    global _lib
    if _lib is None:
        path = path or build()
        _lib = C.CDLL(path)
        P = C.c_void_p
        cfgp = C.POINTER(OrcCfg)
        _lib.orc_expert_bytes.restype = C.c_size_t
        _lib.orc_expert_bytes.argtypes = [cfgp]
        _lib.orc_section_offsets.argtypes = [cfgp, C.POINTER(C.c_size_t)]
        _lib.orc_f32_to_bf16.restype = C.c_uint16
        _lib.orc_f32_to_bf16.argtypes = [C.c_float]
        _lib.orc_bf16_to_f64.restype = C.c_double
        _lib.orc_bf16_to_f64.argtypes = [C.c_uint16]
        _lib.orc_f64_to_bf16.restype = C.c_uint16
        _lib.orc_f64_to_bf16.argtypes = [C.c_double]
        _lib.orc_prenorm.argtypes = [cfgp, P, P, C.c_int, P]
        _lib.orc_quantize_expert.restype = C.c_int
        _lib.orc_quantize_expert.argtypes = [cfgp, P, P, P, P]
        _lib.orc_dequant.restype = C.c_double
        _lib.orc_dequant.argtypes = [cfgp, P, C.c_int, C.c_int, C.c_int]
        _lib.orc_code.restype = C.c_int
        _lib.orc_code.argtypes = [cfgp, P, C.c_int, C.c_int, C.c_int]
        _lib.orc_dequant_matrix.argtypes = [cfgp, P, C.c_int, P]
        _lib.orc_router.argtypes = [cfgp, P, P, P, C.c_int, P, P, P]
        _lib.orc_topk.argtypes = [cfgp, P, C.c_int, P, P, P]
        _lib.orc_expert_ffn.argtypes = [cfgp, P, P, P]
        _lib.orc_expert_ffn_fma_form.argtypes = [cfgp, P, P, P]
        _lib.orc_expert_act.argtypes = [cfgp, P, P, P]
        _lib.orc_shared_ffn.argtypes = [cfgp, P, P, P, P, P]
        _lib.orc_layer_forward.argtypes = [cfgp, P, P, P, P, P, P, P, P, P, C.c_int,
                                           P, P, P, P, P, P]
        _lib.orc_layer_forward_ex.argtypes = [cfgp, P, P, P, P, P, P, P, P, P, P, P, C.c_int,
                                              P, P, P, P, P, P]
    return _lib


def cfg(hidden, inter, n_experts, top_k, bits=4, group=64, eps=1e-6, has_shared=1):
    return OrcCfg(hidden, inter, n_experts, top_k, bits, group, eps, has_shared)


def _p(a):
    return None if a is None else a.ctypes.data_as(C.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def expert_bytes(c):
    return lib().orc_expert_bytes(C.byref(c))


def section_offsets(c):
    off = (C.c_size_t * 6)()
    lib().orc_section_offsets(C.byref(c), off)
    return [int(v) for v in off]


def f32_to_bf16(a):
    a = np.asarray(a, dtype=np.float32)
    f = lib().orc_f32_to_bf16
    return np.array([f(float(v)) for v in a.ravel()], dtype=np.uint16).reshape(a.shape)


def f64_to_bf16(a):
    a = np.asarray(a, dtype=np.float64)
    f = lib().orc_f64_to_bf16
    return np.array([f(float(v)) for v in a.ravel()], dtype=np.uint16).reshape(a.shape)


def prenorm(c, h_bf16, gamma_bf16):
    """x = h / sqrt(mean(h^2) + eps) * gamma per token, in double [T][H]."""
    h = _c(h_bf16, np.uint16)
    g = _c(gamma_bf16, np.uint16)
    T = h.shape[0]
    assert h.shape == (T, c.hidden) and g.shape == (c.hidden,)
    out = np.zeros((T, c.hidden), dtype=np.float64)
    lib().orc_prenorm(C.byref(c), _p(h), _p(g), T, _p(out))
    return out


def bf16_to_f64(a):
    a = np.asarray(a, dtype=np.uint16)
    return (a.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def quantize_expert(c, w_gate, w_up, w_down):
    wg, wu, wd = _c(w_gate, np.float32), _c(w_up, np.float32), _c(w_down, np.float32)
    assert wg.shape == (c.inter, c.hidden) and wu.shape == wg.shape
    assert wd.shape == (c.hidden, c.inter)
    out = np.zeros(expert_bytes(c), dtype=np.uint8)
    rc = lib().orc_quantize_expert(C.byref(c), _p(wg), _p(wu), _p(wd), _p(out))
    assert rc == 0
    return out


def dequant(c, blob, m, row, col):
    return lib().orc_dequant(C.byref(c), _p(blob), m, row, col)


def code(c, blob, m, row, col):
    return lib().orc_code(C.byref(c), _p(blob), m, row, col)


def dequant_matrix(c, blob, m):
    rows, cols = (c.hidden, c.inter) if m == 2 else (c.inter, c.hidden)
    out = np.zeros((rows, cols), dtype=np.float64)
    lib().orc_dequant_matrix(C.byref(c), _p(blob), m, _p(out))
    return out


def router(c, x_bf16, wr_bf16, bias=None):
    x = _c(x_bf16, np.uint16)
    wr = _c(wr_bf16, np.uint16)
    T = x.shape[0]
    b = None if bias is None else _c(bias, np.float32)
    logits = np.zeros((T, c.n_experts), dtype=np.float32)
    idx = np.zeros((T, c.top_k), dtype=np.int32)
    w = np.zeros((T, c.top_k), dtype=np.float32)
    lib().orc_router(C.byref(c), _p(x), _p(wr), _p(b), T, _p(logits), _p(idx), _p(w))
    return logits, idx, w


def topk(c, logits):
    l = _c(logits, np.float32)
    T = l.shape[0]
    idx = np.zeros((T, c.top_k), dtype=np.int32)
    w = np.zeros((T, c.top_k), dtype=np.float32)
    w64 = np.zeros((T, c.top_k), dtype=np.float64)
    lib().orc_topk(C.byref(c), _p(l), T, _p(idx), _p(w), _p(w64))
    return idx, w, w64


def expert_ffn(c, blob, x):
    x = _c(x, np.float64)
    y = np.zeros(c.hidden, dtype=np.float64)
    lib().orc_expert_ffn(C.byref(c), _p(blob), _p(x), _p(y))
    return y


def expert_ffn_fma_form(c, blob, x):
    x = _c(x, np.float64)
    y = np.zeros(c.hidden, dtype=np.float64)
    lib().orc_expert_ffn_fma_form(C.byref(c), _p(blob), _p(x), _p(y))
    return y


def expert_act(c, blob, x):
    x = _c(x, np.float64)
    a = np.zeros(c.inter, dtype=np.float64)
    lib().orc_expert_act(C.byref(c), _p(blob), _p(x), _p(a))
    return a


def shared_ffn(c, wg, wu, wd, x):
    x = _c(x, np.float64)
    y = np.zeros(c.hidden, dtype=np.float64)
    lib().orc_shared_ffn(C.byref(c), _p(_c(wg, np.uint16)), _p(_c(wu, np.uint16)),
                         _p(_c(wd, np.uint16)), _p(x), _p(y))
    return y


def layer_forward(c, experts, wr, bias, shared_gate, shared_up, shared_down, gamma,
                  x, residual, idx_in=None, w_in=None, shared_blob=None, shared_gate_w=None):
    """experts: list (length E) of uint8 blobs (entries may repeat).
    shared_blob: the shared expert packed like the routed ones (replaces the
    bf16 weights); shared_gate_w: bf16 [H], the shared output scaled by
    sigmoid(x . shared_gate_w)."""
    x = _c(x, np.uint16)
    T = x.shape[0]
    blobs = [_c(b, np.uint8) for b in experts]
    ptrs = (C.c_void_p * len(blobs))(*[b.ctypes.data for b in blobs])
    idx = np.zeros((T, c.top_k), dtype=np.int32)
    w = np.zeros((T, c.top_k), dtype=np.float32)
    h = np.zeros((T, c.hidden), dtype=np.float64)
    yn = np.zeros((T, c.hidden), dtype=np.float64)
    sg = None if shared_gate is None else _c(shared_gate, np.uint16)
    su = None if shared_up is None else _c(shared_up, np.uint16)
    sd = None if shared_down is None else _c(shared_down, np.uint16)
    bb = None if bias is None else _c(bias, np.float32)
    ii = None if idx_in is None else _c(idx_in, np.int32)
    wi = None if w_in is None else _c(w_in, np.float64)
    sb = None if shared_blob is None else _c(shared_blob, np.uint8)
    sgw = None if shared_gate_w is None else _c(shared_gate_w, np.uint16)
    lib().orc_layer_forward_ex(C.byref(c), C.cast(ptrs, C.c_void_p), _p(_c(wr, np.uint16)),
                               _p(bb), _p(sg), _p(su), _p(sd), _p(sb), _p(sgw), _p(_c(gamma, np.uint16)),
                               _p(x), _p(_c(residual, np.uint16)), T, _p(ii), _p(wi),
                               _p(idx), _p(w), _p(h), _p(yn))
    return idx, w, h, yn


def layer_forward_prenorm(c, experts, wr, bias, shared_gate, shared_up, shared_down, gamma,
                          gamma_pre, h_in):
    """The layer with the RMSNorm before it: x = bf16(prenorm(h_in)), then
    the layer on x with h_in as the residual.  Returns (x_bf16, idx, w, h, y)."""
    x = f64_to_bf16(prenorm(c, h_in, gamma_pre))
    return (x,) + tuple(layer_forward(c, experts, wr, bias, shared_gate, shared_up, shared_down,
                                      gamma, x, h_in))
