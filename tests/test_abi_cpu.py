"""CPU-side checks of the C-ABI library: it loads, exports every symbol the
header declares, the host packer matches the oracle's packer bit for bit,
and argument checks reject bad calls before touching a GPU."""
import ctypes as C
import os
import re
import subprocess

import numpy as np
import pytest

import oracle as O
import synth as S
import quantized_expert_ffn_03_b200 as M
from conftest import ROOT


def _declared_symbols():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            text = open(os.path.join(ROOT, "include", fn)).read()
            text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
            names |= set(re.findall(r"\b(moe_[a-z0-9_]+)\s*\(", text))
    return sorted(names)


def test_library_exports_every_declared_symbol():
    syms = _declared_symbols()
    assert len(syms) >= 15
    out = subprocess.run(["nm", "-D", "--defined-only", M.LIB_PATH], capture_output=True, text=True,
                         check=True).stdout
    exported = set(re.findall(r" T (moe_[a-z0-9_]+)$", out, flags=re.M))
    missing = [s for s in syms if s not in exported]
    assert not missing, missing
    for s in syms:
        assert hasattr(M.lib(), s)


def test_binding_names_match_header():
    for s in _declared_symbols():
        assert s in M.EXPORTS, s


@pytest.mark.parametrize("H,I,bits", [(4096, 1024, 4), (4096, 1024, 2), (256, 128, 4), (320, 192, 2),
                                      (64, 64, 4)])
def test_layout_matches_oracle(H, I, bits):
    cfg = M.config(H, I, 16, 2, bits=bits)
    oc = O.cfg(H, I, 16, 2, bits=bits)
    assert M.moe_packed_expert_bytes(cfg) == O.expert_bytes(oc)
    assert M.moe_packed_layout(cfg) == O.section_offsets(oc)


def test_packed_size_config_matches_pages():
    assert M.moe_packed_expert_bytes(M.config(4096, 1024, 512, 4, bits=4)) == 7077888
    assert M.moe_packed_expert_bytes(M.config(4096, 1024, 512, 4, bits=2)) == 3932160


@pytest.mark.parametrize("bits", [4, 2])
@pytest.mark.parametrize("H,I", [(256, 128), (320, 192)])
def test_host_packer_matches_oracle_bitwise(bits, H, I):
    s = S.LayerShape("t", H, I, 4, 2, bits=bits)
    cfg = M.config(H, I, 4, 2, bits=bits)
    oc = O.cfg(H, I, 4, 2, bits=bits)
    ws = [S.expert_weights(s, e) for e in range(3)]
    # planted edge groups: constant, all zero, a single outlier, exact halves
    ws[1][0][0, :64] = 0.125
    ws[1][1][2, 64:128] = 0.0
    ws[1][2][5, :64] = 0.0
    ws[1][2][5, 7] = 3.0
    ws[2][0][1, :64] = np.arange(64, dtype=np.float32) * np.float32(0.5)
    wg = np.stack([w[0] for w in ws])
    wu = np.stack([w[1] for w in ws])
    wd = np.stack([w[2] for w in ws])
    got = M.moe_pack_experts(cfg, wg, wu, wd)
    for e in range(3):
        ref = O.quantize_expert(oc, wg[e], wu[e], wd[e])
        assert np.array_equal(got[e], ref), e
    # a sub-range of experts
    part = M.moe_pack_experts(cfg, wg, wu, wd, e_begin=1, e_count=2)
    assert np.array_equal(part, got[1:])


def test_host_packer_full_size_expert_matches_oracle():
    s = S.QWEN_4BIT
    cfg = M.config(s.hidden, s.inter, s.n_experts, s.top_k, bits=4)
    oc = O.cfg(s.hidden, s.inter, s.n_experts, s.top_k, bits=4)
    wg, wu, wd = S.expert_weights(s, 17)
    got = M.moe_pack_experts(cfg, wg, wu, wd)[0]
    assert got.nbytes == 7077888
    assert np.array_equal(got, O.quantize_expert(oc, wg, wu, wd))


def test_argument_checks_without_gpu():
    lib = M.lib()
    bad = M.config(4096, 1024, 512, 4, bits=3)
    assert lib.moe_packed_expert_bytes(C.byref(bad)) == 0
    good = M.config(256, 128, 16, 2)
    st = lib.moe_pack_experts(C.byref(bad), None, None, None, 0, 1, None, 0)
    assert st == 2 and "bits" in M.last_error()
    st = lib.moe_pack_experts(C.byref(good), None, None, None, 0, 1, None, 0)
    assert st == 1
    # more tokens than one launch takes run in chunks; the argument checks
    # still come first (a NULL expert table is refused before any device work)
    wts = M.MoeLayerWeights()
    st = lib.moe_layer_forward(C.byref(good), C.byref(wts), 16, 16, 9, 16, 16, None, None, 256, 1 << 20, None)
    assert st == 1 and "NULL" in M.last_error()
    # a traced call is one launch: at most one chunk of tokens
    st = lib.moe_layer_forward_traced(C.byref(good), C.byref(wts), 16, 16, 9, 16, 16, 256, 1 << 20, 16, 1 << 20,
                                      None)
    assert st == 2 and "at most" in M.last_error()
    # below 32 tokens the workspace is one chunk's (the fused kernel's
    # chunks); from 32 it covers the batched path, which grows with T
    assert lib.moe_layer_workspace_bytes(C.byref(good), 31) == lib.moe_layer_workspace_bytes(C.byref(good), 8)
    assert lib.moe_layer_workspace_bytes(C.byref(good), 2048) == lib.moe_layer_batched_workspace_bytes(
        C.byref(good), 2048)
    assert lib.moe_layer_batched_workspace_bytes(C.byref(good), 2048) > \
        2 * lib.moe_layer_batched_workspace_bytes(C.byref(good), 512)
    # the batched call checks its arguments before any device work too
    st = lib.moe_layer_forward_batched(C.byref(good), C.byref(wts), 16, 16, 40, 16, 16, None, None, 256, 1 << 20,
                                       None)
    assert st == 1 and "NULL" in M.last_error()
    # T == 0 is a no-op that touches nothing
    st = lib.moe_layer_forward(C.byref(good), None, None, None, 0, None, None, None, None, None, 0, None)
    assert st == 0
    # the streamed call refuses a bad shape or a NULL cache before any device work
    st = lib.moe_layer_forward_streamed(C.byref(bad), C.byref(wts), 16, 16, 1, 16, 16, None, None, None, 0, 256,
                                        1 << 20, None)
    assert st == 2
    st = lib.moe_layer_forward_streamed(C.byref(good), C.byref(wts), 16, 16, 1, 16, 16, None, None, None, 0, 256,
                                        1 << 20, None)
    assert st == 1 and "cache" in M.last_error()
    k_gt_e = M.config(256, 128, 4, 8)
    st = lib.moe_layer_forward(C.byref(k_gt_e), C.byref(wts), 16, 16, 1, 16, 16, None, None, 256, 1 << 20, None)
    assert st == 2
    assert lib.moe_layer_workspace_bytes(C.byref(good), 4) > 256
