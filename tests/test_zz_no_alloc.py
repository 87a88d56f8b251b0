"""moe_layer_forward_noalloc: the fused layer on the library's built-in
scratch.  Collected last on purpose (the scratch is shared state of the
loaded library); each test also passes alone.

The GPU test compares the allocation-free call with moe_layer_forward (same
inputs, a workspace of its own) on two calls in a row, within the layer
tests' tolerances; the CPU test checks that an oversized shape is refused
with a clear message before any device work."""
from dataclasses import replace

import numpy as np
import pytest

import oracle as O
import synth as S
from layer_setup import TOL_ABS, TOL_REL, DeviceLayer, bf16_to_f64, from_dev_bits, ocfg, to_dev_bits


@pytest.fixture(scope="module")
def M():
    import quantized_expert_ffn_03_b200 as M
    return M


def test_noalloc_rejects_shapes_beyond_the_scratch(M):
    cfg = M.config(4096, 16384, 512, 8, bits=4)
    assert M.moe_layer_workspace_bytes(cfg, 8) > M.NOALLOC_SCRATCH_BYTES
    with pytest.raises(M.MoeError) as ei:
        M.moe_layer_forward_noalloc(cfg, M.MoeLayerWeights(), np.zeros((8, 4096), np.uint16),
                                    np.zeros((8, 4096), np.uint16), np.zeros((8, 4096), np.uint16),
                                    np.zeros((8, 4096), np.uint16), stream=0)
    assert ei.value.status == M.MOE_ERR_WORKSPACE
    assert "scratch" in str(ei.value)


def _close(a_bits, b_bits, what):
    a, b = bf16_to_f64(a_bits), bf16_to_f64(b_bits)
    assert np.all(np.isfinite(a)), what
    err = np.abs(a - b).max()
    rel = np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-30)
    assert err <= TOL_ABS and rel <= TOL_REL, "%s: max-abs %.3g, rel-L2 %.3g" % (what, err, rel)


@pytest.mark.gpu
@pytest.mark.parametrize("shape", [replace(S.TINY, tokens=4), replace(S.QWEN_4BIT, tokens=1)],
                         ids=["tiny_T4", "h4096_T1"])
def test_noalloc_matches_workspace_path_twice(M, shape):
    import torch
    s = shape
    x, res = S.activations(s, step=3)
    # materialise the experts the oracle routes to (the others share a decoy blob)
    dense = S.dense_weights(s)
    _, idx_o, _ = O.router(ocfg(s), x, dense["wr"], dense["bias"])
    dl = DeviceLayer(s, expert_ids=idx_o.ravel().tolist(), dense=dense)
    T = x.shape[0]
    xd, rd = to_dev_bits(x), to_dev_bits(res)
    h_ref, y_ref = torch.empty_like(xd), torch.empty_like(xd)
    i_ref = torch.empty((T, s.top_k), dtype=torch.int32, device="cuda")
    w_ref = torch.empty((T, s.top_k), dtype=torch.float32, device="cuda")
    M.moe_layer_forward(dl.cfg, dl.wts, xd, rd, h_ref, y_ref, i_ref, w_ref, workspace=dl.ws)
    torch.cuda.synchronize()
    for call in range(2):
        h, y = torch.full_like(xd, 0x7fc0), torch.full_like(xd, 0x7fc0)
        idx = torch.full((T, s.top_k), -1, dtype=torch.int32, device="cuda")
        w = torch.zeros((T, s.top_k), dtype=torch.float32, device="cuda")
        M.moe_layer_forward_noalloc(dl.cfg, dl.wts, xd, rd, h, y, idx, w)
        torch.cuda.synchronize()
        assert np.array_equal(idx.cpu().numpy(), i_ref.cpu().numpy()), call
        np.testing.assert_allclose(w.cpu().numpy(), w_ref.cpu().numpy(), rtol=2e-6, atol=1e-7)
        _close(from_dev_bits(h), from_dev_bits(h_ref), "h_out call %d" % call)
        _close(from_dev_bits(y), from_dev_bits(y_ref), "y_norm call %d" % call)


@pytest.mark.gpu
def test_noalloc_failed_call_does_not_poison_the_next(M):
    """A call whose expert table holds misaligned pointers fails on the device
    (the kernel checks every chosen pointer before any access); the next good
    call must write its outputs and match moe_layer_forward, whether or not
    the failure was read in between."""
    import torch
    s = S.TINY
    dl = DeviceLayer(s)
    bad_ptr = dl.expert_ptr.clone()
    bad_ptr += 16
    bad = M.layer_weights(bad_ptr, dl.wr, dl.bias, dl.sg, dl.su, dl.sd, dl.gamma)
    x, res = S.activations(s, step=5)
    xd, rd = to_dev_bits(x), to_dev_bits(res)
    h_ref, y_ref = torch.empty_like(xd), torch.empty_like(xd)
    M.moe_layer_forward(dl.cfg, dl.wts, xd, rd, h_ref, y_ref, workspace=dl.ws)
    torch.cuda.synchronize()
    for read_error in (False, True):
        h, y = torch.empty_like(xd), torch.empty_like(xd)
        M.moe_layer_forward_noalloc(dl.cfg, bad, xd, rd, h, y)
        if read_error:
            assert M.moe_noalloc_device_error() == (M.MOE_ERR_DEVICE, 2)
        h, y = torch.full_like(xd, 0x7fc0), torch.full_like(xd, 0x7fc0)
        M.moe_layer_forward_noalloc(dl.cfg, dl.wts, xd, rd, h, y)
        assert M.moe_noalloc_device_error() == (M.MOE_OK, 0)
        _close(from_dev_bits(h), from_dev_bits(h_ref), "h_out after a failed call (read=%s)" % read_error)
        _close(from_dev_bits(y), from_dev_bits(y_ref), "y_norm after a failed call (read=%s)" % read_error)
