"""GPU parity of the CUDA path against the oracle, through the C ABI.

Bars: routing indices exact (on every token whose K-th/(K+1)-th logit gap is
beyond the fp32 rounding bound, and always exact against the oracle's top-K
on the device's own logits); outputs within max-abs 2e-2 and relative L2
5e-3 of the oracle; packers bit-exact; repeated runs bit-identical."""
from dataclasses import replace

import numpy as np
import pytest

import oracle as O
import synth as S
from layer_setup import (DeviceLayer, bf16_to_f64, check_layer, from_dev_bits, mcfg, ocfg,
                         oracle_forward, to_dev_bits)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def M():
    import quantized_expert_ffn_03_b200 as M
    return M


# ---- packers ------------------------------------------------------------------------

@pytest.mark.parametrize("bits", [4, 2])
@pytest.mark.parametrize("H,I", [(256, 128), (320, 192), (4096, 1024)])
def test_device_packer_matches_host_and_oracle(M, bits, H, I):
    import torch
    s = S.LayerShape("p", H, I, 4, 2, bits=bits)
    cfg = mcfg(s)
    n = 2
    ws = [S.expert_weights(s, e) for e in range(n)]
    wg = np.stack([w[0] for w in ws])
    wu = np.stack([w[1] for w in ws])
    wd = np.stack([w[2] for w in ws])
    wg[0, 0, :64] = 0.5  # constant group
    host = M.moe_pack_experts(cfg, wg, wu, wd)
    out = torch.full((n * M.moe_packed_expert_bytes(cfg),), 0xAB, dtype=torch.uint8, device="cuda")
    M.moe_pack_experts_device(cfg, torch.from_numpy(wg).cuda(), torch.from_numpy(wu).cuda(),
                              torch.from_numpy(wd).cuda(), out)
    dev = out.cpu().numpy().reshape(n, -1)
    assert np.array_equal(dev, host)
    if H <= 320:
        assert np.array_equal(dev[1], O.quantize_expert(ocfg(s), wg[1], wu[1], wd[1]))


# ---- router ---------------------------------------------------------------------------

@pytest.mark.parametrize("E,K,H", [(16, 2, 256), (512, 4, 4096), (20, 3, 320), (16, 16, 256)])
def test_router_topk_matches_oracle(M, E, K, H):
    s = S.LayerShape("r", H, 128, E, K, tokens=8, routing="zipf")
    dl_dense = S.dense_weights(s)
    import torch
    x, _ = S.activations(s)
    cfg = mcfg(s)
    xd, wr = to_dev_bits(x), to_dev_bits(dl_dense["wr"])
    bias = torch.from_numpy(dl_dense["bias"]).cuda()
    idx = torch.empty((8, K), dtype=torch.int32, device="cuda")
    w = torch.empty((8, K), dtype=torch.float32, device="cuda")
    ws = torch.empty(M.moe_router_workspace_bytes(cfg, 8), dtype=torch.uint8, device="cuda")
    M.moe_router_topk(cfg, xd, wr, bias, idx, w, workspace=ws)
    lg = torch.empty((8, E), dtype=torch.float32, device="cuda")
    idx2 = torch.empty_like(idx)
    w2 = torch.empty_like(w)
    M.moe_router_topk(cfg, xd, wr, bias, idx2, w2, logits_out=lg)
    torch.cuda.synchronize()
    assert torch.equal(idx, idx2) and torch.equal(w, w2)
    lg = lg.cpu().numpy()
    oi, ow, ow64 = O.topk(ocfg(s), lg)
    assert np.array_equal(idx.cpu().numpy(), oi)
    np.testing.assert_allclose(w.cpu().numpy(), ow64, rtol=2e-6, atol=1e-7)
    lo, _, _ = O.router(ocfg(s), x, dl_dense["wr"], dl_dense["bias"])
    from layer_setup import router_error_bound
    assert np.all(np.abs(lg.astype(np.float64) - lo) <= router_error_bound(s, x, dl_dense["wr"], lo))


def test_topk_from_logits_ties_and_nan(M):
    import torch
    E, K, T = 40, 5, 6
    g = np.random.default_rng(0)
    logits = g.integers(-2, 3, size=(T, E)).astype(np.float32)
    logits[0] = 0.0
    logits[1, 7] = np.nan
    logits[2, :] = -np.inf
    logits[2, 9] = 1.0
    cfg = M.config(64, 64, E, K)
    idx = torch.empty((T, K), dtype=torch.int32, device="cuda")
    w = torch.empty((T, K), dtype=torch.float32, device="cuda")
    M.moe_topk_from_logits(cfg, torch.from_numpy(logits).cuda(), idx, w)
    torch.cuda.synchronize()
    oi, _, ow64 = O.topk(O.cfg(64, 64, E, K), logits)
    assert np.array_equal(idx.cpu().numpy(), oi)
    wg = w.cpu().numpy()
    fin = np.isfinite(ow64)
    np.testing.assert_allclose(wg[fin], ow64[fin], rtol=2e-6, atol=1e-7)


# ---- whole layer ------------------------------------------------------------------------

TINY_CASES = {
    "tiny_4bit_T4": S.TINY,
    "tiny_2bit_T4": replace(S.TINY, bits=2),
    "tiny_zipf_T1": replace(S.TINY, tokens=1, routing="zipf"),
    "tiny_T8": replace(S.TINY, tokens=8),
    "no_shared": replace(S.TINY, has_shared=0),
    "k1": replace(S.TINY, top_k=1),
    "k_eq_e": replace(S.TINY, top_k=16, tokens=4),
    "ragged_320x192_e20": S.LayerShape("ragged", 320, 192, 20, 3, tokens=3, routing="zipf"),
    "h2048_i1536": S.LayerShape("h2k", 2048, 1536, 12, 2, tokens=2, routing="zipf"),
    "h5120_i64_2bit": S.LayerShape("wide", 5120, 64, 8, 2, bits=2, tokens=2),
}


@pytest.mark.parametrize("name", sorted(TINY_CASES))
def test_layer_matches_oracle_small(M, name):
    s = TINY_CASES[name]
    dl = DeviceLayer(s)
    x, res = S.activations(s)
    check_layer(dl, x, res)


def test_layer_is_deterministic_and_host_path_matches(M):
    import torch
    s = S.TINY
    dl = DeviceLayer(s)
    x, res = S.activations(s, step=3)
    a = dl.forward(x, res)
    b = dl.forward(x, res)
    for u, v in zip(a, b):
        assert np.array_equal(u, v)
    hw = torch.zeros(M.moe_layer_host_workspace_bytes(dl.cfg, s.tokens), dtype=torch.uint8, device="cuda")
    M.moe_workspace_init(hw)
    xh = torch.from_numpy(x.view(np.int16)).pin_memory()
    rh = torch.from_numpy(res.view(np.int16)).pin_memory()
    hh = torch.empty_like(xh).pin_memory()
    yh = torch.empty_like(xh).pin_memory()
    M.moe_layer_forward_host(dl.cfg, dl.wts, xh, rh, hh, yh, hw)
    assert np.array_equal(hh.numpy().view(np.uint16), a[0])
    assert np.array_equal(yh.numpy().view(np.uint16), a[1])
    # the asynchronous calls: separate buffers, and x|residual, h_out|y_norm
    # packed in one host buffer each (one copy each way)
    hh2, yh2 = torch.zeros_like(hh).pin_memory(), torch.zeros_like(yh).pin_memory()
    M.moe_layer_forward_host_async(dl.cfg, dl.wts, xh, rh, hh2, yh2, hw)
    torch.cuda.synchronize()
    assert np.array_equal(hh2.numpy().view(np.uint16), a[0])
    assert np.array_equal(yh2.numpy().view(np.uint16), a[1])
    inp = torch.from_numpy(np.stack([x, res]).view(np.int16)).pin_memory()
    out = torch.zeros_like(inp).pin_memory()
    M.moe_layer_forward_host_packed(dl.cfg, dl.wts, inp, out, hw)
    torch.cuda.synchronize()
    assert np.array_equal(out[0].numpy().view(np.uint16), a[0])
    assert np.array_equal(out[1].numpy().view(np.uint16), a[1])


def test_layer_uniform_zero_router_picks_lowest_indices(M):
    s = replace(S.TINY, tokens=2)
    dense = S.dense_weights(s)
    dense = dict(dense, wr=np.zeros_like(dense["wr"]), bias=np.zeros_like(dense["bias"]))
    dl = DeviceLayer(s, dense=dense)
    x, res = S.activations(s)
    h, y, idx, w = dl.forward(x, res)
    assert (idx == np.arange(s.top_k)).all()
    assert (w == np.float32(1.0 / s.top_k)).all()
    check_layer(dl, x, res)


def test_empty_batch_is_noop(M):
    import torch
    s = S.TINY
    dl = DeviceLayer(s)
    z = torch.empty((0, s.hidden), dtype=torch.int16, device="cuda")
    M.moe_layer_forward(dl.cfg, dl.wts, z, z, z, z, workspace=dl.ws)
    torch.cuda.synchronize()


@pytest.mark.parametrize("bits", [4, 2])
def test_layer_full_size_matches_oracle(M, bits):
    """The benchmark's launch configuration: H=4096, E=512, K=4, I=1024, T=1,
    Zipf-biased router.  Only the experts the oracle routes to are
    materialised; the oracle computes every output."""
    s = S.QWEN_4BIT if bits == 4 else S.QWEN_2BIT
    dense = S.dense_weights(s)
    steps = [S.activations(s, step=k) for k in range(3)]
    need = set()
    oc = ocfg(s)
    for x, _ in steps:
        _, idx, _ = O.router(oc, x, dense["wr"], dense["bias"])
        need |= set(idx.ravel().tolist())
    dl = DeviceLayer(s, expert_ids=sorted(need), dense=dense)
    blobs = dl.oracle_blobs()
    for e in dl.ids:
        assert np.array_equal(blobs[e], dl.host_blobs[e])
    for x, res in steps:
        check_layer(dl, x, res, blobs=blobs)


def test_layer_full_size_four_tokens(M):
    s = replace(S.QWEN_4BIT, tokens=4)
    dense = S.dense_weights(s)
    x, res = S.activations(s, step=11)
    _, idx, _ = O.router(ocfg(s), x, dense["wr"], dense["bias"])
    dl = DeviceLayer(s, expert_ids=idx.ravel().tolist(), dense=dense)
    check_layer(dl, x, res)


# ---- failure paths (no fault, no hang) ------------------------------------------------------

def test_bounded_wait_times_out_and_context_survives(M):
    import torch
    ws = torch.zeros(4096, dtype=torch.uint8, device="cuda")
    M.moe_selftest_bounded_wait(ws, timeout_ns=2_000_000)
    st, detail = M.moe_device_error(ws)
    assert st == 6 and detail == 1
    st, detail = M.moe_device_error(ws)
    assert st == 0
    dl = DeviceLayer(S.TINY)
    x, res = S.activations(S.TINY)
    check_layer(dl, x, res)


def test_misaligned_expert_pointer_is_reported(M):
    import torch
    s = S.TINY
    dl = DeviceLayer(s)
    bad = dl.expert_ptr.clone()
    bad += 16
    wts = M.layer_weights(bad, dl.wr, dl.bias, dl.sg, dl.su, dl.sd, dl.gamma)
    x, res = S.activations(s)
    xd, rd = to_dev_bits(x), to_dev_bits(res)
    h, y = torch.empty_like(xd), torch.empty_like(xd)
    M.moe_layer_forward(dl.cfg, wts, xd, rd, h, y, workspace=dl.ws)
    st, detail = M.moe_device_error(dl.ws)
    assert st == 8 and detail == 2
    check_layer(dl, x, res)
