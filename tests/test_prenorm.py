"""GPU parity of the layer with the RMSNorm before it folded in
(moe_layer_forward_prenorm) against the oracle: x = bf16(prenorm(h)) then
the layer on x with h as the residual.

Bars: x_out equal to the oracle's correctly rounded x except where the exact
value lies within the fp32 evaluation error of a bf16 rounding boundary
(there one bf16 unit apart); routing exact on every token whose top K+1
oracle logits are further apart than the router's rounding bound plus the
effect of those boundary cases; outputs within the layer tolerance of the
oracle under the device's routing."""
from dataclasses import replace

import numpy as np
import pytest

import oracle as O
import synth as S
from layer_setup import (DeviceLayer, assert_outputs_close, bf16_to_f64, from_dev_bits, ocfg, oracle_forward,
                         router_error_bound, to_dev_bits)

pytestmark = pytest.mark.gpu

# relative error of the fp32 evaluation of h * inv * gamma: the sum of
# squares (short per-thread chains, a warp tree, a few partials: about 30
# units of 2^-24, halved by the square root), the divide, root, reciprocal
# and two products; 2^-16 leaves a wide margin
FP32_REL = 2.0 ** -16


@pytest.fixture(scope="module")
def M():
    import quantized_expert_ffn_03_b200 as M
    return M


def _near_boundary(xe):
    """Elements whose exact value lies within FP32_REL of a bf16 rounding
    boundary (a midpoint between neighbours): only there may a correctly
    computed fp32 value round to the other neighbour."""
    a = np.abs(xe)
    e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    ulp = 2.0 ** (e - 7)
    frac = a / ulp - np.floor(a / ulp)
    return (a > 0) & (np.abs(frac - 0.5) * ulp <= FP32_REL * a), ulp


def _run(M, dl, h_bits, gp_bits):
    import torch
    T = h_bits.shape[0]
    h = to_dev_bits(h_bits)
    gp = to_dev_bits(gp_bits)
    x_out, h_out, y = (torch.empty_like(h) for _ in range(3))
    idx = torch.empty((T, dl.s.top_k), dtype=torch.int32, device="cuda")
    w = torch.empty((T, dl.s.top_k), dtype=torch.float32, device="cuda")
    M.moe_layer_forward_prenorm(dl.cfg, dl.wts, gp, h, h_out, y, x_out, idx, w, workspace=dl.ws)
    torch.cuda.synchronize()
    st, detail = M.moe_device_error(dl.ws)
    assert st == 0, (st, detail)
    return from_dev_bits(x_out), from_dev_bits(h_out), from_dev_bits(y), idx.cpu().numpy(), w.cpu().numpy()


def check_prenorm_layer(M, dl, h_bits, gp_bits, blobs=None):
    s = dl.s
    oc = ocfg(s)
    x_dev, h_dev, y_dev, idx, w = _run(M, dl, h_bits, gp_bits)
    # x: the oracle's correctly rounded value, or one unit off at a boundary
    xe = O.prenorm(oc, h_bits, gp_bits)
    x_o = O.f64_to_bf16(xe)
    near, ulp = _near_boundary(xe)
    diff = np.abs(bf16_to_f64(x_dev) - bf16_to_f64(x_o))
    assert np.all((diff == 0) | (near & (diff <= ulp * 1.0000001))), "x_out off the correctly rounded value"
    # routing, against the oracle's logits on its own x
    lo, idx_o, _ = O.router(oc, x_o, dl.dense["wr"], dl.dense["bias"])
    wr = bf16_to_f64(dl.dense["wr"])
    bound = router_error_bound(s, x_o, dl.dense["wr"], lo) + (near * ulp) @ np.abs(wr).T
    K, E = s.top_k, s.n_experts
    for t in range(h_bits.shape[0]):
        order = np.lexsort((np.arange(E), -lo[t].astype(np.float64)))
        top = lo[t, order[:min(K + 1, E)]].astype(np.float64)
        gaps = top[:-1] - top[1:]
        if gaps.size == 0 or np.all(gaps > 2 * bound[t].max()):
            assert np.array_equal(idx[t], idx_o[t]), t
        else:  # a near tie: the device's choice lies within the bound of the oracle's K-th logit
            kth = lo[t, order[K - 1]]
            assert np.all(lo[t, idx[t]] >= kth - 2 * bound[t].max()), t
        lk = lo[t, idx[t]].astype(np.float64)
        wk = np.exp(lk - lk.max())
        wk /= wk.sum()
        np.testing.assert_allclose(w[t], wk, rtol=8 * bound[t].max() + 2e-6, atol=1e-7)
    blobs = dl.oracle_blobs() if blobs is None else blobs
    _, _, h_ref, y_ref = oracle_forward(s, blobs, dl.dense, x_o, h_bits, idx_in=idx, w_in=w.astype(np.float64))
    # h_out carries the residual stream (magnitudes up to ~100 here) and
    # y_norm its normalised form (up to ~30 on the 8x channels): their bf16
    # rounding is part of the bound
    assert_outputs_close(h_dev, h_ref, "h_out", round_rel=2.0 ** -8)
    assert_outputs_close(y_dev, y_ref, "y_norm", round_rel=2.0 ** -8)
    return x_dev


# T = 1 and 4 take the fused kernel (the norm inside it); 12 runs the norm
# kernel and successive fused launches; 40 the norm kernel and the batched path
@pytest.mark.parametrize("T", [1, 4, 12, 40])
def test_prenorm_layer_small(M, T):
    s = replace(S.TINY, tokens=T, routing="zipf")
    dl = DeviceLayer(s, max_tokens=T)
    h, gp = S.prenorm_inputs(s, step=T)
    check_prenorm_layer(M, dl, h, gp)


def test_prenorm_ragged_shape(M):
    s = S.LayerShape("ragged", 320, 192, 20, 3, tokens=3, routing="zipf")
    dl = DeviceLayer(s)
    h, gp = S.prenorm_inputs(s, step=1)
    check_prenorm_layer(M, dl, h, gp)


def test_prenorm_fused_and_kernel_paths_agree(M):
    """The norm inside the fused kernel and the stand-alone norm kernel give
    the same x (up to boundary cases) and so the same layer."""
    s = replace(S.TINY, tokens=12, routing="zipf")
    dl = DeviceLayer(s, max_tokens=12)
    h, gp = S.prenorm_inputs(s, step=5)
    C = M.moe_layer_tokens_per_launch(dl.cfg)
    whole = _run(M, dl, h, gp)[0]   # T = 12 > C: the norm kernel
    parts = np.concatenate([_run(M, dl, h[t:t + C], gp)[0] for t in range(0, 12, C)])
    xe = O.prenorm(ocfg(s), h, gp)
    near, ulp = _near_boundary(xe)
    diff = np.abs(bf16_to_f64(whole) - bf16_to_f64(parts))
    assert np.all((diff == 0) | near)


def test_prenorm_full_size(M):
    """H=4096, E=512, K=4, I=1024 (the decode shape), T = 1 and 4."""
    s = replace(S.QWEN_4BIT, tokens=4)
    dense = S.dense_weights(s)
    oc = ocfg(s)
    cases = [S.prenorm_inputs(s, step=3, tokens=1), S.prenorm_inputs(s, step=4, tokens=4)]
    need = set()
    for h, gp in cases:
        x_o = O.f64_to_bf16(O.prenorm(oc, h, gp))
        _, idx, _ = O.router(oc, x_o, dense["wr"], dense["bias"])
        need |= set(idx.ravel().tolist())
    dl = DeviceLayer(s, expert_ids=sorted(need), dense=dense, max_tokens=4)
    blobs = dl.oracle_blobs()
    for h, gp in cases:
        check_prenorm_layer(M, dl, h, gp, blobs=blobs)


def test_prenorm_argument_errors(M):
    import torch
    s = S.TINY
    dl = DeviceLayer(s)
    h = to_dev_bits(S.prenorm_inputs(s)[0])
    gp = to_dev_bits(S.prenorm_inputs(s)[1])
    y = torch.empty_like(h)
    with pytest.raises(M.MoeError):
        M.moe_layer_forward_prenorm(dl.cfg, dl.wts, gp, h, h, y, y, workspace=dl.ws)  # h_out aliases h_in
    with pytest.raises(M.MoeError):
        M.moe_layer_forward_prenorm(dl.cfg, dl.wts, None, h, torch.empty_like(h), y, torch.empty_like(h),
                                    workspace=dl.ws)
