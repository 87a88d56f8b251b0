"""The batched layer (moe_layer_forward_batched): router GEMM, top-K, pairs
grouped by expert, grouped dequant GEMMs on the tensor cores, shared-expert
GEMMs, combine + residual + RMSNorm.

Routing follows the same rule as the decode path (checked as in check_layer:
exact against the oracle wherever the logits leave no near tie); outputs are
compared with the oracle under the device's own routing, element by element,
within the layer tolerances.  Shapes cover chunks of one expert's tokens
above and below the 128-column tile, experts with a single token, ragged
token counts, both bit widths, no shared expert, and the h4096 layer under
uniform and Zipf routing (where one expert draws far more than 128 tokens)."""
from dataclasses import replace

import numpy as np
import pytest

import oracle as O
import synth as S
from layer_setup import (DeviceLayer, assert_outputs_close, clear_gap_tokens, from_dev_bits, observed_clear_tokens,
                         ocfg, oracle_forward, router_error_bound, to_dev_bits)


@pytest.fixture(scope="module")
def M():
    import quantized_expert_ffn_03_b200 as M
    return M


def run_batched(M, dl, x, res, fn="moe_layer_forward_batched"):
    import torch
    T = x.shape[0]
    s = dl.s
    ws = torch.zeros(max(M.moe_layer_batched_workspace_bytes(dl.cfg, T), M.moe_layer_workspace_bytes(dl.cfg, T)),
                     dtype=torch.uint8, device="cuda")
    M.moe_workspace_init(ws)
    xd, rd = to_dev_bits(x), to_dev_bits(res)
    h, y = torch.full_like(xd, 0x7fc0), torch.full_like(xd, 0x7fc0)
    idx = torch.full((T, s.top_k), -1, dtype=torch.int32, device="cuda")
    w = torch.zeros((T, s.top_k), dtype=torch.float32, device="cuda")
    getattr(M, fn)(dl.cfg, dl.wts, xd, rd, h, y, idx, w, workspace=ws)
    torch.cuda.synchronize()
    st, detail = M.moe_device_error(ws)
    assert st == 0, (st, detail)
    return from_dev_bits(h), from_dev_bits(y), idx.cpu().numpy(), w.cpu().numpy()


def check_batched(M, dl, x, res, sample=None, blobs=None):
    """Routing against the oracle and outputs against the oracle under the
    device's routing; sample: token indices the oracle computes (all if None)."""
    s = dl.s
    h, y, idx, w = run_batched(M, dl, x, res)
    lg, idx_r, _ = dl.router(x)
    lo, idx_o, _ = O.router(ocfg(s), x, dl.dense["wr"], dl.dense["bias"])
    bound = router_error_bound(s, x, dl.dense["wr"], lo)
    assert np.all(np.abs(lg.astype(np.float64) - lo) <= bound + 1e-30)
    clear = clear_gap_tokens(s, lo, bound)
    assert np.array_equal(idx[clear], idx_o[clear])
    seen, dev = observed_clear_tokens(s, lo, lg)
    assert np.array_equal(idx[seen], idx_o[seen])
    assert int((~seen).sum()) == 0
    for t in range(idx.shape[0]):
        lk = lo[t, idx[t]].astype(np.float64)
        wk = np.exp(lk - lk.max())
        # the router GEMM rounds its logits in its own order (tensor-core
        # accumulation), a few times the stand-alone router's observed error
        np.testing.assert_allclose(w[t], wk / wk.sum(), rtol=16 * dev[t] + 2e-5, atol=1e-7)
    tok = np.arange(x.shape[0]) if sample is None else np.asarray(sample)
    blobs = dl.oracle_blobs() if blobs is None else blobs
    _, _, h_ref, y_ref = oracle_forward(s, blobs, dl.dense, x[tok], res[tok], idx_in=idx[tok],
                                        w_in=w[tok].astype(np.float64))
    assert_outputs_close(h[tok], h_ref, "h_out")
    assert_outputs_close(y[tok], y_ref, "y_norm")
    return h, y, idx, w


SMALL = {
    "tiny_T64": replace(S.TINY, tokens=64),
    "tiny_2bit_T37": replace(S.TINY, bits=2, tokens=37),
    "tiny_no_shared_T50": replace(S.TINY, has_shared=0, tokens=50),
    "tiny_zipf_T300": replace(S.TINY, tokens=300, routing="zipf"),  # a hot expert takes > 128 tokens
    "ragged_320x192_e20_T33": S.LayerShape("ragged", 320, 192, 20, 3, tokens=33, routing="zipf"),
}


@pytest.mark.gpu
@pytest.mark.parametrize("name", sorted(SMALL))
def test_batched_matches_oracle_small(M, name):
    s = SMALL[name]
    dl = DeviceLayer(s)
    x, res = S.activations(s, step=1)
    h, y, idx, w = check_batched(M, dl, x, res)
    # tokens per expert span single tokens and, for the Zipf case, more than one tile
    counts = np.bincount(idx.ravel(), minlength=s.n_experts)
    if name == "tiny_zipf_T300":
        assert counts.max() > 128 and (counts == 1).any() or counts.max() > 128
    # deterministic run to run
    h2, y2, idx2, w2 = run_batched(M, dl, x, res)
    assert np.array_equal(h, h2) and np.array_equal(y, y2) and np.array_equal(idx, idx2)


@pytest.mark.gpu
def test_batched_equals_chunked_within_tolerance_and_default_dispatch(M):
    """moe_layer_forward takes the batched path from 32 tokens: its result is
    the batched call's, and within tolerance of the fused kernel's chunks."""
    s = replace(S.TINY, tokens=48)
    dl = DeviceLayer(s)
    x, res = S.activations(s, step=2)
    hb, yb, ib, wb = run_batched(M, dl, x, res)
    hd, yd, idd, wd = run_batched(M, dl, x, res, fn="moe_layer_forward")
    assert np.array_equal(hb, hd) and np.array_equal(yb, yd) and np.array_equal(ib, idd)
    hc, yc, ic, wc = run_batched(M, dl, x, res, fn="moe_layer_forward_chunked")
    same = (ib == ic).all(axis=1)
    assert same.mean() > 0.9
    assert_outputs_close(yb[same], S.bf16_bits_to_f32(yc[same]).astype(np.float64), "y_norm batched vs chunked")


def _h4096_layer(s, x):
    dense = S.dense_weights(s)
    _, idx_o, _ = O.router(ocfg(s), x, dense["wr"], dense["bias"])
    return DeviceLayer(s, expert_ids=idx_o.ravel().tolist(), dense=dense)


@pytest.mark.gpu
@pytest.mark.parametrize("routing,T", [("uniform", 64), ("zipf", 256)])
def test_batched_h4096_matches_oracle_on_sampled_tokens(M, routing, T):
    """The benchmark's layer shape.  Every expert the oracle routes to is
    materialised; the oracle computes a sample of tokens that includes the
    hottest expert's first and last tokens (Zipf: more than one 128-token
    chunk of that expert)."""
    s = replace(S.QWEN_4BIT, tokens=T, routing=routing)
    x, res = S.activations(s, step=3)
    dl = _h4096_layer(s, x)
    h, y, idx, w = run_batched(M, dl, x, res)
    counts = np.bincount(idx.ravel(), minlength=s.n_experts)
    hot = int(counts.argmax())
    users = np.nonzero((idx == hot).any(axis=1))[0]
    sample = sorted(set([0, T - 1, int(users[0]), int(users[-1])] + list(range(1, T, T // 6))))
    if routing == "zipf":
        assert counts.max() > 128
    check_batched(M, dl, x, res, sample=sample)
