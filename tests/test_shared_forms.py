"""GPU parity of the shared expert's optional forms against the oracle: the
output gate (sigmoid(x . g) scaling the shared FFN) and the packed shared
expert (the routed experts' format, run as one more pair per token), through
the fused decode kernel (one launch and successive launches) and the batched
path."""
from dataclasses import replace

import numpy as np
import pytest

import oracle as O
import synth as S
from layer_setup import DeviceLayer, check_layer, ocfg

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def M():
    import quantized_expert_ffn_03_b200 as M
    return M


def _gate(s, scale):
    g = S.rng(s.seed, 0, "shared_out_gate", s.hidden).standard_normal(s.hidden).astype(np.float32)
    return S.f32_to_bf16_bits(g * np.float32(scale))


# T = 1 and 4: one fused launch; 12: successive fused launches; 40: the batched path
@pytest.mark.parametrize("T", [1, 4, 12, 40])
def test_shared_gate_small(M, T):
    s = replace(S.TINY, tokens=T, routing="zipf")
    dl = DeviceLayer(s, max_tokens=T, shared_out_gate=_gate(s, 0.1))
    x, res = S.activations(s, step=T)
    check_layer(dl, x, res)


def test_shared_gate_changes_the_output(M):
    """The gate is applied: the device output with the gate matches the
    gated oracle and differs from the ungated one by the expected amount."""
    s = replace(S.TINY, tokens=2, routing="zipf")
    g = _gate(s, 0.1)
    dl = DeviceLayer(s, shared_out_gate=g)
    x, res = S.activations(s, step=3)
    h, _, idx, w = dl.forward(x, res)
    blobs = dl.oracle_blobs()
    oc = ocfg(s)
    d = dl.dense
    _, _, h_gate, _ = O.layer_forward(oc, blobs, d["wr"], d["bias"], d["shared_gate"], d["shared_up"],
                                      d["shared_down"], d["gamma"], x, res, idx_in=idx, w_in=w.astype(np.float64),
                                      shared_gate_w=g)
    _, _, h_plain, _ = O.layer_forward(oc, blobs, d["wr"], d["bias"], d["shared_gate"], d["shared_up"],
                                       d["shared_down"], d["gamma"], x, res, idx_in=idx, w_in=w.astype(np.float64))
    got = S.bf16_bits_to_f32(h).astype(np.float64)
    assert np.abs(got - h_gate).max() < 2e-2
    # the device output is far closer to the gated oracle than to the ungated one
    assert np.linalg.norm(got - h_gate) < 0.25 * np.linalg.norm(got - h_plain)


def test_shared_gate_full_size(M):
    s = replace(S.QWEN_4BIT, tokens=1)
    dense = S.dense_weights(s)
    x, res = S.activations(s, step=21)
    _, idx, _ = O.router(ocfg(s), x, dense["wr"], dense["bias"])
    dl = DeviceLayer(s, expert_ids=idx.ravel().tolist(), dense=dense, shared_out_gate=_gate(s, 0.02))
    check_layer(dl, x, res)


@pytest.mark.parametrize("gate", [False, True])
@pytest.mark.parametrize("T", [1, 4, 12, 40])
def test_packed_shared_small(M, T, gate):
    s = replace(S.TINY, tokens=T, routing="zipf")
    dl = DeviceLayer(s, max_tokens=T, shared_packed=True, shared_out_gate=_gate(s, 0.1) if gate else None)
    x, res = S.activations(s, step=T + 7)
    check_layer(dl, x, res)


@pytest.mark.parametrize("bits", [4, 2])
def test_packed_shared_full_size(M, bits):
    s = replace(S.QWEN_4BIT if bits == 4 else S.QWEN_2BIT, tokens=2)
    dense = S.dense_weights(s)
    x, res = S.activations(s, step=23)
    _, idx, _ = O.router(ocfg(s), x, dense["wr"], dense["bias"])
    dl = DeviceLayer(s, expert_ids=idx.ravel().tolist(), dense=dense, shared_packed=True,
                     shared_out_gate=_gate(s, 0.02))
    check_layer(dl, x, res)
