"""Batches longer than one launch of the fused kernel (T > 8): the layer runs
on successive chunks of tokens.  Every token's result depends on that token
alone, so a long batch must match the oracle token by token and equal, bit
for bit, the same tokens sent in separate calls of one chunk each."""
from dataclasses import replace

import numpy as np
import pytest

import oracle as O
import synth as S
from layer_setup import DeviceLayer, check_layer, ocfg


@pytest.mark.gpu
def test_long_batch_matches_oracle_tiny():
    s = replace(S.TINY, tokens=20)  # chunks of 8, 8 and 4 tokens
    dl = DeviceLayer(s)
    x, res = S.activations(s, step=2)
    check_layer(dl, x, res)


@pytest.mark.gpu
def test_long_batch_matches_oracle_and_its_chunks_h4096():
    import quantized_expert_ffn_03_b200 as M
    s = replace(S.QWEN_4BIT, tokens=16)
    dense = S.dense_weights(s)
    x, res = S.activations(s, step=4)
    _, idx_o, _ = O.router(ocfg(s), x, dense["wr"], dense["bias"])
    dl = DeviceLayer(s, expert_ids=idx_o.ravel().tolist(), dense=dense)
    C = M.moe_layer_tokens_per_launch(dl.cfg)
    assert 1 <= C <= 8
    # token by token against the oracle (routing and outputs)
    check_layer(dl, x, res)
    h, y, idx, w = dl.forward(x, res)  # ceil(16 / C) launches
    parts = [dl.forward(x[a:a + C], res[a:a + C]) for a in range(0, 16, C)]
    assert np.array_equal(h, np.concatenate([p[0] for p in parts]))
    assert np.array_equal(y, np.concatenate([p[1] for p in parts]))
    assert np.array_equal(idx, np.concatenate([p[2] for p in parts]))
    assert np.array_equal(w, np.concatenate([p[3] for p in parts]))
