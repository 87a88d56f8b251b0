"""Pins of the CPU oracle against facts fixed outside it.

Each test ties one oracle function to something it does not compute itself:
sizes the pages print, values worked out by hand, brute force on tiny inputs,
closed forms, or special cases that reduce to numpy/scipy routines.
"""
import os

import numpy as np
import pytest
from scipy.special import expit, softmax

import oracle as O
import synth as S
from conftest import GOLDEN


def _read_kv(path):
    out = {}
    for line in open(path):
        line = line.split("#")[0].strip()
        if line:
            k, v = [p.strip() for p in line.split("=")]
            out[k] = float(v)
    return out


# ---- sizes and layout -------------------------------------------------------

def test_expert_size_matches_pages():
    g = _read_kv(os.path.join(GOLDEN, "expert_sizes.txt"))
    c4 = O.cfg(int(g["hidden"]), int(g["inter"]), int(g["experts_per_layer"]),
               int(g["top_k"]), bits=4, group=int(g["group"]))
    c2 = O.cfg(int(g["hidden"]), int(g["inter"]), int(g["experts_per_layer"]),
               int(g["top_k"]), bits=2, group=int(g["group"]))
    b4, b2 = O.expert_bytes(c4), O.expert_bytes(c2)
    assert b4 == g["expert_mib_4bit"] * 2**20  # 6.75 MiB exactly
    n = g["layers"] * g["experts_per_layer"]
    gib = 2.0**30
    # whole-model totals, experts plus the resident non-expert weights
    assert abs((n * b4 / gib + g["non_expert_gb"]) / g["total_gb_4bit"] - 1) < 0.03
    assert abs((n * b2 / gib + g["non_expert_gb"]) / g["total_gb_2bit"] - 1) < 0.03


def test_section_offsets_by_hand():
    for line in open(os.path.join(GOLDEN, "section_offsets.txt")):
        line = line.split("#")[0].split()
        if not line:
            continue
        H, I, b, G = map(int, line[:4])
        offs = list(map(int, line[4:10]))
        total = int(line[10])
        c = O.cfg(H, I, 4, 2, bits=b, group=G)
        assert O.section_offsets(c) == offs, line
        assert O.expert_bytes(c) == total, line


def _hand_cases():
    cases, cur = [], None
    for line in open(os.path.join(GOLDEN, "hand_packed.txt")):
        f = line.split("#")[0].split()
        if not f:
            continue
        if f[0] == "cfg":
            cur = dict(cfg=tuple(map(int, f[1:4])), bytes=[], expect=[])
            cases.append(cur)
        elif f[0] == "byte":
            cur["bytes"].append((int(f[1]), int(f[2]), int(f[3], 16)))
        elif f[0] == "expect":
            cur["expect"].append((int(f[1]), int(f[2]), int(f[3]), float(f[4])))
    return cases


@pytest.mark.parametrize("case", _hand_cases(), ids=lambda c: "H%d_I%d_b%d" % c["cfg"])
def test_hand_packed_dequant(case):
    H, I, b = case["cfg"]
    c = O.cfg(H, I, 4, 2, bits=b)
    blob = np.zeros(O.expert_bytes(c), dtype=np.uint8)
    off = O.section_offsets(c)
    for sec, pos, val in case["bytes"]:
        blob[off[sec] + pos] = val
    for m, row, col, val in case["expect"]:
        assert O.dequant(c, blob, m, row, col) == val, (m, row, col)


# ---- bf16 rounding ------------------------------------------------------------

def test_bf16_round_closed_cases():
    f = lambda v: int(O.f32_to_bf16(np.float32(v)))
    assert f(1.0) == 0x3F80
    assert f(1.0 + 2.0**-8) == 0x3F80          # tie, even stays
    assert f(1.0 + 3 * 2.0**-8) == 0x3F82      # tie, odd rounds up
    assert f(1.0 + 2.0**-8 + 2.0**-20) == 0x3F81
    assert f(-2.0) == 0xC000
    assert f(np.inf) == 0x7F80
    assert np.isnan(O.bf16_to_f64(f(np.nan)))


def test_bf16_round_is_nearest():
    # brute force: the chosen bf16 is the closest of its two neighbours
    g = np.random.default_rng(1)
    v = (g.standard_normal(3000) * 10.0 ** g.integers(-6, 6, 3000)).astype(np.float32)
    for x in v:
        h = int(O.f32_to_bf16(x))
        cand = [h - 1, h, h + 1]
        d = [abs(O.bf16_to_f64(np.uint16(k & 0xFFFF)) - float(x)) for k in cand]
        assert d[1] <= min(d[0], d[2])


# ---- quantiser ----------------------------------------------------------------

@pytest.mark.parametrize("bits", [4, 2])
def test_quantizer_picks_nearest_code(bits):
    c = O.cfg(128, 64, 4, 2, bits=bits)
    g = np.random.default_rng(7)
    wg = (g.standard_normal((64, 128)) * 0.02).astype(np.float32)
    wg[3, :64] = 0.25                       # constant group: scale 0, codes 0
    wg[5, 64:] = np.linspace(-1, 1, 64)     # evenly spread group
    wu = (g.standard_normal((64, 128)) * 0.5).astype(np.float32)
    wd = (g.standard_normal((128, 64)) * 0.02).astype(np.float32)
    blob = O.quantize_expert(c, wg, wu, wd)
    qmax = 2**bits - 1
    ties = 0
    for m, w in ((0, wg), (1, wu), (2, wd)):
        rows, cols = w.shape
        for r in range(rows):
            for grp in range(cols // 64):
                seg = w[r, grp * 64:(grp + 1) * 64]
                # scale and bias from the dequantised values of two codes of the group
                i0 = int(np.argmin([O.code(c, blob, m, r, grp * 64 + i) for i in range(64)]))
                i1 = int(np.argmax([O.code(c, blob, m, r, grp * 64 + i) for i in range(64)]))
                q0, q1 = O.code(c, blob, m, r, grp * 64 + i0), O.code(c, blob, m, r, grp * 64 + i1)
                d0, d1 = O.dequant(c, blob, m, r, grp * 64 + i0), O.dequant(c, blob, m, r, grp * 64 + i1)
                s = (d1 - d0) / (q1 - q0) if q1 != q0 else 0.0
                beta = d0 - q0 * s
                # scale and bias follow min and max of the group
                assert s == O.bf16_to_f64(O.f32_to_bf16(np.float32((seg.max() - seg.min()) / np.float32(qmax))))
                assert beta == O.bf16_to_f64(O.f32_to_bf16(seg.min()))
                for i in range(64):
                    q = O.code(c, blob, m, r, grp * 64 + i)
                    assert 0 <= q <= qmax
                    if s == 0:
                        assert q == 0
                        continue
                    dist = np.abs(np.arange(qmax + 1) * s + beta - float(seg[i]))
                    best = int(np.argmin(dist))
                    if q != best:  # only a near tie may go either way
                        assert abs(dist[q] - dist[best]) < 1e-6 * s
                        ties += 1
    assert ties < 5


@pytest.mark.parametrize("bits", [4, 2])
def test_quantize_roundtrip_error(bits):
    c = O.cfg(256, 128, 4, 2, bits=bits)
    wg, wu, wd = S.expert_weights(S.TINY, 1)
    blob = O.quantize_expert(c, wg, wu, wd)
    for m, w in ((0, wg), (1, wu), (2, wd)):
        dq = O.dequant_matrix(c, blob, m)
        rows, cols = w.shape
        grp = w.reshape(rows, cols // 64, 64)
        rng_ = (grp.max(-1) - grp.min(-1)).astype(np.float64)
        step = rng_ / (2**bits - 1)
        bound = 0.5 * step + 2.0**-7 * (rng_ + np.abs(grp.min(-1))) + 1e-12
        err = np.abs(dq - w).reshape(rows, cols // 64, 64).max(-1)
        assert (err <= bound).all()


# ---- router ---------------------------------------------------------------------

def _brute_topk(l, K):
    key = [(-(-np.inf if np.isnan(v) else float(v)), e) for e, v in enumerate(l)]
    return [e for _, e in sorted(key)[:K]]


def test_topk_bruteforce_with_ties():
    g = np.random.default_rng(3)
    for E, K in ((16, 2), (16, 16), (37, 5), (512, 4), (8, 1)):
        c = O.cfg(64, 64, E, K)
        logits = g.integers(-3, 4, size=(20, E)).astype(np.float32)  # many exact ties
        logits[0, :] = 1.0                                             # all tied
        logits[1, 5 % E] = np.nan
        idx, w, w64 = O.topk(c, logits)
        for t in range(20):
            sel = _brute_topk(logits[t], K)
            assert list(idx[t]) == sel
            ls = np.where(np.isnan(logits[t, sel]), -np.inf, logits[t, sel]).astype(np.float64)
            np.testing.assert_allclose(w64[t], softmax(ls), rtol=1e-14, atol=0)
            assert abs(w64[t].sum() - 1.0) < 1e-14
            assert abs(float(np.sum(w[t], dtype=np.float64)) - 1.0) <= K * 2.0**-24


def test_topk_k_equals_e_is_softmax():
    g = np.random.default_rng(4)
    E = 16
    c = O.cfg(64, 64, E, E)
    logits = g.standard_normal((3, E)).astype(np.float32)
    idx, w, w64 = O.topk(c, logits)
    for t in range(3):
        p = softmax(logits[t].astype(np.float64))
        np.testing.assert_allclose(w64[t], p[idx[t]], rtol=1e-14)
        assert sorted(idx[t]) == list(range(E))


def test_router_logits_match_numpy():
    s = S.TINY
    c = O.cfg(s.hidden, s.inter, s.n_experts, s.top_k)
    d = S.dense_weights(s)
    x, _ = S.activations(s)
    bias = S.router_bias(S.LayerShape("z", 256, 128, 16, 2, routing="zipf"))
    logits, idx, w = O.router(c, x, d["wr"], bias)
    ref = S.bf16_bits_to_f32(x).astype(np.float64) @ S.bf16_bits_to_f32(d["wr"]).astype(np.float64).T
    ref = (ref + bias.astype(np.float64)).astype(np.float32)
    # same double sum up to summation order: at most one float ulp apart
    assert np.all(np.abs(logits - ref) <= np.spacing(np.abs(ref)))
    for t in range(x.shape[0]):
        assert list(idx[t]) == _brute_topk(logits[t], s.top_k)


# ---- expert FFN -------------------------------------------------------------------

def _np_ffn(c, blob, x):
    Wg, Wu, Wd = (O.dequant_matrix(c, blob, m) for m in range(3))
    g, u = Wg @ x, Wu @ x
    return Wd @ (g * expit(g) * u), g * expit(g) * u


@pytest.mark.parametrize("bits", [4, 2])
def test_expert_ffn_matches_numpy(bits):
    c = O.cfg(320, 192, 4, 2, bits=bits)  # H != I catches a transposed operand
    g = np.random.default_rng(5)
    wg = (g.standard_normal((192, 320)) * 0.05).astype(np.float32)
    wu = (g.standard_normal((192, 320)) * 0.05).astype(np.float32)
    wd = (g.standard_normal((320, 192)) * 0.05).astype(np.float32)
    blob = O.quantize_expert(c, wg, wu, wd)
    x = g.standard_normal(320)
    y_ref, a_ref = _np_ffn(c, blob, x)
    np.testing.assert_allclose(O.expert_act(c, blob, x), a_ref, rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(O.expert_ffn(c, blob, x), y_ref, rtol=1e-11, atol=1e-13)


def test_fma_form_identity():
    c = O.cfg(256, 128, 4, 2, bits=4)
    wg, wu, wd = S.expert_weights(S.TINY, 2)
    blob = O.quantize_expert(c, wg, wu, wd)
    x = np.random.default_rng(6).standard_normal(256)
    a = O.expert_ffn(c, blob, x)
    b = O.expert_ffn_fma_form(c, blob, x)
    np.testing.assert_allclose(b, a, rtol=1e-10, atol=1e-13)


def test_shared_ffn_matches_numpy():
    s = S.TINY
    c = O.cfg(s.hidden, s.inter, s.n_experts, s.top_k)
    d = S.dense_weights(s)
    x = np.random.default_rng(8).standard_normal(s.hidden)
    Wg, Wu, Wd = (O.bf16_to_f64(d[k]) for k in ("shared_gate", "shared_up", "shared_down"))
    g, u = Wg @ x, Wu @ x
    ref = Wd @ (g * expit(g) * u)
    np.testing.assert_allclose(O.shared_ffn(c, d["shared_gate"], d["shared_up"], d["shared_down"], x),
                               ref, rtol=1e-11, atol=1e-13)


# ---- whole layer --------------------------------------------------------------------

def _tiny_layer(E=16, K=2, H=256, I=128, bits=4, seed=0):
    s = S.LayerShape("t", H, I, E, K, bits=bits, tokens=3, routing="uniform", seed=seed)
    c = O.cfg(H, I, E, K, bits=bits)
    blobs = [O.quantize_expert(c, *S.expert_weights(s, e)) for e in range(E)]
    d = S.dense_weights(s)
    x, res = S.activations(s)
    return s, c, blobs, d, x, res


def test_one_hot_routing_is_single_expert():
    s, c, blobs, d, x, res = _tiny_layer(K=1)
    j = 11
    bias = np.zeros(s.n_experts, dtype=np.float32)
    bias[j] = 1e4
    idx, w, h, yn = O.layer_forward(c, blobs, d["wr"], bias, d["shared_gate"], d["shared_up"],
                                    d["shared_down"], d["gamma"], x, res)
    assert (idx == j).all() and (w == 1.0).all()
    Wsg, Wsu, Wsd = (O.bf16_to_f64(d[k]) for k in ("shared_gate", "shared_up", "shared_down"))
    for t in range(x.shape[0]):
        xt = O.bf16_to_f64(x[t])
        ye, _ = _np_ffn(c, blobs[j], xt)
        g, u = Wsg @ xt, Wsu @ xt
        ys = Wsd @ (g * expit(g) * u)
        ref = O.bf16_to_f64(res[t]) + ye + ys
        np.testing.assert_allclose(h[t], ref, rtol=1e-10, atol=1e-12)


def test_k_equals_e_uniform_is_dense_average():
    E = 6
    s, c, blobs, d, x, res = _tiny_layer(E=E, K=E, H=128, I=64)
    c.has_shared = 0
    wr0 = np.zeros_like(d["wr"][:E])
    idx, w, h, yn = O.layer_forward(c, blobs, wr0, None, None, None, None, d["gamma"], x, res)
    assert (w == np.float32(1.0 / E)).all()
    for t in range(x.shape[0]):
        xt = O.bf16_to_f64(x[t])
        dense = sum(_np_ffn(c, b, xt)[0] for b in blobs) / E
        np.testing.assert_allclose(h[t], O.bf16_to_f64(res[t]) + dense, rtol=1e-10, atol=1e-12)


def test_rmsnorm_closed_form():
    # all-zero expert and shared weights: h_out is the residual itself
    H, I, E, K = 128, 64, 4, 2
    c = O.cfg(H, I, E, K)
    zero = O.quantize_expert(c, np.zeros((I, H), np.float32), np.zeros((I, H), np.float32),
                             np.zeros((H, I), np.float32))
    zb = np.zeros((I, H), np.uint16)
    gamma = S.f32_to_bf16_bits(np.linspace(0.5, 2.0, H).astype(np.float32))
    cval = 0.75
    x = S.f32_to_bf16_bits(np.ones((2, H), np.float32))
    res = S.f32_to_bf16_bits(np.full((2, H), cval, np.float32))
    res[1, ::2] = S.f32_to_bf16_bits(np.float32(-cval))
    idx, w, h, yn = O.layer_forward(c, [zero] * E, np.zeros((E, H), np.uint16), None, zb, zb,
                                    np.zeros((H, I), np.uint16), gamma, x, res)
    np.testing.assert_array_equal(h[0], np.full(H, cval))
    inv = 1.0 / np.sqrt(cval * cval + np.float64(np.float32(1e-6)))
    g = O.bf16_to_f64(gamma)
    np.testing.assert_allclose(yn[0], cval * inv * g, rtol=1e-14)
    np.testing.assert_allclose(yn[1], np.where(np.arange(H) % 2 == 0, -cval, cval) * inv * g, rtol=1e-14)


# ---- the shared expert's gate and packed form ---------------------------------

def _shared_variants(gate_w=None, shared_blob=None, has_shared=1):
    s, c, blobs, d, x, res = _tiny_layer()
    c = O.cfg(c.hidden, c.inter, c.n_experts, c.top_k, bits=c.bits, has_shared=has_shared)
    idx_in = np.array([[1, 2], [3, 4], [5, 0]], np.int32)
    w_in = np.array([[0.6, 0.4], [0.25, 0.75], [0.5, 0.5]])
    _, _, h, _ = O.layer_forward(c, blobs, d["wr"], None, d["shared_gate"], d["shared_up"], d["shared_down"],
                                 d["gamma"], x, res, idx_in=idx_in, w_in=w_in, shared_blob=shared_blob,
                                 shared_gate_w=gate_w)
    return h, x, blobs


def test_shared_gate_closed_forms():
    # the gate scales the shared output by sigmoid(x . g): 1/2 at g = 0;
    # with g = +-sign(x) the logit is +-sum|x| (about 200 here), so the
    # gate is 1 (the ungated layer) or 0 (the layer without a shared expert)
    h_plain, x, _ = _shared_variants()
    h_none, _, _ = _shared_variants(has_shared=0)
    H = x.shape[1]
    h_half, _, _ = _shared_variants(gate_w=np.zeros(H, np.uint16))
    np.testing.assert_allclose(h_half, h_none + 0.5 * (h_plain - h_none), rtol=1e-12, atol=1e-13)
    for t in range(x.shape[0]):
        sgn = np.where(O.bf16_to_f64(x[t]) >= 0, 1.0, -1.0).astype(np.float32)
        up, _, _ = _shared_variants(gate_w=S.f32_to_bf16_bits(sgn))
        dn, _, _ = _shared_variants(gate_w=S.f32_to_bf16_bits(-sgn))
        assert np.sum(np.abs(O.bf16_to_f64(x[t]))) > 100
        np.testing.assert_allclose(up[t], h_plain[t], rtol=1e-12, atol=1e-13)
        np.testing.assert_allclose(dn[t], h_none[t], rtol=1e-12, atol=1e-13)


def test_packed_shared_is_an_expert():
    # the packed shared expert adds expert_ffn(blob, x) with weight 1
    _, x, blobs = _shared_variants()
    h_none, _, _ = _shared_variants(has_shared=0)
    h_pk, _, _ = _shared_variants(shared_blob=blobs[9])
    c = O.cfg(256, 128, 16, 2)
    for t in range(x.shape[0]):
        ys = O.expert_ffn(c, blobs[9], O.bf16_to_f64(x[t]))
        np.testing.assert_allclose(h_pk[t], h_none[t] + ys, rtol=1e-12, atol=1e-13)


# ---- RMSNorm before the layer ------------------------------------------------

def test_prenorm_hand_worked():
    # H = 64, eps = 0: h = (1, 2, 2, 4, 0, ...), sum of squares 25, mean 25/64,
    # root 5/8, so inv = 1.6; gamma = 1 on the first two columns, 0.5 after
    c = O.cfg(64, 64, 4, 2, eps=0.0)
    h = np.zeros((1, 64), np.float32)
    h[0, :4] = [1, 2, 2, 4]
    g = np.full(64, 0.5, np.float32)
    g[:2] = 1.0
    x = O.prenorm(c, S.f32_to_bf16_bits(h), S.f32_to_bf16_bits(g))
    want = np.zeros(64)
    want[:4] = [1.6, 3.2, 1.6, 3.2]
    np.testing.assert_allclose(x[0], want, rtol=1e-15, atol=0)


def test_prenorm_closed_forms():
    H = 128
    c = O.cfg(H, 64, 4, 2)
    eps = np.float64(np.float32(1e-6))
    gamma = S.f32_to_bf16_bits(np.linspace(0.5, 2.0, H).astype(np.float32))
    g = O.bf16_to_f64(gamma)
    # one-hot token: x_j = a / sqrt(a^2 / H + eps) * gamma_j, zero elsewhere
    a, j = 3.0, 17
    h1 = np.zeros(H, np.float32)
    h1[j] = a
    # constant token: x = v / sqrt(v^2 + eps) * gamma
    v = -0.375
    h2 = np.full(H, v, np.float32)
    x = O.prenorm(c, S.f32_to_bf16_bits(np.stack([h1, h2])), gamma)
    want1 = np.zeros(H)
    want1[j] = a / np.sqrt(a * a / H + eps) * g[j]
    np.testing.assert_allclose(x[0], want1, rtol=1e-14, atol=0)
    np.testing.assert_allclose(x[1], v / np.sqrt(v * v + eps) * g, rtol=1e-14)


def test_f64_to_bf16_single_rounding():
    # bf16 keeps 8 significant bits: steps of 2^-7 just above 1
    u = 2.0**-8
    cases = {1.0: 0x3F80, 1.0 + u: 0x3F80,          # tie, to even (down)
             1.0 + 3 * u: 0x3F82,                    # tie, to even (up)
             1.0 + u + 2.0**-40: 0x3F81,             # just above the tie: up
             -2.0: 0xC000, 0.0: 0x0000, 2.0**-130: 0x0008,  # subnormal: 8 units of 2^-133
             3.0e38: 0x7F62}
    for v, want in cases.items():
        assert int(O.f64_to_bf16(np.array([v]))[0]) == want, v
    # on values that are floats, the same as the float rounding
    rng = np.random.default_rng(5)
    f = (rng.standard_normal(2000) * np.exp(rng.uniform(-20, 20, 2000))).astype(np.float32)
    np.testing.assert_array_equal(O.f64_to_bf16(f.astype(np.float64)), S.f32_to_bf16_bits(f))


def test_prenorm_layer_composes():
    # the prenorm layer is the plain layer on x = bf16(prenorm(h)) with residual h
    s, c, blobs, d, x, res = _tiny_layer()
    gp = S.f32_to_bf16_bits(np.linspace(0.8, 1.2, c.hidden).astype(np.float32))
    xn, idx, w, h, yn = O.layer_forward_prenorm(c, blobs, d["wr"], None, d["shared_gate"], d["shared_up"],
                                                d["shared_down"], d["gamma"], gp, res)
    xr = O.prenorm(c, res, gp)
    assert np.all(np.abs(O.bf16_to_f64(xn) - xr) <= np.abs(xr) * 2.0**-8)
    idx2, w2, h2, yn2 = O.layer_forward(c, blobs, d["wr"], None, d["shared_gate"], d["shared_up"],
                                        d["shared_down"], d["gamma"], xn, res)
    np.testing.assert_array_equal(idx, idx2)
    np.testing.assert_array_equal(h, h2)


def test_given_routing_overrides():
    s, c, blobs, d, x, res = _tiny_layer()
    idx_in = np.array([[3, 4], [5, 6], [7, 8]], np.int32)
    w_in = np.array([[0.25, 0.75]] * 3)
    idx, w, h, _ = O.layer_forward(c, blobs, d["wr"], None, d["shared_gate"], d["shared_up"],
                                   d["shared_down"], d["gamma"], x, res, idx_in=idx_in, w_in=w_in)
    assert (idx == idx_in).all()
    t = 1
    xt = O.bf16_to_f64(x[t])
    ys = O.shared_ffn(c, d["shared_gate"], d["shared_up"], d["shared_down"], xt)
    ref = O.bf16_to_f64(res[t]) + 0.25 * O.expert_ffn(c, blobs[5], xt) + 0.75 * O.expert_ffn(c, blobs[6], xt) + ys
    np.testing.assert_allclose(h[t], ref, rtol=1e-12, atol=1e-13)


# ---- hand-worked values (router projection, routed FFN, shared FFN) -------------

def _lines(name):
    for line in open(os.path.join(GOLDEN, name)):
        f = line.split("#")[0].split()
        if f:
            yield f


def test_router_hand_worked():
    """Logits, top-K order and weights of tests/golden/router_hand.txt, every
    value worked out by hand (transposing Wr or dropping the bias changes the
    chosen experts there)."""
    rows = list(_lines("router_hand.txt"))
    H, E, K = map(int, next(f for f in rows if f[0] == "shape")[1:4])
    fill = float(next(f for f in rows if f[0] == "wr_fill")[1])
    T = 1 + max(int(f[1]) for f in rows if f[0] == "x")
    x = np.zeros((T, H), np.float32)
    wr = np.full((E, H), fill, np.float32)
    bias = np.zeros(E, np.float32)
    logit, top = {}, {}
    for f in rows:
        if f[0] == "x":
            x[int(f[1]), int(f[2])] = float(f[3])
        elif f[0] == "wr":
            wr[int(f[1]), int(f[2])] = float(f[3])
        elif f[0] == "bias":
            bias[int(f[1])] = float(f[2])
        elif f[0] == "logit":
            logit[int(f[1]), int(f[2])] = float(f[3])
        elif f[0] == "top":
            top[int(f[1]), int(f[2])] = (int(f[3]), float(f[4]))
    c = O.cfg(H, 64, E, K)
    logits, idx, w = O.router(c, S.f32_to_bf16_bits(x), S.f32_to_bf16_bits(wr), bias)
    for (t, e), v in logit.items():
        assert logits[t, e] == np.float32(v), (t, e, logits[t, e], v)
    _, _, w64 = O.topk(c, logits)
    for (t, k), (e, d) in top.items():
        assert idx[t, k] == e, (t, k)
        assert abs(w64[t, k] - 1.0 / (1.0 + np.exp(-d))) < 1e-15, (t, k)
        assert w[t, k] == np.float32(1.0 / (1.0 + np.exp(-d)))


def _ffn_expect(rows):
    L = np.log(3.0)
    act = {int(f[1]): float(f[2]) * L * L for f in rows if f[0] == "act"}
    y = {int(f[1]): float(f[2]) * L * L for f in rows if f[0] == "y"}
    xs = {int(f[1]): float(f[2]) * L for f in rows if f[0] == "x"}
    return xs, act, y


def _check_vec(got, expect, n):
    ref = np.zeros(n)
    for i, v in expect.items():
        ref[i] = v
    np.testing.assert_allclose(got, ref, rtol=1e-14, atol=1e-14)


def test_expert_ffn_hand_worked():
    """silu(Wg x) * (Wu x) and Wd of it on the hand-packed expert of
    tests/golden/expert_ffn_hand.txt (values are multiples of (ln 3)^2); the
    FMA form of the same product must give the same numbers."""
    rows = list(_lines("expert_ffn_hand.txt"))
    H, I, b = map(int, next(f for f in rows if f[0] == "cfg")[1:4])
    c = O.cfg(H, I, 4, 2, bits=b)
    blob = np.zeros(O.expert_bytes(c), dtype=np.uint8)
    off = O.section_offsets(c)
    for f in rows:
        if f[0] == "byte":
            blob[off[int(f[1])] + int(f[2])] = int(f[3], 16)
    xs, act, y = _ffn_expect(rows)
    x = np.zeros(H)
    for i, v in xs.items():
        x[i] = v
    _check_vec(O.expert_act(c, blob, x), act, I)
    _check_vec(O.expert_ffn(c, blob, x), y, H)
    _check_vec(O.expert_ffn_fma_form(c, blob, x), y, H)


def test_shared_ffn_hand_worked():
    """The bf16 shared expert on the hand-set weights of
    tests/golden/shared_ffn_hand.txt (values are multiples of (ln 3)^2)."""
    rows = list(_lines("shared_ffn_hand.txt"))
    H, I = map(int, next(f for f in rows if f[0] == "shape")[1:3])
    m = {"wg": np.zeros((I, H), np.float32), "wu": np.zeros((I, H), np.float32),
         "wd": np.zeros((H, I), np.float32)}
    for f in rows:
        if f[0] in m:
            m[f[0]][int(f[1]), int(f[2])] = float(f[3])
    xs, act, y = _ffn_expect(rows)
    x = np.zeros(H)
    for i, v in xs.items():
        x[i] = v
    c = O.cfg(H, I, 4, 2)
    got = O.shared_ffn(c, S.f32_to_bf16_bits(m["wg"]), S.f32_to_bf16_bits(m["wu"]),
                       S.f32_to_bf16_bits(m["wd"]), x)
    _check_vec(got, y, H)
