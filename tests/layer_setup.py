"""Helpers shared by the GPU tests: build one MoE layer on the device from the
seeded synthetic inputs, run it through the C ABI, and compare with the
oracle.  The oracle always gets its own quantiser's blobs and the raw inputs;
nothing it sees comes from the CUDA path."""
import numpy as np

import oracle as O
import synth as S

TOL_ABS = 2e-2   # max-abs error against the oracle
TOL_REL = 5e-3   # relative L2 error against the oracle


def mcfg(s):
    import quantized_expert_ffn_03_b200 as M
    return M.config(s.hidden, s.inter, s.n_experts, s.top_k, bits=s.bits, eps=s.eps, has_shared=s.has_shared)


def ocfg(s):
    return O.cfg(s.hidden, s.inter, s.n_experts, s.top_k, bits=s.bits, eps=s.eps, has_shared=s.has_shared)


def to_dev_bits(a):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).cuda()


def from_dev_bits(t):
    return t.cpu().numpy().view(np.uint16)


def bf16_to_f64(bits):
    return S.bf16_bits_to_f32(bits).astype(np.float64)


def router_error_bound(s, x_bits, wr_bits, logits):
    """Rigorous bound on |fp32 logit - exact logit|: 2*gamma_H*sum|x*w| plus
    the rounding of the bias add and of the result."""
    H = s.hidden
    u = 2.0 ** -24
    gam = H * u / (1 - H * u)
    x = bf16_to_f64(x_bits)
    w = bf16_to_f64(wr_bits)
    mag = np.abs(x) @ np.abs(w).T
    return 2 * gam * mag + 4 * u * (np.abs(logits) + 1.0)


def clear_gap_tokens(s, logits_orc, bound):
    """Tokens whose K-th and (K+1)-th logits are further apart than twice the
    bound: on those the chosen set is fixed whatever the rounding order."""
    K, E = s.top_k, s.n_experts
    if K >= E:
        return np.ones(logits_orc.shape[0], bool)
    out = []
    for t in range(logits_orc.shape[0]):
        order = np.lexsort((np.arange(E), -logits_orc[t].astype(np.float64)))
        gap = float(logits_orc[t, order[K - 1]]) - float(logits_orc[t, order[K]])
        out.append(gap > 2 * bound[t].max())
    return np.array(out)


class DeviceLayer:
    """One layer on the device.  expert_ids: the experts to materialise (all
    by default); the others point at a decoy blob (expert ids[0]'s copy)."""

    def __init__(self, s, expert_ids=None, replica=0, max_tokens=8, dense=None, shared_out_gate=None,
                 shared_packed=False):
        import torch
        import quantized_expert_ffn_03_b200 as M
        self.s, self.M = s, M
        self.cfg = mcfg(s)
        ids = list(range(s.n_experts)) if expert_ids is None else sorted(set(int(e) for e in expert_ids))
        self.ids = ids
        nb = M.moe_packed_expert_bytes(self.cfg)
        self.host_blobs = {}
        pool = np.zeros((len(ids) + 1, nb), dtype=np.uint8)
        for j, e in enumerate(ids):
            wg, wu, wd = S.expert_weights(s, e, replica)
            pool[j] = M.moe_pack_experts(self.cfg, wg, wu, wd)[0]
            self.host_blobs[e] = pool[j]
        pool[len(ids)] = pool[0]
        self.pool = torch.from_numpy(pool).cuda()
        base = self.pool.data_ptr()
        slot = {e: j for j, e in enumerate(ids)}
        ptrs = [base + nb * slot.get(e, len(ids)) for e in range(s.n_experts)]
        self.expert_ptr = torch.tensor(ptrs, dtype=torch.int64, device="cuda")
        self.dense = S.dense_weights(s, replica) if dense is None else dense
        d = self.dense
        self.wr = to_dev_bits(d["wr"])
        self.bias = torch.from_numpy(d["bias"]).cuda()
        self.sg = to_dev_bits(d["shared_gate"])
        self.su = to_dev_bits(d["shared_up"])
        self.sd = to_dev_bits(d["shared_down"])
        self.gamma = to_dev_bits(d["gamma"])
        # the shared expert's output gate (bf16 bits [H]) or None
        self.sgate_bits = shared_out_gate
        self.sgate = None if shared_out_gate is None else to_dev_bits(shared_out_gate)
        # the shared expert packed like the routed ones (seeded as expert id E)
        self.shared_blob = None
        self.spacked = None
        if shared_packed:
            wg, wu, wd = S.expert_weights(s, s.n_experts, replica)
            self.shared_blob = M.moe_pack_experts(self.cfg, wg, wu, wd)[0]
            self.spacked = torch.from_numpy(self.shared_blob.copy()).cuda()
        bf = s.has_shared and not shared_packed
        self.wts = M.layer_weights(self.expert_ptr, self.wr, self.bias, self.sg if bf else None,
                                   self.su if bf else None, self.sd if bf else None,
                                   self.gamma, shared_out_gate=self.sgate, shared_packed=self.spacked)
        self.ws = torch.zeros(M.moe_layer_workspace_bytes(self.cfg, max_tokens), dtype=torch.uint8,
                              device="cuda")
        M.moe_workspace_init(self.ws)

    def forward(self, x_bits, res_bits):
        import torch
        T = x_bits.shape[0]
        x, r = to_dev_bits(x_bits), to_dev_bits(res_bits)
        h = torch.empty_like(x)
        y = torch.empty_like(x)
        idx = torch.empty((T, self.s.top_k), dtype=torch.int32, device="cuda")
        w = torch.empty((T, self.s.top_k), dtype=torch.float32, device="cuda")
        self.M.moe_layer_forward(self.cfg, self.wts, x, r, h, y, idx, w, workspace=self.ws)
        torch.cuda.synchronize()
        st, detail = self.M.moe_device_error(self.ws)
        assert st == 0, (st, detail)
        return from_dev_bits(h), from_dev_bits(y), idx.cpu().numpy(), w.cpu().numpy()

    def router(self, x_bits):
        import torch
        T = x_bits.shape[0]
        x = to_dev_bits(x_bits)
        idx = torch.empty((T, self.s.top_k), dtype=torch.int32, device="cuda")
        w = torch.empty((T, self.s.top_k), dtype=torch.float32, device="cuda")
        logits = torch.empty((T, self.s.n_experts), dtype=torch.float32, device="cuda")
        self.M.moe_router_topk(self.cfg, x, self.wr, self.bias, idx, w, logits_out=logits)
        torch.cuda.synchronize()
        return logits.cpu().numpy(), idx.cpu().numpy(), w.cpu().numpy()

    def oracle_blobs(self):
        """The oracle's own quantisation of the materialised experts."""
        oc = ocfg(self.s)
        blobs = {}
        for e in self.ids:
            blobs[e] = O.quantize_expert(oc, *S.expert_weights(self.s, e))
        first = blobs[self.ids[0]]
        return [blobs.get(e, first) for e in range(self.s.n_experts)]


def oracle_forward(s, blobs, dense, x_bits, res_bits, idx_in=None, w_in=None, shared_gate_w=None,
                   shared_blob=None):
    d = dense
    sh = s.has_shared
    return O.layer_forward(ocfg(s), blobs, d["wr"], d["bias"], d["shared_gate"] if sh else None,
                           d["shared_up"] if sh else None, d["shared_down"] if sh else None,
                           d["gamma"], x_bits, res_bits, idx_in=idx_in, w_in=w_in,
                           shared_gate_w=shared_gate_w if sh else None,
                           shared_blob=shared_blob if sh else None)


def assert_outputs_close(got_bits, ref, what, round_rel=0.0):
    """Element-wise |got - ref| <= TOL_ABS + round_rel * |ref| and relative
    L2 <= TOL_REL.  round_rel covers the bf16 rounding of outputs whose
    magnitude is far above 1 (2^-8: twice the half unit of a bf16)."""
    g = bf16_to_f64(got_bits)
    assert np.all(np.isfinite(g)), what
    excess = np.abs(g - ref) - round_rel * np.abs(ref)
    err = excess.max()
    rel = np.linalg.norm(g - ref) / max(np.linalg.norm(ref), 1e-30)
    assert err <= TOL_ABS and rel <= TOL_REL, "%s: max-abs beyond rounding %.3g, rel-L2 %.3g" % (what, err, rel)
    return err, rel


def observed_clear_tokens(s, logits_orc, logits_dev, margin=4.0):
    """Tokens on which a device routing is fixed by the oracle's logits alone:
    the device's logits of the token differ from the oracle's by at most d
    (observed on the stand-alone router; the fused kernel's own rounding is of
    the same size, hence the margin), and the oracle's K+1 largest logits are
    more than margin*d apart pairwise-adjacent, so neither the chosen set nor
    its order can differ.  The others are near ties at the device's rounding."""
    K, E = s.top_k, s.n_experts
    out, dev = [], []
    for t in range(logits_orc.shape[0]):
        d = float(np.abs(logits_dev[t].astype(np.float64) - logits_orc[t].astype(np.float64)).max())
        order = np.lexsort((np.arange(E), -logits_orc[t].astype(np.float64)))
        top = logits_orc[t, order[:min(K + 1, E)]].astype(np.float64)
        gaps = top[:-1] - top[1:]
        # d == 0: the logits came out exact, so ties are exact ties on both sides
        out.append(bool(d == 0.0 or np.all(gaps > margin * d)) if gaps.size else True)
        dev.append(d)
    return np.array(out), np.array(dev)


def check_layer(dl, x_bits, res_bits, blobs=None, max_near_ties=0):
    """Run the device layer and the oracle on the same inputs and compare.
    Routing: the stand-alone router's indices equal the oracle's top-K of its
    own logits, which lie within the rigorous accumulation bound of the
    oracle's; the fused layer's indices equal the oracle's own on every token
    whose top K+1 logits are further apart than the device's rounding can
    swap, and at most max_near_ties tokens may be such near ties (0 on every
    seeded case); its weights match the softmax of the oracle's logits at its
    choice within that rounding.  Outputs: the oracle under the fused layer's
    routing.  Returns (max-abs, rel-L2) of y_norm and the number of near-tie
    tokens."""
    s = dl.s
    blobs = dl.oracle_blobs() if blobs is None else blobs
    h, y, idx, w = dl.forward(x_bits, res_bits)
    lg, idx_r, w_r = dl.router(x_bits)
    idx_o_on_gpu_logits, _, w64_on_gpu = O.topk(ocfg(s), lg)
    assert np.array_equal(idx_r, idx_o_on_gpu_logits)
    np.testing.assert_allclose(w_r, w64_on_gpu, rtol=2e-6, atol=1e-7)
    lo, idx_o, _ = O.router(ocfg(s), x_bits, dl.dense["wr"], dl.dense["bias"])
    bound = router_error_bound(s, x_bits, dl.dense["wr"], lo)
    assert np.all(np.abs(lg.astype(np.float64) - lo) <= bound + 1e-30)
    clear = clear_gap_tokens(s, lo, bound)
    assert np.array_equal(idx[clear], idx_o[clear])
    seen, dev = observed_clear_tokens(s, lo, lg)
    assert np.array_equal(idx[seen], idx_o[seen])
    near = int((~seen).sum())
    assert near <= max_near_ties, "%d near-tie tokens (limit %d)" % (near, max_near_ties)
    for t in range(idx.shape[0]):
        lk = lo[t, idx[t]].astype(np.float64)
        wk = np.exp(lk - lk.max())
        wk /= wk.sum()
        np.testing.assert_allclose(w[t], wk, rtol=8 * dev[t] + 2e-6, atol=1e-7)
    # outputs under the device's routing (equal to the oracle's on clear tokens)
    # the oracle quantises the packed shared expert itself
    sblob = None
    if dl.shared_blob is not None:
        sblob = O.quantize_expert(ocfg(s), *S.expert_weights(s, s.n_experts))
        assert np.array_equal(sblob, dl.shared_blob)
    _, _, h_ref, y_ref = oracle_forward(s, blobs, dl.dense, x_bits, res_bits, idx_in=idx,
                                        w_in=w.astype(np.float64), shared_gate_w=dl.sgate_bits,
                                        shared_blob=sblob)
    assert_outputs_close(h, h_ref, "h_out")
    err = assert_outputs_close(y, y_ref, "y_norm")
    return err, near
