"""Shared set-up for the parity tests: one seeded synthetic MoE layer, the
CUDA library's view of it (through the C ABI) and the oracle's view of it.

Inputs come only from ``sparse_moe_expert_gemv_b200.inputs``; expected values
come only from ``oracle``.  The two sides share the input bytes and nothing
else.
"""
from __future__ import annotations

import numpy as np

import oracle as O
from sparse_moe_expert_gemv_b200 import inputs as I

# tolerances (stated by the workload definition)
OUT_TOL = 2e-2      # max-abs error <= OUT_TOL * RMS(oracle tensor)
W_TOL = 1e-5        # routing weights, absolute
TIE_MARGIN = 1e-5   # oracle k-th vs (k+1)-th fp64 logit gap below which a
                    # token is excluded from the bit-exact routing checks


class LayerSpec:
    """One MoE layer's synthetic weights (router, experts, shared expert)."""

    def __init__(self, *, d, f, E, k, fmt, seed=0, shared=True, zipf=False, layer=0):
        self.d, self.f, self.E, self.k, self.fmt = d, f, E, k, fmt
        self.seed, self.shared, self.zipf, self.layer = seed, shared, zipf, layer
        self.W = I.router_np(seed, E, d, layer)
        self.bias = I.zipf_bias_np(seed, E, layer)[0] if zipf else None
        self._host = {}

    # ---- expert bytes (generator output), host side for the oracle
    def expert(self, e):
        if e not in self._host:
            self._host[e] = I.expert_np(self.seed, self.fmt, self.d, self.f, self.layer, e)
        return self._host[e]

    def set_host_experts(self, codes, scales, mins):
        """Host copies of all E experts (from the torch generator's tensors)."""
        for e in range(self.E):
            self._host[e] = (codes[e], scales[e].view(np.uint16),
                             None if mins is None else mins[e].view(np.uint16))

    def shared_expert(self):
        return I.shared_np(self.seed, self.fmt, self.d, self.f, self.layer) if self.shared else None

    # ---- oracle
    def oracle(self, x_bits, norm=False, eps=1e-6, route_only_experts=None):
        x_bits = np.ascontiguousarray(x_bits, np.uint16)
        # route first (cheap) to know which experts the oracle needs
        h = O.rmsnorm(x_bits, None, eps) if norm else x_bits
        lg = O.router(h, self.W, self.bias)
        idx, _, _ = O.topk(lg, self.k)
        need = sorted(set(idx.reshape(-1).tolist()))
        experts = {e: self.expert(e) for e in need}
        return O.moe_layer(x_bits, fmt=self.fmt, d=self.d, f=self.f, E=self.E, k=self.k,
                           router_w=self.W, router_bias=self.bias, experts=experts,
                           shared=self.shared_expert(), norm=norm, eps=eps)


def load_layer(B, ctx, spec: LayerSpec, layer=0, device="cuda", chunk=64):
    """Generate the layer's experts on the GPU with the input generator and
    load everything through the C ABI.  Returns host copies of the experts."""
    import torch

    B.moe_set_router(ctx, layer, spec.W, spec.bias)
    hc, hs, hm = [], [], []
    for first in range(0, spec.E, chunk):
        n = min(chunk, spec.E - first)
        c, s, m = I.experts_torch(spec.seed, spec.fmt, spec.d, spec.f, spec.layer, first, n,
                                  device)
        B.moe_load_experts(ctx, layer, first, n, c, s, m)
        hc.append(c.cpu().numpy())
        hs.append(s.cpu().numpy())
        hm.append(None if m is None else m.cpu().numpy())
        del c, s, m
    if spec.shared:
        c, s, m = spec.shared_expert()
        B.moe_load_shared(ctx, layer, c, s, m)
    torch.cuda.synchronize()
    codes = np.concatenate(hc)
    scales = np.concatenate(hs)
    mins = None if hm[0] is None else np.concatenate(hm)
    spec.set_host_experts(codes, scales, mins)
    return codes, scales, mins


def rms(a):
    a = np.asarray(a, np.float64)
    return float(np.sqrt(np.mean(a * a))) if a.size else 0.0


def assert_close_rms(got, want, tol=OUT_TOL, what="output"):
    got = np.asarray(got, np.float64)
    want = np.asarray(want, np.float64)
    assert got.shape == want.shape, (got.shape, want.shape)
    if want.size == 0:
        return 0.0
    err = float(np.max(np.abs(got - want)))
    bound = tol * rms(want)
    assert err <= bound, f"{what}: max|err| {err:.3e} > {tol} * RMS {rms(want):.3e}"
    return err / max(rms(want), 1e-300)


def check_routing(gpu_idx, gpu_w, orc, k):
    """Expert sets bit-exact and weights within W_TOL, except near ties.
    Returns the boolean mask of tokens that were checked."""
    ok = orc["margin"] >= TIE_MARGIN
    for t in np.nonzero(ok)[0]:
        assert set(gpu_idx[t].tolist()) == set(orc["idx"][t].tolist()), f"token {t}"
        # compare weights expert by expert
        wo = dict(zip(orc["idx"][t].tolist(), orc["w"][t].tolist()))
        for e, wv in zip(gpu_idx[t].tolist(), gpu_w[t].tolist()):
            assert abs(wv - wo[e]) <= W_TOL, f"token {t} expert {e}: {wv} vs {wo[e]}"
    return ok


def check_buckets(off, perm, orc_idx, E, k, tokens_ok):
    """Bucket contents bit-exact per expert, as the ordered list of tokens
    (the position j of an expert inside a token's top-k is not graded);
    near-tie tokens are dropped from both sides before comparing."""
    T = orc_idx.shape[0]
    _, ooff, operm = O.bucket(orc_idx, E)
    for e in range(E):
        g = [p // k for p in perm[off[e]:off[e + 1]].tolist() if tokens_ok[p // k]]
        o = [p // k for p in operm[ooff[e]:ooff[e + 1]].tolist() if tokens_ok[p // k]]
        assert g == o, f"bucket of expert {e}: {g[:8]} vs {o[:8]}"
    assert off[0] == 0 and off[E] == T * k
