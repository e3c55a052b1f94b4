"""Shared set-up for the parity tests: one seeded synthetic MoE layer, the
CUDA library's view of it (through the C ABI) and the oracle's view of it.

Inputs come only from ``sparse_moe_expert_gemv_b200.inputs``; expected values
come only from ``oracle``.  The two sides share the input bytes and nothing
else.
"""
from __future__ import annotations

import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np

import oracle as O
from sparse_moe_expert_gemv_b200 import inputs as I

# tolerances (stated by the workload definition)
OUT_TOL = 2e-2      # max-abs error <= OUT_TOL * RMS(oracle tensor)
W_TOL = 1e-5        # routing weights, absolute
TIE_MARGIN = 1e-5   # oracle k-th vs (k+1)-th fp64 logit gap below which a
                    # token is excluded from the bit-exact routing checks


def quantised_expert(seed, fmt, d, f, layer, e):
    """An expert whose N(0, 0.02) matrices are encoded by the oracle's
    quantiser (the packed bytes both sides then consume)."""
    mats = I.expert_weights_np(seed, d, f, layer, e)
    parts = [O.quantize(fmt, W) for W in mats]
    codes = np.concatenate([p[0] for p in parts])
    scales = np.concatenate([p[1] for p in parts])
    mins = None if fmt == O.Q4 else np.concatenate([p[2] for p in parts])
    return codes, scales, mins


class LayerSpec:
    """One MoE layer's synthetic weights (router, experts, shared expert).

    weights: "codes" -- the generator's packed codes (``inputs.expert_np``);
    "quantised" -- N(0, 0.02) matrices encoded by the oracle's quantiser,
    for the experts in ``quantise`` (all when None; the others keep the
    generator's codes); "uniform" -- uniform code bytes (every code value)."""

    def __init__(self, *, d, f, E, k, fmt, seed=0, shared=True, zipf=False, layer=0,
                 weights="codes", quantise=None):
        self.d, self.f, self.E, self.k, self.fmt = d, f, E, k, fmt
        self.seed, self.shared, self.zipf, self.layer = seed, shared, zipf, layer
        self.weights, self.quantise = weights, quantise
        self.W = I.router_np(seed, E, d, layer)
        self.bias = I.zipf_bias_np(seed, E, layer)[0] if zipf else None
        self._host = {}

    def special(self, e):
        """Whether expert e (SHARED_INDEX for the shared one) differs from
        the generator's codes."""
        if self.weights == "codes":
            return False
        return self.quantise is None or e in self.quantise

    def _make(self, e):
        if self.special(e):
            if self.weights == "quantised":
                return quantised_expert(self.seed, self.fmt, self.d, self.f, self.layer, e)
            return I.expert_uniform_codes_np(self.seed, self.fmt, self.d, self.f, self.layer, e)
        return I.expert_np(self.seed, self.fmt, self.d, self.f, self.layer, e)

    # ---- expert bytes, host side for the oracle
    def expert(self, e):
        if e not in self._host:
            self._host[e] = self._make(e)
        return self._host[e]

    def set_host_experts(self, codes, scales, mins):
        """Host copies of all E experts (from the torch generator's tensors)."""
        for e in range(self.E):
            self._host[e] = (codes[e], scales[e].view(np.uint16),
                             None if mins is None else mins[e].view(np.uint16))

    def shared_expert(self):
        if not self.shared:
            return None
        if "shared" not in self._host:
            self._host["shared"] = self._make(I.SHARED_INDEX)
        return self._host["shared"]

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
    # experts that are not the generator's codes: host bytes, one by one
    for e in range(spec.E):
        if spec.special(e):
            spec._host.pop(e, None)
            c, s, m = spec.expert(e)
            B.moe_load_experts(ctx, layer, e, 1, c, s, m)
    return codes, scales, mins


# ------------------------------------------------- oracle on many host cores
def oracle_threads():
    return max(1, min(32, os.cpu_count() or 1))


def router_parallel(h_bits, W, bias=None, threads=None):
    """O.router over row chunks on a thread pool (the C oracle runs without
    the GIL); the result is the oracle's, row for row."""
    h_bits = np.ascontiguousarray(h_bits, np.uint16)
    n = threads or oracle_threads()
    chunks = np.array_split(np.arange(h_bits.shape[0]), n)
    with ThreadPoolExecutor(n) as ex:
        parts = list(ex.map(lambda r: O.router(h_bits[r], W, bias), [c for c in chunks if c.size]))
    return np.concatenate(parts)


def oracle_rows(spec, x_bits, rows, threads=None, norm=False):
    """The oracle's whole layer on the given rows (tokens are independent),
    in chunks on a thread pool.  Returns (delta [n, d], x_out [n, d] bits,
    margin [n]) in the order of ``rows``."""
    rows = np.asarray(rows)
    n = min(threads or oracle_threads(), max(1, rows.size))
    chunks = [c for c in np.array_split(np.arange(rows.size), n) if c.size]

    def one(c):
        out = spec.oracle(x_bits[rows[c]], norm=norm)
        return out["delta"], out["x_out"], out["margin"]

    with ThreadPoolExecutor(len(chunks)) as ex:
        parts = list(ex.map(one, chunks))
    return (np.concatenate([p[0] for p in parts]), np.concatenate([p[1] for p in parts]),
            np.concatenate([p[2] for p in parts]))


def covering_sample(idx, E, tile=128, n_hot=3):
    """Tokens (sorted) such that, in the expert-grouped order of the pairs
    (each expert's tokens ascending), every expert's first and last
    ``tile``-row tile holds a sampled token, every tile of the ``n_hot``
    experts with most tokens does, and so do each expert's first and last
    token (the edges of its first and last tiles).  Chosen greedily, so one
    token covers the tiles of all its experts."""
    T, k = idx.shape
    lists = [[] for _ in range(E)]
    for t in range(T):
        for e in idx[t]:
            lists[int(e)].append(t)
    counts = np.array([len(l) for l in lists])
    hot = set(np.argsort(-counts, kind="stable")[:n_hot].tolist())
    need = {}   # (expert, tile) -> tokens of that tile
    must = set()
    for e in range(E):
        L = lists[e]
        if not L:
            continue
        nt = (len(L) + tile - 1) // tile
        tiles = range(nt) if e in hot else sorted({0, nt - 1})
        for m in tiles:
            need[(e, m)] = set(L[m * tile:(m + 1) * tile])
        must.add(L[0])
        must.add(L[-1])
    chosen = set(must)
    open_ = {key for key, toks in need.items() if not (toks & chosen)}
    while open_:
        score = {}
        for key in open_:
            for t in need[key]:
                score[t] = score.get(t, 0) + 1
        best = min(score, key=lambda t: (-score[t], t))
        chosen.add(best)
        open_ = {key for key in open_ if best not in need[key]}
    return np.array(sorted(chosen))


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


def bf16_ulp(v):
    """Spacing of bf16 values at magnitude |v| (normal range)."""
    a = np.maximum(np.abs(np.asarray(v, np.float64)), 2.0 ** -126)
    return 2.0 ** (np.floor(np.log2(a)) - 7)


def assert_close_residual(got_bits, want_bits, tol=OUT_TOL, what="residual x"):
    """The layer's bf16 output x = bf16(x_in + delta).  Two sums that agree
    within the tolerance can still round to neighbouring bf16 values, so the
    bound is tol * RMS plus one bf16 ulp at the element's magnitude; the
    strict check is the one on delta, before this rounding."""
    got = I.bf16_bits_to_f32(got_bits).astype(np.float64)
    want = I.bf16_bits_to_f32(want_bits).astype(np.float64)
    assert got.shape == want.shape, (got.shape, want.shape)
    if want.size == 0:
        return
    bound = tol * rms(want) + bf16_ulp(np.maximum(np.abs(got), np.abs(want)))
    bad = np.abs(got - want) > bound
    assert not bad.any(), (f"{what}: {int(bad.sum())} elements beyond tol*RMS + 1 ulp, "
                           f"max|err| {np.abs(got - want).max():.3e}")


def check_routing(gpu_idx, gpu_w, orc, k):
    """Expert sets bit-exact and weights within W_TOL, except near ties.
    Returns the boolean mask of tokens that were checked."""
    ok = orc["margin"] >= TIE_MARGIN
    for t in np.nonzero(ok)[0]:
        assert set(gpu_idx[t].tolist()) == set(orc["idx"][t].tolist()), (
            f"token {t}: oracle margin {orc['margin'][t]:.3e}, gpu only "
            f"{sorted(set(gpu_idx[t].tolist()) - set(orc['idx'][t].tolist()))}, oracle only "
            f"{sorted(set(orc['idx'][t].tolist()) - set(gpu_idx[t].tolist()))}")
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
