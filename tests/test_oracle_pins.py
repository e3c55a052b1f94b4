"""Pins for the CPU oracle, against things other than the oracle itself.

Each test ties one oracle function to a closed form, an invariant, a brute
force enumeration on a tiny input, a library routine that the case reduces
to, or a number printed on the pages.  They are chosen so that a plausible
slip (dropped term, wrong sign, swapped gate/up, transposed down matrix,
wrong nibble order, tie broken the wrong way) fails at least one of them.
"""
import itertools
import math

import numpy as np
import pytest
import torch
from scipy.special import expit

import oracle as O
from sparse_moe_expert_gemv_b200 import inputs as I
from tests._golden import read_kv

RNG = np.random.default_rng(1234)


# ------------------------------------------------------------ encodings
def test_f16_roundtrip_matches_numpy_float16():
    # numpy's float64 -> float16 cast is IEEE round-to-nearest-even
    vals = np.concatenate([
        RNG.normal(0, 1, 2000), RNG.normal(0, 1e-5, 500), RNG.normal(0, 3e4, 200),
        np.array([0.0, -0.0, 65504.0, 65519.99, 65520.0, 1e-8, 2.0 ** -24,
                  2.0 ** -25, 3 * 2.0 ** -26, 2.0 ** -14, 1.0 + 2.0 ** -11,
                  1.0 + 3 * 2.0 ** -11, -2047.5, 2049.0]),
    ])
    with np.errstate(over="ignore"):
        wants = vals.astype(np.float16).view(np.uint16)
    for v, want in zip(vals, wants):
        want = int(want)
        assert O.f64_to_f16(v) == want, v
    for b in range(0, 1 << 16, 7):
        e = (b >> 10) & 0x1F
        if e == 31:
            continue
        want = float(np.array([b], np.uint16).view(np.float16)[0])
        assert O.f16_to_f64(b) == want


def test_bf16_matches_torch_for_float32_values():
    # torch's float32 -> bfloat16 cast is round-to-nearest-even; for inputs
    # that are exact float32 values there is no double rounding
    vals = np.concatenate([RNG.normal(0, 1, 3000), RNG.normal(0, 1e30, 100),
                           RNG.normal(0, 1e-30, 100)]).astype(np.float32)
    vals = np.concatenate([vals, np.array([1 + 2 ** -8, 1 + 3 * 2 ** -8, 1 - 2 ** -9,
                                           3.3895313e38], np.float32)])
    want = torch.from_numpy(vals).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    for v, w in zip(vals, want):
        assert O.f64_to_bf16(float(v)) == int(w)
        back = torch.from_numpy(np.array([w], np.uint16).view(np.int16)).view(torch.bfloat16)
        assert O.bf16_to_f64(int(w)) == float(back.float()[0])


# -------------------------------------------------------------- formats
def test_q4_dequant_worked_example():
    # row of 32 weights (one group); byte 0 = 0x9F: low nibble 15 -> element
    # 0 = (15-8)*s, high nibble 9 -> element 1 = (9-8)*s; s = 0.5
    codes = np.full(16, 0x88, np.uint8)
    codes[0] = 0x9F
    codes[15] = 0x0F  # element 30 = +7 s, element 31 = -8 s
    s = np.array([O.f64_to_f16(0.5)], np.uint16)
    W = O.dequant(O.Q4, codes, s, None, 1, 32)[0]
    assert W[0] == 3.5 and W[1] == 0.5
    assert W[30] == 3.5 and W[31] == -4.0
    assert np.all(W[2:30] == 0.0)


def test_q2_dequant_worked_example():
    # one group of 64; byte 0 = 0b11_10_01_00 -> elements 0..3 have q = 0,1,2,3
    codes = np.zeros(16, np.uint8)
    codes[0] = 0b11100100
    codes[15] = 0b00000011  # element 60 -> q=3
    s = np.array([O.f64_to_f16(0.25)], np.uint16)
    m = np.array([O.f64_to_f16(-1.0)], np.uint16)
    W = O.dequant(O.Q2, codes, s, m, 1, 64)[0]
    assert list(W[:4]) == [-1.0, -0.75, -0.5, -0.25]
    assert W[60] == -0.25 and W[61] == -1.0


def _exact_q4(R, K):
    # s a power of two (exact in fp16), levels in [-7,7], each group holds +-7
    q = RNG.integers(-7, 8, size=(R, K))
    q[:, ::32] = 7 * RNG.choice([-1, 1], size=(R, K // 32))
    s = 2.0 ** RNG.integers(-9, -4, size=(R, K // 32))
    return q * np.repeat(s, 32, axis=1)


def _exact_q2(R, K):
    q = RNG.integers(0, 4, size=(R, K))
    q[:, ::64] = 0
    q[:, 1::64] = 3
    s = 2.0 ** RNG.integers(-7, -3, size=(R, K // 64))
    m = -RNG.integers(1, 9, size=(R, K // 64)) * 2.0 ** -6
    return q * np.repeat(s, 64, axis=1) + np.repeat(m, 64, axis=1)


@pytest.mark.parametrize("fmt", [O.Q4, O.Q2])
def test_quant_roundtrip_exact_on_representable(fmt):
    W = _exact_q4(6, 128) if fmt == O.Q4 else _exact_q2(6, 128)
    c, s, m = O.quantize(fmt, W)
    assert np.array_equal(O.dequant(fmt, c, s, m, 6, 128), W)


@pytest.mark.parametrize("fmt", [O.Q4, O.Q2])
def test_quant_idempotent_and_error_bound(fmt):
    G = O.GROUP[fmt]
    W = RNG.normal(0, 0.02, size=(8, 256))
    c, s, m = O.quantize(fmt, W)
    Wq = O.dequant(fmt, c, s, m, 8, 256)
    c2, s2, m2 = O.quantize(fmt, Wq)
    assert np.array_equal(c, c2) and np.array_equal(s, s2)
    if fmt == O.Q2:
        assert np.array_equal(m, m2)
    sv = np.array([O.f16_to_f64(b) for b in s]).reshape(8, 256 // G)
    bound = np.repeat(sv, G, axis=1) / 2
    assert np.all(np.abs(W - Wq) <= bound + 1e-15)


def test_q4_zero_group_encodes_to_level_zero():
    c, s, _ = O.quantize(O.Q4, np.zeros((1, 32)))
    assert s[0] == 0 and np.all(c == 0x88)


def _q4_levels(codes):
    lo = (codes & 0xF).astype(np.int64) - 8
    hi = (codes >> 4).astype(np.int64) - 8
    return np.stack([lo, hi], 1).reshape(-1)


def test_q4_rounding_ties_go_to_even_level():
    # max|w| = 7 * 2^-4, so s = 2^-4 exactly and w / s is exact: the group
    # holds w/s = +-0.5, +-1.5, +-2.5, +-3.5, +-4.5 (exact halves).  Round half
    # to even gives 0, 2, 2, 4, 4 (and the negatives); half away from zero
    # would give 1, 2, 3, 4, 5 and floor(x + 0.5) 1, 2, 3, 4, 5 / 0, -1, -2, -3, -4.
    s = 2.0 ** -4
    halves = np.array([0.5, 1.5, 2.5, 3.5, 4.5])
    w = np.zeros(32)
    w[0] = 7.0 * s
    w[1:6] = halves * s
    w[6:11] = -halves * s
    w[11] = -7.0 * s
    c, sc, _ = O.quantize(O.Q4, w[None, :])
    assert O.f16_to_f64(int(sc[0])) == s
    q = _q4_levels(c)
    assert list(q[1:6]) == [0, 2, 2, 4, 4]
    assert list(q[6:11]) == [0, -2, -2, -4, -4]
    assert q[0] == 7 and q[11] == -7


def test_q2_rounding_ties_go_to_even_code():
    # m = 0, max = 3 * 2^-3: s = 2^-3 exactly; (w - m) / s = 0.5, 1.5, 2.5
    # round half to even -> 0, 2, 2 (half away from zero: 1, 2, 3)
    s = 2.0 ** -3
    w = np.zeros(64)
    w[1] = 3.0 * s
    w[2:5] = np.array([0.5, 1.5, 2.5]) * s
    c, sc, mn = O.quantize(O.Q2, w[None, :])
    assert O.f16_to_f64(int(sc[0])) == s and O.f16_to_f64(int(mn[0])) == 0.0
    q = np.array([(c[i // 4] >> (2 * (i % 4))) & 3 for i in range(64)])
    assert list(q[2:5]) == [0, 2, 2]
    assert q[1] == 3 and q[0] == 0


def test_q4_clamp_reaches_level_minus_8_on_subnormal_scale():
    # max|w| / 7 = 2.5 * 2^-24 lies halfway between the fp16 subnormals 2 and
    # 3 * 2^-24 and rounds to 2 * 2^-24 (even): then w / s = -7 * 1.25 = -8.75
    # for the largest-magnitude element, clamped to the lowest level -8, and
    # +8.75 for its positive twin, clamped to +7.
    amax = 7.0 * 2.5 * 2.0 ** -24
    w = np.zeros(32)
    w[0] = -amax
    w[1] = amax
    c, sc, _ = O.quantize(O.Q4, w[None, :])
    assert int(sc[0]) == 2  # fp16 bits of 2 * 2^-24
    q = _q4_levels(c)
    assert q[0] == -8 and q[1] == 7
    assert np.all(q[2:] == 0)


def test_page_expert_byte_counts_match_shape():
    g = read_kv("page_expert_bytes.txt")
    d, f = 2048, 768
    weights = 3 * d * f
    per_expert = g["expert_mb_per_token"] * 1e6 / (g["layers"] * g["active_per_token"])
    per_slot = g["cache_slot_mib"] * 2 ** 20 / g["cache_slots"]
    assert abs(per_expert - per_slot) / per_slot < 1e-3  # the two pages' figures agree
    bits = per_expert * 8 / weights
    # a 2-bit-class format: more than bare 2-bit codes, at most this
    # library's Q2 (2 bits + fp16 scale and min per 64)
    q2_bits = 8 * (I.expert_sizes(I.Q2, d, f)[0] + 2 * 2 * I.expert_sizes(I.Q2, d, f)[1]) / weights
    assert 2.0 < bits <= q2_bits
    assert O.code_bytes(O.Q2, f, d) * 3 * 8 / weights == 2.0


# ---------------------------------------------------------------- router
def _bf16(a):
    return I.f32_to_bf16_bits(np.asarray(a, np.float32))


def test_router_matches_blas_matmul():
    T, d, E = 5, 96, 24
    h = _bf16(RNG.normal(0, 1, (T, d)))
    W = RNG.normal(0, 0.02, (E, d)).astype(np.float32)
    b = RNG.normal(0, 1, E).astype(np.float32)
    got = O.router(h, W, b)
    hv = I.bf16_bits_to_f32(h).astype(np.float64)
    want = hv @ W.astype(np.float64).T + b.astype(np.float64)
    assert np.allclose(got, want, rtol=1e-13, atol=1e-13)


def test_router_one_hot_selects_column():
    d, E = 64, 16
    W = RNG.normal(0, 0.02, (E, d)).astype(np.float32)
    h = np.zeros((1, d), np.float32)
    h[0, 17] = 1.0
    assert np.array_equal(O.router(_bf16(h), W)[0], W[:, 17].astype(np.float64))


# ----------------------------------------------------------------- top-k
def _brute_topk_set(l, k):
    # the unique k-subset S whose every member beats every non-member, where
    # "beats" = larger logit, or equal logit and lower index
    E = len(l)
    beats = lambda a, b: l[a] > l[b] or (l[a] == l[b] and a < b)
    found = [S for S in itertools.combinations(range(E), k)
             if all(beats(a, b) for a in S for b in range(E) if b not in S)]
    assert len(found) == 1
    return set(found[0])


def test_topk_brute_force_with_ties():
    for trial in range(200):
        E = int(RNG.integers(2, 11))
        k = int(RNG.integers(1, min(E, 4) + 1))
        l = RNG.integers(-3, 4, size=(1, E)).astype(np.float64)  # many ties
        idx, w, margin = O.topk(l, k)
        assert set(idx[0].tolist()) == _brute_topk_set(l[0], k)
        order = sorted(range(E), key=lambda e: (-l[0, e], e))
        want_margin = math.inf if k == E else l[0, order[k - 1]] - l[0, order[k]]
        assert margin[0] == want_margin


def test_topk_all_equal_takes_lowest_ids():
    idx, w, _ = O.topk(np.zeros((1, 9)), 4)
    assert idx[0].tolist() == [0, 1, 2, 3]
    assert np.allclose(w[0], 0.25, atol=0, rtol=1e-15)


def test_softmax_weights_closed_forms():
    l = RNG.normal(0, 1, (50, 32))
    idx, w, _ = O.topk(l, 6)
    assert np.all(np.abs(w.sum(1) - 1) <= 1e-12)
    sel = np.take_along_axis(l, idx, 1)
    assert np.all(np.diff(sel, axis=1) <= 0) and np.all(np.diff(w, axis=1) <= 0)
    idx2, w2, _ = O.topk(l + 123.25, 6)
    assert np.array_equal(idx, idx2) and np.allclose(w, w2, rtol=1e-12, atol=0)
    # k = 2: w0 = logistic(l0 - l1)  (scipy.special.expit)
    idx, w, _ = O.topk(l, 2)
    sel = np.take_along_axis(l, idx, 1)
    assert np.allclose(w[:, 0], expit(sel[:, 0] - sel[:, 1]), rtol=1e-14, atol=0)
    # k = 1: weight exactly 1
    _, w1, _ = O.topk(l, 1)
    assert np.all(w1 == 1.0)


# -------------------------------------------------------------- bucketing
def test_bucket_brute_force():
    for trial in range(30):
        T, E = int(RNG.integers(1, 20)), int(RNG.integers(2, 17))
        k = int(RNG.integers(1, E + 1))
        idx = np.stack([RNG.permutation(E)[:k] for _ in range(T)]).astype(np.int32)
        cnt, off, perm = O.bucket(idx, E)
        assert cnt.sum() == T * k and off[0] == 0 and off[-1] == T * k
        assert sorted(perm.tolist()) == list(range(T * k))
        for e in range(E):
            want = [t * k + j for t in range(T) for j in range(k) if idx[t, j] == e]
            assert perm[off[e]:off[e + 1]].tolist() == want
            assert cnt[e] == len(want)


# ----------------------------------------------------------------- expert
def test_silu_closed_forms():
    assert O.silu(0.0) == 0.0
    for z in RNG.normal(0, 4, 100):
        assert math.isclose(O.silu(z), z * expit(z), rel_tol=1e-14, abs_tol=1e-300)
        assert math.isclose(O.silu(z) - O.silu(-z), z, rel_tol=1e-13, abs_tol=1e-14)
    assert O.silu(-800.0) == 0.0


def _rand_h(n, d):
    return _bf16(RNG.normal(0, 1, (n, d)))


def test_expert_gate_negation_identity():
    # SiLU(z) - SiLU(-z) = z, so y(Wg) - y(-Wg) = Wd ((Wg h) * (Wu h)):
    # bilinear, no SiLU; pins which matrix is gated and how Wd is applied
    d, f, n = 64, 32, 3
    Wg = RNG.normal(0, 0.2, (f, d)); Wu = RNG.normal(0, 0.2, (f, d))
    Wd = RNG.normal(0, 0.2, (d, f))
    h = _rand_h(n, d)
    hv = I.bf16_bits_to_f32(h).astype(np.float64)
    diff = O.expert(Wg, Wu, Wd, h) - O.expert(-Wg, Wu, Wd, h)
    want = ((hv @ Wg.T) * (hv @ Wu.T)) @ Wd.T
    assert np.allclose(diff, want, rtol=1e-10, atol=1e-12)


def test_expert_zero_and_linearity():
    d, f = 64, 32
    Wg = RNG.normal(0, 0.2, (f, d)); Wu = RNG.normal(0, 0.2, (f, d))
    Wd = RNG.normal(0, 0.2, (d, f))
    h = _rand_h(2, d)
    y = O.expert(Wg, Wu, Wd, h)
    assert np.all(O.expert(np.zeros_like(Wg), Wu, Wd, h) == 0)
    assert np.all(O.expert(Wg, np.zeros_like(Wu), Wd, h) == 0)
    assert np.array_equal(O.expert(Wg, Wu, 2 * Wd, h), 2 * y)  # power of two: exact
    tol = 1e-13 * np.abs(y).max()
    assert np.allclose(O.expert(Wg, 3 * Wu, Wd, h), 3 * y, rtol=0, atol=3 * tol)


@pytest.mark.parametrize("fmt", [O.Q4, O.Q2])
def test_quantised_expert_equals_dense_on_representable(fmt):
    d, f = 128, 64
    mk = _exact_q4 if fmt == O.Q4 else _exact_q2
    Wg, Wu, Wd = mk(f, d), mk(f, d), mk(d, f)
    parts = [O.quantize(fmt, M) for M in (Wg, Wu, Wd)]
    codes = np.concatenate([p[0] for p in parts])
    scales = np.concatenate([p[1] for p in parts])
    mins = np.concatenate([p[2] for p in parts]) if fmt == O.Q2 else None
    g2, u2, d2 = O.dequant_expert(fmt, d, f, codes, scales, mins)
    h = _rand_h(3, d)
    assert np.array_equal(O.expert(g2, u2, d2, h), O.expert(Wg, Wu, Wd, h))


# ------------------------------------------------------------------ layer
def _layer_setup(fmt=O.Q4, d=64, f=64, E=8, T=5, seed=3):
    experts = {e: I.expert_np(seed, fmt, d, f, 0, e) for e in range(E)}
    shared = I.shared_np(seed, fmt, d, f, 0)
    W = I.router_np(seed, E, d)
    x = I.hidden_np(seed, T, d)
    return experts, shared, W, x


def test_layer_identical_experts_sum_to_one():
    # every expert the same -> routed part = Expert(h) for any routing,
    # because the routing weights sum to one; with the shared expert also
    # the same, delta = 2 Expert(h)
    fmt, d, f, E, k = O.Q4, 64, 64, 8, 3
    experts, shared, W, x = _layer_setup(fmt, d, f, E)
    one = experts[2]
    same = {e: one for e in range(E)}
    Wg, Wu, Wd = O.dequant_expert(fmt, d, f, *one)
    y = O.expert(Wg, Wu, Wd, x)
    out = O.moe_layer(x, fmt=fmt, d=d, f=f, E=E, k=k, router_w=W, experts=same)
    assert np.allclose(out["delta"], y, rtol=1e-12, atol=1e-14)
    out2 = O.moe_layer(x, fmt=fmt, d=d, f=f, E=E, k=k, router_w=W, experts=same,
                       shared=one)
    assert np.allclose(out2["delta"], 2 * y, rtol=1e-12, atol=1e-14)


def test_layer_k1_and_residual():
    fmt, d, f, E = O.Q2, 64, 64, 8
    experts, shared, W, x = _layer_setup(fmt, d, f, E)
    out = O.moe_layer(x, fmt=fmt, d=d, f=f, E=E, k=1, router_w=W, experts=experts)
    assert np.all(out["w"] == 1.0)
    for t in range(x.shape[0]):
        e = out["idx"][t, 0]
        y = O.expert(*O.dequant_expert(fmt, d, f, *experts[e]), x[t:t + 1])
        assert np.array_equal(out["delta"][t], y[0])
    xv = I.bf16_bits_to_f32(x).astype(np.float64)
    want = [O.f64_to_bf16(v) for v in (xv + out["delta"]).reshape(-1)]
    assert np.array_equal(out["x_out"].reshape(-1), np.array(want, np.uint16))


def test_layer_is_sum_over_selected_experts():
    # delta[t] = sum_j w_j Expert_{idx_j}(h_t) + Shared(h_t), built from the
    # separately pinned pieces
    fmt, d, f, E, k = O.Q4, 64, 64, 8, 3
    experts, shared, W, x = _layer_setup(fmt, d, f, E)
    out = O.moe_layer(x, fmt=fmt, d=d, f=f, E=E, k=k, router_w=W, experts=experts,
                      shared=shared)
    ys = O.expert(*O.dequant_expert(fmt, d, f, *shared), x)
    for t in range(x.shape[0]):
        acc = ys[t].copy()
        for j in range(k):
            e = out["idx"][t, j]
            acc += out["w"][t, j] * O.expert(*O.dequant_expert(fmt, d, f, *experts[e]),
                                             x[t:t + 1])[0]
        assert np.allclose(out["delta"][t], acc, rtol=1e-12, atol=1e-15)


def test_layer_expert_relabelling_invariance():
    fmt, d, f, E, k = O.Q4, 64, 64, 8, 3
    experts, shared, W, x = _layer_setup(fmt, d, f, E)
    pi = RNG.permutation(E)
    W2 = W[pi]
    ex2 = {e: experts[pi[e]] for e in range(E)}
    a = O.moe_layer(x, fmt=fmt, d=d, f=f, E=E, k=k, router_w=W, experts=experts)
    b = O.moe_layer(x, fmt=fmt, d=d, f=f, E=E, k=k, router_w=W2, experts=ex2)
    assert np.allclose(a["delta"], b["delta"], rtol=1e-12, atol=1e-15)
    assert np.array_equal(pi[b["idx"]], a["idx"])


def test_layer_zero_weights_leave_residual_unchanged():
    fmt, d, f, E, k = O.Q4, 64, 64, 4, 2
    zero = (np.full(3 * f * d // 2, 0x88, np.uint8), np.zeros(3 * f * d // 32, np.uint16), None)
    _, _, W, x = _layer_setup(fmt, d, f, E)
    out = O.moe_layer(x, fmt=fmt, d=d, f=f, E=E, k=k, router_w=W,
                      experts={e: zero for e in range(E)}, shared=zero)
    assert np.all(out["delta"] == 0) and np.array_equal(out["x_out"], x)


def test_rmsnorm_closed_form():
    d = 64
    for a in [0.5, 3.0, 1e-3]:
        x = np.tile(np.array([a, -a], np.float32), d // 2)[None, :]
        h = O.rmsnorm(_bf16(x), None, 1e-6)
        xa = float(I.bf16_bits_to_f32(_bf16(np.array([a])))[0])
        want = O.f64_to_bf16(xa / math.sqrt(xa * xa + 1e-6))
        assert h[0, 0] == want and h[0, 1] == (want | 0x8000)
    # gamma multiplies the normalised value elementwise
    x = _bf16(RNG.normal(0, 2, (3, d)))
    g = np.full(d, 2.0, np.float32)
    h1 = I.bf16_bits_to_f32(O.rmsnorm(x, None, 1e-6))
    h2 = I.bf16_bits_to_f32(O.rmsnorm(x, g, 1e-6))
    assert np.array_equal(2 * h1, h2)  # exact: scaling by 2 commutes with rounding
    # mean of h^2 is one up to bf16 rounding and eps
    assert np.allclose((h1.astype(np.float64) ** 2).mean(1), 1.0, rtol=1e-2)


def test_layer_norm_path_uses_normalised_input():
    fmt, d, f, E, k = O.Q4, 64, 64, 8, 2
    experts, shared, W, x = _layer_setup(fmt, d, f, E)
    out = O.moe_layer(x, fmt=fmt, d=d, f=f, E=E, k=k, router_w=W, experts=experts,
                      norm=True, eps=1e-6)
    h = O.rmsnorm(x, None, 1e-6)
    assert np.array_equal(out["h"], h)
    ref = O.moe_layer(h, fmt=fmt, d=d, f=f, E=E, k=k, router_w=W, experts=experts)
    assert np.array_equal(out["delta"], ref["delta"])
