"""GPU parity of the prefill path (moe_prefill: routing, sort by expert, the
grouped tcgen05 GEMM over dequantised tiles, combine) against the oracle.

Bars as for decode: MoE delta and residual x within max-abs error <= 2e-2 x
RMS; tokens whose oracle k-th/(k+1)-th logit gap is < 1e-5 are excluded.
"""
import numpy as np
import pytest
import torch

import oracle as O
from sparse_moe_expert_gemv_b200 import inputs as I
from tests._harness import TIE_MARGIN, LayerSpec, assert_close_rms, load_layer

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def B():
    from sparse_moe_expert_gemv_b200 import binding
    return binding


def make_ctx(B, spec, max_tokens):
    ctx = B.moe_create(spec.d, spec.f, spec.E, spec.k, spec.fmt)
    B.moe_configure(ctx, 1, 1 if spec.shared else 0, 0, max_tokens)
    return ctx


def to_dev(bits):
    return torch.from_numpy(np.ascontiguousarray(bits, np.uint16).view(np.int16)).cuda()


def run_prefill(B, ctx, spec, x_bits):
    N, d = x_bits.shape[0], spec.d
    x = to_dev(x_bits)
    delta = torch.empty((N, d), dtype=torch.float32, device="cuda")
    B.moe_prefill_delta(ctx, 0, x, N, delta)
    x2 = x.clone()
    B.moe_prefill(ctx, 0, x2, N)
    B.moe_sync(ctx, 120000)
    return delta.cpu().numpy(), x2.cpu().numpy().view(np.uint16)


def check_rows(spec, x_bits, delta, x_out, rows):
    """Oracle on `rows` only (tokens are independent); near ties excluded."""
    lg = O.router(x_bits[rows], spec.W, spec.bias)
    _, _, margin = O.topk(lg, spec.k)
    ok = margin >= TIE_MARGIN
    orc = spec.oracle(x_bits[rows])
    rel = assert_close_rms(delta[rows][ok], orc["delta"][ok], what="MoE delta")
    assert_close_rms(I.bf16_bits_to_f32(x_out[rows][ok]), I.bf16_bits_to_f32(orc["x_out"][ok]),
                     what="residual x")
    return rel, int((~ok).sum())


@pytest.mark.parametrize("zipf", [False, True])
@pytest.mark.parametrize("N", [33, 300, 1000])
def test_prefill_small_layer_all_tokens(B, N, zipf):
    """d=256, f=128, E=16, k=2 + shared: partial and multiple 128-row tiles
    per expert, several shared-expert tiles; every token checked."""
    spec = LayerSpec(d=256, f=128, E=16, k=2, fmt=I.Q4, seed=5, shared=True, zipf=zipf)
    ctx = make_ctx(B, spec, 1024)
    try:
        load_layer(B, ctx, spec)
        x = I.hidden_np(5, N, spec.d, window=77 + N)
        delta, x_out = run_prefill(B, ctx, spec, x)
        rel, ties = check_rows(spec, x, delta, x_out, np.arange(N))
        print(f"N={N} zipf={zipf}: delta max-err/RMS {rel:.2e}, near ties {ties}")
    finally:
        B.moe_destroy(ctx)


def test_prefill_matches_decode_path(B):
    """The grouped GEMM and the GEMV path compute the same layer: equal
    within the output tolerance on every token."""
    spec = LayerSpec(d=256, f=256, E=8, k=2, fmt=I.Q4, seed=9, shared=True)
    ctx = make_ctx(B, spec, 512)
    try:
        load_layer(B, ctx, spec)
        N = 400
        x = to_dev(I.hidden_np(9, N, spec.d, window=3))
        d1 = torch.empty((N, spec.d), dtype=torch.float32, device="cuda")
        d2 = torch.empty_like(d1)
        B.moe_prefill_delta(ctx, 0, x, N, d1)
        B.moe_forward_delta(ctx, 0, x, N, d2)
        B.moe_sync(ctx, 60000)
        assert_close_rms(d1.cpu().numpy(), d2.cpu().numpy(), what="prefill vs decode path")
    finally:
        B.moe_destroy(ctx)


def test_prefill_q2_takes_the_gemv_path(B):
    spec = LayerSpec(d=256, f=128, E=16, k=2, fmt=I.Q2, seed=6, shared=True)
    ctx = make_ctx(B, spec, 256)
    try:
        load_layer(B, ctx, spec)
        x = I.hidden_np(6, 200, spec.d, window=5)
        delta, x_out = run_prefill(B, ctx, spec, x)
        check_rows(spec, x, delta, x_out, np.arange(200))
    finally:
        B.moe_destroy(ctx)


def test_prefill_chunk_8192_zipf_sampled(B):
    """The prefill workload: d=2048, f=768, E=512, top-10 + shared, Q4 g32,
    8192 tokens, Zipf(1.1)-biased routing; 16 sampled tokens against the
    oracle."""
    spec = LayerSpec(d=2048, f=768, E=512, k=10, fmt=I.Q4, seed=0, shared=True, zipf=True)
    ctx = make_ctx(B, spec, 8192)
    try:
        load_layer(B, ctx, spec)
        N = 8192
        x = I.hidden_np(0, N, spec.d, window=4242)
        delta, x_out = run_prefill(B, ctx, spec, x)
        rows = np.sort(np.random.default_rng(1).choice(N, size=16, replace=False))
        rel, ties = check_rows(spec, x, delta, x_out, rows)
        print(f"prefill 8192: delta max-err/RMS {rel:.2e}, near ties {ties}")
        assert np.isfinite(delta).all()
    finally:
        B.moe_destroy(ctx)
