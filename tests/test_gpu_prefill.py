"""GPU parity of the prefill path (moe_prefill: routing, sort by expert, the
grouped tcgen05 GEMM over dequantised tiles, combine) against the oracle.

Bars as for decode: MoE delta within max-abs error <= 2e-2 x RMS, residual x
within that plus one bf16 ulp (its final rounding); tokens whose oracle
k-th/(k+1)-th logit gap is < 1e-5 are excluded.
"""
import numpy as np
import pytest
import torch

import oracle as O
from sparse_moe_expert_gemv_b200 import inputs as I
from tests._harness import (TIE_MARGIN, LayerSpec, assert_close_residual, assert_close_rms,
                            check_buckets, check_routing, covering_sample, load_layer, oracle_rows,
                            router_parallel)

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
    assert_close_residual(x_out[rows][ok], orc["x_out"][ok])
    return rel, int((~ok).sum())


@pytest.mark.parametrize("fmt", [I.Q4, I.Q2])
@pytest.mark.parametrize("zipf", [False, True])
@pytest.mark.parametrize("N", [33, 300, 1000])
def test_prefill_small_layer_all_tokens(B, N, zipf, fmt):
    """d=256, f=128, E=16, k=2 + shared: partial and multiple 128-row tiles
    per expert, several shared-expert tiles; every token checked.  Q2 experts
    are dequantised by the GEMM's own Q2 stage (a code tile per two k-steps)."""
    spec = LayerSpec(d=256, f=128, E=16, k=2, fmt=fmt, seed=5, shared=True, zipf=zipf)
    ctx = make_ctx(B, spec, 1024)
    try:
        load_layer(B, ctx, spec)
        x = I.hidden_np(5, N, spec.d, window=77 + N)
        delta, x_out = run_prefill(B, ctx, spec, x)
        rel, ties = check_rows(spec, x, delta, x_out, np.arange(N))
        print(f"N={N} zipf={zipf}: delta max-err/RMS {rel:.2e}, near ties {ties}")
        # the same chunk's routing and buckets, bit for bit
        out = _route_outputs(N, spec.k, spec.E)
        B.moe_prefill_route(ctx, 0, to_dev(x), N, *out)
        B.moe_sync(ctx, 60000)
        idx, w, off, perm = [t.cpu().numpy() for t in out]
        lg = O.router(x, spec.W, spec.bias)
        oi, ow, om = O.topk(lg, spec.k)
        orc = dict(idx=oi, w=ow, margin=om)
        ok = check_routing(idx, w, orc, spec.k)
        check_buckets(off, perm, oi, spec.E, spec.k, ok)
    finally:
        B.moe_destroy(ctx)


def test_prefill_and_forward_agree(B):
    """moe_prefill and moe_forward on a window of more than 32 tokens run
    the same chunk path (GEMM experts + GEMV experts): equal outputs."""
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
        assert torch.equal(d1, d2)
    finally:
        B.moe_destroy(ctx)


def test_prefill_q2_gemm_and_gemv_experts(B):
    """Q2 experts, 400 tokens over 8 experts: every routed expert is a GEMM
    expert; the same layer with 24 experts and 40 tokens puts most of them
    on the GEMV.  Both against the oracle on every token."""
    for E, N in ((8, 400), (24, 40)):
        spec = LayerSpec(d=256, f=256, E=E, k=2, fmt=I.Q2, seed=9 + E, shared=True)
        ctx = make_ctx(B, spec, 512)
        try:
            load_layer(B, ctx, spec)
            x = I.hidden_np(9, N, spec.d, window=E)
            delta, x_out = run_prefill(B, ctx, spec, x)
            check_rows(spec, x, delta, x_out, np.arange(N))
        finally:
            B.moe_destroy(ctx)


def test_prefill_q2_matches_decode_path_small_windows(B):
    """Q2 experts: a 32-token window (single-launch decode kernel) and the
    same tokens inside a 64-token chunk (GEMM / GEMV experts) agree within
    the output tolerance."""
    spec = LayerSpec(d=256, f=256, E=8, k=2, fmt=I.Q2, seed=9, shared=True)
    ctx = make_ctx(B, spec, 512)
    try:
        load_layer(B, ctx, spec)
        x = to_dev(I.hidden_np(9, 64, spec.d, window=3))
        d1 = torch.empty((64, spec.d), dtype=torch.float32, device="cuda")
        d2 = torch.empty((32, spec.d), dtype=torch.float32, device="cuda")
        B.moe_prefill_delta(ctx, 0, x, 64, d1)
        B.moe_forward_delta(ctx, 0, x[:32], 32, d2)
        B.moe_sync(ctx, 60000)
        assert_close_rms(d1[:32].cpu().numpy(), d2.cpu().numpy(), what="chunk vs decode path")
    finally:
        B.moe_destroy(ctx)


def test_prefill_q2_oracle(B):
    spec = LayerSpec(d=256, f=128, E=16, k=2, fmt=I.Q2, seed=6, shared=True)
    ctx = make_ctx(B, spec, 256)
    try:
        load_layer(B, ctx, spec)
        x = I.hidden_np(6, 200, spec.d, window=5)
        delta, x_out = run_prefill(B, ctx, spec, x)
        check_rows(spec, x, delta, x_out, np.arange(200))
    finally:
        B.moe_destroy(ctx)


# ------------------------------------------------ the 8192-token chunk
@pytest.fixture(scope="module")
def chunk8192(B):
    """The prefill workload: d=2048, f=768, E=512, top-10 + shared, Q4 g32,
    one chunk of 8192 tokens, Zipf(1.1)-biased routing; with the oracle's
    fp64 routing of every token (computed on a thread pool)."""
    spec = LayerSpec(d=2048, f=768, E=512, k=10, fmt=I.Q4, seed=0, shared=True, zipf=True)
    ctx = make_ctx(B, spec, 8192)
    load_layer(B, ctx, spec)
    N = 8192
    x = I.hidden_np(0, N, spec.d, window=4242)
    lg = router_parallel(x, spec.W, spec.bias)
    idx, w, margin = O.topk(lg, spec.k)
    yield ctx, spec, x, dict(idx=idx, w=w, margin=margin)
    B.moe_destroy(ctx)


def _route_outputs(N, k, E):
    return [torch.empty((N, k), dtype=torch.int32, device="cuda"),
            torch.empty((N, k), dtype=torch.float32, device="cuda"),
            torch.empty(E + 1, dtype=torch.int32, device="cuda"),
            torch.empty(N * k, dtype=torch.int32, device="cuda")]


def test_prefill_route_8192_bit_exact(B, chunk8192):
    """The prefill path's own routing (tensor-core router, one warp per token
    top-k, per-expert column scan, scan, scatter) against the oracle on all
    8192 tokens: expert sets and bucket contents bit-exact, weights within
    1e-5, near ties (oracle margin < 1e-5) excluded and counted."""
    ctx, spec, x, orc = chunk8192
    N = x.shape[0]
    out = _route_outputs(N, spec.k, spec.E)
    B.moe_prefill_route(ctx, 0, to_dev(x), N, *out)
    B.moe_sync(ctx, 120000)
    idx, w, off, perm = [t.cpu().numpy() for t in out]
    ok = check_routing(idx, w, orc, spec.k)
    check_buckets(off, perm, orc["idx"], spec.E, spec.k, ok)
    ties = int((~ok).sum())
    print(f"prefill routing, 8192 tokens: near ties {ties}")
    assert ties <= 8


@pytest.mark.parametrize("N", [512, 8192])
def test_moe_route_large_windows_bit_exact(B, chunk8192, N):
    """moe_route on 512 and 8192 tokens (E = 512): the tensor-core router
    path of the multi-launch routing, against the oracle on every token."""
    ctx, spec, x, orc = chunk8192
    out = _route_outputs(N, spec.k, spec.E)
    B.moe_route(ctx, 0, to_dev(x[:N]), N, *out)
    B.moe_sync(ctx, 120000)
    idx, w, off, perm = [t.cpu().numpy() for t in out]
    sub = {key: v[:N] for key, v in orc.items()}
    ok = check_routing(idx, w, sub, spec.k)
    check_buckets(off, perm, sub["idx"], spec.E, spec.k, ok)
    print(f"moe_route N={N}: near ties {int((~ok).sum())}")


def test_prefill_chunk_8192_covering_sample(B, chunk8192):
    """The whole prefill layer at 8192 tokens against the oracle on a
    deterministic sample of tokens that covers every expert's first and last
    128-row GEMM tile (and each expert's first and last row), every tile of
    the three hottest experts, and the shared expert's first and last tiles."""
    ctx, spec, x, orc = chunk8192
    N = x.shape[0]
    delta, x_out = run_prefill(B, ctx, spec, x)
    assert np.isfinite(delta).all()
    rows = np.union1d(covering_sample(orc["idx"], spec.E), [0, 127, 128, N - 129, N - 128, N - 1])
    ok = orc["margin"][rows] >= TIE_MARGIN
    od, ox, _ = oracle_rows(spec, x, rows)
    rel = assert_close_rms(delta[rows][ok], od[ok], what="MoE delta")
    assert_close_residual(x_out[rows][ok], ox[ok])
    print(f"prefill 8192: {rows.size} sampled tokens, delta max-err/RMS {rel:.2e}, "
          f"near ties {int((~ok).sum())}")


def test_prefill_pruned_256_experts(B):
    """A 1024-token chunk of the pruned 256-expert configuration (E a
    multiple of 256: the tensor-core router), Zipf routing; routing and
    buckets on every token, the layer on a covering sample."""
    spec = LayerSpec(d=2048, f=768, E=256, k=10, fmt=I.Q4, seed=0, shared=True, zipf=True)
    ctx = make_ctx(B, spec, 1024)
    try:
        load_layer(B, ctx, spec)
        N = 1024
        x = I.hidden_np(0, N, spec.d, window=2560)
        lg = router_parallel(x, spec.W, spec.bias)
        oi, ow, om = O.topk(lg, spec.k)
        orc = dict(idx=oi, w=ow, margin=om)
        out = _route_outputs(N, spec.k, spec.E)
        B.moe_prefill_route(ctx, 0, to_dev(x), N, *out)
        B.moe_sync(ctx, 60000)
        idx, w, off, perm = [t.cpu().numpy() for t in out]
        ok = check_routing(idx, w, orc, spec.k)
        check_buckets(off, perm, oi, spec.E, spec.k, ok)
        delta, x_out = run_prefill(B, ctx, spec, x)
        rows = covering_sample(oi, spec.E)
        keep = om[rows] >= TIE_MARGIN
        od, ox, _ = oracle_rows(spec, x, rows)
        rel = assert_close_rms(delta[rows][keep], od[keep], what="MoE delta")
        assert_close_residual(x_out[rows][keep], ox[keep])
        print(f"E=256 chunk: {rows.size} sampled, delta max-err/RMS {rel:.2e}, near ties {int((~ok).sum())}")
    finally:
        B.moe_destroy(ctx)


def test_prefill_route_rejects_bad_calls(B):
    spec = LayerSpec(d=256, f=128, E=16, k=2, fmt=I.Q4, seed=5, shared=True)
    ctx = make_ctx(B, spec, 16)  # decode-only context: no prefill buffers
    try:
        load_layer(B, ctx, spec)
        x = to_dev(I.hidden_np(5, 8, spec.d))
        out = _route_outputs(8, spec.k, spec.E)
        with pytest.raises(B.MoeError) as ei:
            B.moe_prefill_route(ctx, 0, x, 8, *out)
        assert ei.value.status == 8  # NOT_SUPPORTED
        with pytest.raises(B.MoeError) as ei:
            B.moe_prefill_route(ctx, 0, x, 0, *out)
        assert ei.value.status == 1
    finally:
        B.moe_destroy(ctx)
