"""Host tier on the GPU: experts' backing copies in pinned host memory, the
HBM slot pool as a cache over them (the engine article "93 token/s on one
8 GB card", section "Expert cache").  Residency only moves where an expert is
read from, so the tiered forward must match the all-HBM context bit for bit;
the copies, hits, misses and the routing trace are checked against the
window's routing."""
import numpy as np
import pytest

from sparse_moe_expert_gemv_b200 import inputs as I
from tests._harness import LayerSpec, assert_close_residual, load_layer

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def B():
    from sparse_moe_expert_gemv_b200 import binding

    return binding

D, F, E, K, L = 256, 128, 64, 4, 3


def _make(B, fmt, tier, n_slots, policy=1, max_tokens=64, zipf=True):
    ctx = B.moe_create(D, F, E, K, fmt)
    if tier:
        B.moe_set_host_tier(ctx, 1, policy, 8.0)
    B.moe_configure(ctx, L, 1, n_slots, max_tokens)
    specs = []
    for layer in range(L):
        spec = LayerSpec(d=D, f=F, E=E, k=K, fmt=fmt, zipf=zipf, layer=layer)
        load_layer(B, ctx, spec, layer=layer)
        specs.append(spec)
    return ctx, specs


def _windows(n, T):
    return [I.hidden_np(0, T, D, window=100 + i) for i in range(n)]


@pytest.mark.parametrize("fmt", [I.Q4, I.Q2])
@pytest.mark.parametrize("policy", [0, 1])
def test_tiered_forward_matches_the_hbm_forward(B, fmt, policy):
    import torch

    # uniform routing: about 14 distinct experts per window, far more over
    # the three layers than the 20 slots hold
    ref, _ = _make(B, fmt, False, 0, zipf=False)
    tier, _ = _make(B, fmt, True, 20, policy=policy, zipf=False)
    try:
        for i, x in enumerate(_windows(12, 4)):
            layer = i % L
            xa = torch.from_numpy(x.view(np.int16).copy()).cuda()
            xb = xa.clone()
            B.moe_forward(ref, layer, xa, 4)
            B.moe_forward_tiered(tier, layer, xb, 4)
            torch.cuda.synchronize()
            assert torch.equal(xa, xb), f"window {i}: tiered output differs"
        B.moe_sync(ref, 60000)
        B.moe_sync(tier, 60000)
        st = B.moe_tier_stats(tier)
        assert st["requests"] == 12
        assert st["misses"] > 0 and st["evictions"] > 0 and st["slots_used"] == 20
        assert st["bytes"] == st["misses"] * B.moe_expert_bytes(D, F, fmt)
    finally:
        B.moe_destroy(ref)
        B.moe_destroy(tier)


def test_tier_counts_follow_the_routing(B, tmp_path):
    """Misses are exactly the window's distinct experts without a slot; a
    window repeated at once hits everywhere; the trace lists the requests."""
    import torch

    ctx, specs = _make(B, I.Q4, True, 40)
    try:
        idx = torch.empty(8 * K, dtype=torch.int32, device="cuda")
        w = torch.empty(8 * K, dtype=torch.float32, device="cuda")
        x = torch.from_numpy(I.hidden_np(0, 8, D, window=7).view(np.int16).copy()).cuda()
        B.moe_route(ctx, 1, x, 8, idx, w, None, None)
        distinct = sorted(set(idx.cpu().numpy().tolist()))
        B.moe_tier_prepare(ctx, 1, idx, 8)
        st = B.moe_tier_stats(ctx)
        assert (st["hits"], st["misses"]) == (0, len(distinct))
        B.moe_tier_prefetch(ctx, 1, idx, 8)      # all resident: nothing to copy
        B.moe_tier_prepare(ctx, 1, idx, 8)
        st = B.moe_tier_stats(ctx)
        assert (st["hits"], st["misses"], st["requests"]) == (2 * len(distinct), len(distinct), 3)
        path = tmp_path / "trace.txt"
        B.moe_tier_dump_trace(ctx, str(path))
        lines = [ln.split() for ln in path.read_text().splitlines() if not ln.startswith("#")]
        assert len(lines) == 3
        for n, ln in enumerate(lines, 1):
            assert list(map(int, ln[:3])) == [n, 1, len(distinct)]
            assert list(map(int, ln[3:])) == distinct
        torch.cuda.synchronize()
    finally:
        B.moe_destroy(ctx)


def test_tiered_forward_against_the_oracle(B):
    """A Zipf-routed window sequence through a pool that holds a fraction of
    the experts, checked against the fp64 oracle."""
    import torch

    ctx, specs = _make(B, I.Q4, True, 20)
    try:
        for i, x in enumerate(_windows(6, 4)):
            layer = (2 * i) % L
            xb = torch.from_numpy(x.view(np.int16).copy()).cuda()
            B.moe_forward_tiered(ctx, layer, xb, 4)
            torch.cuda.synchronize()
            want = specs[layer].oracle(x)["x_out"]
            assert_close_residual(xb.cpu().numpy().view(np.uint16), want, what=f"window {i}")
        B.moe_sync(ctx, 60000)
    finally:
        B.moe_destroy(ctx)


def test_tier_rejects_a_pool_smaller_than_a_window(B):
    import torch

    ctx, _ = _make(B, I.Q4, True, 3)
    try:
        x = torch.from_numpy(I.hidden_np(0, 4, D, window=1).view(np.int16).copy()).cuda()
        with pytest.raises(B.MoeError):
            B.moe_forward_tiered(ctx, 0, x, 4)     # 4 tokens x top-4 need more than 3 slots
        torch.cuda.synchronize()
    finally:
        B.moe_destroy(ctx)


def test_host_tier_call_order(B):
    ctx = B.moe_create(D, F, E, K, I.Q4)
    try:
        with pytest.raises(B.MoeError):
            B.moe_tier_stats(ctx)                  # no host tier
        B.moe_configure(ctx, 1, 0, 8, 16)
        with pytest.raises(B.MoeError):
            B.moe_set_host_tier(ctx, 1, 0, 8.0)    # after configuration
    finally:
        B.moe_destroy(ctx)
