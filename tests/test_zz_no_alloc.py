"""moe_route_static: routing for callers that cannot allocate device memory.

Code that runs under a fixed device-memory budget (its own pool took every
byte up front) or a plugin that only receives raw device pointers cannot
call cudaMalloc, so it cannot create a context.  moe_route_static routes a
window with the router weights passed in as a device pointer and keeps its
scratch in a static device array.  This test checks, on two calls in a row,
that it returns what the context-based moe_route returns for the same input.
It runs last so that a failure here leaves the rest of the suite reported.
"""
import numpy as np
import pytest
import torch

import oracle as O
from sparse_moe_expert_gemv_b200 import inputs as I
from tests._harness import check_buckets, check_routing

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def B():
    from sparse_moe_expert_gemv_b200 import binding
    return binding


@pytest.mark.parametrize("zipf", [False, True])
def test_route_static_matches_moe_route(B, zipf):
    d, f, E, k, T = 2048, 768, 512, 10, 4
    W = I.router_np(0, E, d)
    bias = I.zipf_bias_np(0, E)[0] if zipf else None
    ctx = B.moe_create(d, f, E, k, I.Q4)
    try:
        B.moe_configure(ctx, 1, 0, 0, 32)
        B.moe_set_router(ctx, 0, W, bias)
        Wd = torch.from_numpy(W).cuda()
        bd = torch.from_numpy(bias).cuda() if bias is not None else None
        for window in (0, 1):  # two calls in a row share the static scratch
            x = torch.from_numpy(I.hidden_np(0, T, d, window=window).view(np.int16)).cuda()
            ref = [torch.empty((T, k), dtype=torch.int32, device="cuda"),
                   torch.empty((T, k), dtype=torch.float32, device="cuda"),
                   torch.empty(E + 1, dtype=torch.int32, device="cuda"),
                   torch.empty(T * k, dtype=torch.int32, device="cuda")]
            got = [torch.full_like(t, -7) for t in ref]
            B.moe_route(ctx, 0, x, T, *ref)
            B.moe_route_static(x, T, d, E, k, Wd, bd, *got)
            torch.cuda.synchronize()
            assert torch.equal(got[0], ref[0])
            assert torch.allclose(got[1], ref[1], rtol=0, atol=1e-5)
            assert torch.equal(got[2], ref[2])
            assert torch.equal(got[3], ref[3])
            assert B.moe_route_static_status() == 0
    finally:
        B.moe_destroy(ctx)


@pytest.mark.parametrize("T,d,E,k,zipf", [
    (1, 128, 16, 1, False),      # one token, smallest shapes
    (9, 2048, 1024, 32, False),  # eight warps per CTA, 32 logits per lane, k at its limit
    (32, 2048, 512, 10, True),   # the largest window, Zipf-biased
    (32, 128, 1024, 1, True),
    (9, 128, 16, 16, False),     # k = E
])
def test_route_static_matches_oracle(B, T, d, E, k, zipf):
    """Across the shapes the entry point accepts, its expert sets and
    bucket contents equal the oracle's bit for bit and its weights are
    within 1e-5 (tokens whose oracle k-th and (k+1)-th logits differ by less
    than 1e-5 are excluded and counted)."""
    seed = 30 + T + E
    W = I.router_np(seed, E, d)
    bias = I.zipf_bias_np(seed, E)[0] if zipf else None
    x = I.hidden_np(seed, T, d, window=E)
    out = [torch.full((T, k), -7, dtype=torch.int32, device="cuda"),
           torch.zeros((T, k), dtype=torch.float32, device="cuda"),
           torch.zeros(E + 1, dtype=torch.int32, device="cuda"),
           torch.zeros(T * k, dtype=torch.int32, device="cuda")]
    B.moe_route_static(torch.from_numpy(x.view(np.int16)).cuda(), T, d, E, k,
                       torch.from_numpy(W).cuda(),
                       None if bias is None else torch.from_numpy(bias).cuda(), *out)
    assert B.moe_route_static_status() == 0
    idx, w, off, perm = [t.cpu().numpy() for t in out]
    oi, ow, om = O.topk(O.router(x, W, bias), k)
    ok = check_routing(idx, w, dict(idx=oi, w=ow, margin=om), k)
    check_buckets(off, perm, oi, E, k, ok)
    print(f"T={T} d={d} E={E} k={k}: near ties {int((~ok).sum())}")


def test_route_static_rejects_sizes_beyond_its_scratch(B):
    x = torch.zeros((33, 2048), dtype=torch.int16, device="cuda")
    W = torch.zeros((512, 2048), dtype=torch.float32, device="cuda")
    out = [torch.empty((33, 10), dtype=torch.int32, device="cuda"),
           torch.empty((33, 10), dtype=torch.float32, device="cuda"),
           torch.empty(513, dtype=torch.int32, device="cuda"),
           torch.empty(330, dtype=torch.int32, device="cuda")]
    with pytest.raises(B.MoeError) as ei:
        B.moe_route_static(x, 33, 2048, 512, 10, W, None, *out)  # T > 32
    assert ei.value.status == 1
    with pytest.raises(B.MoeError) as ei:
        B.moe_route_static(x, 4, 4096, 512, 10, W, None, *out)  # d > 2048
    assert ei.value.status == 1
