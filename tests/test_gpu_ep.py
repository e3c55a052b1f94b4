"""Expert parallelism on the GPU: the owner-side call on given routing
(moe_experts_given), the two ends of the exchange (moe_ep_dispatch,
moe_ep_combine) and the layer built from them (``ep.py``).

With the same routing, an owner receives exactly the rows the one-GPU
layer groups for each of its experts, so a sharded layer must reproduce
moe_prefill bit for bit: the R ranks are emulated on this one GPU (the
all-to-all done by slicing; no kernel waits on another), and a world of one
runs the real NCCL all-to-all.  Given routing with fewer experts per row,
or the shared expert alone, is checked against the oracle."""
import numpy as np
import pytest
import torch

import oracle as O
from sparse_moe_expert_gemv_b200 import inputs as I
from tests._harness import LayerSpec, assert_close_rms, load_layer

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def B():
    from sparse_moe_expert_gemv_b200 import binding
    return binding


def to_dev(bits):
    return torch.from_numpy(np.ascontiguousarray(bits, np.uint16).view(np.int16)).cuda()


def make_ctx(B, spec, max_tokens, norm=False):
    ctx = B.moe_create(spec.d, spec.f, spec.E, spec.k, spec.fmt)
    B.moe_configure(ctx, 1, 1 if spec.shared else 0, 0, max_tokens)
    if norm:
        B.moe_set_norm(ctx, 0, None, 1e-6)
    return ctx


def load_owned(B, ctx, spec, first, n):
    """Router, shared expert and experts [first, first + n) only."""
    B.moe_set_router(ctx, 0, spec.W, spec.bias)
    if n:
        c, s, m = I.experts_torch(spec.seed, spec.fmt, spec.d, spec.f, spec.layer, first, n, "cuda")
        B.moe_load_experts(ctx, 0, first, n, c, s, m)
    if spec.shared:
        c, s, m = spec.shared_expert()
        B.moe_load_shared(ctx, 0, c, s, m)
    torch.cuda.synchronize()


SMALL = dict(d=512, f=256, E=64, k=4)
FULL = dict(d=2048, f=768, E=512, k=10)


@pytest.mark.parametrize("fmt", [I.Q4, I.Q2])
@pytest.mark.parametrize("shape,N", [(SMALL, 700), (FULL, 1500)])
def test_given_routing_reproduces_prefill(B, fmt, shape, N):
    """moe_prefill_route's routing fed back through moe_experts_given (all k
    experts and the shared one) gives moe_prefill_delta's output exactly."""
    spec = LayerSpec(fmt=fmt, zipf=True, **shape)
    ctx = make_ctx(B, spec, N)
    try:
        load_layer(B, ctx, spec)
        x = to_dev(I.hidden_np(1, N, spec.d, window=2))
        want = torch.empty((N, spec.d), dtype=torch.float32, device="cuda")
        B.moe_prefill_delta(ctx, 0, x, N, want)
        idx = torch.empty((N, spec.k), dtype=torch.int32, device="cuda")
        w = torch.empty((N, spec.k), dtype=torch.float32, device="cuda")
        B.moe_prefill_route(ctx, 0, x, N, idx, w)
        got = torch.empty_like(want)
        B.moe_experts_given(ctx, 0, x, N, spec.k, idx, w, 1, got)
        B.moe_sync(ctx, 120000)
        assert torch.equal(got, want)
    finally:
        B.moe_destroy(ctx)


@pytest.mark.parametrize("kk,shared", [(2, True), (1, False), (0, True), (4, False)])
def test_given_routing_against_the_oracle(B, kk, shared):
    """Arbitrary given routing (seeded ids, distinct per row; seeded
    weights): delta = sum_j w_j y_j (+ y_shared) against the fp64 oracle's
    experts, on every row."""
    spec = LayerSpec(fmt=I.Q4, zipf=False, shared=True, **SMALL)
    N = 300
    ctx = make_ctx(B, spec, N)
    try:
        load_layer(B, ctx, spec)
        xb = I.hidden_np(2, N, spec.d, window=4)
        rng = np.random.default_rng(7)
        ids = np.stack([rng.choice(spec.E, size=kk, replace=False) for _ in range(N)]).astype(np.int32) \
            if kk else np.zeros((N, 0), np.int32)
        wv = rng.uniform(0.05, 1.0, size=(N, kk)).astype(np.float32)
        # a hot expert (3, in half the rows) so that the grouped GEMM runs as
        # well as the GEMV
        for t in range(N // 2 if kk else 0):
            if 3 not in ids[t]:
                ids[t, 0] = 3
        delta = torch.empty((N, spec.d), dtype=torch.float32, device="cuda")
        B.moe_experts_given(ctx, 0, to_dev(xb), N, kk, torch.from_numpy(ids).cuda(),
                            torch.from_numpy(wv).cuda(), int(shared), delta)
        B.moe_sync(ctx, 120000)
        want = np.zeros((N, spec.d), np.float64)
        for e in sorted(set(ids.reshape(-1).tolist())):
            rows, js = np.nonzero(ids == e)
            Wg, Wu, Wd = O.dequant_expert(spec.fmt, spec.d, spec.f, *spec.expert(e))
            y = O.expert(Wg, Wu, Wd, np.ascontiguousarray(xb[rows]))
            np.add.at(want, rows, wv[rows, js][:, None].astype(np.float64) * y)
        if shared:
            Wg, Wu, Wd = O.dequant_expert(spec.fmt, spec.d, spec.f, *spec.shared_expert())
            want += O.expert(Wg, Wu, Wd, xb)
        assert_close_rms(delta.cpu().numpy(), want, what=f"given routing kk={kk}")
    finally:
        B.moe_destroy(ctx)


def test_given_routing_is_checked(B):
    spec = LayerSpec(fmt=I.Q4, zipf=False, shared=False, **SMALL)
    N = 40
    ctx = make_ctx(B, spec, N)
    try:
        load_owned(B, ctx, spec, 0, 32)          # experts 32..63 not loaded
        x = to_dev(I.hidden_np(0, N, spec.d))
        w = torch.ones((N, 2), dtype=torch.float32, device="cuda")
        out = torch.empty((N, spec.d), dtype=torch.float32, device="cuda")
        base = np.tile(np.array([[1, 2]], np.int32), (N, 1))

        def call(ids, kk=2, shared=0):
            B.moe_experts_given(ctx, 0, x, N, kk, torch.from_numpy(ids).cuda(), w, shared, out)

        call(base)                               # valid
        for bad, status in [(64, B.MOE_ERR_INVALID_ARG), (-1, B.MOE_ERR_INVALID_ARG),
                            (40, B.MOE_ERR_STATE)]:
            ids = base.copy()
            ids[N - 1, 1] = bad
            with pytest.raises(B.MoeError) as ei:
                call(ids)
            assert ei.value.status == status
        dup = base.copy()
        dup[5, 1] = dup[5, 0]
        with pytest.raises(B.MoeError):
            call(dup)                            # an expert twice in one row
        with pytest.raises(B.MoeError):
            call(base, kk=5)                     # kk > k
        with pytest.raises(B.MoeError):
            call(base[:, :0].copy(), kk=0, shared=1)   # no shared expert configured
        B.moe_sync(ctx, 60000)
    finally:
        B.moe_destroy(ctx)


@pytest.mark.parametrize("R", [1, 8])
def test_dispatch_layout(B, R):
    """Send order, positions and counts against a stable sort by owner;
    every sent row is its token's router-input row."""
    spec = LayerSpec(fmt=I.Q4, zipf=True, shared=False, **FULL)
    N = 1000
    ctx = make_ctx(B, spec, 64)
    try:
        xb = I.hidden_np(4, N, spec.d, window=1)
        ids = I.routing_idx_np(0, N, spec.k, spec.E, window=3)
        h = to_dev(xb)
        send_h = torch.empty((N * spec.k, spec.d), dtype=torch.int16, device="cuda")
        send_e = torch.empty(N * spec.k, dtype=torch.int32, device="cuda")
        row_of = torch.empty(N * spec.k, dtype=torch.int32, device="cuda")
        counts = B.moe_ep_dispatch(ctx, torch.from_numpy(ids).cuda(), N, R, h, send_h, send_e, row_of)
        per = spec.E // R
        flat = ids.reshape(-1)
        order = np.concatenate([np.nonzero(flat // per == r)[0] for r in range(R)])
        assert counts == [int((flat // per == r).sum()) for r in range(R)]
        assert np.array_equal(send_e.cpu().numpy(), flat[order])
        ro = row_of.cpu().numpy()
        assert np.array_equal(ro[order], np.arange(order.size))
        sh = send_h.cpu().numpy().view(np.uint16)
        assert np.array_equal(sh, xb[order // spec.k])
        B.moe_sync(ctx, 60000)
    finally:
        B.moe_destroy(ctx)


def test_dispatch_flags_an_invalid_id(B):
    spec = LayerSpec(fmt=I.Q4, zipf=False, shared=False, **SMALL)
    N = 50
    ctx = make_ctx(B, spec, 64)
    try:
        ids = I.routing_idx_np(0, N, spec.k, spec.E, window=0)
        ids[7, 2] = spec.E
        h = to_dev(I.hidden_np(0, N, spec.d))
        send_h = torch.empty((N * spec.k, spec.d), dtype=torch.int16, device="cuda")
        send_e = torch.empty(N * spec.k, dtype=torch.int32, device="cuda")
        row_of = torch.empty(N * spec.k, dtype=torch.int32, device="cuda")
        counts = B.moe_ep_dispatch(ctx, torch.from_numpy(ids).cuda(), N, 2, h, send_h, send_e, row_of)
        assert sum(counts) == N * spec.k - 1
        assert row_of.cpu().numpy()[7 * spec.k + 2] == -1
        with pytest.raises(B.MoeError) as ei:
            B.moe_sync(ctx, 60000)
        assert ei.value.status == B.MOE_ERR_DEVICE
    finally:
        B.moe_destroy(ctx)


def _emulated_vs_one_gpu(B, spec, sizes, R, norm):
    from sparse_moe_expert_gemv_b200.ep import DeviceOps, emulate

    Nt = sum(sizes)
    ref = make_ctx(B, spec, Nt, norm)
    ranks = []
    try:
        load_layer(B, ref, spec)
        per = spec.E // R
        for r in range(R):
            ctx = make_ctx(B, spec, Nt * spec.k, norm)
            load_owned(B, ctx, spec, r * per, per)
            ranks.append(ctx)
        x_all = to_dev(I.hidden_np(5, Nt, spec.d, window=9))
        # one routing of the whole batch, as the one-GPU layer computes it
        h_all = torch.empty_like(x_all)
        B.moe_rmsnorm(ref, 0, x_all, Nt, h_all)
        idx = torch.empty((Nt, spec.k), dtype=torch.int32, device="cuda")
        w = torch.empty((Nt, spec.k), dtype=torch.float32, device="cuda")
        B.moe_prefill_route(ref, 0, h_all, Nt, idx, w)
        want = x_all.clone()
        B.moe_prefill(ref, 0, want, Nt)
        ops = [DeviceOps(B, c, d=spec.d, k=spec.k, E=spec.E, max_tokens=Nt * spec.k,
                         has_shared=spec.shared) for c in ranks]
        bounds = np.cumsum([0] + sizes)
        sl = [slice(int(bounds[r]), int(bounds[r + 1])) for r in range(R)]
        xs = [x_all[s].clone() for s in sl]
        received = emulate(ops, 0, xs, [h_all[s] for s in sl], sizes,
                           [(idx[s].contiguous(), w[s].contiguous()) for s in sl])
        torch.cuda.synchronize()
        for c in [ref] + ranks:
            B.moe_sync(c, 120000)
        for r in range(R):
            e = received[r].cpu().numpy()
            assert ((e // per) == r).all(), f"rank {r} received another rank's expert"
        got = torch.cat(xs)
        assert torch.equal(got, want), f"R={R}: {(got != want).sum().item()} elements differ"
    finally:
        for c in [ref] + ranks:
            B.moe_destroy(c)


@pytest.mark.parametrize("R", [1, 2, 4])
@pytest.mark.parametrize("fmt", [I.Q4, I.Q2])
def test_emulated_ranks_match_one_gpu_small(B, R, fmt):
    spec = LayerSpec(fmt=fmt, zipf=True, **SMALL)
    _emulated_vs_one_gpu(B, spec, [300, 77, 250, 173][:R] if R > 1 else [800], R, norm=True)


def test_emulated_rank_without_tokens(B):
    """Three ranks, the middle one with no tokens of its own: it still
    computes its experts' rows for the others."""
    spec = LayerSpec(fmt=I.Q4, zipf=True, d=512, f=256, E=60, k=4)
    _emulated_vs_one_gpu(B, spec, [400, 0, 200], 3, norm=False)


def test_emulated_ranks_match_one_gpu_full_shape(B):
    """d=2048 f=768 E=512 top-10 + shared, Zipf routing, four ranks of
    uneven size."""
    spec = LayerSpec(fmt=I.Q4, zipf=True, **FULL)
    _emulated_vs_one_gpu(B, spec, [512, 300, 700, 536], 4, norm=False)


def test_world_of_one_over_nccl(B):
    """The distributed layer (ExpertParallelMoE with NCCL's all-to-all) in a
    process group of one: its own routing, dispatch, exchange, experts and
    combine give moe_prefill's result exactly."""
    import os
    import socket

    import torch.distributed as dist
    from sparse_moe_expert_gemv_b200.ep import DeviceOps, Exchange, ExpertParallelMoE

    spec = LayerSpec(fmt=I.Q4, zipf=True, **FULL)
    N = 1024
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0, world_size=1)
    ref = make_ctx(B, spec, N, norm=True)
    ctx = make_ctx(B, spec, N * spec.k, norm=True)
    try:
        load_layer(B, ref, spec)
        load_owned(B, ctx, spec, 0, spec.E)
        x = to_dev(I.hidden_np(6, N, spec.d, window=2))
        want = x.clone()
        B.moe_prefill(ref, 0, want, N)
        layer = ExpertParallelMoE(DeviceOps(B, ctx, d=spec.d, k=spec.k, E=spec.E,
                                            max_tokens=N * spec.k, has_shared=True), Exchange())
        layer.forward(0, x, N)
        torch.cuda.synchronize()
        B.moe_sync(ref, 120000)
        B.moe_sync(ctx, 120000)
        assert torch.equal(x, want)
    finally:
        dist.destroy_process_group()
        B.moe_destroy(ref)
        B.moe_destroy(ctx)


@pytest.mark.parametrize("with_gamma", [False, True])
def test_rmsnorm_call_against_the_oracle(B, with_gamma):
    """moe_rmsnorm (the expert-parallel layer's router input) against the
    oracle's RMSNorm: fp32 inside against fp64, one bf16 rounding each, so
    equal or one bf16 ulp apart; and a copy of x on a layer without a norm."""
    spec = LayerSpec(fmt=I.Q4, zipf=False, shared=False, **SMALL)
    N = 300
    ctx = make_ctx(B, spec, 64)
    try:
        gamma = I.router_np(9, 1, spec.d, 0)[0] * 50.0 + 1.0 if with_gamma else None
        B.moe_set_norm(ctx, 0, gamma, 1e-5)
        xb = I.hidden_np(8, N, spec.d, window=3)
        h = torch.empty((N, spec.d), dtype=torch.int16, device="cuda")
        B.moe_rmsnorm(ctx, 0, to_dev(xb), N, h)
        torch.cuda.synchronize()
        got = h.cpu().numpy().view(np.uint16).astype(np.int64)
        want = O.rmsnorm(xb, gamma, 1e-5).astype(np.int64)
        assert np.array_equal(got >> 15, want >> 15)
        assert np.abs(got - want).max() <= 1
        assert (got == want).mean() >= 0.999
        B.moe_sync(ctx, 60000)
    finally:
        B.moe_destroy(ctx)
    ctx = make_ctx(B, spec, 64)   # no norm configured: h is x
    try:
        B.moe_set_router(ctx, 0, spec.W, spec.bias)
        x = to_dev(I.hidden_np(8, 40, spec.d))
        h = torch.empty_like(x)
        B.moe_rmsnorm(ctx, 0, x, 40, h)
        torch.cuda.synchronize()
        assert torch.equal(h, x)
    finally:
        B.moe_destroy(ctx)


@pytest.mark.parametrize("fmt", [I.Q4, I.Q2])
def test_one_rank_chain_into_delta(B, fmt):
    """The expert-parallel steps by hand at one rank, ending in
    moe_ep_combine's delta form: route, dispatch, the owner's experts (one
    expert per row, fp16 outputs), the shared expert, combine; equal to
    moe_prefill_delta bit for bit."""
    spec = LayerSpec(fmt=fmt, zipf=True, **SMALL)
    N = 600
    ref = make_ctx(B, spec, N)
    ctx = make_ctx(B, spec, N * spec.k)
    try:
        load_layer(B, ref, spec)
        load_owned(B, ctx, spec, 0, spec.E)
        x = to_dev(I.hidden_np(3, N, spec.d, window=6))
        want = torch.empty((N, spec.d), dtype=torch.float32, device="cuda")
        B.moe_prefill_delta(ref, 0, x, N, want)
        idx = torch.empty((N, spec.k), dtype=torch.int32, device="cuda")
        w = torch.empty((N, spec.k), dtype=torch.float32, device="cuda")
        B.moe_prefill_route(ctx, 0, x, N, idx, w)
        P = N * spec.k
        send_h = torch.empty((P, spec.d), dtype=torch.int16, device="cuda")
        send_e = torch.empty(P, dtype=torch.int32, device="cuda")
        row_of = torch.empty(P, dtype=torch.int32, device="cuda")
        counts = B.moe_ep_dispatch(ctx, idx, N, 1, x, send_h, send_e, row_of)
        assert counts == [P]
        y = torch.empty((P, spec.d), dtype=torch.float16, device="cuda")
        B.moe_experts_rows(ctx, 0, send_h, P, send_e, y)
        ysh = torch.empty((N, spec.d), dtype=torch.float32, device="cuda")
        B.moe_experts_given(ctx, 0, x, N, 0, None, None, 1, ysh)
        got = torch.empty_like(want)
        B.moe_ep_combine(ctx, N, w, y, row_of, ysh, delta=got)
        with pytest.raises(B.MoeError):
            B.moe_ep_combine(ctx, N, w, y, row_of, ysh)            # neither x nor delta
        with pytest.raises(B.MoeError):
            B.moe_ep_combine(ctx, N, w, y, row_of, ysh, x=x, delta=got)   # both
        torch.cuda.synchronize()
        B.moe_sync(ref, 60000)
        B.moe_sync(ctx, 60000)
        assert torch.equal(got, want)
    finally:
        B.moe_destroy(ref)
        B.moe_destroy(ctx)


@pytest.mark.parametrize("fmt,N", [(I.Q2, 256), (I.Q4, 1500)])
def test_chunk_path_under_graph_capture(B, fmt, N):
    """The chunk path forks its GEMV experts to a second stream and joins
    them before the combine; captured in a CUDA graph and replayed, it must
    give the eager result bit for bit."""
    spec = LayerSpec(fmt=fmt, zipf=True, **FULL)
    ctx = make_ctx(B, spec, N)
    try:
        load_layer(B, ctx, spec)
        x = to_dev(I.hidden_np(2, N, spec.d, window=8))
        eager = torch.empty((N, spec.d), dtype=torch.float32, device="cuda")
        B.moe_prefill_delta(ctx, 0, x, N, eager)
        torch.cuda.synchronize()
        out = torch.zeros_like(eager)
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            B.moe_prefill_delta(ctx, 0, x, N, out, stream=s)   # warm-up on the capture stream
        torch.cuda.current_stream().wait_stream(s)
        torch.cuda.synchronize()
        out.zero_()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            B.moe_prefill_delta(ctx, 0, x, N, out)
        for _ in range(2):
            out.zero_()
            g.replay()
            torch.cuda.synchronize()
            assert torch.equal(out, eager)
        B.moe_sync(ctx, 60000)
    finally:
        B.moe_destroy(ctx)
