"""GPU parity: the CUDA library (through the C ABI) against the CPU oracle on
the same seeded inputs.

Bars: expert-id sets and bucket contents bit-exact (tokens whose oracle
k-th/(k+1)-th fp64 logit gap is < 1e-5 are excluded and counted); routing
weights within 1e-5; MoE outputs within max-abs error <= 2e-2 * RMS.
"""
from concurrent.futures import ThreadPoolExecutor

import numpy as np
import pytest
import torch

import oracle as O
from sparse_moe_expert_gemv_b200 import inputs as I
from tests._harness import (TIE_MARGIN, LayerSpec, assert_close_residual, assert_close_rms,
                            check_buckets, check_routing, load_layer, oracle_threads)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def B():
    from sparse_moe_expert_gemv_b200 import binding
    return binding


def make_ctx(B, spec, *, max_tokens, L=1, n_slots=0):
    ctx = B.moe_create(spec.d, spec.f, spec.E, spec.k, spec.fmt)
    B.moe_configure(ctx, L, 1 if spec.shared else 0, n_slots, max_tokens)
    return ctx


def to_dev(bits):
    return torch.from_numpy(np.ascontiguousarray(bits, np.uint16).view(np.int16)).cuda()


def to_bits(t):
    return t.cpu().numpy().view(np.uint16)


def run(B, ctx, spec, x_bits, layer=0):
    T, d, k, E = x_bits.shape[0], spec.d, spec.k, spec.E
    x = to_dev(x_bits)
    idx = torch.empty((T, k), dtype=torch.int32, device="cuda")
    w = torch.empty((T, k), dtype=torch.float32, device="cuda")
    off = torch.empty(E + 1, dtype=torch.int32, device="cuda")
    perm = torch.empty(T * k, dtype=torch.int32, device="cuda")
    B.moe_route(ctx, layer, x, T, idx, w, off, perm)
    delta = torch.empty((T, d), dtype=torch.float32, device="cuda")
    B.moe_forward_delta(ctx, layer, x, T, delta)
    x2 = x.clone()
    B.moe_forward(ctx, layer, x2, T)
    B.moe_sync(ctx, 120000)
    return dict(idx=idx.cpu().numpy(), w=w.cpu().numpy(), off=off.cpu().numpy(),
                perm=perm.cpu().numpy(), delta=delta.cpu().numpy(), x_out=to_bits(x2))


def check(out, orc, spec, sample=None):
    """Routing on all tokens; outputs on `sample` rows (oracle computed on those)."""
    ok = check_routing(out["idx"], out["w"], orc["route"], spec.k)
    check_buckets(out["off"], out["perm"], orc["route"]["idx"], spec.E, spec.k, ok)
    rows = np.arange(out["delta"].shape[0]) if sample is None else sample
    keep = ok[rows]
    got_d = out["delta"][rows][keep]
    want_d = orc["out"]["delta"][keep]
    rel = assert_close_rms(got_d, want_d, what="MoE delta")
    assert_close_residual(out["x_out"][rows][keep], orc["out"]["x_out"][keep])
    return rel, int((~ok).sum())


def oracle_for(spec, x_bits, sample=None):
    """Routing (fp64) of every token; the full layer on the sampled rows."""
    lg = O.router(x_bits, spec.W, spec.bias)
    idx, w, margin = O.topk(lg, spec.k)
    rows = np.arange(x_bits.shape[0]) if sample is None else sample
    out = spec.oracle(x_bits[rows])
    return dict(route=dict(idx=idx, w=w, margin=margin), out=out)


# ------------------------------------------------------------- config 1
def test_tiny_layer_seed0(B):
    """d=256, f=128, E=16, top-2, T=4, Q4 g32, no shared expert, seed 0."""
    spec = LayerSpec(d=256, f=128, E=16, k=2, fmt=I.Q4, seed=0, shared=False)
    ctx = make_ctx(B, spec, max_tokens=64)
    try:
        load_layer(B, ctx, spec)
        x = I.hidden_np(0, 4, 256)
        out = run(B, ctx, spec, x)
        check(out, oracle_for(spec, x), spec)
    finally:
        B.moe_destroy(ctx)


@pytest.mark.parametrize("fmt", [I.Q4, I.Q2])
def test_tiny_layer_oracle_quantised_weights(B, fmt):
    """The tiny workload exactly as stated: expert matrices drawn from
    N(0, 0.02) and encoded by the oracle's quantiser (Q4 symmetric g32 fp16
    scale; the same shape in Q2 asymmetric g64), d=256, f=128, E=16, top-2,
    T=4, seed 0, loaded through moe_load_experts from host memory."""
    spec = LayerSpec(d=256, f=128, E=16, k=2, fmt=fmt, seed=0, shared=False, weights="quantised")
    ctx = make_ctx(B, spec, max_tokens=64)
    try:
        load_layer(B, ctx, spec)
        x = I.hidden_np(0, 4, 256)
        out = run(B, ctx, spec, x)
        rel, _ = check(out, oracle_for(spec, x), spec)
        print(f"fmt {fmt}: delta max-err/RMS {rel:.2e}")
    finally:
        B.moe_destroy(ctx)


def test_decode_window_oracle_quantised_weights(B):
    """One decode window (d=2048, f=768, E=512, top-10 + shared, Q4, T=4)
    whose selected experts and shared expert are N(0, 0.02) matrices encoded
    by the oracle's quantiser.  Only those experts reach the output, so the
    others keep the generator's codes."""
    d, f, E, k = 2048, 768, 512, 10
    x = I.hidden_np(0, 4, d, window=11)
    W = I.router_np(0, E, d)
    need, _, _ = O.topk(O.router(x, W), k)
    need = set(need.reshape(-1).tolist()) | {I.SHARED_INDEX}
    spec = LayerSpec(d=d, f=f, E=E, k=k, fmt=I.Q4, seed=0, shared=True, weights="quantised",
                     quantise=need)
    with ThreadPoolExecutor(oracle_threads()) as ex:  # encode them on the host cores
        list(ex.map(spec.expert, sorted(need - {I.SHARED_INDEX})))
    spec.shared_expert()
    ctx = make_ctx(B, spec, max_tokens=64)
    try:
        load_layer(B, ctx, spec)
        out = run(B, ctx, spec, x)
        rel, ties = check(out, oracle_for(spec, x), spec)
        print(f"quantised window: delta max-err/RMS {rel:.2e}, near ties {ties}")
    finally:
        B.moe_destroy(ctx)


@pytest.mark.parametrize("fmt", [I.Q4, I.Q2])
@pytest.mark.parametrize("T", [5, 37])
def test_every_code_value(B, fmt, T):
    """Experts whose code bytes are uniform: all 16 Q4 nibbles (level -8
    included) and all four Q2 codes occur, in every position of the
    fragment layout.  T = 5 runs the single-launch kernel, T = 37 the
    multi-launch path."""
    spec = LayerSpec(d=256, f=256, E=16, k=4, fmt=fmt, seed=13, shared=True, weights="uniform")
    ctx = make_ctx(B, spec, max_tokens=64)
    try:
        load_layer(B, ctx, spec)
        codes = spec.expert(0)[0]
        if fmt == I.Q4:
            vals = np.concatenate([codes & 0xF, codes >> 4])
            assert set(np.unique(vals).tolist()) == set(range(16))
        else:
            vals = np.concatenate([(codes >> (2 * i)) & 3 for i in range(4)])
            assert set(np.unique(vals).tolist()) == set(range(4))
        x = I.hidden_np(13, T, 256, window=T)
        out = run(B, ctx, spec, x)
        rel, _ = check(out, oracle_for(spec, x), spec)
        print(f"fmt {fmt} T={T}: delta max-err/RMS {rel:.2e}")
    finally:
        B.moe_destroy(ctx)


@pytest.mark.parametrize("fmt", [I.Q4, I.Q2])
def test_every_code_value_prefill_gemm(B, fmt):
    """The same uniform codes through the grouped tcgen05 GEMM (its own
    fp16 dequantisation of every Q4 nibble and every Q2 code)."""
    spec = LayerSpec(d=256, f=256, E=16, k=4, fmt=fmt, seed=14, shared=True, weights="uniform")
    ctx = make_ctx(B, spec, max_tokens=512)
    try:
        load_layer(B, ctx, spec)
        N = 300
        x = I.hidden_np(14, N, 256, window=1)
        xd = to_dev(x)
        delta = torch.empty((N, 256), dtype=torch.float32, device="cuda")
        B.moe_prefill_delta(ctx, 0, xd, N, delta)
        B.moe_sync(ctx, 60000)
        orc = spec.oracle(x)
        ok = orc["margin"] >= TIE_MARGIN
        assert_close_rms(delta.cpu().numpy()[ok], orc["delta"][ok], what="MoE delta")
    finally:
        B.moe_destroy(ctx)


@pytest.mark.parametrize("fmt", [I.Q4, I.Q2])
@pytest.mark.parametrize("shared", [False, True])
@pytest.mark.parametrize("T", [1, 5, 13, 37])
def test_small_layer_ragged(B, fmt, shared, T):
    """E = 40 (not a multiple of 32), k = 3; T ragged against the 8-token
    mma columns and the 16-token jobs."""
    spec = LayerSpec(d=256, f=256, E=40, k=3, fmt=fmt, seed=7, shared=shared)
    ctx = make_ctx(B, spec, max_tokens=64)
    try:
        load_layer(B, ctx, spec)
        x = I.hidden_np(7, T, 256, window=T)
        out = run(B, ctx, spec, x)
        check(out, oracle_for(spec, x), spec)
    finally:
        B.moe_destroy(ctx)


@pytest.mark.parametrize("fmt", [I.Q4, I.Q2])
@pytest.mark.parametrize("T", [12, 40])
def test_multi_launch_path_d_not_multiple_of_256(B, fmt, T):
    """d = 128 (not a multiple of 256): windows of more than 32 tokens take
    the multi-launch routing and GEMV kernels, since the grouped GEMM's down
    items are 256 features wide."""
    spec = LayerSpec(d=128, f=256, E=24, k=3, fmt=fmt, seed=17, shared=True)
    ctx = make_ctx(B, spec, max_tokens=64)
    try:
        load_layer(B, ctx, spec)
        x = I.hidden_np(17, T, 128, window=T)
        out = run(B, ctx, spec, x)
        check(out, oracle_for(spec, x), spec)
    finally:
        B.moe_destroy(ctx)


# ------------------------------------------------------------- config 2
@pytest.fixture(scope="module")
def decode_q4(B):
    spec = LayerSpec(d=2048, f=768, E=512, k=10, fmt=I.Q4, seed=0, shared=True)
    ctx = make_ctx(B, spec, max_tokens=64)
    load_layer(B, ctx, spec)
    yield ctx, spec
    B.moe_destroy(ctx)


@pytest.mark.parametrize("window", [0, 1, 2])
def test_decode_layer_q4_T4(B, decode_q4, window):
    """d=2048, f=768, E=512, top-10 + shared, Q4 g32, T=4, uniform routing."""
    ctx, spec = decode_q4
    x = I.hidden_np(0, 4, 2048, window=window)
    out = run(B, ctx, spec, x)
    rel, ties = check(out, oracle_for(spec, x), spec)
    print(f"window {window}: delta max-err/RMS {rel:.2e}, near ties {ties}")


def test_decode_q4_full_max_tokens(B, decode_q4):
    """T = max_tokens (64), outputs checked on a sample of rows."""
    ctx, spec = decode_q4
    x = I.hidden_np(0, 64, 2048, window=99)
    out = run(B, ctx, spec, x)
    sample = np.array([0, 1, 17, 31, 32, 50, 63])
    check(out, oracle_for(spec, x, sample), spec, sample)


@pytest.mark.parametrize("T", [16, 32])
def test_decode_q4_wide_windows(B, decode_q4, T):
    """Windows of 16 and 32 tokens: the 32-token window no longer fits the
    single-launch kernel's staging area next to the weight rings, so each
    CTA re-stages only its own jobs' token rows after routing."""
    ctx, spec = decode_q4
    x = I.hidden_np(0, T, 2048, window=300 + T)
    out = run(B, ctx, spec, x)
    sample = np.array([0, T // 2, T - 1])
    rel, ties = check(out, oracle_for(spec, x, sample), spec, sample)
    print(f"T={T}: delta max-err/RMS {rel:.2e}, near ties {ties}")


def test_deterministic(B, decode_q4):
    ctx, spec = decode_q4
    x = I.hidden_np(0, 4, 2048, window=5)
    a = run(B, ctx, spec, x)
    b = run(B, ctx, spec, x)
    for key in a:
        assert np.array_equal(a[key], b[key]), key


# ------------------------------------------------------------- config 3
@pytest.fixture(scope="module")
def decode_q2_zipf(B):
    spec = LayerSpec(d=2048, f=768, E=512, k=10, fmt=I.Q2, seed=0, shared=True, zipf=True)
    ctx = make_ctx(B, spec, max_tokens=320)
    load_layer(B, ctx, spec)
    yield ctx, spec
    B.moe_destroy(ctx)


@pytest.mark.parametrize("T", [1, 2, 3, 4, 5])
def test_decode_q2_zipf_64_sequences(B, decode_q2_zipf, T):
    """Q2 g64 asym, Zipf(1.1)-biased routing, window T, 64 sequences in one
    call (N = 64 T tokens).  Routing checked on every token, outputs on 12
    sampled tokens."""
    ctx, spec = decode_q2_zipf
    N = 64 * T
    x = I.hidden_np(0, N, 2048, window=1000 + T)
    out = run(B, ctx, spec, x)
    rng = np.random.default_rng(T)
    sample = np.sort(rng.choice(N, size=min(12, N), replace=False))
    rel, ties = check(out, oracle_for(spec, x, sample), spec, sample)
    print(f"T={T}: delta max-err/RMS {rel:.2e}, near ties {ties}")


# ------------------------------------------------------------ edge cases
def test_k_equals_E(B):
    spec = LayerSpec(d=128, f=128, E=16, k=16, fmt=I.Q4, seed=3, shared=True)
    ctx = make_ctx(B, spec, max_tokens=16)
    try:
        load_layer(B, ctx, spec)
        x = I.hidden_np(3, 9, 128)
        check(run(B, ctx, spec, x), oracle_for(spec, x), spec)
    finally:
        B.moe_destroy(ctx)


def test_k1(B):
    spec = LayerSpec(d=128, f=256, E=32, k=1, fmt=I.Q2, seed=4, shared=False)
    ctx = make_ctx(B, spec, max_tokens=16)
    try:
        load_layer(B, ctx, spec)
        x = I.hidden_np(4, 11, 128)
        out = run(B, ctx, spec, x)
        assert np.all(out["w"] == 1.0)
        check(out, oracle_for(spec, x), spec)
    finally:
        B.moe_destroy(ctx)


def test_equal_logits_go_to_lower_id(B):
    """Router rows duplicated: equal logits; the lower expert id must win,
    exactly as in the oracle."""
    spec = LayerSpec(d=256, f=128, E=24, k=4, fmt=I.Q4, seed=5, shared=False)
    spec.W[8:16] = spec.W[0:8]      # experts e and e+8 tie for e < 8
    spec.W[16:24] = spec.W[0:8]
    ctx = make_ctx(B, spec, max_tokens=16)
    try:
        load_layer(B, ctx, spec)
        x = I.hidden_np(5, 10, 256)
        out = run(B, ctx, spec, x)
        orc = oracle_for(spec, x)
        # ties at the k boundary are real ties here: compare the whole sets
        assert np.array_equal(np.sort(out["idx"], 1), np.sort(orc["route"]["idx"], 1))
        # a tie always goes to the lower id: an id e >= 8 is only selected
        # together with its lower twin e - 8 (same logit)
        for row in out["idx"]:
            sel = set(row.tolist())
            assert all(e - 8 in sel for e in sel if e >= 8), row
        check(out, orc, spec)
    finally:
        B.moe_destroy(ctx)


@pytest.mark.parametrize("T", [1, 4, 8])
def test_equal_logits_split_topk_outputs(B, T):
    """The decode kernel's top-k splits a token over several warps at
    T <= 8 (4 warps at T <= 4, 2 at T = 8) and merges their candidates.
    Router rows are triplicated (experts e, e+8, e+16 have equal logits),
    so the twins of one row fall into different warps' parts: only the
    lower id may be taken.  A wrong twin changes the output (its weights
    differ), and tokens whose distinct logits are well separated are
    compared against the oracle, exact ties included."""
    spec = LayerSpec(d=256, f=128, E=24, k=4, fmt=I.Q4, seed=15, shared=True)
    spec.W[8:16] = spec.W[0:8]
    spec.W[16:24] = spec.W[0:8]
    ctx = make_ctx(B, spec, max_tokens=16)
    try:
        load_layer(B, ctx, spec)
        x = I.hidden_np(15, T, 256, window=T)
        delta = torch.empty((T, spec.d), dtype=torch.float32, device="cuda")
        B.moe_forward_delta(ctx, 0, to_dev(x), T, delta)
        B.moe_sync(ctx, 60000)
        lg = O.router(x, spec.W, spec.bias)[:, :8]          # the 8 distinct logits
        top = -np.sort(-lg, axis=1)
        # k = 4 takes the three copies of the best row and the lowest copy of
        # the second: fp32 can only disagree if these rows nearly tie
        sep = np.minimum(top[:, 0] - top[:, 1], top[:, 1] - top[:, 2]) >= 1e-5
        assert sep.any()
        orc = spec.oracle(x)
        assert_close_rms(delta.cpu().numpy()[sep], orc["delta"][sep], what="MoE delta")
    finally:
        B.moe_destroy(ctx)


@pytest.mark.parametrize("path", ["decode", "multi", "prefill"])
def test_near_tie_count_matches_oracle(B, path):
    """Planted near ties: experts 0-2 are always selected (bias +10) and
    experts 3 and 4 always rank k-th and (k+1)-th (bias +5); their router rows
    are equal except in column 0, where they differ by 1.0.  Tokens with
    x[t, 0] = 0 therefore tie exactly at the k boundary and every other token
    is 0.5 apart there.  The device's near-tie count (moe_stats.near_ties)
    must equal the number of tokens whose oracle margin is below 1e-5."""
    T = {"decode": 16, "multi": 37, "prefill": 37}[path]
    spec = LayerSpec(d=256, f=128, E=32, k=4, fmt=I.Q4, seed=16, shared=True)
    spec.bias = np.zeros(32, np.float32)
    spec.bias[:3] = 10.0
    spec.bias[3:5] = 5.0
    spec.W[4] = spec.W[3]
    spec.W[4, 0] = spec.W[3, 0] + 1.0
    x = I.hidden_np(16, T, 256, window=T).copy()
    half = int(I.f32_to_bf16_bits(np.array([0.5], np.float32))[0])
    x[:, 0] = half
    ties = [1, 4, 5, 11] + ([33] if T > 33 else [])
    x[ties, 0] = 0
    ctx = make_ctx(B, spec, max_tokens=64)
    try:
        load_layer(B, ctx, spec)
        orc = spec.oracle(x)
        assert int((orc["margin"] < TIE_MARGIN).sum()) == len(ties)
        assert np.all((orc["margin"] < 1e-9) | (orc["margin"] > 1e-2))  # nothing in between
        st0 = B.moe_get_stats(ctx)
        delta = torch.empty((T, 256), dtype=torch.float32, device="cuda")
        if path == "prefill":
            B.moe_prefill_delta(ctx, 0, to_dev(x), T, delta)
        else:
            B.moe_forward_delta(ctx, 0, to_dev(x), T, delta)
        B.moe_sync(ctx, 60000)
        st1 = B.moe_get_stats(ctx)
        assert st1["near_ties"] - st0["near_ties"] == len(ties)
        ok = orc["margin"] >= TIE_MARGIN
        assert_close_rms(delta.cpu().numpy()[ok], orc["delta"][ok], what="MoE delta")
    finally:
        B.moe_destroy(ctx)


def test_one_hot_expert_many_jobs(B):
    """A large bias sends every token to expert 7: one expert with T tokens,
    split into several 16-token jobs."""
    spec = LayerSpec(d=256, f=128, E=16, k=2, fmt=I.Q4, seed=6, shared=True)
    spec.bias = np.zeros(16, np.float32)
    spec.bias[7] = 50.0
    ctx = make_ctx(B, spec, max_tokens=64)
    try:
        load_layer(B, ctx, spec)
        x = I.hidden_np(6, 61, 256)
        out = run(B, ctx, spec, x)
        assert np.all(out["idx"][:, 0] == 7)
        check(out, oracle_for(spec, x), spec)
    finally:
        B.moe_destroy(ctx)


def test_bucket_only_bit_exact(B):
    E, k, T = 512, 10, 200
    spec = LayerSpec(d=128, f=128, E=E, k=k, fmt=I.Q4, shared=False)
    ctx = make_ctx(B, spec, max_tokens=T)
    try:
        idx = I.routing_idx_np(11, T, k, E)
        cnt, off, perm = O.bucket(idx, E)
        d_off = torch.empty(E + 1, dtype=torch.int32, device="cuda")
        d_perm = torch.empty(T * k, dtype=torch.int32, device="cuda")
        B.moe_bucket(ctx, torch.from_numpy(idx).cuda(), T, d_off, d_perm)
        B.moe_sync(ctx, 60000)
        assert np.array_equal(d_off.cpu().numpy(), off)
        assert np.array_equal(d_perm.cpu().numpy(), perm)
    finally:
        B.moe_destroy(ctx)


def test_bucket_bad_expert_sets_status(B):
    E, k, T = 64, 2, 8
    spec = LayerSpec(d=128, f=128, E=E, k=k, fmt=I.Q4, shared=False)
    ctx = make_ctx(B, spec, max_tokens=T)
    try:
        idx = I.routing_idx_np(12, T, k, E)
        idx[3, 1] = E + 5
        d_off = torch.empty(E + 1, dtype=torch.int32, device="cuda")
        d_perm = torch.empty(T * k, dtype=torch.int32, device="cuda")
        B.moe_bucket(ctx, torch.from_numpy(idx).cuda(), T, d_off, d_perm)
        with pytest.raises(B.MoeError) as ei:
            B.moe_sync(ctx, 60000)
        assert ei.value.status == 6  # MOE_ERR_DEVICE
        B.moe_sync(ctx, 60000)       # status was cleared
    finally:
        B.moe_destroy(ctx)


# ------------------------------------------------------------- residency
def test_residency_table_does_not_change_results(B):
    spec = LayerSpec(d=256, f=128, E=32, k=4, fmt=I.Q4, seed=8, shared=True)
    ctx = make_ctx(B, spec, max_tokens=32, L=2, n_slots=20)
    try:
        load_layer(B, ctx, spec, layer=0)
        spec1 = LayerSpec(d=256, f=128, E=32, k=4, fmt=I.Q4, seed=8, shared=True, layer=1)
        load_layer(B, ctx, spec1, layer=1)
        x = I.hidden_np(8, 24, 256)
        base = run(B, ctx, spec, x, layer=0)
        st0 = B.moe_get_stats(ctx)
        table = np.full(2 * 32, -1, np.int32)
        rng = np.random.default_rng(0)
        chosen = rng.choice(64, size=20, replace=False)
        table[chosen] = np.arange(20)
        B.moe_set_slots(ctx, table)
        res = run(B, ctx, spec, x, layer=0)
        for key in base:
            assert np.array_equal(base[key], res[key]), key
        st1 = B.moe_get_stats(ctx)
        # three routed calls per run(); every pair is a hit or a miss
        resident = set(int(c) for c in chosen if c < 32)
        pairs = res["idx"].reshape(-1)
        hits = sum(1 for e in pairs if int(e) in resident)
        assert (st1["hits"] - st0["hits"]) == 2 * hits
        assert (st1["misses"] - st0["misses"]) == 2 * (len(pairs) - hits)
        assert st1["last_T"] == 24
        assert np.array_equal(np.bincount(pairs, minlength=32), st1["expert_count"])
        check(res, oracle_for(spec, x), spec)
    finally:
        B.moe_destroy(ctx)


def test_corrupt_slot_is_reported_not_trapped(B):
    """A slot id beyond the pool, written past the host checks, is caught on
    the device: the kernel uses the backing copy and moe_sync reports
    MOE_ERR_BAD_SLOT."""
    spec = LayerSpec(d=256, f=128, E=16, k=16, fmt=I.Q4, seed=9, shared=False)
    ctx = make_ctx(B, spec, max_tokens=8, n_slots=4)
    try:
        load_layer(B, ctx, spec)
        x = I.hidden_np(9, 4, 256)
        B.moe_debug_poke_slot(ctx, 0, 3, 4 + 1000)
        xd = to_dev(x)
        delta = torch.empty((4, 256), dtype=torch.float32, device="cuda")
        B.moe_forward_delta(ctx, 0, xd, 4, delta)
        with pytest.raises(B.MoeError) as ei:
            B.moe_sync(ctx, 60000)
        assert ei.value.status == 5  # MOE_ERR_BAD_SLOT
        orc = oracle_for(spec, x)
        assert_close_rms(delta.cpu().numpy(), orc["out"]["delta"])
    finally:
        B.moe_destroy(ctx)


def test_decode_barrier_wait_runs_out_and_recovers(B):
    """A bounded device wait made to run out: the test hook gives the next
    single-launch decode a first grid barrier that cannot complete (poll
    limit ~16 K).  The kernel reports the give-up and leaves; moe_sync
    returns MOE_ERR_DEVICE with the timeout bit, resets the barrier counters,
    and the next calls match the oracle.  No fault or hang is involved."""
    spec = LayerSpec(d=256, f=128, E=16, k=2, fmt=I.Q4, seed=18, shared=True)
    ctx = make_ctx(B, spec, max_tokens=32)
    try:
        load_layer(B, ctx, spec)
        x = I.hidden_np(18, 4, 256)
        orc = oracle_for(spec, x)
        check(run(B, ctx, spec, x), orc, spec)          # before
        B.moe_debug_stall_next_decode(ctx, 1 << 14)
        delta = torch.empty((4, 256), dtype=torch.float32, device="cuda")
        B.moe_forward_delta(ctx, 0, to_dev(x), 4, delta)
        with pytest.raises(B.MoeError) as ei:
            B.moe_sync(ctx, 60000)
        assert ei.value.status == 6 and "0x8" in str(ei.value)
        B.moe_sync(ctx, 60000)                          # status cleared
        for _ in range(2):                              # after: counters reset
            check(run(B, ctx, spec, x), orc, spec)
    finally:
        B.moe_destroy(ctx)


@pytest.mark.parametrize("T", [4, 40])
def test_pruned_256_expert_layer(B, T):
    """The pruned "Coder" configuration of the engine article's performance
    validation (256 of the 512 experts kept, 10 active): d=2048, f=768,
    E=256, top-10 + shared, Q4; a decode window and a 40-token window."""
    spec = LayerSpec(d=2048, f=768, E=256, k=10, fmt=I.Q4, seed=0, shared=True)
    ctx = make_ctx(B, spec, max_tokens=64)
    try:
        load_layer(B, ctx, spec)
        x = I.hidden_np(0, T, 2048, window=256 + T)
        sample = None if T <= 4 else np.array([0, 7, T // 2, T - 1])
        rel, ties = check(run(B, ctx, spec, x), oracle_for(spec, x, sample), spec, sample)
        print(f"E=256 T={T}: delta max-err/RMS {rel:.2e}, near ties {ties}")
    finally:
        B.moe_destroy(ctx)


def test_sync_times_out_on_stalled_stream(B, decode_q4):
    ctx, spec = decode_q4
    x = to_dev(I.hidden_np(0, 4, 2048))
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        torch.cuda._sleep(2_000_000_000)  # a bounded busy kernel (~1 s)
        B.moe_forward(ctx, 0, x, 4, stream=s)
    with pytest.raises(B.MoeError) as ei:
        B.moe_sync(ctx, 20)
    assert ei.value.status == 7  # MOE_ERR_TIMEOUT
    B.moe_sync(ctx, -1)
    torch.cuda.synchronize()


def test_invalid_arguments(B):
    spec = LayerSpec(d=128, f=128, E=8, k=2, fmt=I.Q4, shared=False)
    ctx = make_ctx(B, spec, max_tokens=8)
    try:
        x = torch.zeros((9, 128), dtype=torch.int16, device="cuda")
        with pytest.raises(B.MoeError) as ei:
            B.moe_forward(ctx, 0, x, 4)
        assert ei.value.status == 4  # router/experts not loaded: STATE
        load_layer(B, ctx, spec)
        for T in (0, 9):
            with pytest.raises(B.MoeError) as ei:
                B.moe_forward(ctx, 0, x, T)
            assert ei.value.status == 1
        with pytest.raises(B.MoeError):
            B.moe_forward(ctx, 1, x, 4)  # no layer 1
        with pytest.raises(B.MoeError):
            B.moe_configure(ctx, 2, 0, 0, 8)  # already configured
        with pytest.raises(B.MoeError):
            B.moe_set_slots(ctx, np.full(8, 3, np.int32))  # no slot pool
    finally:
        B.moe_destroy(ctx)
    with pytest.raises(B.MoeError):
        B.moe_create(100, 128, 8, 2, 1)  # d not a multiple of 128
    with pytest.raises(B.MoeError):
        B.moe_create(128, 128, 8, 9, 1)  # k > E


# ------------------------------------------------------ RMSNorm + stack
def test_stack_with_norm_matches_layers_and_oracle(B):
    """3 layers with RMSNorm: moe_forward_stack (one CUDA graph) equals the
    layer-by-layer calls bit for bit; each layer matches the oracle when fed
    the GPU's input to that layer (teacher forcing)."""
    L, d, f, E, k = 3, 256, 128, 32, 4
    specs = [LayerSpec(d=d, f=f, E=E, k=k, fmt=I.Q4, seed=21, shared=True, zipf=True, layer=l)
             for l in range(L)]
    ctx = B.moe_create(d, f, E, k, I.Q4)
    B.moe_configure(ctx, L, 1, 8, 16)
    try:
        for l, sp in enumerate(specs):
            load_layer(B, ctx, sp, layer=l)
            B.moe_set_norm(ctx, l, None, 1e-6)
        table = np.full(L * E, -1, np.int32)
        table[[0, 5, 33, 34, 70, 90, 95, 64]] = np.arange(8)
        B.moe_set_slots(ctx, table)
        x0 = I.hidden_np(21, 12, d)
        xs = [x0]
        cur = to_dev(x0)
        for l in range(L):
            B.moe_forward(ctx, l, cur, 12)
            B.moe_sync(ctx, 60000)
            xs.append(to_bits(cur))
        xg = to_dev(x0)
        B.moe_forward_stack(ctx, xg, 12)       # records the graph
        B.moe_sync(ctx, 60000)
        assert np.array_equal(to_bits(xg), xs[-1])
        xg.copy_(to_dev(x0))
        B.moe_forward_stack(ctx, xg, 12)       # replays it
        B.moe_sync(ctx, 60000)
        assert np.array_equal(to_bits(xg), xs[-1])
        for l in range(L):
            # teacher forcing: the oracle gets the GPU's input to layer l
            orc = specs[l].oracle(xs[l], norm=True)
            ok = orc["margin"] >= 1e-5
            delta = torch.empty((12, d), dtype=torch.float32, device="cuda")
            B.moe_forward_delta(ctx, l, to_dev(xs[l]), 12, delta)
            B.moe_sync(ctx, 60000)
            assert_close_rms(delta.cpu().numpy()[ok], orc["delta"][ok], what=f"layer {l} delta")
            assert_close_residual(xs[l + 1][ok], orc["x_out"][ok], what=f"layer {l} x")
            # the router input is RMSNorm(x), as the decode kernel computed it
            # (fp32 inside, bf16 round to nearest even) against the oracle's
            # (fp64 inside): equal, or one bf16 ulp apart where the fp32
            # result sits within rounding of a bf16 halfway point
            hg = torch.empty((12, d), dtype=torch.int16, device="cuda")
            B.moe_debug_last_h(ctx, hg, 12)
            torch.cuda.synchronize()
            hg = hg.cpu().numpy().view(np.uint16).astype(np.int64)
            ho = orc["h"].astype(np.int64)
            # same-sign bf16 bit patterns differ by their distance in ulps
            assert np.array_equal(hg >> 15, ho >> 15), f"layer {l}: sign of h"
            assert np.abs(hg - ho).max() <= 1, f"layer {l}: h differs by more than one ulp"
            assert (hg == ho).mean() >= 0.999, f"layer {l}: exact {(hg == ho).mean():.5f}"
    finally:
        B.moe_destroy(ctx)
