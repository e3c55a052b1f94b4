"""Expert parallelism: the experts of each layer sharded by id over the
ranks of a process group (one process per GPU), the tokens data-parallel.

Rank r owns experts [r E/R, (r+1) E/R) of every layer; router and shared
expert are replicated.  Per layer and rank, the engine article's per-layer
flow ("93 token/s on one 8 GB card", section "Architecture overview":
route, run the selected experts, combine into the residual) becomes:

1. ``h = RMSNorm(x)`` (``moe_rmsnorm``) and the routing of the rank's own
   tokens (``moe_prefill_route``; ``moe_route`` for windows of <= 32 tokens);
2. ``moe_ep_dispatch``: each (token, expert) pair's router-input row, grouped
   by the expert's owner, and the rows' expert ids;
3. an all-to-all of those rows and ids (the split sizes are exchanged first);
4. each owner runs its experts on the rows it received
   (``moe_experts_rows``: one expert per row, each row's output y in fp16);
5. an all-to-all of the outputs back to their source ranks, and the shared
   expert on the rank's own rows (``moe_experts_given`` with no routed
   experts);
6. ``moe_ep_combine``: ``x <- bf16(x + sum_j w_j y_j + y_shared)``, j in
   order, with the one-GPU combine's arithmetic.

The owners receive exactly the rows the one-GPU layer would group for each
expert, so with the same routing the sharded layer reproduces
``moe_prefill`` bit for bit.  Every step of the layer is a library kernel;
this module allocates buffers and calls the collectives.  The collectives
are NCCL's ``all_to_all_single`` (no peer-memory kernel of this library
reads another GPU's memory).
"""
from __future__ import annotations

import torch
import torch.distributed as dist


class DeviceOps:
    """The layer's steps on one context, each a call into the library."""

    def __init__(self, B, ctx, *, d, k, E, max_tokens, has_shared, device="cuda"):
        self.B, self.ctx = B, ctx
        self.d, self.k, self.E = d, k, E
        self.max_tokens, self.has_shared, self.device = max_tokens, has_shared, device
        self.last_rows = 0    # rows of the last experts() call

    def norm(self, layer, x, N):
        h = torch.empty_like(x)
        self.B.moe_rmsnorm(self.ctx, layer, x, N, h)
        return h

    def route(self, layer, h, N):
        idx = torch.empty((N, self.k), dtype=torch.int32, device=self.device)
        w = torch.empty((N, self.k), dtype=torch.float32, device=self.device)
        if N > 32:
            self.B.moe_prefill_route(self.ctx, layer, h, N, idx, w)
        else:
            self.B.moe_route(self.ctx, layer, h, N, idx, w)
        return idx, w

    def dispatch(self, idx, h, N, n_ranks):
        P = N * self.k
        send_h = torch.empty((P, self.d), dtype=h.dtype, device=self.device)
        send_e = torch.empty(P, dtype=torch.int32, device=self.device)
        row_of = torch.empty(P, dtype=torch.int32, device=self.device)
        counts = self.B.moe_ep_dispatch(self.ctx, idx, N, n_ranks, h, send_h, send_e, row_of)
        return send_h, send_e, row_of, counts

    def experts(self, layer, rows_h, M, rows_e):
        """y [M, d] fp16: row i's output of expert rows_e[i] (M may be 0), in
        the fp16 the chunk path keeps expert outputs in.  More rows than the
        context holds run in slices of max_tokens rows."""
        self.last_rows = M
        y = torch.empty((M, self.d), dtype=torch.float16, device=self.device)
        for a in range(0, M, self.max_tokens):
            n = min(self.max_tokens, M - a)
            self.B.moe_experts_rows(self.ctx, layer, rows_h[a:a + n], n, rows_e[a:a + n], y[a:a + n])
        return y

    def shared(self, layer, h, N):
        if not self.has_shared:
            return None
        ysh = torch.empty((N, self.d), dtype=torch.float32, device=self.device)
        for a in range(0, N, self.max_tokens):
            n = min(self.max_tokens, N - a)
            self.B.moe_experts_given(self.ctx, layer, h[a:a + n], n, 0, None, None, 1, ysh[a:a + n])
        return ysh

    def combine(self, N, w, y, row_of, y_shared, x):
        self.B.moe_ep_combine(self.ctx, N, w, y, row_of, y_shared, x=x)


def _as_rows_of_bytes(t):
    """A [n, ...] tensor as [n, row bytes] uint8 (the all-to-all splits count
    rows); n may be 0."""
    row = 1
    for s in t.shape[1:]:
        row *= s
    if t.shape[0] == 0:
        return torch.empty((0, row * t.element_size()), dtype=torch.uint8, device=t.device)
    return t.contiguous().reshape(t.shape[0], row).view(torch.uint8)


class Exchange:
    """All-to-all of row blocks over a torch.distributed process group."""

    def __init__(self, group=None):
        self.group = group
        self.world = dist.get_world_size(group)
        self.rank = dist.get_rank(group)
        backend = dist.get_backend(group)
        self.device = torch.device("cuda", torch.cuda.current_device()) if backend == "nccl" \
            else torch.device("cpu")

    def counts(self, send_counts):
        send = torch.tensor(send_counts, dtype=torch.int64, device=self.device)
        recv = torch.empty_like(send)
        dist.all_to_all_single(recv, send, group=self.group)
        return [int(v) for v in recv.tolist()]

    def rows(self, send, send_counts, recv_counts):
        """Rows [sum(send_counts), ...] split by destination -> the rows this
        rank receives, ordered by source rank."""
        src = _as_rows_of_bytes(send[:sum(send_counts)])
        out = torch.empty((sum(recv_counts), src.shape[1]), dtype=torch.uint8, device=src.device)
        dist.all_to_all_single(out, src, output_split_sizes=list(recv_counts),
                               input_split_sizes=list(send_counts), group=self.group)
        return out.view(send.dtype).reshape((sum(recv_counts),) + tuple(send.shape[1:]))


class ExpertParallelMoE:
    """One rank's view of expert-parallel MoE layers (``ops`` on this rank's
    context, ``exchange`` over the process group)."""

    def __init__(self, ops, exchange, on_phase=None):
        self.ops, self.ex = ops, exchange
        self.on_phase = on_phase   # optional callable(name), called after each phase

    def _mark(self, name):
        if self.on_phase is not None:
            self.on_phase(name)

    def forward(self, layer, x, N):
        """x [N, d] bf16, in place: x <- x + MoE(norm(x)) for this rank's
        tokens.  N may be 0: the rank still serves its experts to the others
        and takes part in every collective."""
        if N == 0:
            self._serve_only(layer, x)
            return
        h = self.ops.norm(layer, x, N)
        idx, w = self.ops.route(layer, h, N)
        self._mark("route")
        self.forward_routed(layer, x, h, N, idx, w)

    def _serve_only(self, layer, x):
        """A step with no tokens of this rank's own: empty send blocks, the
        owner's work for the other ranks, nothing to combine."""
        ops, ex = self.ops, self.ex
        zero = [0] * ex.world
        recv_counts = ex.counts(zero)
        d = x.shape[1]
        rows_h = ex.rows(x.new_empty((0, d)), zero, recv_counts)
        rows_e = ex.rows(torch.empty(0, dtype=torch.int32, device=x.device), zero, recv_counts)
        self._mark("exchange")
        y = ops.experts(layer, rows_h, sum(recv_counts), rows_e)
        self._mark("experts")
        ex.rows(y, recv_counts, zero)
        self._mark("return")

    def forward_routed(self, layer, x, h, N, idx, w):
        ops, ex = self.ops, self.ex
        send_h, send_e, row_of, send_counts = ops.dispatch(idx, h, N, ex.world)
        self._mark("dispatch")
        recv_counts = ex.counts(send_counts)
        rows_h = ex.rows(send_h, send_counts, recv_counts)
        rows_e = ex.rows(send_e, send_counts, recv_counts)
        self._mark("exchange")
        M = sum(recv_counts)
        y = ops.experts(layer, rows_h, M, rows_e)   # M may be 0: an empty output of the ops' row type
        self._mark("experts")
        y_back = ex.rows(y, recv_counts, send_counts)
        self._mark("return")
        y_shared = ops.shared(layer, h, N)
        self._mark("shared")
        ops.combine(N, w, y_back, row_of, y_shared, x)
        self._mark("combine")


def emulate(ops_by_rank, layer, xs, hs, Ns, routings):
    """R ranks' expert-parallel layer in one process, the all-to-all done by
    slicing (one device standing in for R): the same steps as
    ``ExpertParallelMoE.forward_routed``, rank by rank.  xs are updated in
    place.  Returns the rows each rank received (for inspection)."""
    R = len(ops_by_rank)

    def plan(r):
        if Ns[r] == 0:  # nothing to send: empty blocks of the same row types
            h = hs[r]
            return (h.new_empty((0, h.shape[1])), torch.empty(0, dtype=torch.int32, device=h.device),
                    torch.empty(0, dtype=torch.int32, device=h.device), [0] * R)
        return ops_by_rank[r].dispatch(routings[r][0], hs[r], Ns[r], R)

    plans = [plan(r) for r in range(R)]
    splits = [p[3] for p in plans]

    def a2a(bufs, split):
        out = []
        for dst in range(R):
            parts = []
            for src in range(R):
                off = sum(split[src][:dst])
                parts.append(bufs[src][off:off + split[src][dst]])
            out.append(torch.cat(parts))
        return out

    rows_h = a2a([p[0] for p in plans], splits)
    rows_e = a2a([p[1] for p in plans], splits)
    recv = [[splits[src][dst] for src in range(R)] for dst in range(R)]
    ys = []
    for r in range(R):
        M = sum(recv[r])
        ys.append(ops_by_rank[r].experts(layer, rows_h[r], M, rows_e[r]))
    y_back = a2a(ys, recv)
    for r in range(R):
        if Ns[r] == 0:
            continue
        ops = ops_by_rank[r]
        ops.combine(Ns[r], routings[r][1], y_back[r], plans[r][2], ops.shared(layer, hs[r], Ns[r]), xs[r])
    return rows_e
