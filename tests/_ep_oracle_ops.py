"""The steps of an expert-parallel layer computed by the oracle on the CPU,
with the interface of ``sparse_moe_expert_gemv_b200.ep.DeviceOps``: lets the
layer's exchange choreography (split sizes, all-to-all order, the way back,
the combine in j order) run as gloo ranks without a GPU.  A rank holds the
dequantised weights of its own experts only; a row sent to the wrong owner
raises."""
from __future__ import annotations

import numpy as np
import torch

import oracle as O


class OracleOps:
    def __init__(self, spec, rank, world, norm=False, eps=1e-6):
        self.spec, self.rank, self.world = spec, rank, world
        self.d, self.k, self.E = spec.d, spec.k, spec.E
        self.norm_on, self.eps = norm, eps
        per = spec.E // world
        self.owned = range(rank * per, (rank + 1) * per)
        self._w = {}
        self.received = []       # expert ids of the rows this rank computed
        self.last_delta = None

    def _weights(self, e):
        if e not in self._w:
            c, s, m = self.spec.shared_expert() if e == "shared" else self.spec.expert(e)
            self._w[e] = O.dequant_expert(self.spec.fmt, self.d, self.spec.f, c, s, m)
        return self._w[e]

    def norm(self, layer, x, N):
        xb = x.numpy().view(np.uint16)
        h = O.rmsnorm(xb, None, self.eps) if self.norm_on else xb.copy()
        return torch.from_numpy(h.view(np.int16))

    def route(self, layer, h, N):
        lg = O.router(h.numpy().view(np.uint16), self.spec.W, self.spec.bias)
        idx, w, _ = O.topk(lg, self.k)
        return torch.from_numpy(idx), torch.from_numpy(w)

    def dispatch(self, idx, h, N, n_ranks):
        per = self.E // n_ranks
        flat = idx.numpy().reshape(-1)
        order = np.concatenate([np.nonzero(flat // per == r)[0] for r in range(n_ranks)])
        row_of = np.empty(flat.size, np.int64)
        row_of[order] = np.arange(order.size)
        counts = [int(np.sum(flat // per == r)) for r in range(n_ranks)]
        send_h = h[torch.from_numpy(order // self.k)]
        send_e = torch.from_numpy(flat[order].astype(np.int32))
        return send_h, send_e, torch.from_numpy(row_of), counts

    def experts(self, layer, rows_h, M, rows_e):
        e_np = rows_e.numpy()
        hb = rows_h.numpy().view(np.uint16)
        y = np.zeros((M, self.d), np.float64)
        for e in sorted(set(e_np.tolist())):
            if e not in self.owned:
                raise AssertionError(f"rank {self.rank} received a row of expert {e}")
            rows = np.nonzero(e_np == e)[0]
            Wg, Wu, Wd = self._weights(e)
            y[rows] = O.expert(Wg, Wu, Wd, np.ascontiguousarray(hb[rows]))
        self.received.extend(e_np.tolist())
        return torch.from_numpy(y)

    def shared(self, layer, h, N):
        if not self.spec.shared:
            return None
        Wg, Wu, Wd = self._weights("shared")
        return torch.from_numpy(O.expert(Wg, Wu, Wd, h.numpy().view(np.uint16)))

    def combine(self, N, w, y, row_of, y_shared, x):
        """The oracle's combine: j order, then the shared expert, then the
        residual add with one bf16 rounding."""
        yv, wv, ro = y.numpy(), w.numpy(), row_of.numpy()
        acc = np.zeros((N, self.d), np.float64)
        for t in range(N):
            for j in range(self.k):
                acc[t] += wv[t, j] * yv[ro[t * self.k + j]]
        if y_shared is not None:
            acc += y_shared.numpy()
        self.last_delta = acc
        xb = x.numpy().view(np.uint16)
        to64, to16 = np.vectorize(O.bf16_to_f64), np.vectorize(O.f64_to_bf16)
        xb[...] = to16(to64(xb) + acc).astype(np.uint16)
