"""Expert parallelism on the CPU: the layer's exchange (dispatch by owner,
split sizes, all-to-all there and back, combine in j order) as gloo ranks,
each rank's steps computed by the oracle with only its own experts' weights.
Every rank's output must equal the oracle's one-process layer on the whole
batch exactly: the sharding moves rows, it must not change any sum."""
import json
import os
import sys

import numpy as np
import pytest

from tests.test_bench_multirank_cpu import free_port, launch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

RANK_PROG = r"""
import json, os, sys
sys.path.insert(0, sys.argv[1])
import numpy as np, torch
import torch.distributed as dist
from sparse_moe_expert_gemv_b200 import inputs as I
from sparse_moe_expert_gemv_b200.ep import Exchange, ExpertParallelMoE
from tests._harness import LayerSpec
from tests._ep_oracle_ops import OracleOps
cfg = json.loads(sys.argv[2])
rank, world = int(os.environ["RANK"]), int(os.environ["WORLD_SIZE"])
dist.init_process_group("gloo", rank=rank, world_size=world)
spec = LayerSpec(d=cfg["d"], f=cfg["f"], E=cfg["E"], k=cfg["k"], fmt=cfg["fmt"], zipf=True,
                 shared=cfg["shared"])
sizes = cfg["sizes"]
x_all = I.hidden_np(3, sum(sizes), cfg["d"], window=5)
a = sum(sizes[:rank])
x = torch.from_numpy(x_all[a:a + sizes[rank]].view(np.int16).copy())
ops = OracleOps(spec, rank, world, norm=cfg["norm"])
ExpertParallelMoE(ops, Exchange()).forward(0, x, sizes[rank])
dist.barrier()
dist.destroy_process_group()
delta = ops.last_delta if ops.last_delta is not None else np.zeros((0, cfg["d"]))
np.savez(os.path.join(sys.argv[3], f"rank{rank}.npz"), x=x.numpy().view(np.uint16),
         delta=delta, received=np.array(ops.received, np.int64))
print(json.dumps({"rank": rank, "rows": len(ops.received)}))
"""


@pytest.mark.parametrize("world,E,sizes,shared,norm", [
    (2, 16, [37, 20], True, False),
    (3, 24, [9, 1, 30], False, True),
    (3, 24, [0, 25, 12], True, False),   # a rank with no tokens of its own still serves
    (4, 32, [11, 0, 6, 19], True, True),
])
def test_expert_parallel_gloo_ranks_match_the_one_process_layer(tmp_path, world, E, sizes, shared,
                                                                 norm):
    from sparse_moe_expert_gemv_b200 import inputs as I
    from tests._harness import LayerSpec
    import oracle as O

    cfg = dict(d=256, f=128, E=E, k=4, fmt=O.Q4, sizes=sizes, shared=shared, norm=norm)
    outs = launch(["-c", RANK_PROG, ROOT, json.dumps(cfg), str(tmp_path)], world, free_port())
    for rc, out, err in outs:
        assert rc == 0, err[-3000:]
    spec = LayerSpec(d=256, f=128, E=E, k=4, fmt=O.Q4, zipf=True, shared=shared)
    x_all = I.hidden_np(3, sum(sizes), 256, window=5)
    want = spec.oracle(x_all, norm=norm)
    per = E // world
    rows = 0
    for r in range(world):
        got = np.load(tmp_path / f"rank{r}.npz")
        a = sum(sizes[:r])
        sl = slice(a, a + sizes[r])
        assert np.array_equal(got["x"], want["x_out"][sl]), f"rank {r}: residual differs"
        assert np.array_equal(got["delta"], want["delta"][sl]), f"rank {r}: delta differs"
        # each owner computed exactly the pairs of its experts, from every rank
        rec = np.sort(got["received"])
        idx = want["idx"].reshape(-1)
        assert np.array_equal(rec, np.sort(idx[(idx // per) == r]))
        rows += rec.size
    assert rows == sum(sizes) * 4


EMPTY_PROG = r"""
import json, os, sys
sys.path.insert(0, sys.argv[1])
import numpy as np, torch
import torch.distributed as dist
import oracle as O
from sparse_moe_expert_gemv_b200 import inputs as I
from sparse_moe_expert_gemv_b200.ep import Exchange, ExpertParallelMoE
from tests._harness import LayerSpec
from tests._ep_oracle_ops import OracleOps

class FirstHalfRouting(OracleOps):
    # every token picks experts from rank 0's half only: rank 1 receives no rows
    def route(self, layer, h, N):
        t = np.arange(N)[:, None]
        j = np.arange(self.k)[None, :]
        idx = ((3 * t + 5 * j) % (self.E // 2)).astype(np.int32)
        w = np.full((N, self.k), 1.0 / self.k)
        return torch.from_numpy(idx), torch.from_numpy(w)

rank, world = int(os.environ["RANK"]), int(os.environ["WORLD_SIZE"])
dist.init_process_group("gloo", rank=rank, world_size=world)
spec = LayerSpec(d=256, f=128, E=16, k=4, fmt=O.Q4, zipf=False, shared=True)
N = 7
x = torch.from_numpy(I.hidden_np(4, N, 256, window=rank).view(np.int16).copy())
ops = FirstHalfRouting(spec, rank, world)
ExpertParallelMoE(ops, Exchange()).forward(0, x, N)
dist.barrier()
dist.destroy_process_group()
np.savez(os.path.join(sys.argv[2], f"rank{rank}.npz"), x=x.numpy().view(np.uint16), delta=ops.last_delta,
         received=np.array(ops.received, np.int64))
"""


def test_a_rank_that_receives_no_rows(tmp_path):
    """Rank 1 owns experts nobody selects: it sends its tokens' rows, receives
    none, computes nothing, and still gets its outputs back."""
    import oracle as O
    from sparse_moe_expert_gemv_b200 import inputs as I
    from tests._harness import LayerSpec

    outs = launch(["-c", EMPTY_PROG, ROOT, str(tmp_path)], 2, free_port())
    for rc, out, err in outs:
        assert rc == 0, err[-3000:]
    spec = LayerSpec(d=256, f=128, E=16, k=4, fmt=O.Q4, zipf=False, shared=True)
    N, k = 7, 4
    for r in range(2):
        got = np.load(tmp_path / f"rank{r}.npz")
        assert got["received"].size == (2 * N * k if r == 0 else 0)
        xb = I.hidden_np(4, N, 256, window=r)
        idx = (3 * np.arange(N)[:, None] + 5 * np.arange(k)[None, :]) % 8
        acc = np.zeros((N, 256))
        for j in range(k):
            for t in range(N):
                Wg, Wu, Wd = O.dequant_expert(spec.fmt, 256, 128, *spec.expert(int(idx[t, j])))
                acc[t] += (1.0 / k) * O.expert(Wg, Wu, Wd, xb[t:t + 1])[0]
        Wg, Wu, Wd = O.dequant_expert(spec.fmt, 256, 128, *spec.shared_expert())
        acc += O.expert(Wg, Wu, Wd, xb)
        assert np.array_equal(got["delta"], acc)
