"""Host tier replacement policy (moe_tier_sim_*: host code only, no GPU).

The engine article ("93 token/s on one 8 GB card", section "Expert cache")
keeps a model's hot experts in a fixed set of device slots and brings misses
in; the user report "EPYC 7B13 + 2x RTX 3090" makes that cache adaptive.
These tests pin the policy the library uses for its HBM slot pool when the
experts' backing copies live in host memory."""
import random

import pytest

from sparse_moe_expert_gemv_b200 import binding as B


def test_lru_evicts_the_least_recently_used():
    s = B.TierSim(4, B.TIER_LRU, 64.0, 100)
    assert s.request([1, 2, 3]) == (3, [0, 1, 2])   # three free slots
    assert s.request([4, 5]) == (2, [3, 0])         # slot 3 free; 1, 2, 3 tie: slot 0 (key 1) goes
    assert s.request([2]) == (0, [1])               # hit
    assert s.request([1, 6]) == (2, [2, 0])         # LRU: key 3 (slot 2); keys 5 and 4 tie: slot 0
    assert s.counts() == {"hits": 1, "misses": 7, "evictions": 3}


@pytest.mark.parametrize("policy", [B.TIER_LRU, B.TIER_ADAPTIVE])
def test_a_request_never_evicts_its_own_experts(policy):
    rng = random.Random(7)
    n_keys, n_slots = 300, 40
    s = B.TierSim(n_slots, policy, 16.0, n_keys)
    resident = {}
    for _ in range(400):
        keys = rng.sample(range(n_keys), rng.randint(1, n_slots))
        misses, slots = s.request(keys)
        assert len(set(slots)) == len(keys)                  # distinct slots
        assert all(0 <= x < n_slots for x in slots)
        assert misses == sum(1 for kk in keys if kk not in resident)
        for kk, sl in zip(keys, slots):                      # the resident map after the request
            for other in [o for o, v in resident.items() if v == sl and o != kk]:
                del resident[other]
            resident[kk] = sl
        assert len(resident) <= n_slots


def test_prefetch_keeps_the_previous_request_resident():
    s = B.TierSim(6, B.TIER_LRU, 64.0, 100)
    _, prev = s.request([10, 11, 12])
    _, _ = s.request([13, 14, 15])                            # fills the pool
    misses, _ = s.request([20, 21, 22], protect_prev=True)    # may only evict 10, 11, 12
    assert misses == 3
    _, again = s.request([13, 14, 15])
    assert sorted(again) == sorted(set(again))                # still resident: all hits
    assert s.counts()["hits"] == 3


def test_requests_beyond_the_pool_are_refused():
    s = B.TierSim(4, B.TIER_ADAPTIVE, 64.0, 100)
    with pytest.raises(B.MoeError):
        s.request([1, 2, 3, 4, 5])
    s.request([1, 2, 3])
    with pytest.raises(B.MoeError):                           # only one slot may be taken
        s.request([5, 6], protect_prev=True)
    with pytest.raises(ValueError):
        s.request([1, 1])                                     # keys must be distinct
    with pytest.raises(ValueError):
        s.request([100])                                      # key out of range


def _hit_rate(policy):
    """A hot set used every third request, two scans of new experts between:
    LRU evicts the hot set during the second scan, a use-count policy keeps
    it (the pool holds the hot set plus one scan)."""
    hot = list(range(50))
    nxt = 1000
    s = B.TierSim(160, policy, 64.0, 100000)
    hot_hits = hot_total = 0
    for rnd in range(40):
        misses, _ = s.request(hot)
        if rnd >= 2:
            hot_total += len(hot)
            hot_hits += len(hot) - misses
        for _ in range(2):
            s.request(list(range(nxt, nxt + 100)))
            nxt += 100
    return hot_hits / hot_total


def test_adaptive_policy_resists_scans():
    lru, adaptive = _hit_rate(B.TIER_LRU), _hit_rate(B.TIER_ADAPTIVE)
    assert lru < 0.5
    assert adaptive == 1.0


def test_bad_sim_arguments():
    with pytest.raises(ValueError):
        B.TierSim(0, B.TIER_LRU, 64.0, 10)
    with pytest.raises(ValueError):
        B.TierSim(4, 7, 64.0, 10)
