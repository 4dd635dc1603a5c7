"""The library's expert-cache replacement policy against the oracle's LRU
replay, on the CPU: the cache runs policy-only (device < 0: no memory, no
copies, no CUDA calls) and both sides see the same random traces."""
import ctypes
import random

import pytest

import expert_ffn_layer_route_b200 as moe
from oracle.lru import LRUReplay

STAT_KEYS = ("lookups", "hits", "misses", "evictions", "prefetch_issued", "prefetch_used")


def _policy_cache(L, E, C):
    return moe.ExpertCache(L, E, C, 1 << 20, device=-1)


@pytest.mark.parametrize("seed", range(6))
def test_policy_matches_oracle_replay_on_random_traces(seed):
    rng = random.Random(seed)
    L, E, C = rng.choice([(1, 8, 3), (3, 16, 5), (2, 64, 16), (4, 32, 8)])
    lib = _policy_cache(L, E, C)
    ref = LRUReplay(L, E, C)
    zipf = [1.0 / (i + 1) ** 1.1 for i in range(E)]
    for step in range(60):
        layer = rng.randrange(L)
        n = rng.randint(0, 2 * C)  # sometimes more than the capacity: waves
        experts = [rng.choices(range(E), weights=zipf)[0] for _ in range(n)]
        if rng.random() < 0.35:
            lib.prefetch(layer, experts)
            ref.prefetch(layer, experts)
        else:
            lib.lookup(layer, experts, None)
            ref.lookup(layer, experts)
        got = lib.stats()
        assert {k: got[k] for k in STAT_KEYS} == ref.stats, (step, layer, experts)
        for l in range(L):
            assert lib.slot_map(l) == ref.slot_map(l)
    lib.close()


def test_policy_mode_validates_expert_ids():
    lib = _policy_cache(2, 8, 3)
    with pytest.raises(moe.MoeError):
        lib.lookup(0, [8], None)
    with pytest.raises(moe.MoeError):
        lib.prefetch(2, [1])
    assert lib.host_expert(0, 0) is None and lib.slot_base(0) is None
    lib.close()
