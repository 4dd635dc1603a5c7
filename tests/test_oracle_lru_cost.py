"""Pins for the LRU replay (a hand-worked trace), for the decode cost model
(the numbers printed on the Galactus page) and for the verification-block
accounting (brute force over acceptance patterns, special cases)."""
import itertools
import json
import os

import numpy as np
import pytest

from oracle import cost
from oracle.lru import LRUReplay, replay

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "galactus_cost_model.json")


def test_lru_hand_worked_trace():
    # capacity 3, one layer of 6 experts; worked by hand step by step:
    # 1 lookup [0,1]: miss 0->s0, miss 1->s1
    # 2 lookup [1,2]: hit 1, miss 2->s2
    # 3 lookup [3]:   miss, LRU among {0,1,2} is 0 -> 3 takes s0 (evict 0)
    # 4 prefetch [0,4]: 0 evicts LRU 1 -> s1; 4 evicts LRU 2 -> s2
    # 5 lookup [0,3,5]: hit 0 (prefetched, used), hit 3, miss 5 evicts 4 -> s2
    r = replay([("lookup", 0, [1, 0]), ("lookup", 0, [2, 1]), ("lookup", 0, [3]),
                ("prefetch", 0, [4, 0]), ("lookup", 0, [5, 3, 0])], 1, 6, 3)
    assert r.stats == {"lookups": 8, "hits": 3, "misses": 5, "evictions": 4,
                       "prefetch_issued": 2, "prefetch_used": 1}
    assert r.slot_map(0) == [1, -1, -1, 0, -1, 2]
    assert r.copies == [(0, 0, 0), (0, 1, 1), (0, 2, 2), (0, 3, 0), (0, 0, 1), (0, 4, 2), (0, 5, 2)]


def test_lru_waves_when_need_exceeds_capacity():
    # need of 5 with 3 slots: wave [0,1,2] fills s0..s2; wave [3,4] evicts 0 then 1
    r = LRUReplay(2, 6, 3)
    r.lookup(1, [4, 3, 2, 1, 0])
    assert r.slot_map(1) == [-1, -1, 2, 0, 1, -1]
    assert r.stats["misses"] == 5 and r.stats["evictions"] == 2
    assert r.slot_map(0) == [-1] * 6  # other layers untouched


def test_lru_layers_are_independent_and_prefetch_of_resident_is_noop():
    r = LRUReplay(2, 4, 2)
    r.lookup(0, [0, 1])
    assert r.prefetch(0, [1]) == 0
    r.lookup(1, [2])
    assert r.slot_map(0) == [0, 1, -1, -1] and r.slot_map(1) == [-1, -1, 0, -1]
    assert r.stats["prefetch_issued"] == 0


def test_cost_model_reproduces_page_numbers():
    g = json.load(open(GOLDEN))
    for model, rate in g["decode_tokens_per_s"].items():
        row = g["rows_ms"][model]
        t_ms = round(1000.0 / rate)  # "The measured times are reciprocals of the August decode rates"
        assert t_ms == row["T"], model
        lo = cost.residual(row["T"], row["S"][1])
        hi = cost.residual(row["T"], row["S"][0])
        assert (lo, hi) == tuple(row["C"]), model
    k = g["kimi_traffic"]
    assert cost.streaming_time(k["bytes"], k["bandwidth"]) * 1000 == pytest.approx(k["S_ms_about"])
    w = g["glm_what_if"]
    assert cost.token_time(w["C_ms"], w["S_ms"], 1.0) == w["T_ms"]
    assert round(cost.tokens_per_second(w["T_ms"] / 1000.0), 2) == w["tok_s"]
    s_new = round(w["S_ms"] * (1 - w["traffic_cut"]))
    assert s_new == w["S_new_ms_about"]
    t_new = cost.token_time(w["C_ms"], s_new, 1.0)
    assert t_new == w["T_new_ms"]
    assert round(cost.tokens_per_second(t_new / 1000.0), 2) == w["tok_s_new"]
    assert round(w["tok_s_new"] / w["tok_s"] - 1, 2) == w["throughput_gain_about"]


def pin_expected_accepted(fn):
    """The closed form against brute force over every accept/reject pattern of
    the drafts (probability of each pattern times its output tokens), and the
    special cases: alpha = 0 is ordinary decode (one token), alpha = 1 accepts
    every draft."""
    for depth in range(0, 6):
        for alpha in (0.0, 0.3, 0.7, 0.95, 1.0):
            brute = 0.0
            for pat in itertools.product([0, 1], repeat=depth):
                p = np.prod([alpha if a else 1 - alpha for a in pat]) if depth else 1.0
                brute += p * cost.accepted_in_block(np.array(pat))
            if abs(fn(depth, alpha) - brute) > 1e-12:
                return False
        if fn(depth, 0.0) != 1.0 or fn(depth, 1.0) != depth + 1:
            return False
    return True


def test_expected_accepted_matches_brute_force():
    assert pin_expected_accepted(cost.expected_accepted)


def test_accepted_in_block_and_union():
    assert cost.accepted_in_block(np.array([1, 1, 0, 1])) == 3  # stops at the first rejection
    assert cost.accepted_in_block(np.array([0, 1, 1])) == 1
    assert cost.accepted_in_block(np.array([], dtype=bool)) == 1
    assert cost.expert_union(np.array([[3, 1], [1, 7], [3, 7]])) == 3
    assert cost.bytes_per_accepted_token(300.0, 2.5) == 120.0


def test_verification_pins_reject_planted_mistakes():
    # one draft too few in the sum, and acceptance that does not stop at a rejection
    assert not pin_expected_accepted(lambda d, a: float(sum(a ** i for i in range(d))))
    assert not pin_expected_accepted(lambda d, a: 1.0 + d * a)


def test_library_verification_accounting_matches_oracle():
    """The package's verification-block counters against the oracle's pinned ones."""
    from expert_ffn_layer_route_b200 import verify as V
    rng = np.random.default_rng(9)
    for _ in range(200):
        depth = int(rng.integers(0, 7))
        flags = rng.random(depth) < 0.6
        assert V.accepted_tokens(flags.tolist()) == cost.accepted_in_block(flags)
        alpha = float(rng.random())
        assert V.expected_accepted_tokens(depth, alpha) == pytest.approx(cost.expected_accepted(depth, alpha),
                                                                         rel=1e-14)
    assert V.bytes_per_accepted_token(300.0, 2.5) == cost.bytes_per_accepted_token(300.0, 2.5)
