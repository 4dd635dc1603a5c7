"""bench.py's per-kernel sampling (host logic): which timed steps carry CUDA
events, and the launch count of the timed region scaled up from them."""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import bench  # noqa: E402


def test_long_runs_sample_sparsely_short_runs_every_step():
    assert bench.profile_every(2000) == 50
    assert bench.profile_every(500) == 50
    assert bench.profile_every(499) == 10
    assert bench.profile_every(100) == 10
    assert bench.profile_every(99) == 1
    assert bench.profile_every(3) == 1


def test_every_long_run_keeps_at_least_ten_samples():
    for steps in (100, 250, 499, 500, 1000, 2000, 5000):
        every = bench.profile_every(steps)
        sampled = [i for i in range(steps) if i > 0 and i % every == 0]
        assert len(sampled) >= 9, steps


def test_launch_count_scales_from_the_sampled_steps():
    # five launches per layer call, recorded on the sampled steps only
    for steps in (7, 120, 1000, 2000):
        every = bench.profile_every(steps)
        sampled = len([i for i in range(steps) if i > 0 and i % every == 0])
        prof = {"route_prep_small": (sampled, 1.0), "ffn_stage1_gate_up": (sampled, 1.0),
                "prep_h": (sampled, 1.0), "ffn_stage2_down": (sampled, 1.0), "combine": (sampled, 1.0)}
        assert bench.launches_per_step(prof, steps) == 5 * steps
