"""Host logic of the per-step candidate count and the per-rank sweep.

sampled_softmax.py: CANDIDATES_BY_STAGE and candidate_count_at (count of each
step), CandidateBuilder.reset (rank r of N starts its sweep at V * r // N)
and CandidateBuilder._negatives (each build moves the sweep past the window
it drew). The count schedule is pinned to the step ranges the page prints for
its default run; the sweep is pinned to the oracle's candidate builds chained
over steps.
"""

import json
import os

import numpy as np
import pytest

from oracle import sampled_ce as oc
from sampled_softmax_cross_b200 import schedule as sc
from sampled_softmax_cross_b200 import workloads as wl

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def test_default_run_counts_match_the_printed_ranges():
    g = json.load(open(os.path.join(GOLDEN, "schedule_default_run.json")))
    b = [tuple(x) for x in g["boundaries"]]
    for r in g["ranges"]:
        got = {sc.candidate_count_at(b, s) for s in range(r["first"], r["last"] + 1)}
        assert got == {r["P"]}, (r, got)


def test_workload_steps_fall_in_their_stage_counts():
    b = [tuple(x) for x in json.load(open(os.path.join(GOLDEN, "schedule_default_run.json")))["boundaries"]]
    for name in ("stage0", "stage2_early", "stage2_late"):
        w = wl.WORKLOADS[name]
        assert sc.candidate_count_at(b, w.step) == w.P, name


def test_count_splits_stage_into_equal_parts():
    b = [(0, 10), (10, 19)]
    counts = {1: (4, 5, 6)}
    got = [sc.candidate_count_at(b, s, counts) for s in range(10, 19)]
    assert got == [4, 4, 4, 5, 5, 5, 6, 6, 6]
    assert sc.candidate_count_at(b, 3, counts) == 0  # stage 0 not listed: full softmax
    assert sc.stage_index(b, 19) == 1 and sc.stage_index(b, 500) == 1


def test_sweep_reset_staggers_ranks():
    V = 50304
    assert [sc.NegativeSweep(V, r, 8).offset for r in range(8)] == [0, 6288, 12576, 18864,
                                                                   25152, 31440, 37728, 44016]
    s = sc.NegativeSweep(V, 3, 4)
    s.advance(1000)
    s.reset()
    assert s.offset == 37728
    with pytest.raises(ValueError):
        sc.NegativeSweep(V, 2, 2)


@pytest.mark.parametrize("rank,world", [(0, 1), (1, 2), (3, 4)])
def test_sweep_follows_chained_oracle_builds(rank, world):
    """Chaining the oracle's builds through NegativeSweep reproduces the
    oracle's own next-offset chain, including steps that draw nothing."""
    V, T = 5003, 700
    rng = np.random.default_rng(rank + 10 * world)
    sweep = sc.NegativeSweep(V, rank, world)
    off = (V * rank) // world
    for step, P in enumerate([900, 900, 1400, 0, 2000, 2000]):
        targets = rng.integers(-1, V, T)
        D = np.unique(targets[targets >= 0]).size
        P = P or D  # a step whose targets fill C exactly draws no window
        _, _, _, info = oc.build_candidates(targets, V, P, sweep.offset)
        assert sweep.offset == off
        sweep.advance(info["draw"])
        off = info["next_offset"]
        assert sweep.offset == off, step
    assert off != (V * rank) // world


def test_sweep_windows_of_consecutive_builds_abut():
    """With no targets, build j+1's negatives are the next sweep positions
    after build j's window: over V // draw builds no class repeats within the
    union of windows, and the union of windows tiles the sweep."""
    V, P = 1009, 40
    sweep = sc.NegativeSweep(V)
    seen = []
    draws = 0
    while draws + oc.window_length(P, V) <= V:
        cand, _, _, info = oc.build_candidates(np.full(3, -1), V, P, sweep.offset)
        seen.extend(cand.tolist())
        sweep.advance(info["draw"])
        draws += info["draw"]
    assert len(seen) == len(set(seen))
    assert sweep.offset == draws % V
