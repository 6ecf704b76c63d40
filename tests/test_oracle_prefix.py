"""Pins for the oracle's prefix-target positions (oracle.sampled_ce.prefix_positions).

sampled_softmax.py, module docstring and CandidateBuilder.build: the prefix
target of a token is prefix_table[target]; the loss receives its position in
C, or -1 when it is not in C ("no prefix", a class outside C, an ignored
token). Checked against hand-worked fixtures, a brute-force search of C for
every token, and the invariant that a prefix table never changes C.
"""

import json
import os

import numpy as np
import pytest

from oracle import sampled_ce as oc

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def brute_prefix(prefix_table, targets, candidates):
    """Position of each token's prefix class by a linear scan of C."""
    out = []
    for t in targets:
        p = -1 if t < 0 else int(prefix_table[t])
        pos = -1
        if p >= 0:
            for j, c in enumerate(candidates):
                if c == p:
                    pos = j
                    break
        out.append(pos)
    return np.array(out, dtype=np.int64)


@pytest.mark.parametrize("case", json.load(open(os.path.join(GOLDEN, "prefix_hand_worked.json")))["cases"],
                         ids=lambda c: c["name"])
def test_hand_worked_fixtures(case):
    cand, _, vpos, _ = oc.build_candidates(np.array(case["targets"]), case["V"], case["P"],
                                           case["offset"], case["stride"])
    got = oc.prefix_positions(np.array(case["prefix_table"]), np.array(case["targets"]), vpos)
    assert got.tolist() == case["prefix_pos"]


@pytest.mark.parametrize("seed", range(6))
def test_brute_force_tiny_random(seed):
    rng = np.random.default_rng(seed)
    V = int(rng.integers(5, 60))
    T = int(rng.integers(0, 40))
    targets = rng.integers(-1, V, T)
    D = np.unique(targets[targets >= 0]).size
    P = int(rng.integers(max(D, 1), V + 1))
    table = rng.integers(-1, V, V)
    cand, _, vpos, _ = oc.build_candidates(targets, V, P, int(rng.integers(0, 3 * V)), 1)
    got = oc.prefix_positions(table, targets, vpos)
    assert np.array_equal(got, brute_prefix(table, targets, cand))
    # where a position is given, C holds the token's prefix class there
    hit = got >= 0
    assert np.array_equal(cand[got[hit]], table[targets[hit]])


def test_prefix_table_never_changes_the_candidate_set():
    rng = np.random.default_rng(11)
    V, P = 1009, 400
    targets = rng.integers(-1, 300, 500)
    table = (np.arange(V) + 500) % V  # every prefix class lies outside the targets' range
    cand, _, vpos, _ = oc.build_candidates(targets, V, P, 17, 20011)
    got = oc.prefix_positions(table, targets, vpos)
    in_c = np.isin(table[targets[targets >= 0]], cand)
    assert np.array_equal(got[targets >= 0] >= 0, in_c)
    assert not in_c.all()  # some prefix classes are outside C and dropped
    cand2, _, _, _ = oc.build_candidates(targets, V, P, 17, 20011)
    assert np.array_equal(cand, cand2)


def test_rejections():
    vpos = np.array([0, -1, 1, -1])
    with pytest.raises(oc.OracleError) as e:
        oc.prefix_positions(np.array([0, 1, 4, 2]), np.array([2]), vpos)
    assert e.value.code == "bad_index"
    with pytest.raises(oc.OracleError) as e:
        oc.prefix_positions(np.array([0, 1, 2, 2]), np.array([4]), vpos)
    assert e.value.code == "bad_index"
    with pytest.raises(oc.OracleError):
        oc.prefix_positions(np.array([0, 1, 2]), np.array([1]), vpos)


def test_planted_sentinel_mistake_is_caught():
    """Dropping the 'no prefix' sentinel makes -1 wrap to the last class's position."""
    targets = np.array([0, 1, 2])
    table = np.array([-1, 2, 3, 1])
    vpos = np.array([0, 1, 2, 3])  # C = every class
    good = oc.prefix_positions(table, targets, vpos)
    planted = vpos[table[targets]]  # no sentinel: -1 indexes vpos[-1] = 3
    assert good.tolist() == [-1, 2, 3]
    assert not np.array_equal(planted, good)
    assert np.array_equal(good, brute_prefix(table, targets, np.arange(4)))
