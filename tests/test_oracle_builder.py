"""Pins for the oracle's candidate-set build (sampled_softmax.py, CandidateBuilder).

Each test checks the oracle against something other than itself: hand-worked
fixtures, a brute-force walk written with different arithmetic (repeated
addition instead of multiplication, Python sets instead of bitmaps), the
permutation property of the stride sweep, and invariants of the result.
"""

import json
import math
import os
import random

import numpy as np
import pytest

from oracle import sampled_ce as oc
from sampled_softmax_cross_b200 import workloads as wl

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _load(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


# --------------------------------------------------------------------------
# brute force: walk the sweep one position at a time with Python ints
# --------------------------------------------------------------------------


def brute_build(targets, V, P, offset, stride):
    """The page's definition with plain Python loops and sets.

    The sweep class is advanced by repeated addition of ``stride`` (mod V),
    never by multiplication; the window length uses integer tenths.
    """
    present = set(t for t in targets if t != -1)
    D = len(present)
    assert D <= P
    need = P - D
    chosen = []
    draw = 0
    fallback = False
    if need:
        draw = min(V, (need * 17) // 10 + 256)
        # class at position ``offset`` by repeated addition from position 0
        cls = 0
        for _ in range(offset % V):
            cls = (cls + stride) % V
        survivors = []
        for _ in range(draw):
            if cls not in present:
                survivors.append(cls)
            cls = (cls + stride) % V
        if len(survivors) >= need:
            chosen = survivors[:need]
        else:
            fallback = True
            free = [c for c in range(V) if c not in present]
            step = max(1, len(free) // need)
            chosen = [free[i] for i in range(0, len(free), step)][:need]
    cset = sorted(present | set(chosen))
    vpos = {c: j for j, c in enumerate(cset)}
    tpos = [vpos[t] if t != -1 else -1 for t in targets]
    return cset, tpos, dict(D=D, need=need, draw=draw, used_fallback=fallback,
                            next_offset=(offset % V + draw) % V)


def _check_same(targets, V, P, offset, stride):
    cand, tpos, vpos, info = oc.build_candidates(np.array(targets), V, P, offset, stride)
    bc, bt, binfo = brute_build(list(targets), V, P, offset, stride)
    assert cand.tolist() == bc
    assert tpos.tolist() == bt
    assert info == binfo
    expect_vpos = [-1] * V
    for j, c in enumerate(bc):
        expect_vpos[c] = j
    assert vpos.tolist() == expect_vpos
    return info


# --------------------------------------------------------------------------


def test_stride_sweep_is_a_permutation():
    V = wl.VOCAB
    assert math.gcd(oc.NEGATIVE_STRIDE, V) == 1
    s = oc.stride_class(np.arange(V), V)
    assert np.array_equal(np.sort(s), np.arange(V))


def test_stride_class_matches_repeated_addition():
    V, stride = wl.VOCAB, oc.NEGATIVE_STRIDE
    k = np.arange(3 * V + 17)
    s = oc.stride_class(k, V, stride)
    cls = 0
    for i in range(k.size):
        assert s[i] == cls
        cls = (cls + stride) % V


@pytest.mark.parametrize("case", _load("builder_hand_worked.json")["cases"], ids=lambda c: c["name"])
def test_hand_worked_fixtures(case):
    V, P = case["V"], case["P"]
    if "targets" in case:
        targets = np.array(case["targets"])
    else:
        keep = [c for c in range(V) if c not in set(case["targets_all_except"])]
        targets = np.array(keep + [-1] * case["targets_extra_ignored"])
    cand, tpos, vpos, info = oc.build_candidates(targets, V, P, case["offset"], case["stride"])
    if "candidates" in case:
        assert cand.tolist() == case["candidates"]
    else:
        assert cand.tolist() == [c for c in range(V) if c not in set(case["candidates_all_except"])]
    if "vocab_pos" in case:
        assert vpos.tolist() == case["vocab_pos"]
    if "target_pos" in case:
        assert tpos.tolist() == case["target_pos"]
    for key in ("D", "need", "draw", "used_fallback", "next_offset"):
        assert info[key] == case[key], key


@pytest.mark.parametrize("V,stride", [(7, 3), (13, 5), (101, 20011), (263, 2)])
def test_brute_force_tiny_random(V, stride):
    rng = random.Random(V * 1000 + stride)
    for _ in range(150):
        T = rng.randint(0, 3 * V)
        targets = [rng.randrange(-1, V) for _ in range(T)]
        D = len(set(t for t in targets if t != -1))
        P = rng.randint(max(1, D), V)
        offset = rng.randrange(0, 5 * V)
        _check_same(targets, V, P, offset, stride)


@pytest.mark.parametrize("V,stride", [(1009, 20011), (2003, 7), (50304, 20011)])
def test_brute_force_forced_fallback(V, stride):
    """Targets packed into the front of the window force the fallback branch."""
    rng = random.Random(V)
    hits = 0
    for trial in range(12):
        offset = rng.randrange(V)
        need = rng.randint(1, 40)
        draw = min(V, (need * 17) // 10 + 256)
        # mark all but a few window positions, so the window runs dry
        keep_free = rng.randint(0, need - 1)
        window = [(stride * ((offset + k) % V)) % V for k in range(draw)]
        free_in_window = set(rng.sample(window, keep_free))
        targets = [c for c in window if c not in free_in_window]
        targets += [rng.randrange(V) for _ in range(rng.randint(0, 50))]
        D = len(set(targets))
        P = min(V, D + need)
        rng.shuffle(targets)
        info = _check_same(targets, V, P, offset, stride)
        hits += info["used_fallback"]
    assert hits >= 8


def test_window_integer_form_matches_float_form():
    # The device computes draw with integer tenths; the page uses int(need * 1.7).
    need = np.arange(0, 1 << 20)
    float_form = (need * 1.7).astype(np.int64)
    assert np.array_equal(float_form, (17 * need) // 10)
    for n in (0, 1, 9, 10, 11, 29440, 50304, (1 << 20) - 1):
        assert oc.window_length(n, 1 << 30) == (17 * n) // 10 + 256


@pytest.mark.parametrize("name", list(wl.WORKLOADS))
def test_invariants_on_workloads(name):
    w = wl.WORKLOADS[name]
    _, _, targets = wl.workload_inputs(w)
    cand, tpos, vpos, info = oc.build_candidates(targets, w.V, w.P, w.offset)
    V, P = w.V, w.P
    valid = targets >= 0
    assert cand.size == P
    assert np.all(np.diff(cand) > 0)
    assert np.isin(targets[valid], cand).all()
    assert np.array_equal(vpos[cand], np.arange(P))
    off = np.ones(V, bool)
    off[cand] = False
    assert np.all(vpos[off] == -1)
    assert np.array_equal(tpos[valid], vpos[targets[valid]])
    assert np.all(tpos[~valid] == -1)
    assert info["D"] == np.unique(targets[valid]).size
    if P == V:
        assert np.array_equal(cand, np.arange(V))
    negatives = np.setdiff1d(cand, targets[valid])
    assert negatives.size == info["need"]
    if not info["used_fallback"] and info["need"]:
        window = oc.stride_class(w.offset + np.arange(info["draw"]), V)
        assert np.isin(negatives, window).all()


def test_full_vocabulary_is_identity():
    V = 50304
    t = np.array([5, 5, -1, 50303, 0], dtype=np.int64)
    cand, tpos, vpos, info = oc.build_candidates(t, V, V, 12345)
    assert np.array_equal(cand, np.arange(V))
    assert np.array_equal(vpos, np.arange(V))
    assert tpos.tolist() == [5, 5, -1, 50303, 0]


def test_distinct_targets_fill_exactly():
    t = np.array([40, 3, 3, 17, -1, 40])
    cand, tpos, vpos, info = oc.build_candidates(t, 101, 3, 7, 20011)
    assert cand.tolist() == [3, 17, 40]
    assert info["draw"] == 0 and info["next_offset"] == 7


@pytest.mark.parametrize("targets,V,P,stride,code", [
    ([1, 2, 3], 7, 2, 3, "too_many_targets"),
    ([1, -2], 7, 3, 3, "bad_target"),
    ([1, 7], 7, 3, 3, "bad_target"),
    ([1], 7, 8, 3, "invalid_arg"),
    ([1], 7, 0, 3, "invalid_arg"),
    ([1], 8, 3, 2, "stride_not_coprime"),
    ([1], 50304, 3, 3, "stride_not_coprime"),
])
def test_rejections(targets, V, P, stride, code):
    with pytest.raises(oc.OracleError) as e:
        oc.build_candidates(np.array(targets), V, P, 0, stride)
    assert e.value.code == code


def test_empty_microbatch():
    cand, tpos, vpos, info = oc.build_candidates(np.zeros(0, np.int64), 50304, 2048, 99)
    assert info["D"] == 0 and info["need"] == 2048
    s = oc.stride_class(99 + np.arange(2048), 50304)
    assert np.array_equal(cand, np.sort(s))
    assert tpos.size == 0


def test_planted_window_mistake_is_caught(monkeypatch):
    """A wrong window start (offset + 1) in the oracle fails the fixtures."""
    orig = oc.pick_negatives

    def shifted(mark, need, offset, V, stride):
        return orig(mark, need, offset + 1, V, stride)

    monkeypatch.setattr(oc, "pick_negatives", shifted)
    case = _load("builder_hand_worked.json")["cases"][0]
    cand, _, _, _ = oc.build_candidates(np.array(case["targets"]), case["V"], case["P"],
                                        case["offset"], case["stride"])
    assert cand.tolist() != case["candidates"]
