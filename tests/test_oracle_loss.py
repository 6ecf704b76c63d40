"""Pins for the oracle's loss and gradients.

Pinned against: a library full-softmax cross-entropy when P = V, the closed
form for uniform logits (log P; the handout's log 5 example), invariance to a
per-row logit shift, a pure-Python math.fsum evaluation, central finite
differences, torch.autograd in float64, the token-weighted split across
microbatches, and the zero patterns and sum identities of the gradients.
Planted mistakes in the oracle (a dropped one-hot term, a
flipped sign, a mean over all rows) must each fail one of these checks.
"""

import json
import math
import os

import numpy as np
import pytest
import torch

from oracle import sampled_ce as oc

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def small_case(T=12, d=6, V=40, P=16, seed=0, n_ignored=3, offset=5):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((T, d))
    lm = rng.standard_normal((V, d)) / math.sqrt(d)
    targets = rng.integers(0, V, T)
    if n_ignored:
        targets[rng.choice(T, n_ignored, replace=False)] = -1
    D = np.unique(targets[targets >= 0]).size
    P = max(P, D)
    return x, lm, targets, P, offset


def loss_of(x, lm, targets, P, offset, stride=20011):
    """Scalar loss with C held fixed (C depends on the targets only)."""
    cand, tpos, vpos, _ = oc.build_candidates(targets, lm.shape[0], P, offset, stride)
    loss, _, _, _ = oc.sampled_ce_forward(x, oc.gather_rows(lm, cand), tpos)
    return loss


def test_full_vocabulary_equals_library_cross_entropy():
    x, lm, targets, _, _ = small_case(T=64, d=16, V=200, seed=1, n_ignored=9)
    V = lm.shape[0]
    out = oc.sampled_ce(x, lm, targets, V, offset=123)
    logits = torch.from_numpy(x @ lm.T)
    ref = torch.nn.functional.cross_entropy(logits, torch.from_numpy(targets).long(),
                                            ignore_index=-1)
    assert out["loss"] == pytest.approx(ref.item(), rel=1e-13)
    lse_ref = torch.logsumexp(logits, dim=1).numpy()
    np.testing.assert_allclose(out["lse"], lse_ref, rtol=1e-13)


def test_uniform_logits_give_log5_golden():
    g = json.load(open(os.path.join(GOLDEN, "loss_uniform_log5.json")))
    T = len(g["targets"])
    x = np.zeros((T, g["d"]))
    rng = np.random.default_rng(0)
    lm = rng.standard_normal((g["V"], g["d"]))
    out = oc.sampled_ce(x, lm, np.array(g["targets"]), g["P"])
    assert out["n_valid"] == g["n_valid"]
    assert math.isclose(out["loss"], g["loss"], rel_tol=1e-12)


@pytest.mark.parametrize("P", [3, 16, 40])
def test_zero_input_closed_form(P):
    x, lm, targets, P0, offset = small_case(T=10, d=5, V=40, seed=2, n_ignored=2)
    P = max(P, np.unique(targets[targets >= 0]).size)
    x = np.zeros_like(x)
    gl = 0.75
    out = oc.sampled_ce(x, lm, targets, P, offset, grad_loss=gl)
    assert math.isclose(out["loss"], math.log(P), rel_tol=1e-14)
    n = out["n_valid"]
    tpos = out["target_pos"]
    z = np.zeros((x.shape[0], P))
    G = oc.dlogits(z, out["lse"], tpos, gl / n)
    expect = np.full_like(G, gl / n / P)
    for i, t in enumerate(tpos):
        if t < 0:
            expect[i] = 0
        else:
            expect[i, t] -= gl / n
    np.testing.assert_allclose(G, expect, rtol=1e-13, atol=1e-16)


def test_row_shift_invariance():
    x, lm, targets, P, offset = small_case(T=9, d=4, V=30, seed=3)
    base = oc.sampled_ce(x, lm, targets, P, offset)
    c = np.linspace(-7.0, 9.0, x.shape[0])
    xa = np.concatenate([x, c[:, None]], axis=1)
    lma = np.concatenate([lm, np.ones((lm.shape[0], 1))], axis=1)
    shifted = oc.sampled_ce(xa, lma, targets, P, offset)
    assert shifted["loss"] == pytest.approx(base["loss"], rel=1e-12)
    np.testing.assert_allclose(shifted["lse"] - c, base["lse"], rtol=1e-12)
    np.testing.assert_allclose(shifted["dx"][:, :-1], base["dx"], rtol=1e-9, atol=1e-14)


def test_fsum_brute_force():
    x, lm, targets, P, offset = small_case(T=7, d=5, V=25, seed=4, n_ignored=2)
    out = oc.sampled_ce(x, lm, targets, P, offset)
    cand, tpos = out["candidates"], out["target_pos"]
    total, n = [], 0
    for i in range(x.shape[0]):
        z = [math.fsum(x[i, k] * lm[c, k] for k in range(x.shape[1])) for c in cand]
        lse = math.log(math.fsum(math.exp(v) for v in z))
        assert out["lse"][i] == pytest.approx(lse, rel=1e-13)
        if tpos[i] >= 0:
            total.append(lse - z[tpos[i]])
            n += 1
    assert out["loss"] == pytest.approx(math.fsum(total) / n, rel=1e-13)


def test_token_weighted_split_matches_whole():
    x, lm, targets, P, offset = small_case(T=20, d=6, V=50, seed=5, n_ignored=6)
    whole = oc.sampled_ce(x, lm, targets, P, offset)
    cand, tpos = whole["candidates"], whole["target_pos"]
    w_c = oc.gather_rows(lm, cand)
    n_total = int((tpos >= 0).sum())
    parts = []
    for sl in (slice(0, 3), slice(3, 20)):
        _, _, rows, _ = oc.sampled_ce_forward(x[sl], w_c, tpos[sl])
        parts.append(rows.sum() / n_total)
    assert sum(parts) == pytest.approx(whole["loss"], rel=1e-13)


def _finite_difference_check(oracle_mod, seed=6):
    x, lm, targets, P, offset = small_case(T=8, d=5, V=20, P=12, seed=seed, n_ignored=2)
    gl = 1.3
    V = lm.shape[0]
    cand, tpos, vpos, _ = oracle_mod.build_candidates(targets, V, P, offset)
    w_c = oracle_mod.gather_rows(lm, cand)
    _, lse, _, _ = oracle_mod.sampled_ce_forward(x, w_c, tpos)
    dx, dW = oracle_mod.sampled_ce_backward(gl, x, w_c, cand, tpos, lse, V)
    h = 1e-6
    num_dx = np.zeros_like(x)
    for idx in np.ndindex(*x.shape):
        xp, xm = x.copy(), x.copy()
        xp[idx] += h
        xm[idx] -= h
        num_dx[idx] = gl * (loss_of(xp, lm, targets, P, offset) - loss_of(xm, lm, targets, P, offset)) / (2 * h)
    num_dW = np.zeros_like(lm)
    for idx in np.ndindex(*lm.shape):
        lp, lmn = lm.copy(), lm.copy()
        lp[idx] += h
        lmn[idx] -= h
        num_dW[idx] = gl * (loss_of(x, lp, targets, P, offset) - loss_of(x, lmn, targets, P, offset)) / (2 * h)
    err_x = np.abs(dx - num_dx).max() / np.abs(num_dx).max()
    err_w = np.abs(dW - num_dW).max() / np.abs(num_dW).max()
    return err_x, err_w


def test_finite_differences():
    err_x, err_w = _finite_difference_check(oc)
    assert err_x < 1e-6 and err_w < 1e-6, (err_x, err_w)


def test_torch_autograd_float64():
    x, lm, targets, P, offset = small_case(T=10, d=7, V=30, P=14, seed=7, n_ignored=3)
    gl = 0.6
    out = oc.sampled_ce(x, lm, targets, P, offset, grad_loss=gl)
    cand = torch.from_numpy(out["candidates"])
    xt = torch.from_numpy(x).requires_grad_(True)
    lmt = torch.from_numpy(lm).requires_grad_(True)
    logits = xt @ lmt[cand].T
    tp = torch.from_numpy(out["target_pos"])
    loss = torch.nn.functional.cross_entropy(logits, tp, ignore_index=-1)
    (gl * loss).backward()
    assert out["loss"] == pytest.approx(loss.item(), rel=1e-13)
    np.testing.assert_allclose(out["dx"], xt.grad.numpy(), rtol=1e-11, atol=1e-15)
    np.testing.assert_allclose(out["dW"], lmt.grad.numpy(), rtol=1e-11, atol=1e-15)


def test_gradient_invariants():
    x, lm, targets, P, offset = small_case(T=30, d=8, V=64, P=24, seed=8, n_ignored=7)
    out = oc.sampled_ce(x, lm, targets, P, offset)
    cand, tpos = out["candidates"], out["target_pos"]
    w_c = oc.gather_rows(lm, cand)
    z = x @ w_c.T
    G = oc.dlogits(z, out["lse"], tpos, 1.0 / out["n_valid"])
    np.testing.assert_allclose(G.sum(axis=1), 0.0, atol=1e-15)
    assert np.all(G[tpos < 0] == 0)
    assert np.all(out["dx"][tpos < 0] == 0)
    off = np.ones(lm.shape[0], bool)
    off[cand] = False
    assert np.all(out["dW"][off] == 0)
    np.testing.assert_allclose(out["dW"][cand].sum(axis=0), 0.0, atol=1e-14)


def test_all_ignored_gives_zero():
    x, lm, _, _, _ = small_case(T=6, d=4, V=20)
    targets = np.full(6, -1)
    out = oc.sampled_ce(x, lm, targets, 8, 3)
    assert out["loss"] == 0.0 and out["n_valid"] == 0
    assert np.all(out["dx"] == 0) and np.all(out["dW"] == 0)


def test_row_and_column_samples_match_whole():
    x, lm, targets, P, offset = small_case(T=40, d=6, V=80, P=30, seed=9, n_ignored=5)
    gl = 0.9
    out = oc.sampled_ce(x, lm, targets, P, offset, grad_loss=gl)
    w_c = oc.gather_rows(lm, out["candidates"])
    rows = np.array([0, 7, 39])
    lse_r, loss_r = oc.rows_forward(x[rows], w_c, out["target_pos"][rows])
    np.testing.assert_allclose(lse_r, out["lse"][rows], rtol=1e-14)
    np.testing.assert_allclose(loss_r, out["loss_rows"][rows], rtol=1e-14)
    scale = gl / out["n_valid"]
    np.testing.assert_allclose(oc.dx_rows(x[rows], w_c, out["target_pos"][rows], out["lse"][rows], scale),
                               out["dx"][rows], rtol=1e-12, atol=1e-16)
    cols = np.array([0, 5, 29])
    np.testing.assert_allclose(oc.dw_c_rows(x, w_c, out["target_pos"], out["lse"], scale, cols, chunk=7),
                               out["dW"][out["candidates"][cols]], rtol=1e-12, atol=1e-16)


# ---- planted mistakes: each must fail a pin ---------------------------------


def test_planted_dropped_onehot_fails_finite_differences(monkeypatch):
    def no_onehot(z, lse, target_pos, scale):
        g = np.exp(z - lse[:, None])
        g[np.asarray(target_pos) < 0] = 0.0
        return scale * g

    monkeypatch.setattr(oc, "dlogits", no_onehot)
    err_x, err_w = _finite_difference_check(oc)
    assert err_x > 1e-2 or err_w > 1e-2


def test_planted_sign_flip_fails_finite_differences(monkeypatch):
    orig = oc.sampled_ce_backward

    def wrong_sign(*a, **k):
        dx, dW = orig(*a, **k)
        return -dx, dW

    monkeypatch.setattr(oc, "sampled_ce_backward", wrong_sign)
    err_x, _ = _finite_difference_check(oc)
    assert err_x > 1.0


def test_planted_mean_over_all_rows_fails_library_check(monkeypatch):
    orig = oc.sampled_ce_forward

    def all_rows(x, w_c, target_pos, chunk=1024):
        loss, lse, rows, n = orig(x, w_c, target_pos, chunk)
        return float(rows.sum() / len(rows)), lse, rows, n

    monkeypatch.setattr(oc, "sampled_ce_forward", all_rows)
    with pytest.raises(AssertionError):
        test_full_vocabulary_equals_library_cross_entropy()
