"""GPU: larger seeded random shapes against the oracle, sampled.

Six cases with T in [15000, 50000), d a multiple of 8 (of 16 in e4m3) up to
768, V in [20000, 120000) and P up to 30000: sizes where the backward GEMMs
pick 512-row tiles for some shapes and 256-row tiles for others, with ragged
tails in every dimension; every third case runs the e4m3 forward. Integers
are compared in full, loss and lse on every row, dX on rows from every
256-row tile and dW on candidate columns from every 256-column tile (plus
random ones), with the element-wise gradient bounds.
"""

import numpy as np
import pytest

from oracle import sampled_ce as oc
from sampled_softmax_cross_b200 import workloads as wl

from gpu_common import (LOSS_ATOL, LOSS_RTOL, LSE_ATOL, check_grad, run_path, sample_cols,
                        sample_rows)

pytestmark = pytest.mark.gpu


def _case(i):
    rng = np.random.default_rng(5000 + i)
    e4m3 = i % 3 == 2
    d = int(rng.integers(4, 49)) * (16 if e4m3 else 8)
    V = int(rng.integers(20000, 120000))
    T = int(rng.integers(15000, 50000))
    s = float(rng.uniform(1.0, 1.3))
    x, lm, t = wl.make_inputs(T, d, V, s, float(rng.uniform(0, 0.05)), 5000 + i)
    D = np.unique(t[t >= 0]).size
    P = int(rng.integers(max(D, 1), min(V, 30000) + 1))
    off = int(rng.integers(0, 4 * V))
    return x, lm, t, P, off, e4m3


@pytest.mark.parametrize("i", range(6))
def test_large_random_shape_matches_oracle(i):
    x, lm, t, P, off, e4m3 = _case(i)
    T, V = x.shape[0], lm.shape[0]
    g = run_path(x, lm, t, P, off, precision="e4m3" if e4m3 else "bf16")
    assert g["status"][0] == 0 and g["status"][8] == 0, g["status"]
    cand, tpos, vpos, _ = oc.build_candidates(t, V, P, off)
    assert np.array_equal(g["candidates"], cand)
    assert np.array_equal(g["target_pos"], tpos)
    assert np.array_equal(g["vocab_pos"], vpos)
    x64 = wl.bits_to_f64(x)
    w_c = oc.gather_rows(wl.bits_to_f64(lm), cand)
    lx, lw = x64, w_c
    if e4m3:  # the logits come from the e4m3 codes; the gradient GEMMs stay bf16
        _, _, lx = oc.quantize_e4m3(x64)
        _, _, lw = oc.quantize_e4m3(w_c)
    loss, lse, _, n = oc.sampled_ce_forward(lx, lw, tpos)
    assert g["n_valid"] == n
    assert abs(g["loss"] - loss) <= LOSS_RTOL * abs(loss) + LOSS_ATOL, (g["loss"], loss)
    assert np.max(np.abs(g["lse"] - lse)) <= LSE_ATOL
    rng = np.random.default_rng(i)
    rows = sample_rows(T, 256, rng)
    dx_o = oc.dx_rows(x64[rows], w_c, tpos[rows], lse[rows], 1.0 / n, logit_x_rows=lx[rows],
                      logit_w=lw)
    check_grad(wl.bits_to_f64(g["dx_bits"][rows]), dx_o, "dx rows")
    cols = sample_cols(P, tpos, 128, rng)
    dw_o = oc.dw_c_rows(x64, w_c, tpos, lse, 1.0 / n, cols, logit_x=lx, logit_w=lw)
    check_grad(wl.bits_to_f64(g["dW_bits"][cand[cols]]), dw_o, "dW rows")
    in_c = np.zeros(V, bool)
    in_c[cand] = True
    assert np.all(g["dW_bits"][~in_c] == 0)
    assert np.all(g["dx_bits"][tpos < 0] == 0)
