"""GPU: seeded random shapes against the oracle, both precisions.

Forty small cases drawn from one seeded generator: T, d, V, P, the stride,
the offset, the Zipf exponent, the ignored fraction and the upstream gradient
all vary, with ragged tails in every dimension. Every case is compared in
full (candidate set and positions bit-exact; loss, lse, dX, dW within the
stated tolerances).
"""

import math

import numpy as np
import pytest

from oracle import sampled_ce as oc
from sampled_softmax_cross_b200 import workloads as wl

from gpu_common import compare_full, run_path

pytestmark = pytest.mark.gpu


def _case(i):
    rng = np.random.default_rng(1000 + i)
    e4m3 = i % 4 == 3
    d = int(rng.integers(1, 33)) * (16 if e4m3 else 8)
    V = int(rng.integers(300, 6000))
    stride = int(rng.choice([20011, 7, 101, 65537]))
    while math.gcd(stride, V) != 1:
        V += 1
    T = int(rng.integers(1, 700))
    s = float(rng.uniform(0.9, 1.4))
    x, lm, t = wl.make_inputs(T, d, V, s, float(rng.uniform(0, 0.3)), 1000 + i)
    D = np.unique(t[t >= 0]).size
    P = int(rng.integers(max(D, 1), V + 1))
    off = int(rng.integers(0, 4 * V))
    grad = float(rng.choice([1.0, 0.5, 3.0]))
    return x, lm, t, P, off, stride, grad, e4m3


@pytest.mark.parametrize("i", range(40))
def test_random_shape_matches_oracle(i):
    x, lm, t, P, off, stride, grad, e4m3 = _case(i)
    g = run_path(x, lm, t, P, off, stride=stride, grad=grad,
                 precision="e4m3" if e4m3 else "bf16")
    fn = oc.sampled_ce_e4m3 if e4m3 else oc.sampled_ce
    o = fn(wl.bits_to_f64(x), wl.bits_to_f64(lm), t, P, off, stride, grad_loss=grad)
    compare_full(g, o, t)
