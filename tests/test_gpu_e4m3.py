"""GPU parity of the e4m3 logits variant against the oracle's e4m3 path.

* ss_quantize_e4m3: codes and scale bit-exact against the oracle's quantizer
  (OCP E4M3, nearest even, saturating; one power-of-two scale per tensor),
  over magnitudes that reach the subnormal codes, exact ties and zeros.
* ss_ce_forward_e4m3 + ss_ce_backward: candidate build bit-exact; loss, lse,
  dX and dW within the same tolerances as the bf16 path, against the oracle
  run on the same quantized operands (the only differences left are fp32
  accumulation order and the bf16 rounding of E); small ragged shapes in
  full, the headline workload on all rows (loss, lse) and sampled rows and
  columns (dX, dW); rows that take the exact fix-up path.
"""

import numpy as np
import pytest
import torch

from oracle import sampled_ce as oc
from sampled_softmax_cross_b200 import capi
from sampled_softmax_cross_b200 import workloads as wl

from gpu_common import (LOSS_ATOL, LOSS_RTOL, LSE_ATOL, check_grad, compare_full, dev_bf16,
                        run_path, sample_cols, sample_rows)

pytestmark = pytest.mark.gpu


def _quantize_gpu(bits):
    src = dev_bf16(bits.reshape(-1))
    dst = torch.empty(src.numel(), dtype=torch.uint8, device="cuda")
    scale = torch.zeros(1, dtype=torch.float32, device="cuda")
    scratch = torch.full((8,), 7, dtype=torch.int32, device="cuda")
    capi.ss_quantize_e4m3(src, dst, scale, scratch)
    torch.cuda.synchronize()
    return dst.cpu().numpy(), float(scale.item())


def _check_quantize(values):
    values = np.asarray(values, dtype=np.float32)
    values = np.concatenate([values, np.zeros(-values.size % 8, np.float32)])  # n % 8 == 0
    bits = wl.bf16_bits(values)
    codes, scale = _quantize_gpu(bits)
    o_codes, k, _ = oc.quantize_e4m3(wl.bits_to_f64(bits))
    assert scale == 2.0 ** k
    bad = np.flatnonzero(codes != o_codes.reshape(-1))
    assert bad.size == 0, (bad[:8], wl.bits_to_f64(bits).reshape(-1)[bad[:8]], codes[bad[:8]],
                           o_codes.reshape(-1)[bad[:8]])


@pytest.mark.parametrize("scale", [1e-3, 1.0, 37.0, 1e4])
def test_quantize_matches_oracle(scale):
    rng = np.random.default_rng(int(scale * 1000) % 9973)
    v = rng.standard_normal(40000) * scale
    v[:4000] *= 10.0 ** rng.uniform(-6, 0, 4000)  # down into the subnormal codes
    v[4000:4100] = 0.0
    _check_quantize(v)


def test_quantize_grid_points_ties_and_saturation():
    grid = np.array([oc.e4m3_decode(c) for c in range(256)])
    grid = grid[~np.isnan(grid)]
    pos = np.sort(grid[grid > 0])
    mids = (pos[:-1] + pos[1:]) / 2  # exact ties (representable in bf16)
    v = np.concatenate([grid, mids, -mids, [448.0]])  # amax 448: scale 2^0
    _check_quantize(v)
    _check_quantize(np.zeros(64))  # all zero: scale 1, codes 0


def _e4m3_oracle(x, lm, t, P, off, grad=1.0):
    return oc.sampled_ce_e4m3(wl.bits_to_f64(x), wl.bits_to_f64(lm), t, P, off, grad_loss=grad)


SMALL = [
    (512, 128, 50304, 2048, 0, 1.0),
    (1000, 208, 5003, 3000, 1, 1.0),
    (777, 144, 4099, 1001, 2, 2.5),
    (129, 16, 300, 257, 4, 0.5),
    (2048, 768, 20023, 4096, 5, 1.0),
]


@pytest.mark.parametrize("T,d,V,P,seed,grad", SMALL)
def test_e4m3_small_shapes_match_oracle(T, d, V, P, seed, grad):
    x, lm, t = wl.make_inputs(T, d, V, 1.1, 0.05, seed)
    assert np.unique(t[t >= 0]).size <= P
    off = (seed * 7919) % V
    g = run_path(x, lm, t, P, off, grad=grad, precision="e4m3")
    o = _e4m3_oracle(x, lm, t, P, off, grad)
    compare_full(g, o, t)
    # the quantization is visible: the bf16 path's loss differs
    ob = oc.sampled_ce(wl.bits_to_f64(x), wl.bits_to_f64(lm), t, P, off)
    assert abs(g["loss"] - ob["loss"]) > abs(g["loss"] - o["loss"])


def test_e4m3_one_k_block_forward_with_many_tiles():
    """d = 128: one 128-deep K block of e4m3 codes per forward tile (the
    dynamic tile schedule's producer furthest ahead), 1024 tiles."""
    T, d, V, P, seed = 8192, 128, 20000, 8192, 44
    x, lm, t = wl.make_inputs(T, d, V, 1.1, 0.05, seed)
    g = run_path(x, lm, t, P, 17, precision="e4m3")
    o = _e4m3_oracle(x, lm, t, P, 17)
    compare_full(g, o, t)


def test_e4m3_rows_with_huge_loss_are_recomputed_exactly():
    T, d, V, P, seed = 300, 64, 1000, 384, 21
    x, lm, t = wl.make_inputs(T, d, V, 1.1, 0.05, seed)
    xf = wl.bits_to_f32(x).copy()
    lmf = wl.bits_to_f32(lm)
    cand, _, _, _ = oc.build_candidates(t, V, P, 0)
    for i in (3, 77, 150):
        a = int(cand[(np.searchsorted(cand, t[i]) + 5) % P]) if t[i] >= 0 else int(cand[5])
        if t[i] < 0:
            t[i] = int(cand[0])
        diff = lmf[a] - lmf[t[i]]
        xf[i] = 60.0 * diff / (diff @ diff)
    x = wl.bf16_bits(xf)
    g = run_path(x, lm, t, P, 0, precision="e4m3")
    o = _e4m3_oracle(x, lm, t, P, 0)
    assert max(o["loss_rows"][[3, 77, 150]]) > 40
    compare_full(g, o, t)


def test_e4m3_headline_workload():
    w = wl.WORKLOADS["stage2_late"]
    x_bits, lm_bits, t = wl.workload_inputs(w)
    g = run_path(x_bits, lm_bits, t, w.P, w.offset, precision="e4m3")
    assert g["status"][0] == 0 and g["status"][8] == 0, g["status"]
    cand, tpos, vpos, _ = oc.build_candidates(t, w.V, w.P, w.offset)
    assert np.array_equal(g["candidates"], cand) and np.array_equal(g["target_pos"], tpos)

    x = wl.bits_to_f64(x_bits)
    w_c = oc.gather_rows(wl.bits_to_f64(lm_bits), cand)
    _, _, xq = oc.quantize_e4m3(x)
    _, _, wq = oc.quantize_e4m3(w_c)
    loss, lse, _, n = oc.sampled_ce_forward(xq, wq, tpos)
    assert g["n_valid"] == n
    assert abs(g["loss"] - loss) <= LOSS_RTOL * abs(loss) + LOSS_ATOL, (g["loss"], loss)
    assert np.max(np.abs(g["lse"] - lse)) <= LSE_ATOL

    rng = np.random.default_rng(w.seed + 200)
    scale = 1.0 / n
    rows = sample_rows(w.T, 512, rng)
    dx_o = oc.dx_rows(x[rows], w_c, tpos[rows], lse[rows], scale, logit_x_rows=xq[rows],
                      logit_w=wq)
    check_grad(wl.bits_to_f64(g["dx_bits"][rows]), dx_o, "dx rows")
    cols = sample_cols(w.P, tpos, 256, rng)
    dw_o = oc.dw_c_rows(x, w_c, tpos, lse, scale, cols, logit_x=xq, logit_w=wq)
    check_grad(wl.bits_to_f64(g["dW_bits"][cand[cols]]), dw_o, "dW rows")


def test_e4m3_stage0_compared_in_full():
    """stage0 at full size (T=16384, d=768, P=10240) in e4m3: every output
    against the oracle's e4m3 path -- codes, candidate set and positions bit
    for bit, loss, lse, and every element of dX and dW."""
    w = wl.WORKLOADS["stage0"]
    x, lm, t = wl.workload_inputs(w)
    g = run_path(x, lm, t, w.P, w.offset, precision="e4m3")
    o = _e4m3_oracle(x, lm, t, w.P, w.offset)
    compare_full(g, o, t)


def test_e4m3_empty_microbatch_and_full_vocabulary():
    lm = wl.bf16_bits(np.random.default_rng(0).standard_normal((512, 64), dtype=np.float32))
    g = run_path(np.zeros((0, 64), np.uint16), lm, np.zeros(0, np.int32), 100, 4,
                 precision="e4m3")
    assert g["loss"] == 0.0 and g["n_valid"] == 0 and np.all(g["dW_bits"] == 0)
    # P = V: C is the whole vocabulary, the e4m3 loss is the full CE on e4m3 logits
    x, lm, t = wl.make_inputs(300, 64, 777, 1.1, 0.05, 8)
    g = run_path(x, lm, t, 777, 0, precision="e4m3")
    o = _e4m3_oracle(x, lm, t, 777, 0)
    assert np.array_equal(o["candidates"], np.arange(777))
    compare_full(g, o, t)
