"""GPU: prefix-target positions, the per-step driver, and the bounded-wait failure path.

* ss_prefix_positions against the oracle, bit for bit (sampled_softmax.py,
  CandidateBuilder.build: prefix target -> position in C, -1 if absent).
* SampledSoftmaxSteps over several steps whose count changes (and ends on the
  full softmax, P = V): every step's candidate set must equal the oracle's
  build at the offset the oracle's own previous build left (CandidateBuilder
  .reset / ._negatives), and the loss and gradients must match the oracle.
* ss_selftest_wait_limit: a kernel wait that nothing completes must end with
  SS_ERR_KERNEL_TIMEOUT in the status words after its time limit, the other
  warp must leave through the abort flag, and the context must stay usable
  (a full path runs and matches the oracle afterwards).
"""

import numpy as np
import pytest
import torch

from oracle import sampled_ce as oc
from sampled_softmax_cross_b200 import capi
from sampled_softmax_cross_b200 import schedule as sc
from sampled_softmax_cross_b200 import workloads as wl

from gpu_common import (LOSS_RTOL, LSE_ATOL, check_grad, compare_full, dev_bf16,
                        run_build, run_path)

pytestmark = pytest.mark.gpu


def _i32(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).cuda()


def _gpu_prefix(table, targets, vocab_pos, V):
    pp = torch.full((max(targets.size, 1),), -7, dtype=torch.int32, device="cuda")
    st = torch.zeros(capi.DEV_STATUS_WORDS, dtype=torch.int32, device="cuda")
    capi.ss_prefix_positions(_i32(table), _i32(targets), _i32(vocab_pos), V, pp, st)
    torch.cuda.synchronize()
    return pp[:targets.size].cpu().numpy(), st.tolist()


@pytest.mark.parametrize("kind", ["small", "stage2_late"])
def test_prefix_positions_match_oracle(kind):
    rng = np.random.default_rng(21)
    if kind == "small":
        V, P, off = 1009, 900, 5
        targets = rng.integers(-1, V, 1500).astype(np.int32)
        targets = np.where(np.isin(targets, np.unique(targets)[:780]) | (targets < 0), targets, -1)
    else:
        w = wl.WORKLOADS[kind]
        V, P, off = w.V, w.P, w.offset
        _, _, targets = wl.workload_inputs(w)
    table = rng.integers(-1, V, V).astype(np.int32)
    table[rng.random(V) < 0.1] = -1
    cand, tpos, vpos, st = run_build(targets, V, P, off)
    assert st[0] == 0
    got, st2 = _gpu_prefix(table, targets, vpos, V)
    want = oc.prefix_positions(table, targets, oc.build_candidates(targets, V, P, off)[2])
    assert st2[8] == 0
    assert np.array_equal(got, want)
    hit = got >= 0
    assert hit.any() and (~hit & (targets >= 0)).any()
    assert np.array_equal(cand[got[hit]], table[targets[hit]])


def test_prefix_positions_report_bad_entries():
    V, P = 100, 60
    rng = np.random.default_rng(3)
    targets = rng.integers(-1, 40, 300).astype(np.int32)
    targets[5] = 7
    table = rng.integers(-1, V, V).astype(np.int32)
    table[7] = 150  # outside [-1, V)
    _, _, vpos, st = run_build(targets, V, P, 0)
    assert st[0] == 0
    got, st2 = _gpu_prefix(table, targets, vpos, V)
    assert st2[8] == capi.STATUS["SS_ERR_BAD_INDEX"] and st2[9] == 2
    clean = table.copy()
    clean[7] = -1
    want = oc.prefix_positions(clean, targets, vpos)
    assert np.array_equal(got, want)
    assert np.all(got[targets == 7] == -1)


def test_prefix_positions_empty_microbatch():
    got, st = _gpu_prefix(np.zeros(10, np.int32), np.zeros(0, np.int32), np.zeros(10, np.int32), 10)
    assert got.size == 0 and st[8] == 0


def test_steps_driver_chains_the_sweep_across_counts():
    T, d, V = 640, 128, 5003
    boundaries = [(0, 3), (3, 7), (7, 9)]
    counts = {0: (1024,), 1: (1536, 2048)}  # stage 2: full softmax
    x_bits, lm_bits, _ = wl.make_inputs(T, d, V, 1.1, 0.05, 30)
    x, lm = dev_bf16(x_bits), dev_bf16(lm_bits)
    x64, lm64 = wl.bits_to_f64(x_bits), wl.bits_to_f64(lm_bits)
    drv = sc.SampledSoftmaxSteps(boundaries, T, d, V, rank=1, world=2, counts_by_stage=counts)
    rng = np.random.default_rng(31)
    off = V // 2
    seen_p = []
    for step in range(9):
        targets = wl.zipf_targets(rng, V, T, 1.1).astype(np.int32)
        targets[rng.random(T) < 0.05] = -1
        ce = drv.step(step, _i32(targets), x, lm)
        torch.cuda.synchronize()
        P = sc.candidate_count_at(boundaries, step, counts) or V
        seen_p.append(P)
        assert ce.P == P
        o = oc.sampled_ce(x64, lm64, targets, P, off)
        st = ce.status()
        assert st[0] == 0 and st[8] == 0, st
        assert np.array_equal(ce.candidates.cpu().numpy(), o["candidates"]), step
        assert np.array_equal(ce.target_pos[:T].cpu().numpy(), o["target_pos"]), step
        assert st[5] == o["info"]["next_offset"]
        loss = float(ce.loss.item())
        assert abs(loss - o["loss"]) <= LOSS_RTOL * abs(o["loss"]), (step, loss, o["loss"])
        assert np.max(np.abs(ce.lse[:T].cpu().numpy() - o["lse"])) <= LSE_ATOL
        dx = wl.bits_to_f64(ce.dx[:T].view(torch.int16).cpu().numpy().view(np.uint16))
        check_grad(dx, o["dx"], f"dx step {step}")
        off = o["info"]["next_offset"]
    drv.settle()
    assert drv.sweep.offset == off
    assert seen_p == [1024, 1024, 1024, 1536, 1536, 2048, 2048, V, V]
    drv.reset()
    assert drv.sweep.offset == V // 2


def test_wait_limit_selftest_reports_timeout_and_context_survives():
    st = torch.zeros(capi.DEV_STATUS_WORDS, dtype=torch.int32, device="cuda")
    capi.ss_selftest_wait_limit(st)
    torch.cuda.synchronize()
    s = st.tolist()
    assert s[8] == capi.STATUS["SS_ERR_KERNEL_TIMEOUT"] and s[9] == 107, s
    assert s[10] == 1, s  # the second warp left through the abort flag
    assert 1900 <= s[11] <= 3000, s  # the first warp waited out its 2 s limit
    # first error wins: a second run leaves [8..9] as they are
    capi.ss_selftest_wait_limit(st)
    torch.cuda.synchronize()
    assert st.tolist()[8:10] == [s[8], s[9]]
    # the context is still usable: a full path matches the oracle
    x, lm, t = wl.make_inputs(700, 128, 3001, 1.1, 0.05, 41)
    g = run_path(x, lm, t, 1200, 9)
    o = oc.sampled_ce(wl.bits_to_f64(x), wl.bits_to_f64(lm), t, 1200, 9)
    compare_full(g, o, t)
