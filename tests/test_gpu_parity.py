"""GPU parity: the CUDA path through the C ABI against the float64 oracle.

Small and ragged shapes are compared element by element with a full oracle
run. The five named workloads are run at full size in the launch
configuration the benchmark times: their integer outputs are compared in full;
stage0 (T=16384, P=10240) and the headline stage2_late (T=49152, P=24576) are
compared in full, every element of dX and dW included; the other two compare
loss and lse on all rows and dX / dW on rows and candidate columns sampled so
that every GEMM tile is hit, which the oracle computes one by one. The
gathered rows W_C are compared with lm_head[C] bit for bit.
"""

import json
import os

import numpy as np
import pytest
import torch

from oracle import sampled_ce as oc
from sampled_softmax_cross_b200 import capi
from sampled_softmax_cross_b200 import workloads as wl

from gpu_common import (LOSS_RTOL, LSE_ATOL, check_build, check_grad, compare_full,
                        dev_bf16, host_bits, run_build, run_path, sample_cols, sample_rows)

pytestmark = pytest.mark.gpu
GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def oracle_run(x_bits, lm_bits, targets, P, offset, stride=20011, grad=1.0):
    return oc.sampled_ce(wl.bits_to_f64(x_bits), wl.bits_to_f64(lm_bits), targets, P, offset,
                         stride, grad_loss=grad)


def random_case(T, d, V, P, seed, ignore_frac=0.05, zipf_s=1.1):
    x, lm, t = wl.make_inputs(T, d, V, zipf_s, ignore_frac, seed)
    D = np.unique(t[t >= 0]).size
    assert D <= P
    return x, lm, t


# ----------------------------------------------------------- candidate build --

@pytest.mark.parametrize("name", list(wl.WORKLOADS))
def test_builder_bit_exact_on_workloads(name):
    w = wl.WORKLOADS[name]
    _, _, targets = wl.workload_inputs(w)
    check_build(targets, w.V, w.P, w.offset)


@pytest.mark.parametrize("case", json.load(open(os.path.join(GOLDEN, "builder_hand_worked.json")))["cases"],
                         ids=lambda c: c["name"])
def test_builder_hand_worked(case):
    V = case["V"]
    if "targets" in case:
        t = np.array(case["targets"], np.int32)
    else:
        keep = [c for c in range(V) if c not in set(case["targets_all_except"])]
        t = np.array(keep + [-1] * case["targets_extra_ignored"], np.int32)
    info = check_build(t, V, case["P"], case["offset"], case["stride"])
    assert info["used_fallback"] == case["used_fallback"]


def test_builder_random_small_vocabularies():
    rng = np.random.default_rng(11)
    for V, stride in ((7, 3), (13, 5), (101, 20011), (263, 2), (1009, 20011), (5003, 20011)):
        for _ in range(6):
            T = int(rng.integers(0, 3 * V))
            t = rng.integers(-1, V, T).astype(np.int32)
            D = np.unique(t[t >= 0]).size
            P = int(rng.integers(max(1, D), V + 1))
            check_build(t, V, P, int(rng.integers(0, 4 * V)), stride)


@pytest.mark.parametrize("V", [1009, 50304])
def test_builder_forced_fallback(V):
    rng = np.random.default_rng(V)
    hits = 0
    for _ in range(6):
        off = int(rng.integers(V))
        need = int(rng.integers(1, 40))
        draw = min(V, (17 * need) // 10 + 256)
        window = oc.stride_class(off + np.arange(draw), V)
        keep_free = rng.choice(window, size=int(rng.integers(0, need)), replace=False)
        t = np.setdiff1d(window, keep_free).astype(np.int32)
        t = np.concatenate([t, rng.integers(0, V, 37).astype(np.int32), [-1, -1]]).astype(np.int32)
        rng.shuffle(t)
        D = np.unique(t[t >= 0]).size
        info = check_build(t, V, min(V, D + need), off)
        hits += info["used_fallback"]
    assert hits >= 4


def test_builder_edge_cases():
    check_build(np.zeros(0, np.int32), 50304, 2048, 99)                      # empty microbatch
    check_build(np.full(1000, -1, np.int32), 50304, 4096, 5)                  # all ignored
    t = np.array([3, 17, 40, 3, -1], np.int32)
    info = check_build(t, 101, 3, 7)                                          # D == P
    assert info["draw"] == 0
    check_build(np.array([0, 50303, 7], np.int32), 50304, 50304, 123)         # P == V
    V = capi.MAX_VOCAB                                                        # largest vocabulary
    rng = np.random.default_rng(3)
    check_build(rng.integers(-1, V, 100000).astype(np.int32), V, 200000, 777, 20011)
    check_build(rng.integers(0, 1000, 7).astype(np.int32), 1000, 999, 1, 7)   # T % 4 != 0


def test_builder_device_errors():
    _, _, _, st = run_build(np.array([1, 2, 3, 4], np.int32), 100, 3, 0)
    assert st[0] == capi.STATUS["SS_ERR_TOO_MANY_TARGETS"] and st[1] == 4
    cand, tpos, vpos, st = run_build(np.array([1, 2, 100, 5, -2], np.int32), 100, 10, 0)
    assert st[0] == capi.STATUS["SS_ERR_BAD_TARGET"] and st[6] == 2
    assert np.all(cand == -1) and np.all(tpos == -1) and np.all(vpos == -1)
    with pytest.raises(capi.SampledCEError) as e:
        run_build(np.array([1], np.int32), 50304, 8, 0, stride=6)
    assert e.value.name == "SS_ERR_STRIDE_NOT_COPRIME"


# ------------------------------------------------- full comparison, small --

SMALL = [
    # (T, d, V, P, seed, grad) -- several tiles and ragged tails in every dim
    (512, 128, 50304, 2048, 0, 1.0),
    (1000, 200, 5003, 3000, 1, 1.0),
    (777, 136, 4099, 1001, 2, 2.5),
    (300, 64, 1000, 1000, 3, 1.0),
    (129, 8, 300, 257, 4, 0.5),
    (2048, 768, 20023, 4096, 5, 1.0),
]


@pytest.mark.parametrize("T,d,V,P,seed,grad", SMALL)
def test_small_shapes_match_oracle(T, d, V, P, seed, grad):
    x, lm, t = random_case(T, d, V, P, seed)
    off = (seed * 7919) % V
    g = run_path(x, lm, t, P, off, grad=grad)
    o = oracle_run(x, lm, t, P, off, grad=grad)
    compare_full(g, o, t)


def _edge_case(kind):
    rng = np.random.default_rng(hash(kind) % (1 << 32))
    if kind == "one_token":
        x, lm, t = random_case(1, 64, 1000, 10, 21)
        return x, lm, t, 10, 3
    if kind == "one_class":  # P = 1: C = {the only target}; softmax 1, loss 0, gradients 0
        x, lm, _ = wl.make_inputs(200, 64, 500, 1.1, 0.0, 22)
        t = np.full(200, 7, np.int32)
        t[::9] = -1
        return x, lm, t, 1, 11
    if kind == "one_target_class":  # D = 1, P - 1 negatives
        x, lm, _ = wl.make_inputs(300, 96, 2000, 1.1, 0.0, 23)
        return x, lm, np.full(300, 1234, np.int32), 300, 5
    if kind == "wide_d":  # K = 4096 in the forward: 64 K blocks per tile
        x, lm, t = random_case(256, 4096, 3001, 700, 24)
        return x, lm, t, 700, 17
    if kind == "max_vocab":  # V = SS_MAX_VOCAB, P = V / 4
        V = capi.MAX_VOCAB
        x, lm, t = random_case(256, 64, V, V // 4, 25)
        return x, lm, t, V // 4, 123457
    if kind == "huge_offset":  # a 64-bit offset, reduced mod V
        x, lm, t = random_case(500, 64, 5003, 1500, 26)
        return x, lm, t, 1500, (1 << 40) + 5
    raise ValueError(kind)


@pytest.mark.parametrize("kind", ["one_token", "one_class", "one_target_class", "wide_d",
                                  "max_vocab", "huge_offset"])
def test_edge_shapes_match_oracle(kind):
    x, lm, t, P, off = _edge_case(kind)
    g = run_path(x, lm, t, P, off)
    o = oracle_run(x, lm, t, P, off)
    compare_full(g, o, t)
    if kind == "one_class":  # exactly 0 up to fp32 rounding of z_target - ref
        assert abs(g["loss"]) <= 1e-6
        assert np.max(np.abs(wl.bits_to_f64(g["dx_bits"]))) <= 1e-6


@pytest.mark.parametrize("T,d,V,P,seed", [
    (8192, 64, 20000, 8192, 41),   # forward: d = 64, one K block; 1024 tiles
    (32768, 768, 64, 64, 42),      # dX: K = P = 64, one K block; 384 tiles
    (64, 768, 50304, 40000, 43),   # dW: K = T = 64, one K block; 471 tiles
])
def test_one_k_block_gemms_with_many_tiles_compared_in_full(T, d, V, P, seed):
    """A tile with a single K block lets the dynamic tile schedule's producer
    run furthest ahead of the warps that read its tile ring (the ring's size
    is set by that case); each shape gives one GEMM a single K block and more
    tiles than CTA pairs, compared in full."""
    x, lm, t = random_case(T, d, V, P, seed)
    off = (seed * 7919) % V
    g = run_path(x, lm, t, P, off)
    o = oracle_run(x, lm, t, P, off)
    compare_full(g, o, t)


def test_tiny_workload_matches_oracle():
    w = wl.WORKLOADS["tiny"]
    x, lm, t = wl.workload_inputs(w)
    g = run_path(x, lm, t, w.P, w.offset)
    o = oracle_run(x, lm, t, w.P, w.offset)
    compare_full(g, o, t)


def test_all_ignored_and_zero_grad():
    x, lm, _ = random_case(256, 64, 2000, 512, 9)
    t = np.full(256, -1, np.int32)
    g = run_path(x, lm, t, 512, 3)
    assert g["loss"] == 0.0 and g["n_valid"] == 0
    assert np.all(g["dx_bits"] == 0) and np.all(g["dW_bits"] == 0)
    x, lm, t = random_case(256, 64, 2000, 512, 10)
    g = run_path(x, lm, t, 512, 3, grad=0.0)
    assert np.all(wl.bits_to_f64(g["dx_bits"]) == 0) and np.all(wl.bits_to_f64(g["dW_bits"]) == 0)


def test_empty_microbatch():
    lm = wl.bf16_bits(np.random.default_rng(0).standard_normal((500, 64), dtype=np.float32))
    g = run_path(np.zeros((0, 64), np.uint16), lm, np.zeros(0, np.int32), 100, 4)
    assert g["loss"] == 0.0 and g["n_valid"] == 0
    assert np.all(g["dW_bits"] == 0)


def test_uniform_logits_give_log_p():
    T, d, V, P = 300, 64, 3000, 1024
    _, lm, t = random_case(T, d, V, P, 12)
    x = np.zeros((T, d), np.uint16)
    g = run_path(x, lm, t, P, 0)
    assert abs(g["loss"] - np.log(P)) <= 1e-6 * np.log(P)
    assert np.max(np.abs(g["lse"] - np.log(P))) <= 1e-5


def test_rows_with_huge_loss_are_recomputed_exactly():
    """Rows whose target logit lies ~120 below another candidate's.

    The forward stores exp(z - z_target); such rows overflow it and take the
    exact recomputation path. lse, loss and gradients must still match the
    oracle, on those rows and on the rest.
    """
    T, d, V, P, seed = 300, 64, 1000, 384, 21
    x, lm, t = random_case(T, d, V, P, seed)
    xf = wl.bits_to_f32(x).copy()
    lmf = wl.bits_to_f32(lm)
    rng = np.random.default_rng(seed)
    cand, _, _, _ = oc.build_candidates(t, V, P, 0)
    for i in (3, 77, 150):                 # valid rows: push another class far above the target
        a = int(cand[(np.searchsorted(cand, t[i]) + 5) % P]) if t[i] >= 0 else int(cand[5])
        if t[i] < 0:
            t[i] = int(cand[0])
        diff = lmf[a] - lmf[t[i]]
        xf[i] = 60.0 * diff / (diff @ diff)
    t[200] = -1                             # an ignored row far from its reference class
    diff = lmf[int(cand[7])] - lmf[int(cand[0])]
    xf[200] = 60.0 * diff / (diff @ diff)
    x = wl.bf16_bits(xf)
    assert np.unique(t[t >= 0]).size <= P
    g = run_path(x, lm, t, P, 0)
    o = oracle_run(x, lm, t, P, 0)
    assert np.all(np.isfinite(g["lse"]))
    assert max(o["loss_rows"][[3, 77, 150]]) > 50      # the rows really are extreme
    compare_full(g, o, t)
    np.testing.assert_allclose(g["lse"][[3, 77, 150, 200]], o["lse"][[3, 77, 150, 200]], atol=LSE_ATOL)


def test_backward_can_be_repeated():
    x, lm, t = random_case(700, 128, 3001, 1024, 22)
    T, d, V, P = 700, 128, 3001, 1024
    ce = capi.SampledCE(T, d, V, P)
    xt = torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).cuda()
    lt = torch.from_numpy(lm.view(np.int16)).view(torch.bfloat16).cuda()
    ce.build(torch.from_numpy(t).cuda(), 5)
    ce.forward(xt, lt)
    ce.backward()
    dx1, dw1 = ce.dx.clone(), ce.dW.clone()
    ce.grad_loss.fill_(2.0)
    ce.backward()
    torch.cuda.synchronize()
    assert torch.equal(ce.dx.float(), (2 * dx1.float()).bfloat16().float())
    assert torch.equal(ce.dW.float(), (2 * dw1.float()).bfloat16().float())


def test_backward_repeated_with_more_tiles_than_pairs():
    """Here both backward GEMMs have several times more tiles than CTA pairs
    (on 148 SMs: dX 471 and dW 354 tiles of 256 x 256 for 74 pairs), so most
    tiles come from the dynamic schedule's counters: a second backward after
    one forward must find its counters reset (dX resets dW's, dW resets dX's)
    and compute every tile again."""
    T, d, V, P = 40000, 768, 50304, 30000
    x, lm, t = random_case(T, d, V, P, 31)
    ce = capi.SampledCE(T, d, V, P)
    xt = torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).cuda()
    lt = torch.from_numpy(lm.view(np.int16)).view(torch.bfloat16).cuda()
    ce.build(torch.from_numpy(t).cuda(), 5)
    ce.forward(xt, lt)
    ce.backward()
    dx1, dw1 = ce.dx.clone(), ce.dW.clone()
    for g in (2.0, 0.5):
        ce.grad_loss.fill_(g)
        ce.backward()
        torch.cuda.synchronize()
        assert ce.status()[8] == 0
        assert torch.equal(ce.dx.float(), (g * dx1.float()).bfloat16().float())
        assert torch.equal(ce.dW.float(), (g * dw1.float()).bfloat16().float())


def test_deterministic():
    x, lm, t = random_case(1000, 200, 5003, 3000, 13)
    a = run_path(x, lm, t, 3000, 17)
    b = run_path(x, lm, t, 3000, 17)
    assert a["loss"] == b["loss"]
    assert np.array_equal(a["lse"], b["lse"])
    assert np.array_equal(a["dx_bits"], b["dx_bits"])
    assert np.array_equal(a["dW_bits"], b["dW_bits"])


def test_kernel_timing_records_every_kernel():
    x, lm, t = random_case(512, 128, 5000, 1024, 14)
    capi.ss_timing_reset()
    capi.ss_timing_enable(True)
    try:
        run_path(x, lm, t, 1024, 0)
    finally:
        capi.ss_timing_enable(False)
    rec = capi.ss_timing_read()
    capi.ss_timing_reset()
    names = ("build_mark", "build_emit", "gather", "ref_logits", "fwd_gemm_ce", "row_pass",
             "loss_finalize", "dx_gemm", "dw_gemm_scatter")
    for k in names:
        assert rec[k][0] == 1 and rec[k][1] > 0, (k, rec)
    assert set(rec) == set(names), rec  # the dW GEMM writes the zero rows itself
    capi.ss_timing_enable(True, gemms_only=True)
    try:
        run_path(x, lm, t, 1024, 0)
    finally:
        capi.ss_timing_enable(False)
    rec = capi.ss_timing_read()
    capi.ss_timing_reset()
    assert set(rec) == {"fwd_gemm_ce", "dx_gemm", "dw_gemm_scatter"}, rec


# ------------------------------------------------ full-size workloads --

@pytest.mark.parametrize("name", ["stage2_early", "stage2_late", "full_softmax"])
def test_full_size_workload(name):
    """Full size, the benchmark's launch configuration: integers in full, loss
    and lse on every row, dX on rows from every M tile, dW on the first and
    last column of every candidate tile plus random and target columns."""
    w = wl.WORKLOADS[name]
    x_bits, lm_bits, t = wl.workload_inputs(w)
    g = run_path(x_bits, lm_bits, t, w.P, w.offset)
    assert g["status"][0] == 0 and g["status"][8] == 0, g["status"]

    cand, tpos, vpos, info = oc.build_candidates(t, w.V, w.P, w.offset)
    assert np.array_equal(g["candidates"], cand)
    assert np.array_equal(g["target_pos"], tpos)
    assert np.array_equal(g["vocab_pos"], vpos)

    x = wl.bits_to_f64(x_bits)
    w_c = oc.gather_rows(wl.bits_to_f64(lm_bits), cand)
    loss, lse, _, n = oc.sampled_ce_forward(x, w_c, tpos)
    assert g["n_valid"] == n
    assert abs(g["loss"] - loss) <= LOSS_RTOL * abs(loss), (g["loss"], loss)
    assert np.max(np.abs(g["lse"] - lse)) <= LSE_ATOL

    rng = np.random.default_rng(w.seed + 100)
    scale = 1.0 / n
    rows = sample_rows(w.T, 768, rng)
    dx_o = oc.dx_rows(x[rows], w_c, tpos[rows], lse[rows], scale)
    check_grad(wl.bits_to_f64(g["dx_bits"][rows]), dx_o, "dx rows")

    cols = sample_cols(w.P, tpos, 512, rng)
    dw_o = oc.dw_c_rows(x, w_c, tpos, lse, scale, cols)
    check_grad(wl.bits_to_f64(g["dW_bits"][cand[cols]]), dw_o, "dW rows")

    in_c = np.zeros(w.V, bool)
    in_c[cand] = True
    assert np.all(g["dW_bits"][~in_c] == 0)
    assert np.all(g["dx_bits"][tpos < 0] == 0)


@pytest.mark.parametrize("name", ["stage0", "stage2_late"])
def test_full_size_workload_compared_in_full(name):
    """Every output of a full-size workload against a full float64 oracle run:
    candidate set and positions bit for bit, loss, lse of every row, and every
    element of dX and of dW (rows in C; +0.0 bits elsewhere)."""
    w = wl.WORKLOADS[name]
    x_bits, lm_bits, t = wl.workload_inputs(w)
    g = run_path(x_bits, lm_bits, t, w.P, w.offset)
    o = oracle_run(x_bits, lm_bits, t, w.P, w.offset)
    compare_full(g, o, t)


def test_ragged_512_row_backward_tiles_compared_in_full():
    """T = 45000 and P = 20000 (d = 768): both backward GEMMs run on 512-row
    tiles (4 and 2 waves of CTA pairs, against 8 and 4 with 256-row tiles), and
    neither T nor P is a multiple of 512, so the last tile of each has rows
    past the end (456 and 32 rows in it). Every output against the oracle."""
    T, d, V, P = 45000, 768, 50304, 20000
    x, lm, t = wl.make_inputs(T, d, V, 1.05, 0.01, 45)
    assert np.unique(t[t >= 0]).size <= P
    g = run_path(x, lm, t, P, 777)
    o = oracle_run(x, lm, t, P, 777)
    compare_full(g, o, t)


@pytest.mark.parametrize("name,d", [("tiny", None), ("stage0", None), ("stage2_early", None),
                                    ("stage2_late", None), ("full_softmax", None),
                                    ("ragged_d", 200)])
def test_gathered_rows_are_an_exact_copy(name, d):
    """W_C = lm_head[C] is a byte copy (SampledSoftmax._gather_rows): the rows the
    forward leaves in the workspace equal lm_head[C] bit for bit."""
    if name == "ragged_d":
        x_bits, lm_bits, t = wl.make_inputs(700, d, 3001, 1.1, 0.05, 41)
        V, P, off = 3001, 1111, 29
    else:
        w = wl.WORKLOADS[name]
        x_bits, lm_bits, t = wl.workload_inputs(w)
        V, P, off = w.V, w.P, w.offset
    T, dd = x_bits.shape
    for precision in ("bf16", "e4m3") if dd % 16 == 0 else ("bf16",):
        ce = capi.SampledCE(T, dd, V, P, precision=precision)
        ce.build(torch.from_numpy(t).cuda(), off)
        ce.forward(dev_bf16(x_bits), dev_bf16(lm_bits))
        torch.cuda.synchronize()
        st = ce.status()
        assert st[0] == 0 and st[8] == 0, st
        cand = ce.candidates.cpu().numpy()
        o0 = capi.ss_workspace_wc_offset(T, dd, V, P)
        assert o0 >= 0 and o0 % 16 == 0
        w_c = host_bits(ce.workspace[o0:o0 + P * dd * 2].view(torch.bfloat16).view(P, dd))
        assert np.array_equal(w_c, lm_bits[cand]), (name, precision)
