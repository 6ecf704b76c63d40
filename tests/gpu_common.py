"""Shared helpers for the GPU parity tests (not collected by pytest).

Runs the CUDA path through the C ABI (via the ctypes binding) and the float64
oracle on the same seeded inputs, and holds the tolerances:

* candidate set, target/vocab positions, builder info, dW zero pattern:
  bit-exact;
* loss: relative 1e-3, plus an absolute 1e-6 for losses at or near 0 (P = 1,
  where the exact loss is 0 and the GPU's is the log of 1 + the fp32 rounding
  difference between the tensor-core logit and the fp32 target logit);
  lse: absolute 1e-3 (both come from fp32 accumulators);
* dX and dW (rows in C): three bounds, all from the stated gradient tolerance
  2e-2 (bf16 outputs from bf16 logits): the relative Frobenius error; the
  largest absolute error over the largest |expected| entry; and, for every
  element, |got - want| <= GRAD_ROW_RTOL * max|want in its row| +
  GRAD_ATOL_FRAC * max|want| -- so a localised error (one wrong tile, chunk
  or row) fails even where the norm over the rest would dilute it. Row
  maxima differ by orders of magnitude (dW rows of frequent targets against
  rows of negatives), so the floor is kept at 1e-6 of the global maximum; it
  only matters for rows that are exactly zero.
"""

from __future__ import annotations

import numpy as np
import torch

from oracle import sampled_ce as oc
from sampled_softmax_cross_b200 import capi
from sampled_softmax_cross_b200 import workloads as wl

LOSS_RTOL = 1e-3
LOSS_ATOL = 1e-6
LSE_ATOL = 1e-3
GRAD_RTOL = 2e-2
GRAD_ROW_RTOL = 2e-2
GRAD_ATOL_FRAC = 1e-6
GRAD_ZERO_ATOL = 1e-6


def dev_bf16(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def host_bits(t: torch.Tensor) -> np.ndarray:
    return t.view(torch.int16).cpu().numpy().view(np.uint16)


def run_build(targets: np.ndarray, V: int, P: int, offset: int, stride: int = 20011):
    T = targets.size
    dev = torch.device("cuda")
    ws = torch.empty(capi.ss_build_workspace_bytes(V), dtype=torch.uint8, device=dev)
    cand = torch.empty(P, dtype=torch.int32, device=dev)
    tpos = torch.empty(max(T, 1), dtype=torch.int32, device=dev)
    vpos = torch.empty(V, dtype=torch.int32, device=dev)
    st = torch.zeros(capi.DEV_STATUS_WORDS, dtype=torch.int32, device=dev)
    t = torch.from_numpy(np.ascontiguousarray(targets, dtype=np.int32)).cuda()
    capi.ss_build_candidates(t, V, P, offset, stride, cand, tpos, vpos, st, ws)
    torch.cuda.synchronize()
    return cand.cpu().numpy(), tpos[:T].cpu().numpy(), vpos.cpu().numpy(), st.tolist()


def check_build(targets, V, P, offset, stride=20011):
    cand, tpos, vpos, st = run_build(targets, V, P, offset, stride)
    ocand, otpos, ovpos, info = oc.build_candidates(targets, V, P, offset, stride)
    assert st[0] == 0, st
    assert np.array_equal(cand, ocand)
    assert np.array_equal(tpos, otpos)
    assert np.array_equal(vpos, ovpos)
    assert st[1:6] == [info["D"], info["need"], int(info["used_fallback"]), info["draw"],
                       info["next_offset"]], (st, info)
    assert st[7] == P
    return info


def run_path(x_bits, lm_bits, targets, P, offset, stride=20011, grad=1.0, precision="bf16"):
    """build + forward + backward on the GPU; numpy results."""
    T, d = x_bits.shape
    V = lm_bits.shape[0]
    ce = capi.SampledCE(T, d, V, P, precision=precision)
    x = dev_bf16(x_bits) if T else torch.empty((1, d), dtype=torch.bfloat16, device="cuda")
    lm = dev_bf16(lm_bits)
    t = torch.from_numpy(np.ascontiguousarray(targets, dtype=np.int32)).cuda()
    ce.grad_loss.fill_(grad)
    ce.step(t, x, lm, offset, stride)
    torch.cuda.synchronize()
    return dict(
        candidates=ce.candidates.cpu().numpy(), target_pos=ce.target_pos[:T].cpu().numpy(),
        vocab_pos=ce.vocab_pos.cpu().numpy(), status=ce.status(), loss=float(ce.loss.item()),
        n_valid=int(ce.n_valid.item()), lse=ce.lse[:T].cpu().numpy().astype(np.float64),
        dx_bits=host_bits(ce.dx[:T]), dW_bits=host_bits(ce.dW))


def rel_fro(got: np.ndarray, want: np.ndarray) -> float:
    den = np.linalg.norm(want)
    return float(np.linalg.norm(got - want) / den) if den > 0 else float(np.linalg.norm(got))


def grad_errors(got: np.ndarray, want: np.ndarray) -> dict:
    """Error figures of a gradient block (rows = dX rows or dW rows)."""
    err = np.abs(got - want)
    gmax = float(np.max(np.abs(want))) if want.size else 0.0
    rmax = np.max(np.abs(want), axis=1) if want.size else np.zeros(0)
    nz = rmax > 0
    row_ratio = float(np.max(np.max(err[nz], axis=1) / rmax[nz])) if np.any(nz) else 0.0
    return {"rel_fro": rel_fro(got, want),
            "max_abs_over_max": float(err.max() / gmax) if gmax > 0 else float(err.max(initial=0)),
            "row_ratio": row_ratio}


def check_grad(got: np.ndarray, want: np.ndarray, what: str) -> dict:
    """Assert the three gradient bounds (module docstring) on a [rows, d] block.

    A block whose exact value is all zero (P = 1, where softmax minus one-hot
    vanishes) has no scale to be relative to: there |got| <= 1e-6 instead,
    the room the fp32 difference between the two target logits leaves.
    """
    e = grad_errors(got, want)
    if want.size == 0 or not np.any(want):
        assert float(np.max(np.abs(got), initial=0.0)) <= GRAD_ZERO_ATOL, (what, e)
        return e
    assert e["rel_fro"] <= GRAD_RTOL, (what, e)
    assert e["max_abs_over_max"] <= GRAD_RTOL, (what, e)
    gmax = float(np.max(np.abs(want)))
    bound = GRAD_ROW_RTOL * np.max(np.abs(want), axis=1, keepdims=True) + GRAD_ATOL_FRAC * gmax
    bad = np.argwhere(np.abs(got - want) > bound)
    assert bad.size == 0, (what, e, "first elements over the bound (row, col):", bad[:5].tolist())
    return e


def sample_rows(T: int, k: int, rng) -> np.ndarray:
    """Rows for a sampled dX check: one in every 256-row tile (the GEMM's M
    tile of a CTA pair) plus its last row, the ragged tail, and k random ones."""
    tiles = np.arange(0, T, 256)
    per_tile = np.minimum(tiles + rng.integers(0, 256, tiles.size), T - 1)
    extra = rng.choice(T, size=min(T, k), replace=False)
    return np.unique(np.concatenate([[0, T - 1], per_tile, np.minimum(tiles + 255, T - 1), extra]))


def sample_cols(P: int, tpos: np.ndarray, k: int, rng) -> np.ndarray:
    """Candidate positions for a sampled dW check: the first and last column of
    every 256-column tile, P - 1, 32 target positions and k random ones."""
    tiles = np.arange(0, P, 256)
    tgt = np.unique(tpos[tpos >= 0])
    tgt = rng.choice(tgt, size=min(tgt.size, 32), replace=False) if tgt.size else tgt
    extra = rng.choice(P, size=min(P, k), replace=False)
    return np.unique(np.concatenate([[P - 1], tiles, np.minimum(tiles + 255, P - 1), tgt,
                                     extra])).astype(np.int64)


def compare_full(g: dict, o: dict, targets: np.ndarray):
    """Element-by-element comparison against a full oracle run."""
    assert g["status"][0] == 0 and g["status"][8] == 0, g["status"]
    assert np.array_equal(g["candidates"], o["candidates"])
    assert np.array_equal(g["target_pos"], o["target_pos"])
    assert np.array_equal(g["vocab_pos"], o["vocab_pos"])
    assert g["n_valid"] == o["n_valid"]
    if o["n_valid"]:
        assert abs(g["loss"] - o["loss"]) <= LOSS_RTOL * abs(o["loss"]) + LOSS_ATOL, (g["loss"],
                                                                                   o["loss"])
    else:
        assert g["loss"] == 0.0
    if targets.size:
        assert np.max(np.abs(g["lse"] - o["lse"])) <= LSE_ATOL
    dx = wl.bits_to_f64(g["dx_bits"])
    ex = check_grad(dx, o["dx"], "dx")
    ign = o["target_pos"] < 0
    assert np.all(g["dx_bits"][ign] == 0)
    in_c = np.zeros(g["dW_bits"].shape[0], bool)
    in_c[o["candidates"]] = True
    assert np.all(g["dW_bits"][~in_c] == 0)  # +0.0 bits outside C
    dW = wl.bits_to_f64(g["dW_bits"])
    ew = check_grad(dW[in_c], o["dW"][in_c], "dW")
    return {"dx": ex, "dW": ew}
