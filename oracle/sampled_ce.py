"""Float64 CPU oracle for the shared-negatives sampled-softmax CE LM head.

TEST INFRASTRUCTURE. Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import or run
anything under ``oracle/``. The product path (the C-ABI library and its
Python binding) never calls it, and this module shares no code with it.

What it follows, step by step:

* ``sampled_softmax.py`` (modded-nanogpt track_1_short), module docstring
  "What"/"Why" and ``CandidateBuilder.build`` / ``CandidateBuilder._negatives``:
  the candidate set C, the stride-permutation negatives, the fallback, the
  ascending order of C and the class -> position maps.
* ``sampled_softmax.py``, ``SampledSoftmax._gather_rows``: the row gather
  ``lm_head[C]`` and the inverse map (-1 off C).
* "Learning Triton One Kernel at a Time: Softmax", sections "Definition"
  (max-shifted softmax) and "Gradient" (softmax minus one-hot for CE).
* Handout #16 CPU checks (``16_optimization_checks.py``), ``lm_gradient``:
  the loss is the sum of per-token losses over the valid targets divided by
  their count; ignored positions add neither loss nor gradient.

Readings where the pages are silent are listed beside each function. Every
function here is pinned by ``tests/test_oracle_*.py`` against brute force,
closed forms, a library routine, finite differences or hand-worked fixtures.

Floating point is float64 throughout; bf16 inputs arrive as their exact
float64 values. A library matmul (BLAS) serves as the dense contraction step.
"""

from __future__ import annotations

import math

import numpy as np

NEGATIVE_STRIDE = 20011

# Window length factor and pad: draw = min(V, floor(1.7 need) + 256) positions
# (sampled_softmax.py, CandidateBuilder._negatives).
WINDOW_FACTOR = 1.7
WINDOW_PAD = 256


class OracleError(Exception):
    """A case the method rejects; ``code`` names which check failed."""

    def __init__(self, code: str, msg: str):
        super().__init__(f"{code}: {msg}")
        self.code = code


# ---------------------------------------------------------------------------
# Candidate set (integer part)
# ---------------------------------------------------------------------------


def stride_class(k: np.ndarray, V: int, stride: int = NEGATIVE_STRIDE) -> np.ndarray:
    """Class at sweep position k: (stride * k) mod V, for k taken mod V.

    sampled_softmax.py, NEGATIVE_STRIDE and CandidateBuilder.__init__: the
    sweep is k * stride mod V, a permutation of [0, V) when gcd(stride, V) = 1.
    """
    k = np.asarray(k, dtype=np.int64) % V
    return (np.int64(stride) * k) % V


def window_length(need: int, V: int) -> int:
    """How many sweep positions one draw consumes (CandidateBuilder._negatives)."""
    return min(V, int(need * WINDOW_FACTOR) + WINDOW_PAD)


def pick_negatives(mark: np.ndarray, need: int, offset: int, V: int, stride: int):
    """``need`` distinct unmarked classes, as CandidateBuilder._negatives draws them.

    The window is the next ``draw`` positions of the stride sweep starting at
    ``offset``. Classes already marked (the targets) are skipped; the first
    ``need`` survivors, in sweep order, are the negatives. When the window
    holds fewer than ``need`` survivors, the fallback walks all unmarked
    classes in ascending order and keeps every s-th one, starting with the
    first, s = max(1, floor(#unmarked / need)), until it has ``need``.

    Returns (negatives, draw, used_fallback). ``mark`` is not modified: the
    window is tested against the targets' marks only, as on the page.
    """
    draw = window_length(need, V)
    window = stride_class(offset + np.arange(draw, dtype=np.int64), V, stride)
    survivors = window[~mark[window]]
    if survivors.size >= need:
        return survivors[:need], draw, False
    free = np.flatnonzero(~mark)
    if free.size < need:
        raise OracleError("no_free_classes", f"{need} negatives wanted, {free.size} unmarked classes left")
    step = max(1, free.size // need)
    return free[::step][:need], draw, True


def build_candidates(targets: np.ndarray, V: int, P: int, offset: int = 0,
                     stride: int = NEGATIVE_STRIDE):
    """Candidate set C and its maps for one microbatch (CandidateBuilder.build).

    Steps, in the page's order:
      1. mark the classes that occur as targets (``-1`` = none, skipped);
      2. num_targets D = number of marked classes; D > P is an error;
      3. if D != P, mark P - D negatives from the stride window (pick_negatives);
      4. C = the marked classes in ascending order;
      5. vocab_pos[c] = position of c in C, -1 for classes outside C;
         target_pos[i] = vocab_pos[targets[i]], -1 for ignored tokens.

    Readings: the only ignore marker is -1 (any other negative value, or a
    value >= V, is rejected); the window start is ``offset mod V``; when D = P
    no window is consumed (draw = 0) and the next offset equals the offset.

    Returns (candidates int64 [P], target_pos int64 [T], vocab_pos int64 [V], info).
    info = dict(D, need, draw, used_fallback, next_offset).
    """
    targets = np.asarray(targets, dtype=np.int64)
    if V < 1 or P < 1 or P > V:
        raise OracleError("invalid_arg", f"need 1 <= P <= V, got P={P}, V={V}")
    if math.gcd(stride, V) != 1:
        raise OracleError("stride_not_coprime", f"gcd({stride}, {V}) != 1")
    bad = (targets < -1) | (targets >= V)
    if bad.any():
        raise OracleError("bad_target", f"target {int(targets[bad][0])} outside [-1, {V})")
    offset = int(offset) % V

    mark = np.zeros(V, dtype=bool)
    valid = targets >= 0
    mark[targets[valid]] = True
    D = int(mark.sum())
    if D > P:
        raise OracleError("too_many_targets", f"{D} distinct targets > P={P}")
    need = P - D
    draw, used_fallback = 0, False
    if need:
        negatives, draw, used_fallback = pick_negatives(mark, need, offset, V, stride)
        mark[negatives] = True

    candidates = np.flatnonzero(mark).astype(np.int64)
    assert candidates.size == P
    vocab_pos = np.full(V, -1, dtype=np.int64)
    vocab_pos[candidates] = np.arange(P, dtype=np.int64)
    target_pos = np.full(targets.shape, -1, dtype=np.int64)
    target_pos[valid] = vocab_pos[targets[valid]]
    info = dict(D=D, need=need, draw=draw, used_fallback=used_fallback,
                next_offset=(offset + draw) % V)
    return candidates, target_pos, vocab_pos, info


def prefix_positions(prefix_table: np.ndarray, targets: np.ndarray,
                     vocab_pos: np.ndarray) -> np.ndarray:
    """Where each token's prefix target sits in C (CandidateBuilder.build, and
    the SampledLoss field ``prefix_pos``; module docstring: a token whose
    prefix class is not in C gets no prefix target; it never adds a class).

    Steps, in the page's order:
      1. prefix target of token i = prefix_table[targets[i]];
      2. its position = vocab_pos[prefix target], where the class map gives -1
         for classes outside C and for the "no prefix" marker -1 (the page
         keeps a sentinel entry at index V that stays -1 for this).

    Reading: an ignored token (target -1) has no prefix target, so its
    position is -1 (the page's ``np.take`` would wrap -1 to the table's last
    entry; the kernel reads -1 targets as no-ops either way). Table entries
    and targets outside [-1, V) are rejected.

    Returns prefix_pos int64 [T].
    """
    prefix_table = np.asarray(prefix_table, dtype=np.int64)
    targets = np.asarray(targets, dtype=np.int64)
    vocab_pos = np.asarray(vocab_pos, dtype=np.int64)
    V = vocab_pos.size
    if prefix_table.size != V:
        raise OracleError("invalid_arg", f"prefix table of {prefix_table.size} entries, V={V}")
    if ((targets < -1) | (targets >= V)).any():
        raise OracleError("bad_index", "target outside [-1, V)")
    if ((prefix_table < -1) | (prefix_table >= V)).any():
        raise OracleError("bad_index", "prefix class outside [-1, V)")
    pos = np.append(vocab_pos, -1)  # entry V: the "no prefix" sentinel
    valid = targets >= 0
    prefix_targets = np.full(targets.shape, -1, dtype=np.int64)
    prefix_targets[valid] = prefix_table[targets[valid]]
    return pos[prefix_targets]  # -1 indexes the sentinel


# ---------------------------------------------------------------------------
# Loss and gradients (floating-point part)
# ---------------------------------------------------------------------------


def gather_rows(lm_head: np.ndarray, candidates: np.ndarray) -> np.ndarray:
    """W_C = lm_head[C] (SampledSoftmax._gather_rows); rows in C's order."""
    return np.asarray(lm_head)[np.asarray(candidates, dtype=np.int64)]


def _row_chunks(T: int, chunk: int):
    for r0 in range(0, T, chunk):
        yield r0, min(T, r0 + chunk)


def sampled_ce_forward(x: np.ndarray, w_c: np.ndarray, target_pos: np.ndarray,
                       chunk: int = 1024):
    """Loss over the P-wide vocabulary C (module docstring "What").

    z = x @ W_C^T; lse_i = m_i + ln sum_j exp(z_ij - m_i) with m_i the row max
    (max-shifted softmax, "Learning Triton ... Softmax", "Definition");
    loss_i = lse_i - z_{i, target_pos_i} for valid rows; the loss is
    sum(loss_i) / n over the n valid rows, 0 when n = 0 (Handout #16,
    ``lm_gradient``: sum of per-token losses over the valid-target count).

    Readings: no correction term is added (the page says the loss is biased);
    lse is reported for every row, ignored rows included.

    Returns (loss float, lse float64 [T], loss_rows float64 [T] (0 where
    ignored), n_valid int).
    """
    x = np.asarray(x, dtype=np.float64)
    w_c = np.asarray(w_c, dtype=np.float64)
    tpos = np.asarray(target_pos, dtype=np.int64)
    T = x.shape[0]
    lse = np.zeros(T)
    loss_rows = np.zeros(T)
    for r0, r1 in _row_chunks(T, chunk):
        z = x[r0:r1] @ w_c.T
        m = z.max(axis=1)
        lse[r0:r1] = m + np.log(np.exp(z - m[:, None]).sum(axis=1))
        tp = tpos[r0:r1]
        ok = tp >= 0
        rows = np.flatnonzero(ok)
        loss_rows[r0 + rows] = lse[r0 + rows] - z[rows, tp[rows]]
    n = int((tpos >= 0).sum())
    loss = float(loss_rows.sum() / n) if n else 0.0
    return loss, lse, loss_rows, n


def dlogits(z: np.ndarray, lse: np.ndarray, target_pos: np.ndarray, scale: float) -> np.ndarray:
    """G = scale * (softmax(z) - onehot(target_pos)); zero rows where ignored.

    "Learning Triton ... Softmax", "Gradient": for cross-entropy the softmax
    gradient reduces to probabilities minus the one-hot target. ``scale`` is
    g / n, the upstream gradient over the valid-token count.
    """
    tpos = np.asarray(target_pos, dtype=np.int64)
    g = np.exp(z - lse[:, None])
    rows = np.flatnonzero(tpos >= 0)
    g[rows, tpos[rows]] -= 1.0
    g[tpos < 0] = 0.0
    return scale * g


def sampled_ce_backward(grad_loss: float, x: np.ndarray, w_c: np.ndarray,
                        candidates: np.ndarray, target_pos: np.ndarray,
                        lse: np.ndarray, V: int, chunk: int = 1024,
                        logit_x: np.ndarray | None = None, logit_w: np.ndarray | None = None):
    """dX = G @ W_C and the dense lm_head gradient dW (zeros outside C).

    Module docstring of sampled_softmax.py: the two gradient GEMMs, and an
    lm_head gradient over every vocabulary row that is zero off C.
    dW_C = G^T @ x is accumulated over row chunks; dW[C_j] = dW_C[j].
    G comes from the logits z = logit_x @ logit_w^T, by default x and W_C
    themselves (the e4m3 variant passes its quantized operands here).

    Returns (dx float64 [T,d], dW float64 [V,d]).
    """
    x = np.asarray(x, dtype=np.float64)
    w_c = np.asarray(w_c, dtype=np.float64)
    lx = x if logit_x is None else np.asarray(logit_x, dtype=np.float64)
    lw = w_c if logit_w is None else np.asarray(logit_w, dtype=np.float64)
    tpos = np.asarray(target_pos, dtype=np.int64)
    T, d = x.shape
    n = int((tpos >= 0).sum())
    scale = grad_loss / n if n else 0.0
    dx = np.zeros((T, d))
    dw_c = np.zeros_like(w_c)
    for r0, r1 in _row_chunks(T, chunk):
        z = lx[r0:r1] @ lw.T
        g = dlogits(z, lse[r0:r1], tpos[r0:r1], scale)
        dx[r0:r1] = g @ w_c
        dw_c += g.T @ x[r0:r1]
    dW = np.zeros((V, d))
    dW[np.asarray(candidates, dtype=np.int64)] = dw_c
    return dx, dW


def sampled_ce(x, lm_head, targets, P, offset=0, stride=NEGATIVE_STRIDE, grad_loss=1.0,
               chunk=1024):
    """Whole path for one microbatch: build C, gather, loss, gradients."""
    lm_head = np.asarray(lm_head, dtype=np.float64)
    V = lm_head.shape[0]
    cand, tpos, vpos, info = build_candidates(targets, V, P, offset, stride)
    w_c = gather_rows(lm_head, cand)
    loss, lse, loss_rows, n = sampled_ce_forward(x, w_c, tpos, chunk)
    dx, dW = sampled_ce_backward(grad_loss, x, w_c, cand, tpos, lse, V, chunk)
    return dict(candidates=cand, target_pos=tpos, vocab_pos=vpos, info=info, loss=loss,
                lse=lse, loss_rows=loss_rows, n_valid=n, dx=dx, dW=dW)


# ---------------------------------------------------------------------------
# e4m3 variant: the logits GEMM on 8-bit floating-point operands
# ---------------------------------------------------------------------------
#
# sampled_softmax.py keeps the candidate rows as float8 e4m3 (SampledLoss.rows,
# rows_t) and runs the logits through torch._scaled_mm; the scales are not on
# the page. Readings for this variant:
#   * format: OCP 8-bit floating point, E4M3 -- 1 sign bit, 4 exponent bits
#     (bias 7), 3 mantissa bits, subnormals below 2^-6, no infinities, the
#     codes S.1111.111 are NaN, largest finite magnitude 448;
#   * rounding: to nearest, ties to even, finite results saturate at +-448;
#   * scale: one power of two per tensor (x, and W_C of the step): the
#     smallest 2^k with amax * 2^-k <= 448, so scaling is exact and the codes
#     are round(v * 2^-k); 2^0 for an all-zero tensor; k kept in [-126, 127];
#   * only the logits GEMM uses them: z = (x_q 2^kx)(w_q 2^kw)^T; the softmax,
#     loss and G follow from that z, and the gradient GEMMs use the bf16 x and
#     W_C as in the bf16 path (the page does not give G's precision).

E4M3_MAX = 448.0


def e4m3_decode(code: int) -> float:
    """Value of an e4m3 code from its bit fields (NaN for S.1111.111)."""
    code = int(code) & 0xFF
    sign = -1.0 if code & 0x80 else 1.0
    e = (code >> 3) & 0xF
    m = code & 0x7
    if e == 0xF and m == 0x7:
        return math.nan
    if e == 0:
        return sign * (m / 8.0) * 2.0 ** -6
    return sign * (1.0 + m / 8.0) * 2.0 ** (e - 7)


def e4m3_round(v: np.ndarray) -> np.ndarray:
    """Round to the e4m3 grid: nearest, ties to even, saturating at +-448.

    In the binade [2^e, 2^(e+1)) the grid spacing is 2^(e-3); below 2^-6 it
    is 2^-9 (subnormals). Division by the spacing is exact (a power of two)
    and numpy's round is half-to-even.
    """
    v = np.asarray(v, dtype=np.float64)
    a = np.abs(v)
    _, ex = np.frexp(a)  # a = f * 2^ex with f in [0.5, 1): floor(log2 a) = ex - 1
    e = np.maximum(ex - 1, -6)
    q = np.ldexp(1.0, e - 3)
    r = np.minimum(np.round(a / q) * q, E4M3_MAX)
    return np.where(np.signbit(v), -r, r)


def e4m3_encode(r: np.ndarray) -> np.ndarray:
    """Codes of values already on the e4m3 grid (e4m3_round's output)."""
    r = np.asarray(r, dtype=np.float64)
    a = np.abs(r)
    sub = a < 2.0 ** -6
    _, ex = np.frexp(np.where(sub, 1.0, a))
    e = ex - 1
    mant_norm = np.round((np.where(sub, 1.0, a) / np.ldexp(1.0, e) - 1.0) * 8.0)
    exp_field = np.where(sub, 0, e + 7)
    mant = np.where(sub, np.round(a / 2.0 ** -9), mant_norm)
    code = (exp_field.astype(np.int64) << 3) | mant.astype(np.int64)
    code = np.where(np.signbit(r), code | 0x80, code)
    return code.astype(np.uint8)


def e4m3_scale_exponent(amax: float) -> int:
    """The k of the per-tensor scale 2^k: smallest k with amax <= 448 * 2^k,
    kept in [-126, 127] so that 2^k and 2^-k are normal fp32 numbers (the
    device scales by multiplying with them); 0 for an all-zero tensor."""
    amax = float(amax)
    if not amax > 0.0:
        return 0
    _, ex = math.frexp(amax)
    k = ex - 9
    while amax > math.ldexp(E4M3_MAX, k):
        k += 1
    while amax <= math.ldexp(E4M3_MAX, k - 1):
        k -= 1
    return min(max(k, -126), 127)


def quantize_e4m3(a: np.ndarray):
    """Per-tensor e4m3 quantization: (codes uint8, k, dequantized float64)."""
    a = np.asarray(a, dtype=np.float64)
    k = e4m3_scale_exponent(np.max(np.abs(a)) if a.size else 0.0)
    r = e4m3_round(np.ldexp(a, -k))
    return e4m3_encode(r), k, np.ldexp(r, k)


def sampled_ce_e4m3(x, lm_head, targets, P, offset=0, stride=NEGATIVE_STRIDE, grad_loss=1.0,
                    chunk=1024):
    """Whole path with the logits GEMM on e4m3 operands (readings above)."""
    lm_head = np.asarray(lm_head, dtype=np.float64)
    x = np.asarray(x, dtype=np.float64)
    V = lm_head.shape[0]
    cand, tpos, vpos, info = build_candidates(targets, V, P, offset, stride)
    w_c = gather_rows(lm_head, cand)
    xq_codes, kx, xq = quantize_e4m3(x)
    wq_codes, kw, wq = quantize_e4m3(w_c)
    loss, lse, loss_rows, n = sampled_ce_forward(xq, wq, tpos, chunk)
    dx, dW = sampled_ce_backward(grad_loss, x, w_c, cand, tpos, lse, V, chunk,
                                 logit_x=xq, logit_w=wq)
    return dict(candidates=cand, target_pos=tpos, vocab_pos=vpos, info=info, loss=loss,
                lse=lse, loss_rows=loss_rows, n_valid=n, dx=dx, dW=dW,
                x_codes=xq_codes, kx=kx, w_codes=wq_codes, kw=kw)


# ---------------------------------------------------------------------------
# Row / column samples for full-size checks
# ---------------------------------------------------------------------------


def rows_forward(x_rows: np.ndarray, w_c: np.ndarray, tpos_rows: np.ndarray):
    """lse and per-row loss for a subset of rows (same definitions as above)."""
    loss, lse, loss_rows, _ = sampled_ce_forward(x_rows, w_c, tpos_rows)
    return lse, loss_rows


def dx_rows(x_rows, w_c, tpos_rows, lse_rows, scale, logit_x_rows=None, logit_w=None):
    """dX for a subset of rows: G_rows @ W_C (G from logit_x_rows @ logit_w^T,
    by default x_rows and W_C)."""
    lx = x_rows if logit_x_rows is None else logit_x_rows
    lw = w_c if logit_w is None else logit_w
    z = np.asarray(lx, dtype=np.float64) @ np.asarray(lw, dtype=np.float64).T
    return dlogits(z, lse_rows, tpos_rows, scale) @ w_c


def dw_c_rows(x, w_c, target_pos, lse, scale, cols, chunk=1024, logit_x=None, logit_w=None):
    """dW_C[j] for j in ``cols`` only: sum_i G_ij x_i, over all rows (G from
    logit_x @ logit_w^T, by default x and W_C)."""
    x = np.asarray(x, dtype=np.float64)
    lx = x if logit_x is None else np.asarray(logit_x, dtype=np.float64)
    w_sel = np.asarray(w_c if logit_w is None else logit_w, dtype=np.float64)[cols]
    tpos = np.asarray(target_pos, dtype=np.int64)
    out = np.zeros((len(cols), x.shape[1]))
    col_of = {int(c): k for k, c in enumerate(cols)}
    for r0, r1 in _row_chunks(x.shape[0], chunk):
        z = lx[r0:r1] @ w_sel.T
        p = np.exp(z - lse[r0:r1, None])
        tp = tpos[r0:r1]
        for r in np.flatnonzero(tp >= 0):
            k = col_of.get(int(tp[r]))
            if k is not None:
                p[r, k] -= 1.0
        p[tp < 0] = 0.0
        out += (scale * p).T @ x[r0:r1]
    return out
