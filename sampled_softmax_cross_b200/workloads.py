"""Seeded synthetic workloads for the sampled-softmax cross-entropy LM head.

This module only draws random inputs; it holds none of the method's
arithmetic. Both the float64 oracle (under ``oracle/``) and the CUDA path use
it, so the two sides always see the same bits.

The five named workloads follow the shapes of the modded-nanogpt training
track that ``sampled_softmax.py`` (module docstring, "Schedule") describes:
a 50304-class vocabulary, microbatches of up to 24 x 2048 tokens, and
candidate counts of 10240, 14336 and 24576 (plus the full-softmax limit
P = V). Token targets are Zipf-distributed over the class ids so that a
24 x 2048 microbatch holds roughly 11k distinct classes, the figure the same
docstring quotes for batch 24.

Recipe (one ``numpy.random.default_rng(seed)`` per workload, drawn in this
order):

1. ``x = standard_normal((T, d), float32)`` rounded to bf16 (nearest-even);
2. ``lm_head = standard_normal((V, d), float32) / sqrt(d)`` rounded to bf16;
3. ``targets = choice(V, T, p)`` with ``p[k] ~ (k + 1) ** -s`` (int32);
4. ``round(ignore_frac * T)`` positions, drawn without replacement, set to -1.

The negative-window offset is ``(step * P) mod V``.
"""

from __future__ import annotations

import dataclasses
import math

import numpy as np

VOCAB = 50304
NEGATIVE_STRIDE = 20011


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    T: int
    d: int
    V: int
    P: int
    zipf_s: float
    ignore_frac: float
    seed: int
    step: int

    @property
    def offset(self) -> int:
        return (self.step * self.P) % self.V

    @property
    def flops(self) -> int:
        """Dense-contraction FLOPs of one forward + backward: 6 * T * d * P."""
        return 6 * self.T * self.d * self.P


WORKLOADS = {
    w.name: w
    for w in (
        Workload("tiny", 512, 128, VOCAB, 2048, 1.1, 0.05, 0, 0),
        Workload("stage0", 16384, 768, VOCAB, 10240, 1.1, 0.02, 1, 7),
        Workload("stage2_early", 49152, 768, VOCAB, 14336, 1.05, 0.01, 2, 681),
        Workload("stage2_late", 49152, 768, VOCAB, 24576, 1.05, 0.01, 3, 965),
        Workload("full_softmax", 49152, 768, VOCAB, 50304, 1.1, 0.0, 4, 0),
    )
}

HEADLINE = "stage2_late"


def bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round finite float32 values to bf16 (nearest, ties to even); uint16 bits."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)
    lsb = (u >> np.uint32(16)) & np.uint32(1)
    return ((u + np.uint32(0x7FFF) + lsb) >> np.uint32(16)).astype(np.uint16)


def bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """Exact float64 values of bf16 bit patterns."""
    u = bits.astype(np.uint32) << np.uint32(16)
    return u.view(np.float32).astype(np.float64)


def bits_to_f32(bits: np.ndarray) -> np.ndarray:
    u = bits.astype(np.uint32) << np.uint32(16)
    return u.view(np.float32)


def zipf_targets(rng: np.random.Generator, V: int, T: int, s: float) -> np.ndarray:
    w = (np.arange(V, dtype=np.float64) + 1.0) ** (-s)
    return rng.choice(V, size=T, p=w / w.sum()).astype(np.int32)


def make_inputs(T: int, d: int, V: int, zipf_s: float, ignore_frac: float, seed: int):
    """(x_bits [T,d] u16, lm_head_bits [V,d] u16, targets [T] i32) for one seed."""
    rng = np.random.default_rng(seed)
    x = bf16_bits(rng.standard_normal((T, d), dtype=np.float32))
    lm = bf16_bits(rng.standard_normal((V, d), dtype=np.float32) / np.float32(math.sqrt(d)))
    targets = zipf_targets(rng, V, T, zipf_s)
    n_ignored = int(round(ignore_frac * T))
    if n_ignored:
        targets[rng.choice(T, size=n_ignored, replace=False)] = -1
    return x, lm, targets


def workload_inputs(w: Workload | str):
    if isinstance(w, str):
        w = WORKLOADS[w]
    return make_inputs(w.T, w.d, w.V, w.zipf_s, w.ignore_frac, w.seed)
