"""GPU: one step (build, forward, backward) captured in a CUDA graph.

The three C-ABI calls enqueue kernels only (no allocation, no host
synchronisation, launch attributes set on the first call), so a caller can
capture a whole step once and replay it, instead of paying the launches every
step. A replay must give bit for bit what the eager calls give, and a replay
after new inputs are written into the same buffers must give what the eager
calls give on those inputs.
"""

import numpy as np
import pytest
import torch

from sampled_softmax_cross_b200 import capi
from sampled_softmax_cross_b200 import workloads as wl

from gpu_common import dev_bf16

pytestmark = pytest.mark.gpu


def _outputs(ce):
    return [t.clone() for t in (ce.candidates, ce.target_pos, ce.vocab_pos, ce.loss, ce.lse,
                                ce.n_valid, ce.dx, ce.dW, ce.dev_status)]


def _scribble(ce):
    for t in (ce.candidates, ce.target_pos, ce.vocab_pos, ce.n_valid):
        t.fill_(-5)
    ce.loss.fill_(123.0)
    ce.lse.fill_(-1.0)
    ce.dx.fill_(7.0)
    ce.dW.fill_(7.0)


def _same(a, b):
    for u, v in zip(a, b):
        assert torch.equal(u.view(torch.uint8), v.view(torch.uint8))


def test_step_replays_from_a_cuda_graph():
    T, d, V, P, off = 2048, 256, 20023, 4096, 777
    ins = []
    for seed in (61, 62):
        x_bits, lm_bits, t = wl.make_inputs(T, d, V, 1.1, 0.03, seed)
        ins.append((dev_bf16(x_bits), dev_bf16(lm_bits), torch.from_numpy(t).cuda()))
    x, lm, t = (u.clone() for u in ins[0])
    ce = capi.SampledCE(T, d, V, P)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        ce.step(t, x, lm, off)  # eager: also sets the launch attributes once
    torch.cuda.synchronize()
    eager0 = _outputs(ce)

    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        ce.step(t, x, lm, off)
    torch.cuda.synchronize()

    _scribble(ce)
    g.replay()
    torch.cuda.synchronize()
    _same(_outputs(ce), eager0)

    # new inputs in the captured buffers: the replay follows them
    for dst, src in zip((x, lm, t), ins[1]):
        dst.copy_(src)
    _scribble(ce)
    g.replay()
    torch.cuda.synchronize()
    replayed = _outputs(ce)
    with torch.cuda.stream(s):
        ce.step(t, x, lm, off)
    torch.cuda.synchronize()
    _same(replayed, _outputs(ce))
    assert not torch.equal(replayed[3], eager0[3])  # a different loss
    del g
