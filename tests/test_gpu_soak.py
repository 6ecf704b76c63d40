"""GPU: many steps in a row, two independent steps on two streams at once, and
steps while another stream's kernel holds SMs.

compute-sanitizer's race checker is not available here, so these look for
races the way a long training run would meet them: results that change from
one repetition to the next (the persistent GEMMs' barrier phases wrap many
times per launch and across launches), or that depend on what another
stream runs at the same time (the workspace entry points keep no state
between calls, so two workspaces on two streams must not interfere; the
allocation-free build is the one exception, with one scratch array per device
that every call shares, and is not run on two streams here). The GEMMs hand
their tiles to CTA pairs dynamically, so a pair whose SMs another kernel
still holds takes fewer tiles: which pair computes which tile then changes
from step to step, and the results must not.
"""

import hashlib

import numpy as np
import pytest
import torch

from sampled_softmax_cross_b200 import capi
from sampled_softmax_cross_b200 import workloads as wl

from gpu_common import dev_bf16

pytestmark = pytest.mark.gpu


def _digest(ce):
    h = hashlib.sha1()
    for t in (ce.loss, ce.lse, ce.dx, ce.dW, ce.candidates, ce.target_pos):
        h.update(t.view(torch.uint8).cpu().numpy().tobytes())
    return h.hexdigest()


def _inputs(T, d, V, seed):
    x, lm, t = wl.make_inputs(T, d, V, 1.1, 0.02, seed)
    return dev_bf16(x), dev_bf16(lm), torch.from_numpy(t).cuda()


def test_many_steps_are_bit_identical():
    T, d, V, P = 8192, 768, 50304, 8192
    x, lm, t = _inputs(T, d, V, 81)
    ce = capi.SampledCE(T, d, V, P)
    ce.step(t, x, lm, 1234)
    torch.cuda.synchronize()
    first = _digest(ce)
    losses = torch.empty(200, dtype=torch.float32, device="cuda")
    for k in range(200):
        ce.step(t, x, lm, 1234)
        losses[k] = ce.loss[0]
    torch.cuda.synchronize()
    st = ce.status()
    assert st[0] == 0 and st[8] == 0, st
    assert torch.all(losses == losses[0]).item()
    assert _digest(ce) == first


@pytest.mark.parametrize("precision", ["bf16", "e4m3"])
def test_two_streams_match_one_stream(precision):
    shapes = [(4096, 768, 20023, 6144, 91), (3000, 512, 50304, 4096, 92)]
    sets = []
    for T, d, V, P, seed in shapes:
        sets.append((capi.SampledCE(T, d, V, P, precision=precision), _inputs(T, d, V, seed)))
    # one stream, one after the other
    ref = []
    for ce, (x, lm, t) in sets:
        ce.step(t, x, lm, 77)
        torch.cuda.synchronize()
        ref.append(_digest(ce))
    # two streams, interleaved, several times
    streams = [torch.cuda.Stream(), torch.cuda.Stream()]
    for s in streams:
        s.wait_stream(torch.cuda.current_stream())
    for _ in range(5):
        for (ce, (x, lm, t)), s in zip(sets, streams):
            with torch.cuda.stream(s):
                ce.step(t, x, lm, 77, stream=s)
    torch.cuda.synchronize()
    for (ce, _), want in zip(sets, ref):
        assert ce.status()[8] == 0
        assert _digest(ce) == want


@pytest.mark.parametrize("precision", ["bf16", "e4m3"])
def test_steps_with_sms_held_by_another_stream_match(precision):
    """A bf16 matmul on another stream, started at a varying point of each
    step, holds SMs while the step's persistent GEMMs start (all three have
    more tiles than CTA pairs here); every step equals the undisturbed one
    bit for bit."""
    T, d, V, P = 16384, 768, 50304, 16384
    ce = capi.SampledCE(T, d, V, P, precision=precision)
    x, lm, t = _inputs(T, d, V, 93)
    ce.step(t, x, lm, 5)
    torch.cuda.synchronize()
    outs = (ce.dx, ce.dW, ce.loss, ce.lse, ce.candidates, ce.target_pos)
    ref = [a.clone() for a in outs]
    g = torch.Generator(device="cuda").manual_seed(94)
    a = torch.randn(8192, 8192, device="cuda", dtype=torch.bfloat16, generator=g)
    side = torch.cuda.Stream()
    main = torch.cuda.current_stream()

    def hold():
        side.wait_stream(main)
        with torch.cuda.stream(side):
            a @ a

    rng = np.random.default_rng(95)
    for _ in range(12):
        where = int(rng.integers(0, 3))
        if where == 0:
            hold()
        ce.build(t, 5)
        if where == 1:
            hold()
        ce.forward(x, lm)
        if where == 2:
            hold()
        ce.backward()
        assert all(torch.equal(u, v) for u, v in zip(outs, ref))
    torch.cuda.synchronize()
    assert ce.status()[8] == 0
