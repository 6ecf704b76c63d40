"""The allocation-free candidate build against the regular one.

Some callers cannot give the library a workspace: their device memory is
fixed once their set-up ends (a server or trainer whose caching allocator
already holds all the memory it may use, a hook that must not allocate).
ss_build_candidates_noalloc serves them with its scratch in a fixed array
inside the library. Through the C ABI it must give the same candidate set,
positions and status words as ss_build_candidates, bit for bit, on calls made
one after another (the second call reuses the array the first one left).
"""

import numpy as np
import pytest
import torch

from sampled_softmax_cross_b200 import build_lib, capi
from sampled_softmax_cross_b200 import workloads as wl

pytestmark = pytest.mark.gpu


def _buffers(T, V, P):
    dev = torch.device("cuda")
    return (torch.full((P,), -7, dtype=torch.int32, device=dev),
            torch.full((max(T, 1),), -7, dtype=torch.int32, device=dev),
            torch.full((V,), -7, dtype=torch.int32, device=dev),
            torch.zeros(capi.DEV_STATUS_WORDS, dtype=torch.int32, device=dev))


def _both(targets: np.ndarray, V: int, P: int, offset: int, stride: int = 20011):
    T = targets.size
    t = torch.from_numpy(np.ascontiguousarray(targets, dtype=np.int32)).cuda()
    ws = torch.empty(capi.ss_build_workspace_bytes(V), dtype=torch.uint8, device="cuda")
    ref = _buffers(T, V, P)
    capi.ss_build_candidates(t, V, P, offset, stride, *ref, ws)
    got = _buffers(T, V, P)
    capi.ss_build_candidates_noalloc(t, V, P, offset, stride, *got)
    torch.cuda.synchronize()
    for a, b in zip(ref, got):
        assert torch.equal(a, b)
    return [x.cpu() for x in got]


def test_noalloc_matches_workspace_build_on_consecutive_calls():
    build_lib.build()
    capi.load()
    w = wl.WORKLOADS["stage2_late"]
    _, _, t_big = wl.workload_inputs(w)
    first = _both(t_big, w.V, w.P, w.offset)
    assert first[3][0].item() == 0 and first[3][7].item() == w.P
    # second call right after: smaller vocabulary, the array still holds the
    # first call's words beyond the ones this call uses
    rng = np.random.default_rng(5)
    t_small = rng.integers(-1, 1009, 1500).astype(np.int32)  # 781 distinct
    second = _both(t_small, 1009, 900, 17)
    assert second[3][0].item() == 0
    # third call: the full-size workload again, after the small one
    third = _both(t_big, w.V, w.P, w.offset)
    for a, b in zip(first, third):
        assert torch.equal(a, b)


def test_noalloc_reports_device_errors_like_the_regular_build():
    build_lib.build()
    _, _, _, st = _both(np.array([1, 2, 3, 4], np.int32), 100, 3, 0)
    assert st[0].item() == capi.STATUS["SS_ERR_TOO_MANY_TARGETS"]


def test_noalloc_rejects_vocabulary_beyond_its_scratch():
    build_lib.build()
    lib = capi.load()
    t = torch.zeros(4, dtype=torch.int32, device="cuda")
    out = torch.zeros(16, dtype=torch.int32, device="cuda")
    r = lib.ss_build_candidates_noalloc(t.data_ptr(), 4, capi.MAX_VOCAB + 1, 8, 0, 20011,
                                        out.data_ptr(), out.data_ptr(), out.data_ptr(),
                                        out.data_ptr(), None)
    assert r == capi.STATUS["SS_ERR_INVALID_ARG"]
