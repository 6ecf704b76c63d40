"""C-ABI library: loads, exports every declared symbol, host-side checks.

No kernel runs here: each call below is rejected by the host-side argument
checks before any CUDA call, or is a pure host query.
"""

import ctypes
import os
import re

import pytest

from sampled_softmax_cross_b200 import build_lib, capi

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "sampled_ce.h")


@pytest.fixture(scope="module")
def lib():
    build_lib.build()
    return capi.load()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(ss_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_three_calls():
    names = declared_functions()
    for n in ("ss_build_candidates", "ss_ce_forward", "ss_ce_backward", "ss_workspace_bytes"):
        assert n in names


def test_every_declared_symbol_is_exported(lib):
    names = declared_functions()
    assert names
    for n in names:
        assert hasattr(lib, n), n
    assert set(capi.EXPORTS) == set(names)


def test_status_strings(lib):
    assert capi.ss_status_string(0) == "ok"
    for code in range(1, 12):
        assert capi.ss_status_string(code) != "unknown status"
    assert capi.ss_status_string(999) == "unknown status"
    assert capi.ss_version() >= 10000


def test_wc_offset_lies_inside_the_workspace(lib):
    for T, d, V, P in ((512, 128, 50304, 2048), (49152, 768, 50304, 24576), (0, 8, 10, 1),
                       (700, 200, 3001, 1111)):
        off = capi.ss_workspace_wc_offset(T, d, V, P)
        assert off >= 0 and off % 1024 == 0
        assert off + P * d * 2 <= capi.ss_workspace_bytes(T, d, V, P)
        assert off + P * d * 2 <= capi.ss_workspace_bytes_e4m3(T, d, V, P) or d % 16
    assert capi.ss_workspace_wc_offset(512, 127, 50304, 2048) == -1
    assert capi.ss_workspace_wc_offset(512, 128, 50304, 50305) == -1


def test_workspace_bytes_rejects_bad_sizes(lib):
    assert capi.ss_workspace_bytes(512, 128, 50304, 2048) > 0
    assert capi.ss_workspace_bytes(512, 127, 50304, 2048) == 0   # d % 8
    assert capi.ss_workspace_bytes(512, 128, 50304, 50305) == 0  # P > V
    assert capi.ss_workspace_bytes(512, 128, 50304, 0) == 0
    assert capi.ss_workspace_bytes(-1, 128, 50304, 2048) == 0
    assert capi.ss_workspace_bytes(0, 128, 50304, 2048) > 0
    assert capi.ss_workspace_bytes(512, 128, (1 << 19) + 1, 2048) == 0


def test_workspace_holds_logits_and_rows(lib):
    T, d, V, P = 49152, 768, 50304, 24576
    ws = capi.ss_workspace_bytes(T, d, V, P)
    # E' [T,P] + W_C [P,d] + x' [T,d] (bf16), two partial row sums per 256-column
    # tile, per-row words, the row
    # pass's per-block partial sums (4096 x 16 B), builder bitmap
    need = (T * P * 2 + P * d * 2 + T * d * 2 + 2 * ((P + 255) // 256) * T * 4 + 4 * T * 4
            + 4096 * 16)
    assert need <= ws <= need + 2 * ((V + 31) // 32) * 4 + 64 * 1024
    # padded logit rows when P is not a multiple of 8
    assert capi.ss_workspace_bytes(100, 64, 5000, 1001) >= 100 * 1008 * 2


def _raw(lib, fn, *args):
    return getattr(lib, fn)(*args)


@pytest.mark.parametrize("T,V,P,stride,offset,code", [
    (10, 100, 0, 20011, 0, "SS_ERR_INVALID_ARG"),
    (10, 100, 101, 20011, 0, "SS_ERR_INVALID_ARG"),
    (10, 0, 1, 20011, 0, "SS_ERR_INVALID_ARG"),
    (10, (1 << 19) + 1, 8, 20011, 0, "SS_ERR_INVALID_ARG"),
    (10, 100, 10, 20011, -1, "SS_ERR_INVALID_ARG"),
    (10, 100, 10, 0, 0, "SS_ERR_INVALID_ARG"),
    (10, 100, 10, 10, 0, "SS_ERR_STRIDE_NOT_COPRIME"),
    (10, 50304, 10, 3, 0, "SS_ERR_STRIDE_NOT_COPRIME"),
])
def test_build_host_rejections(lib, T, V, P, stride, offset, code):
    fake = ctypes.c_void_p(1 << 20)  # never dereferenced: rejected before any CUDA call
    r = lib.ss_build_candidates(fake, T, V, P, offset, stride, fake, fake, fake, fake, fake,
                                1 << 30, None)
    assert r == capi.STATUS[code]


def test_build_rejects_null_and_misaligned(lib):
    a = ctypes.c_void_p(1 << 20)
    r = lib.ss_build_candidates(None, 10, 100, 10, 0, 20011, a, a, a, a, a, 1 << 30, None)
    assert r == capi.STATUS["SS_ERR_INVALID_ARG"]
    mis = ctypes.c_void_p((1 << 20) + 4)
    r = lib.ss_build_candidates(mis, 10, 100, 10, 0, 20011, a, a, a, a, a, 1 << 30, None)
    assert r == capi.STATUS["SS_ERR_MISALIGNED"]
    r = lib.ss_build_candidates(a, 10, 100, 10, 0, 20011, a, a, a, a, a, 16, None)
    assert r == capi.STATUS["SS_ERR_WORKSPACE_TOO_SMALL"]


def test_forward_backward_host_rejections(lib):
    a = ctypes.c_void_p(1 << 20)
    mis = ctypes.c_void_p((1 << 20) + 8)
    ws = capi.ss_workspace_bytes(512, 128, 50304, 2048)
    f = lib.ss_ce_forward
    assert f(a, a, a, a, 512, 100, 50304, 2048, a, a, a, a, a, ws, None) == capi.STATUS["SS_ERR_INVALID_ARG"]
    assert f(a, a, a, a, 512, 128, 50304, 2048, a, a, a, a, a, ws - 1, None) == capi.STATUS["SS_ERR_WORKSPACE_TOO_SMALL"]
    assert f(mis, a, a, a, 512, 128, 50304, 2048, a, a, a, a, a, ws, None) == capi.STATUS["SS_ERR_MISALIGNED"]
    assert f(a, None, a, a, 512, 128, 50304, 2048, a, a, a, a, a, ws, None) == capi.STATUS["SS_ERR_INVALID_ARG"]
    b = lib.ss_ce_backward
    assert b(a, a, a, a, 512, 128, 50304, 50305, a, a, a, a, ws, None) == capi.STATUS["SS_ERR_INVALID_ARG"]
    assert b(a, a, a, a, 512, 128, 50304, 2048, a, mis, a, a, ws, None) == capi.STATUS["SS_ERR_MISALIGNED"]
    assert b(None, a, a, a, 512, 128, 50304, 2048, a, a, a, a, ws, None) == capi.STATUS["SS_ERR_INVALID_ARG"]


def test_missing_library_fails_loudly(tmp_path, monkeypatch):
    monkeypatch.setattr(capi, "_lib", None)
    with pytest.raises(capi.LibraryNotBuilt):
        capi.load(str(tmp_path / "nope.so"))


def test_prefix_and_selftest_host_rejections(lib):
    a = ctypes.c_void_p(1 << 20)  # never dereferenced: rejected before any CUDA call
    f = lib.ss_prefix_positions
    assert f(a, a, a, 10, 0, a, a, None) == capi.STATUS["SS_ERR_INVALID_ARG"]  # V < 1
    assert f(a, a, a, -1, 100, a, a, None) == capi.STATUS["SS_ERR_INVALID_ARG"]  # T < 0
    assert f(a, a, a, 10, capi.MAX_VOCAB + 1, a, a, None) == capi.STATUS["SS_ERR_INVALID_ARG"]
    assert f(None, a, a, 10, 100, a, a, None) == capi.STATUS["SS_ERR_INVALID_ARG"]
    assert f(a, None, a, 10, 100, a, a, None) == capi.STATUS["SS_ERR_INVALID_ARG"]
    assert f(a, a, a, 10, 100, a, None, None) == capi.STATUS["SS_ERR_INVALID_ARG"]
    assert lib.ss_selftest_wait_limit(None, None) == capi.STATUS["SS_ERR_INVALID_ARG"]


def test_e4m3_host_rejections(lib):
    a = ctypes.c_void_p(1 << 20)  # never dereferenced: rejected before any CUDA call
    ws = capi.ss_workspace_bytes_e4m3(512, 128, 50304, 2048)
    assert ws > capi.ss_workspace_bytes(512, 128, 50304, 2048) + 512 * 128 + 2048 * 128 - 1
    assert capi.ss_workspace_bytes_e4m3(512, 136, 50304, 2048) == 0  # d % 16
    f = lib.ss_ce_forward_e4m3
    assert f(a, a, a, a, 512, 136, 50304, 2048, a, a, a, a, a, ws, None) == capi.STATUS["SS_ERR_INVALID_ARG"]
    assert f(a, a, a, a, 512, 128, 50304, 2048, a, a, a, a, a, ws - 1, None) == \
        capi.STATUS["SS_ERR_WORKSPACE_TOO_SMALL"]
    q = lib.ss_quantize_e4m3
    assert q(a, 12, a, a, a, None) == capi.STATUS["SS_ERR_INVALID_ARG"]  # n % 8
    assert q(a, 16, a, None, a, None) == capi.STATUS["SS_ERR_INVALID_ARG"]
    assert q(ctypes.c_void_p((1 << 20) + 8), 16, a, a, a, None) == capi.STATUS["SS_ERR_MISALIGNED"]


def test_bounds_checked_build_exports_the_same_symbols():
    """The bounds-checked variant (SS_BOUNDS_CHECK=1) builds from the same
    sources and exports every declared entry point."""
    path = build_lib.build(bounds_check=True)
    assert path.endswith("libsampled_ce_bounds.so") and os.path.exists(path)
    blib = ctypes.CDLL(path)
    for n in declared_functions():
        assert hasattr(blib, n), n
