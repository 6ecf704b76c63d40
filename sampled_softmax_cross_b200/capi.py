"""ctypes binding of ``libsampled_ce.so`` (declared in ``include/sampled_ce.h``).

Argument marshalling only: every function forwards to the C entry point of the
same name with device pointers taken from torch tensors (torch provides device
memory and streams; all arithmetic runs in the library's CUDA kernels). A
missing library raises ``LibraryNotBuilt`` on first use; there is no fallback.
"""

from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
# The library to load: the in-tree build, or another build of the same
# sources named by SAMPLED_CE_LIB (the bounds-checked debug build, say).
LIB_PATH = os.environ.get("SAMPLED_CE_LIB") or os.path.join(_PKG, "libsampled_ce.so")

DEV_STATUS_WORDS = 16
DEFAULT_STRIDE = 20011
MAX_VOCAB = 1 << 19

STATUS_NAMES = {
    0: "SS_OK", 1: "SS_ERR_INVALID_ARG", 2: "SS_ERR_BAD_TARGET", 3: "SS_ERR_TOO_MANY_TARGETS",
    4: "SS_ERR_NO_FREE_CLASSES", 5: "SS_ERR_STRIDE_NOT_COPRIME", 6: "SS_ERR_WORKSPACE_TOO_SMALL",
    7: "SS_ERR_MISALIGNED", 8: "SS_ERR_CUDA", 9: "SS_ERR_UNSUPPORTED_DEVICE",
    10: "SS_ERR_KERNEL_TIMEOUT", 11: "SS_ERR_BAD_INDEX",
}
STATUS = {v: k for k, v in STATUS_NAMES.items()}

EXPORTS = (
    "ss_workspace_bytes", "ss_build_workspace_bytes", "ss_build_candidates",
    "ss_build_candidates_noalloc", "ss_ce_forward", "ss_ce_backward",
    "ss_status_string", "ss_last_cuda_error", "ss_version", "ss_timing_enable",
    "ss_timing_reset", "ss_timing_count", "ss_timing_query", "ss_prefix_positions",
    "ss_selftest_wait_limit", "ss_ce_forward_e4m3", "ss_workspace_bytes_e4m3", "ss_quantize_e4m3",
    "ss_workspace_wc_offset",
)


class LibraryNotBuilt(RuntimeError):
    pass


class SampledCEError(RuntimeError):
    def __init__(self, fn: str, code: int, detail: str = ""):
        name = STATUS_NAMES.get(code, str(code))
        super().__init__(f"{fn} returned {name}" + (f": {detail}" if detail else ""))
        self.code = code
        self.name = name


_lib = None

_p = ctypes.c_void_p
_i32 = ctypes.c_int32
_i64 = ctypes.c_int64
_sz = ctypes.c_size_t


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load the library (once) and declare the C signatures."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise LibraryNotBuilt(
            f"{path} is missing: build it with `python -m sampled_softmax_cross_b200.build_lib`")
    lib = ctypes.CDLL(path)
    sig = {
        "ss_workspace_bytes": (_sz, [_i64, _i32, _i32, _i32]),
        "ss_workspace_wc_offset": (_sz, [_i64, _i32, _i32, _i32]),
        "ss_build_workspace_bytes": (_sz, [_i32]),
        "ss_build_candidates": (_i32, [_p, _i64, _i32, _i32, _i64, _i32, _p, _p, _p, _p, _p, _sz, _p]),
        "ss_build_candidates_noalloc": (_i32, [_p, _i64, _i32, _i32, _i64, _i32, _p, _p, _p, _p,
                                                _p]),
        "ss_ce_forward": (_i32, [_p, _p, _p, _p, _i64, _i32, _i32, _i32, _p, _p, _p, _p, _p, _sz, _p]),
        "ss_ce_backward": (_i32, [_p, _p, _p, _p, _i64, _i32, _i32, _i32, _p, _p, _p, _p, _sz,
                                  _p]),
        "ss_prefix_positions": (_i32, [_p, _p, _p, _i64, _i32, _p, _p, _p]),
        "ss_ce_forward_e4m3": (_i32, [_p, _p, _p, _p, _i64, _i32, _i32, _i32, _p, _p, _p, _p, _p,
                                      _sz, _p]),
        "ss_workspace_bytes_e4m3": (_sz, [_i64, _i32, _i32, _i32]),
        "ss_quantize_e4m3": (_i32, [_p, _i64, _p, _p, _p, _p]),
        "ss_selftest_wait_limit": (_i32, [_p, _p]),
        "ss_status_string": (ctypes.c_char_p, [_i32]),
        "ss_last_cuda_error": (ctypes.c_char_p, []),
        "ss_version": (_i32, []),
        "ss_timing_enable": (_i32, [_i32]),
        "ss_timing_reset": (_i32, []),
        "ss_timing_count": (_i32, []),
        "ss_timing_query": (_i32, [_i32, ctypes.c_char_p, _i32, ctypes.POINTER(_i32),
                                   ctypes.POINTER(ctypes.c_double)]),
    }
    for name, (res, args) in sig.items():
        f = getattr(lib, name)
        f.restype = res
        f.argtypes = args
    _lib = lib
    return lib


def _ptr(t) -> int | None:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream) -> int | None:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(fn: str, code: int):
    if code != 0:
        lib = load()
        detail = lib.ss_last_cuda_error().decode() if code == STATUS["SS_ERR_CUDA"] else ""
        raise SampledCEError(fn, code, detail)


def ss_workspace_bytes(T: int, d: int, V: int, P: int) -> int:
    return int(load().ss_workspace_bytes(T, d, V, P))


def ss_workspace_wc_offset(T: int, d: int, V: int, P: int) -> int:
    """Byte offset of W_C [P, d] bf16 in the workspace after a forward (-1: invalid sizes)."""
    off = int(load().ss_workspace_wc_offset(T, d, V, P))
    return -1 if off == (1 << 64) - 1 else off


def ss_build_workspace_bytes(V: int) -> int:
    return int(load().ss_build_workspace_bytes(V))


def ss_build_candidates(targets, V, P, offset, stride, candidates, target_pos, vocab_pos,
                        dev_status, workspace, stream=None):
    T = targets.numel()
    code = load().ss_build_candidates(
        _ptr(targets), T, V, P, offset, stride, _ptr(candidates), _ptr(target_pos),
        _ptr(vocab_pos), _ptr(dev_status), _ptr(workspace), workspace.numel() * workspace.element_size(),
        _stream(stream))
    _check("ss_build_candidates", code)


def ss_build_candidates_noalloc(targets, V, P, offset, stride, candidates, target_pos,
                                vocab_pos, dev_status, stream=None):
    """ss_build_candidates without a workspace (scratch inside the library)."""
    T = targets.numel()
    code = load().ss_build_candidates_noalloc(
        _ptr(targets), T, V, P, offset, stride, _ptr(candidates), _ptr(target_pos),
        _ptr(vocab_pos), _ptr(dev_status), _stream(stream))
    _check("ss_build_candidates_noalloc", code)


def ss_ce_forward(x, lm_head, candidates, target_pos, T, d, V, P, loss, lse, n_valid, dev_status,
                  workspace, stream=None):
    code = load().ss_ce_forward(
        _ptr(x), _ptr(lm_head), _ptr(candidates), _ptr(target_pos), T, d, V, P, _ptr(loss),
        _ptr(lse), _ptr(n_valid), _ptr(dev_status), _ptr(workspace),
        workspace.numel() * workspace.element_size(), _stream(stream))
    _check("ss_ce_forward", code)


def ss_ce_backward(grad_loss, candidates, vocab_pos, n_valid, T, d, V, P, dx, dW, dev_status,
                   workspace, stream=None):
    code = load().ss_ce_backward(
        _ptr(grad_loss), _ptr(candidates), _ptr(vocab_pos), _ptr(n_valid), T, d, V, P, _ptr(dx), _ptr(dW), _ptr(dev_status), _ptr(workspace),
        workspace.numel() * workspace.element_size(), _stream(stream))
    _check("ss_ce_backward", code)


def ss_workspace_bytes_e4m3(T: int, d: int, V: int, P: int) -> int:
    return int(load().ss_workspace_bytes_e4m3(T, d, V, P))


def ss_ce_forward_e4m3(x, lm_head, candidates, target_pos, T, d, V, P, loss, lse, n_valid,
                       dev_status, workspace, stream=None):
    """ss_ce_forward with the logits GEMM on per-tensor e4m3 operands."""
    code = load().ss_ce_forward_e4m3(
        _ptr(x), _ptr(lm_head), _ptr(candidates), _ptr(target_pos), T, d, V, P, _ptr(loss),
        _ptr(lse), _ptr(n_valid), _ptr(dev_status), _ptr(workspace),
        workspace.numel() * workspace.element_size(), _stream(stream))
    _check("ss_ce_forward_e4m3", code)


def ss_quantize_e4m3(src, dst, scale, scratch, stream=None):
    """dst = e4m3 codes of src * 2^-k; scale[0] = 2^k (per-tensor power of two)."""
    code = load().ss_quantize_e4m3(_ptr(src), src.numel(), _ptr(dst), _ptr(scale), _ptr(scratch),
                                   _stream(stream))
    _check("ss_quantize_e4m3", code)


def ss_prefix_positions(prefix_table, targets, vocab_pos, V, prefix_pos, dev_status, stream=None):
    """prefix_pos[i] = position in C of prefix_table[targets[i]], -1 if absent."""
    code = load().ss_prefix_positions(
        _ptr(prefix_table), _ptr(targets), _ptr(vocab_pos), targets.numel(), V, _ptr(prefix_pos),
        _ptr(dev_status), _stream(stream))
    _check("ss_prefix_positions", code)


def ss_selftest_wait_limit(dev_status, stream=None):
    """Run one kernel wait out on purpose; the outcome lands in dev_status[8..11]."""
    _check("ss_selftest_wait_limit", load().ss_selftest_wait_limit(_ptr(dev_status),
                                                                    _stream(stream)))


def ss_status_string(code: int) -> str:
    return load().ss_status_string(code).decode()


def ss_version() -> int:
    return int(load().ss_version())


def ss_timing_enable(on, gemms_only: bool = False):
    """Bracket each launch with CUDA events (only the GEMM launches if gemms_only)."""
    mode = (2 if gemms_only else 1) if on else 0
    _check("ss_timing_enable", load().ss_timing_enable(mode))


def ss_timing_reset():
    _check("ss_timing_reset", load().ss_timing_reset())


def ss_timing_read() -> dict:
    """{kernel name: (launches, total ms)} for the launches recorded so far."""
    lib = load()
    out = {}
    for i in range(lib.ss_timing_count()):
        buf = ctypes.create_string_buffer(64)
        n = _i32()
        ms = ctypes.c_double()
        _check("ss_timing_query", lib.ss_timing_query(i, buf, 64, ctypes.byref(n), ctypes.byref(ms)))
        out[buf.value.decode()] = (n.value, ms.value)
    return out


# ---------------------------------------------------------------------------
# Convenience: buffers for one microbatch, and the three calls in order.
# ---------------------------------------------------------------------------


class SampledCE:
    """Caller-owned device buffers for one (T, d, V, P) shape and the three calls.

    Buffers keep one identity for the object's life, so a step can be captured
    in a CUDA graph by the caller. Nothing here computes; it allocates with
    torch and calls the C ABI.
    """

    def __init__(self, T: int, d: int, V: int, P: int, device="cuda", precision: str = "bf16"):
        if precision not in ("bf16", "e4m3"):
            raise ValueError(f"precision {precision!r}: 'bf16' or 'e4m3' (logits GEMM operands)")
        self.T, self.d, self.V, self.P = T, d, V, P
        self.precision = precision
        dev = torch.device(device)
        ws = (ss_workspace_bytes_e4m3 if precision == "e4m3" else ss_workspace_bytes)(T, d, V, P)
        if ws == 0:
            raise SampledCEError("ss_workspace_bytes", STATUS["SS_ERR_INVALID_ARG"],
                                 f"T={T} d={d} V={V} P={P}")
        self.workspace = torch.empty(ws, dtype=torch.uint8, device=dev)
        self.candidates = torch.empty(P, dtype=torch.int32, device=dev)
        self.target_pos = torch.empty(max(T, 1), dtype=torch.int32, device=dev)
        self.vocab_pos = torch.empty(V, dtype=torch.int32, device=dev)
        self.dev_status = torch.zeros(DEV_STATUS_WORDS, dtype=torch.int32, device=dev)
        self.loss = torch.zeros(1, dtype=torch.float32, device=dev)
        self.lse = torch.empty(max(T, 1), dtype=torch.float32, device=dev)
        self.n_valid = torch.zeros(1, dtype=torch.int32, device=dev)
        self.grad_loss = torch.ones(1, dtype=torch.float32, device=dev)
        self.dx = torch.empty((max(T, 1), d), dtype=torch.bfloat16, device=dev)
        self.dW = torch.empty((V, d), dtype=torch.bfloat16, device=dev)

    def build(self, targets, offset, stride=DEFAULT_STRIDE, stream=None):
        ss_build_candidates(targets, self.V, self.P, offset, stride, self.candidates,
                            self.target_pos, self.vocab_pos, self.dev_status, self.workspace, stream)

    def forward(self, x, lm_head, stream=None):
        fwd = ss_ce_forward_e4m3 if self.precision == "e4m3" else ss_ce_forward
        fwd(x, lm_head, self.candidates, self.target_pos, self.T, self.d, self.V, self.P,
            self.loss, self.lse, self.n_valid, self.dev_status, self.workspace, stream)

    def backward(self, grad_loss=None, stream=None, dW=None):
        """dx into self.dx; dW into self.dW, or into the [V, d] bf16 tensor `dW`."""
        g = self.grad_loss if grad_loss is None else grad_loss
        ss_ce_backward(g, self.candidates, self.vocab_pos, self.n_valid, self.T, self.d, self.V,
                       self.P, self.dx, self.dW if dW is None else dW, self.dev_status,
                       self.workspace, stream)

    def step(self, targets, x, lm_head, offset, stride=DEFAULT_STRIDE, grad_loss=None, stream=None):
        self.build(targets, offset, stride, stream)
        self.forward(x, lm_head, stream)
        self.backward(grad_loss, stream)

    def status(self) -> list[int]:
        return self.dev_status.tolist()
