"""The C ABI from plain C: the header compiles as C99, and a C program that
allocates device memory with the CUDA runtime and calls ss_build_candidates,
ss_ce_forward and ss_ce_backward gives the oracle's results."""

import os
import shutil
import subprocess

import numpy as np
import pytest

from sampled_softmax_cross_b200 import build_lib
from sampled_softmax_cross_b200 import workloads as wl

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "tests", "c_abi", "step_from_c.c")
CUDA = os.environ.get("CUDA_HOME", "/usr/local/cuda")
GCC = shutil.which("gcc")


def _compile(out):
    lib_dir = os.path.dirname(build_lib.build())
    cmd = [GCC, "-std=c99", "-Wall", "-Wextra", "-Werror", "-O2", "-I", os.path.join(ROOT, "include"),
           "-I", os.path.join(CUDA, "include"), SRC, "-L", lib_dir, "-lsampled_ce",
           "-L", os.path.join(CUDA, "lib64"), "-lcudart", f"-Wl,-rpath,{lib_dir}", "-o", out]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr


@pytest.mark.skipif(GCC is None, reason="no gcc")
def test_header_is_c99(tmp_path):
    c = tmp_path / "h.c"
    c.write_text('#include "sampled_ce.h"\nint main(void) { return ss_version() > 0 ? 0 : 1; }\n')
    r = subprocess.run([GCC, "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic",
                        "-fsyntax-only", "-I", os.path.join(ROOT, "include"), str(c)],
                       capture_output=True, text=True)
    assert r.returncode == 0, r.stderr


@pytest.mark.skipif(GCC is None, reason="no gcc")
def test_c_program_builds(tmp_path):
    _compile(str(tmp_path / "step_from_c"))


@pytest.mark.gpu
def test_c_program_matches_oracle(tmp_path):
    from oracle import sampled_ce as oc

    T, d, V, P, off = 640, 128, 5003, 1100, 321
    x, lm, t = wl.make_inputs(T, d, V, 1.1, 0.05, 71)
    inp, out, exe = tmp_path / "in.bin", tmp_path / "out.bin", tmp_path / "step_from_c"
    with open(inp, "wb") as f:
        f.write(np.ascontiguousarray(x).tobytes())
        f.write(np.ascontiguousarray(lm).tobytes())
        f.write(np.ascontiguousarray(t, dtype=np.int32).tobytes())
    _compile(str(exe))
    r = subprocess.run([str(exe), str(inp), str(out), str(T), str(d), str(V), str(P), str(off)],
                       capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stderr
    buf = open(out, "rb").read()
    o = 0

    def take(dtype, n):
        nonlocal o
        a = np.frombuffer(buf, dtype=dtype, count=n, offset=o)
        o += a.nbytes
        return a

    loss = float(take(np.float32, 1)[0])
    n_valid = int(take(np.int32, 1)[0])
    st = take(np.int32, 16)
    cand = take(np.int32, P)
    tpos = take(np.int32, T)
    dx = wl.bits_to_f64(take(np.uint16, T * d).reshape(T, d))
    dW = wl.bits_to_f64(take(np.uint16, V * d).reshape(V, d))
    assert o == len(buf)
    ref = oc.sampled_ce(wl.bits_to_f64(x), wl.bits_to_f64(lm), t, P, off)
    assert st[0] == 0 and st[8] == 0
    assert np.array_equal(cand, ref["candidates"]) and np.array_equal(tpos, ref["target_pos"])
    assert n_valid == ref["n_valid"]
    assert abs(loss - ref["loss"]) <= 1e-3 * abs(ref["loss"])
    assert np.linalg.norm(dx - ref["dx"]) <= 2e-2 * np.linalg.norm(ref["dx"])
    assert np.linalg.norm(dW - ref["dW"]) <= 2e-2 * np.linalg.norm(ref["dW"])
