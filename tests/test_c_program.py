"""The C ABI from plain C: tests/c/abi_demo.c includes only include/nvnorm.h and the CUDA
runtime header and links against libnvnorm.so.

CPU: the program compiles as C99 with every warning an error, and links (so the header is
valid C and its declarations match the exported symbols).  GPU: the program runs
add_rms_norm, rms_norm and layer_norm on device buffers it allocates itself, and its outputs
match the oracle.
"""
import os
import shutil
import subprocess

import numpy as np
import pytest

import oracle
from rope_add_rms_b200 import library_path, synth
from checks import check_bf16

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CUDA = os.environ.get("CUDA_HOME", "/usr/local/cuda")


def build_demo(tmp_path):
    if shutil.which("gcc") is None:
        pytest.skip("gcc is not installed")
    if not os.path.exists(library_path):
        pytest.skip("libnvnorm.so is not built")
    exe = str(tmp_path / "abi_demo")
    libdir = os.path.dirname(library_path)
    cmd = ["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror",
           "-I", os.path.join(ROOT, "include"), "-I", os.path.join(CUDA, "include"),
           os.path.join(ROOT, "tests", "c", "abi_demo.c"), "-o", exe,
           "-L", libdir, "-lnvnorm", "-L", os.path.join(CUDA, "lib64"), "-lcudart",
           f"-Wl,-rpath,{libdir}", f"-Wl,-rpath,{os.path.join(CUDA, 'lib64')}"]
    res = subprocess.run(cmd, capture_output=True, text=True)
    assert res.returncode == 0, res.stderr
    return exe


def test_c_program_builds(tmp_path):
    assert os.path.exists(build_demo(tmp_path))


@pytest.mark.gpu
def test_c_program_runs_and_matches_the_oracle(tmp_path):
    exe = build_demo(tmp_path)
    rows, D = 300, 4096
    inp = synth.add_rms_inputs(rows, D, "bf16", seed=12)
    x, r, w = (synth.to_numpy(inp[k]) for k in ("x", "r", "w"))
    src, dst = tmp_path / "in.bin", tmp_path / "out.bin"
    src.write_bytes(np.concatenate([x.ravel(), r.ravel(), w.ravel()]).astype(np.uint16).tobytes())
    res = subprocess.run([exe, str(rows), str(D), str(src), str(dst)], capture_output=True,
                         text=True, timeout=120)
    assert res.returncode == 0, res.stdout + res.stderr
    out = np.frombuffer(dst.read_bytes(), dtype=np.uint16).reshape(4, rows, D)
    y, h, z, u = out
    y_ref, h_ref = oracle.add_rms_norm(x, r, w, 1e-5)
    assert (h == h_ref).all(), "h is not bit-exact"
    check_bf16(y, y_ref, "y")
    # the next two ops read the device y, which the check above pinned to the oracle's
    check_bf16(z, oracle.rms_norm(y, w, 1e-6), "rms_norm(y)")
    check_bf16(u, oracle.layer_norm(y, w, None, 1e-5), "layer_norm(y)")
