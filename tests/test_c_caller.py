"""The library from plain C: a C program (tests/c/qknorm_c_caller.c) that
includes only include/qknorm.h and the CUDA runtime, links libqknorm.so and
calls qknorm_layerwise on device buffers and qknorm_layerwise_host on
page-locked host buffers.  On the CPU the program must compile and link
against the header and the library; on a GPU both outputs must match the
oracle, and each other bit for bit (the same kernel on the same rows)."""
from __future__ import annotations

import os
import shutil
import subprocess

import numpy as np
import pytest
import torch

import oracle
import workloads
from attention_normalization_b200 import build as qbuild
from tests.conftest import bf16_ulp_distance, to_np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SOURCE = os.path.join(ROOT, "tests", "c", "qknorm_c_caller.c")
CUDA = os.environ.get("CUDA_HOME", "/usr/local/cuda")


def _compile(out_dir: str) -> str:
    qbuild.build(quiet=True)
    exe = os.path.join(out_dir, "qknorm_c_caller")
    lib_dir = os.path.dirname(qbuild.LIBRARY)
    cmd = ["gcc", "-std=c11", "-O2", "-Wall", "-Werror", SOURCE, "-o", exe,
           "-I", os.path.join(ROOT, "include"), "-I", os.path.join(CUDA, "include"),
           "-L", lib_dir, "-lqknorm", f"-Wl,-rpath,{lib_dir}",
           "-L", os.path.join(CUDA, "lib64"), "-lcudart", f"-Wl,-rpath,{os.path.join(CUDA, 'lib64')}"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    return exe


@pytest.mark.skipif(shutil.which("gcc") is None, reason="no C compiler")
def test_c_caller_compiles_and_links(tmp_path):
    assert os.path.exists(_compile(str(tmp_path)))


@pytest.mark.gpu
def test_c_caller_matches_the_oracle(tmp_path):
    exe = _compile(str(tmp_path))
    b = workloads.random_rows(300, 1024, 256, torch.bfloat16, seed=17)
    names = ("q", "k", "gq", "gk", "qo", "ko", "qo_host", "ko_host")
    paths = {n: str(tmp_path / f"{n}.bin") for n in names}
    for n, t in (("q", b.q), ("k", b.k), ("gq", b.gamma_q), ("gk", b.gamma_k)):
        to_np(t).tofile(paths[n])
    chunk = 64  # five chunks, the last one ragged, through two ring slots
    r = subprocess.run([exe, str(b.T), str(b.Hq), str(b.Hk), repr(b.eps), str(chunk)] + [paths[n] for n in names[:4]]
                       + [paths[n] for n in names[4:]], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stdout + r.stderr
    assert "invalid argument" in r.stdout and "ok" in r.stdout
    for n, view, g, H in (("qo", b.q, b.gamma_q, b.Hq), ("ko", b.k, b.gamma_k, b.Hk)):
        got = np.fromfile(paths[n], dtype=np.uint16).reshape(b.T, H)
        want, _, _ = oracle.rmsnorm_rows(to_np(view), H, to_np(g), b.eps)
        assert bf16_ulp_distance(got, want).max() <= 1
        host = np.fromfile(paths[n + "_host"], dtype=np.uint16).reshape(b.T, H)
        assert np.array_equal(host, got), f"{n}: the host-buffer path differs from the device path"
