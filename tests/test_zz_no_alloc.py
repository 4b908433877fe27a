"""The allocation-free projection entry point, through the C-ABI.

``qknorm_qkv_projection_noalloc`` is for callers that cannot allocate device
memory: a serving engine that owns every device allocation and refuses new
ones once it runs, or a latency-critical path on which cudaMalloc's possible
device synchronization is not acceptable.  It keeps the partial sums in a
fixed array inside the library instead of a caller-supplied workspace, and
otherwise runs the same kernels in the same order as
``qknorm_qkv_projection``.  So its output must equal that entry point's bit
for bit.

Two calls run in a row, the second smaller than the first, so the first
call's partial sums are still in the shared array when the second runs.  The
workspace entry point gets a workspace filled with NaN, so a partial sum that
either path reads without having written it shows up as a difference.  Both
calls are also checked against the oracle on sampled rows (projection and
RMS-Norm of the projection, with the bounds of the projection tests; V
columns equal to the plain projection).  The checks run twice: in
this process, after whatever ran before, and in a fresh Python process whose
first library call is this one.

This file is collected last, so a run that stops at its first failure has
run every other test first.
"""
from __future__ import annotations

import os
import subprocess
import sys

import numpy as np
import pytest
import torch

import attention_normalization_b200 as qk
import workloads
from attention_normalization_b200 import _clib
from tests.conftest import to_np
from tests.test_projection import _sample_rows, check_normalized, check_projection

pytestmark = pytest.mark.gpu

DEV = "cuda:0"
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _noalloc(b: workloads.ProjectionBatch, x: torch.Tensor, w: torch.Tensor, qkv: torch.Tensor) -> int:
    lib = qk.capi()
    gq, gk = b.gamma_q.to(DEV), b.gamma_k.to(DEV)
    st = lib.qknorm_qkv_projection_noalloc(x.data_ptr(), x.stride(0), w.data_ptr(), w.stride(0), qkv.data_ptr(),
                                           qkv.stride(0), gq.data_ptr(), gk.data_ptr(), b.T, b.D, b.Hq, b.Hk, b.Hv,
                                           b.eps, _clib.QKN_BF16, torch.cuda.current_stream().cuda_stream)
    torch.cuda.synchronize()
    return st


def run_two_calls() -> None:
    """Two calls in a row, each bit-equal to qknorm_qkv_projection and within
    the projection tests' bounds of the oracle on sampled rows."""
    lib = qk.capi()
    assert lib.qknorm_qkv_projection_noalloc_max_bytes() == 4 << 20
    batches = (workloads.qkv_projection(T=2048, D=512, Hq=4096, Hk=1024, Hv=1024, seed=21),
               workloads.qkv_projection(T=300, D=384, Hq=1024, Hk=512, Hv=256, seed=22))
    for i, b in enumerate(batches):
        x, w = b.x.to(DEV), b.w.to(DEV)
        N = b.Hq + b.Hk + b.Hv
        got = torch.full((b.T, N), float("nan"), dtype=torch.bfloat16, device=DEV)
        assert _noalloc(b, x, w, got) == _clib.QKN_OK, lib.qknorm_last_error().decode()
        need = qk.qkv_workspace_bytes(b.T, b.Hq, b.Hk)
        ws = torch.full(((need + 3) // 4,), float("nan"), dtype=torch.float32, device=DEV)
        ref = qk.qknorm_qkv_projection(x, w, b.gamma_q.to(DEV), b.gamma_k.to(DEV), b.Hq, b.Hk, b.Hv, b.eps,
                                       workspace=ws)
        torch.cuda.synchronize()
        assert qk.device_timeouts() == 0
        g, r = to_np(got.cpu()), to_np(ref.cpu())
        assert np.array_equal(g, r), (f"call {i + 1} ({b.name}): {int(np.sum(g != r))} elements differ from "
                                      "qknorm_qkv_projection")
        # the oracle: its projection checked against the GEMM's stored values
        # (the call rescales Q and K in place, V keeps the projection), its
        # RMS-Norm against the call's Q and K columns
        plain, _, _ = qk.qknorm_qkv_gemm_stats(x, w, b.Hq, b.Hk, b.Hv)
        torch.cuda.synchronize()
        rows = _sample_rows(b.T, 24, seed=300 + i)
        proj = check_projection(b, plain, rows)
        check_normalized(b, proj, got, rows)
        assert torch.equal(got[:, b.Hq + b.Hk:], plain[:, b.Hq + b.Hk:])


def test_noalloc_matches_the_workspace_entry_point_and_the_oracle_on_two_calls():
    run_two_calls()


def test_noalloc_in_a_fresh_process():
    """The same two calls as the first library calls of a new process."""
    r = subprocess.run([sys.executable, "-c", "import tests.test_zz_no_alloc as t; t.run_two_calls()"],
                       cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stdout[-4000:] + r.stderr[-4000:]


def test_noalloc_rejects_a_call_beyond_its_scratch():
    """A workspace beyond the 4 MiB scratch is refused before any launch."""
    b = workloads.ProjectionBatch("too_big", 32769, 64, 4096, 4096, 0, None, None, None, None)
    lib = qk.capi()
    st = lib.qknorm_qkv_projection_noalloc(0x10000, 64, 0x20000000, 64, 0x40000000, 8192, 0x60000000, 0x60010000,
                                           b.T, b.D, b.Hq, b.Hk, b.Hv, 1e-6, _clib.QKN_BF16, None)
    assert st == _clib.QKN_ERR_INVALID_ARG
    assert b"scratch" in lib.qknorm_last_error()
