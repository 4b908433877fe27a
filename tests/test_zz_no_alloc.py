"""The allocation-free projection entry point, through the C-ABI.

``qknorm_qkv_projection_noalloc`` serves callers that cannot allocate device
memory (a host engine that owns every allocation, or a path that cannot take
cudaMalloc's possible device synchronization): it keeps its partial sums in a
fixed array inside the library instead of a caller-supplied workspace.  Its
results must match ``qknorm_qkv_projection`` (same kernels, same order of
operations), checked here within the 1-ulp tolerance the bf16 parity tests use
on two calls in a row, the second smaller than the first so stale partial sums
from the first call are still in the shared array.

This file is named to be collected last.
"""
from __future__ import annotations

import pytest
import torch

import attention_normalization_b200 as qk
import workloads
from attention_normalization_b200 import _clib
from tests.conftest import bf16_ulp_distance, to_np

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def _noalloc(b: workloads.ProjectionBatch, x: torch.Tensor, w: torch.Tensor, qkv: torch.Tensor) -> int:
    lib = qk.capi()
    gq, gk = b.gamma_q.to(DEV), b.gamma_k.to(DEV)
    st = lib.qknorm_qkv_projection_noalloc(x.data_ptr(), x.stride(0), w.data_ptr(), w.stride(0), qkv.data_ptr(),
                                           qkv.stride(0), gq.data_ptr(), gk.data_ptr(), b.T, b.D, b.Hq, b.Hk, b.Hv,
                                           b.eps, _clib.QKN_BF16, torch.cuda.current_stream().cuda_stream)
    torch.cuda.synchronize()
    return st


def test_noalloc_matches_the_workspace_entry_point_on_two_calls():
    lib = qk.capi()
    assert lib.qknorm_qkv_projection_noalloc_max_bytes() == 4 << 20
    for b in (workloads.qkv_projection(T=2048, D=512, Hq=4096, Hk=1024, Hv=1024, seed=21),
              workloads.qkv_projection(T=300, D=384, Hq=1024, Hk=512, Hv=256, seed=22)):
        x, w = b.x.to(DEV), b.w.to(DEV)
        N = b.Hq + b.Hk + b.Hv
        got = torch.empty((b.T, N), dtype=torch.bfloat16, device=DEV)
        assert _noalloc(b, x, w, got) == _clib.QKN_OK, lib.qknorm_last_error().decode()
        ref = qk.qknorm_qkv_projection(x, w, b.gamma_q.to(DEV), b.gamma_k.to(DEV), b.Hq, b.Hk, b.Hv, b.eps)
        torch.cuda.synchronize()
        d = bf16_ulp_distance(to_np(got.cpu()), to_np(ref.cpu()))
        assert d.max() <= 1, f"{b.name}: {int(d.max())} ulp from qknorm_qkv_projection"
    assert qk.device_timeouts() == 0


def test_noalloc_rejects_a_call_beyond_its_scratch():
    """A workspace beyond the 4 MiB scratch is refused before any launch."""
    b = workloads.ProjectionBatch("too_big", 32769, 64, 4096, 4096, 0, None, None, None, None)
    lib = qk.capi()
    st = lib.qknorm_qkv_projection_noalloc(0x10000, 64, 0x20000000, 64, 0x40000000, 8192, 0x60000000, 0x60010000,
                                           b.T, b.D, b.Hq, b.Hk, b.Hv, 1e-6, _clib.QKN_BF16, None)
    assert st == _clib.QKN_ERR_INVALID_ARG
    assert b"scratch" in lib.qknorm_last_error()
