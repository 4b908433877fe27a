"""The QKV projection with Phase A sums in its epilogue, against the oracle.

The tensor-core GEMM (``qknorm_qkv_gemm_stats``) and the projection + QK-Norm
pipeline (``qknorm_qkv_projection``) are compared, through the C-ABI, with the
CPU oracle's double-precision projection (``oracle.project_rows``), its
per-tile squared sums (``oracle.partial_sumsq``) and its RMS-Norm of the
projected rows (``oracle.rmsnorm_rows``).

Tolerances, derived from the arithmetic:

* projection: the GPU forms each dot product of D exact bf16 x bf16 products
  in fp32 in an order of its own, so ``|acc - exact| <= g * sum_d |x_d w_d|``
  with ``g = D u / (1 - D u)`` and ``u = 2^-23`` (allowing for an adder that
  truncates rather than rounds), then rounds once to bf16 (half an ulp).  The
  test checks ``|qkv - exact| <= g * sum|x w| + ulp(|exact| + g * sum|x w|) / 2``
  everywhere, and that qkv is within 1 ulp of the oracle's correctly rounded
  value wherever the accumulation bound is below half an ulp (where the sum
  cancels, the fp32 error can span several ulps of a small result).  The
  worst-case bound is loose for long sums, so the test also asks that 99% of
  the elements sit within 1 ulp, the typical case when rounding errors of
  random sign grow like sqrt(D) u.
* tile sums: a stored value x and the oracle's o differ by at most
  ``delta = bound + ulp(o) / 2``, so each square differs by at most
  ``2|o| delta + delta^2``; the fp32 sum of 256 terms adds at most
  ``256 * 2^-24`` of the sum.
* normalized Q and K: where a projected value sits k ulps from the oracle's,
  x * gamma * r moves by at most 2k ulps of the result (gamma * r can carry x
  across a binade), and the final rounding adds one: ``<= 2k + 1`` ulps, with
  k the element's measured projection distance (taken as 1 where it matched).
"""
from __future__ import annotations

import math

import numpy as np
import pytest
import torch

import attention_normalization_b200 as qk
import oracle
import workloads
from tests.conftest import bf16_ulp_distance, to_np

pytestmark = pytest.mark.gpu

DEV = "cuda:0"
TILE = 256


def _bf16_ulp(mag: np.ndarray) -> np.ndarray:
    """Spacing of bfloat16 values at magnitude `mag` (>= the smallest normal's)."""
    m = np.maximum(np.abs(mag), 2.0 ** -126)
    return np.exp2(np.floor(np.log2(m)) - 7)


def _bits_to_double(bits: np.ndarray) -> np.ndarray:
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def check_projection(b: workloads.ProjectionBatch, qkv_gpu: torch.Tensor, rows: np.ndarray):
    """qkv rows `rows` against the oracle; returns the oracle's bf16 rows."""
    xs, ws = to_np(b.x), to_np(b.w)
    y_bits, y_exact = oracle.project_rows(xs, ws, rows)
    got = to_np(qkv_gpu.cpu()[torch.as_tensor(rows)])
    absdot = np.abs(b.x.double().numpy()[rows]) @ np.abs(b.w.double().numpy()).T
    u = 2.0 ** -23
    g = b.D * u / (1 - b.D * u)
    acc_err = g * absdot
    bound = acc_err + 0.5 * _bf16_ulp(np.abs(y_exact) + acc_err)
    err = np.abs(_bits_to_double(got) - y_exact)
    worst = np.unravel_index(np.argmax(err - bound), err.shape)
    assert np.all(err <= bound), f"projection error {err[worst]:.3g} > bound {bound[worst]:.3g} at {worst}"
    d = bf16_ulp_distance(got, y_bits)
    tight = acc_err <= 0.5 * _bf16_ulp(y_exact)
    assert d[tight].max(initial=0) <= 1, "projection more than 1 ulp from the oracle's rounding"
    # Not a bound but the typical case: with terms of random sign the fp32
    # error grows like sqrt(D) u, far below half an ulp of the result.
    assert np.mean(d <= 1) > 0.99, "projection: fewer than 99% of elements within 1 ulp"
    return y_bits, bound, d


def check_tile_sums(proj, sums_gpu: torch.Tensor, rows: np.ndarray, col0: int, tiles: int):
    """Per-tile squared sums of the projected rows against the oracle's."""
    y_bits, bound, _ = proj
    got = sums_gpu.cpu().double().numpy()[:, rows]  # [tiles, n_rows]
    for p in range(tiles):
        cols = slice(col0 + p * TILE, col0 + (p + 1) * TILE)
        blk = np.ascontiguousarray(y_bits[:, cols])
        ref = oracle.partial_sumsq(blk, TILE, TILE, blk.shape[0])
        o = _bits_to_double(blk)
        delta = bound[:, cols] + 0.5 * _bf16_ulp(o)
        tol = np.sum(2 * np.abs(o) * delta + delta * delta, axis=1) + TILE * 2.0 ** -24 * ref + 1e-30
        err = np.abs(got[p] - ref)
        assert np.all(err <= tol), f"tile {p}: sum error {err.max():.3g} > {tol[np.argmax(err - tol)]:.3g}"


def check_normalized(b: workloads.ProjectionBatch, proj, out_gpu: torch.Tensor, rows: np.ndarray):
    """Q and K columns of the pipeline's output against the oracle's RMS-Norm
    of its own projected rows (full-width divisor)."""
    y_bits, _, dproj = proj
    got = to_np(out_gpu.cpu()[torch.as_tensor(rows)])
    for c0, H, gm, name in ((0, b.Hq, b.gamma_q, "Q"), (b.Hq, b.Hk, b.gamma_k, "K")):
        src = np.ascontiguousarray(y_bits[:, c0:c0 + H])
        ref, _, _ = oracle.rmsnorm_rows(src, H, to_np(gm), b.eps)
        d = bf16_ulp_distance(got[:, c0:c0 + H], ref)
        allowed = 2 * np.maximum(dproj[:, c0:c0 + H], 1) + 1
        assert np.all(d <= allowed), f"normalized {name}: {int((d - allowed).max())} ulp beyond the bound"
        assert np.mean(d <= 1) > 0.99, f"normalized {name}: fewer than 99% of elements within 1 ulp"


def _sample_rows(T: int, n: int, seed: int) -> np.ndarray:
    rng = np.random.default_rng(seed)
    extra = rng.choice(T, size=min(n, T), replace=False)
    return np.unique(np.concatenate([[0, T - 1, min(127, T - 1), min(128, T - 1)], extra]))


@pytest.mark.parametrize("T,D,Hq,Hk,Hv", [
    (200, 320, 512, 256, 256),   # ragged last token tile, 5 k-blocks
    (1, 64, 256, 256, 0),        # one token, one k-block, no V
    (129, 200, 256, 512, 256),   # D not a multiple of the k-block: zero-filled tail
    (300, 8, 256, 256, 512),     # D = 8: one partial k-block
    (128, 1000, 1024, 256, 256),
    (1000, 136, 512, 512, 512),  # 48 tiles
    (2048, 320, 2048, 1024, 1024),  # 256 tiles: more than one per CTA; the ring wraps inside tiles
    (4096, 64, 1024, 1024, 1024),   # 384 tiles of one k-block each: both accumulators cycle often
])
def test_gemm_stats_small_shapes(T, D, Hq, Hk, Hv):
    b = workloads.qkv_projection(T=T, D=D, Hq=Hq, Hk=Hk, Hv=Hv, seed=T + D)
    qkv, qs, ks = qk.qknorm_qkv_gemm_stats(b.x.to(DEV), b.w.to(DEV), Hq, Hk, Hv)
    torch.cuda.synchronize()
    rows = np.arange(T) if T <= 300 else _sample_rows(T, 40, T)
    proj = check_projection(b, qkv, rows)
    check_tile_sums(proj, qs, rows, 0, Hq // TILE)
    check_tile_sums(proj, ks, rows, Hq, Hk // TILE)
    assert qk.device_timeouts() == 0


def test_projection_pipeline_small_and_strided():
    """The full pipeline on padded-stride operands and output; the padding
    columns and the V columns are checked too."""
    b = workloads.qkv_projection(T=333, D=192, Hq=512, Hk=256, Hv=256, seed=9)
    N = b.Hq + b.Hk + b.Hv
    xb = torch.zeros((b.T, b.D + 64), dtype=torch.bfloat16, device=DEV)
    xb[:, :b.D] = b.x.to(DEV)
    wb = torch.zeros((N, b.D + 8), dtype=torch.bfloat16, device=DEV)
    wb[:, :b.D] = b.w.to(DEV)
    ob = torch.full((b.T, N + 16), 7.0, dtype=torch.bfloat16, device=DEV)
    qkv = qk.qknorm_qkv_projection(xb[:, :b.D], wb[:, :b.D], b.gamma_q.to(DEV), b.gamma_k.to(DEV), b.Hq, b.Hk,
                                   b.Hv, b.eps, qkv=ob[:, :N])
    plain, _, _ = qk.qknorm_qkv_gemm_stats(b.x.to(DEV), b.w.to(DEV), b.Hq, b.Hk, b.Hv)
    torch.cuda.synchronize()
    rows = np.arange(b.T)
    proj = check_projection(b, plain, rows)
    check_normalized(b, proj, qkv, rows)
    assert torch.equal(qkv[:, b.Hq + b.Hk:], plain[:, b.Hq + b.Hk:])  # V keeps the projection
    assert torch.all(ob[:, N:] == 7.0)  # padding untouched
    assert qk.device_timeouts() == 0


def test_projection_full_size_sampled_rows():
    """OLMo2-7B-shaped prefill (T=4096, D=4096, 32+32+32 heads of 128): the
    launch the benchmark times, checked on sampled tokens spanning every
    token tile boundary kind."""
    b = workloads.qkv_projection()
    x, w = b.x.to(DEV), b.w.to(DEV)
    plain, qs, ks = qk.qknorm_qkv_gemm_stats(x, w, b.Hq, b.Hk, b.Hv)
    out = qk.qknorm_qkv_projection(x, w, b.gamma_q.to(DEV), b.gamma_k.to(DEV), b.Hq, b.Hk, b.Hv, b.eps)
    torch.cuda.synchronize()
    rows = _sample_rows(b.T, 20, 5)
    proj = check_projection(b, plain, rows)
    check_tile_sums(proj, qs, rows, 0, b.Hq // TILE)
    check_tile_sums(proj, ks, rows, b.Hq, b.Hk // TILE)
    check_normalized(b, proj, out, rows)
    assert qk.device_timeouts() == 0


@pytest.mark.parametrize("T,D,Hq,Hk,Hv", [
    (16284, 3072, 2048, 512, 512),     # X (100 MB) beyond half of L2, W (19 MB) within: one token block per group
    (12000, 4096, 4096, 4096, 2048),   # X (99 MB) and W (84 MB) beyond: groups of ~sqrt(clusters), ragged last
])
def test_projection_rasters_beyond_l2(T, D, Hq, Hk, Hv):
    """Shapes whose operands do not fit in half of L2 run the GEMM in smaller
    raster groups (on a B200: 148 SMs, 126 MB L2); the tiles, their sums and
    the normalized Q and K must not depend on the order.  Checked on sampled
    rows against the oracle, with the ragged last token tile among them, and
    bit for bit between the vector and the scalar apply pass (16-byte aligned
    and unaligned gamma)."""
    plan = qk.qkv_gemm_plan(T, D, Hq, Hk, Hv)
    if plan["clusters"] == 74 and torch.cuda.get_device_properties(DEV).L2_cache_size >= 120 << 20:
        assert plan["group_units"] == (1 if T == 16284 else 7), plan  # the raster the docstring names
    b = workloads.qkv_projection(T=T, D=D, Hq=Hq, Hk=Hk, Hv=Hv, seed=T + D)
    x, w = b.x.to(DEV), b.w.to(DEV)
    gq, gk = b.gamma_q.to(DEV), b.gamma_k.to(DEV)
    plain, qs, ks = qk.qknorm_qkv_gemm_stats(x, w, Hq, Hk, Hv)
    fused = qk.qknorm_qkv_projection(x, w, gq, gk, Hq, Hk, Hv, b.eps)
    two = qk.qknorm_qkv_projection(x, w, _unaligned_copy(gq), _unaligned_copy(gk), Hq, Hk, Hv, b.eps)
    torch.cuda.synchronize()
    assert torch.equal(fused, two)
    rows = _sample_rows(T, 16, T + 2)
    proj = check_projection(b, plain, rows)
    check_tile_sums(proj, qs, rows, 0, Hq // TILE)
    check_tile_sums(proj, ks, rows, Hq, Hk // TILE)
    check_normalized(b, proj, fused, rows)
    assert qk.device_timeouts() == 0


def test_projection_is_deterministic_and_matches_combine_apply():
    """Two runs agree bit for bit, and the pipeline equals gemm_stats followed
    by the public qknorm_combine_apply with 256-column shards (Hq == Hk)."""
    b = workloads.qkv_projection(T=512, D=256, Hq=512, Hk=512, Hv=256, seed=11)
    x, w = b.x.to(DEV), b.w.to(DEV)
    gq, gk = b.gamma_q.to(DEV), b.gamma_k.to(DEV)
    a = qk.qknorm_qkv_projection(x, w, gq, gk, b.Hq, b.Hk, b.Hv, b.eps)
    c = qk.qknorm_qkv_projection(x, w, gq, gk, b.Hq, b.Hk, b.Hv, b.eps)
    plain, qs, ks = qk.qknorm_qkv_gemm_stats(x, w, b.Hq, b.Hk, b.Hv)
    q = plain[:, :b.Hq]
    k = plain[:, b.Hq:b.Hq + b.Hk]
    qo, ko = qk.qknorm_combine_apply(q, k, gq, gk, qs, ks, b.Hq, b.Hk, b.eps)
    torch.cuda.synchronize()
    assert torch.equal(a, c)
    assert torch.equal(a[:, :b.Hq], qo) and torch.equal(a[:, b.Hq:b.Hq + b.Hk], ko)


def _unaligned_copy(t: torch.Tensor) -> torch.Tensor:
    """The same values in a buffer whose start is not 16-byte aligned."""
    buf = torch.empty(t.numel() + 8, dtype=t.dtype, device=t.device)
    v = buf[1:t.numel() + 1]
    v.copy_(t)
    assert v.data_ptr() % 16 != 0
    return v


@pytest.mark.parametrize("T,D,Hq,Hk,Hv", [
    (1000, 136, 1024, 512, 512),    # ragged last token tile; Q and K with different tile counts
    (4096, 64, 2048, 512, 512),     # 8 and 2 partial sums per row
    (129, 64, 256, 256, 0),         # one partial sum per row and tensor
    (2048, 320, 512, 1536, 256),    # K wider than Q
])
def test_aligned_and_unaligned_gamma_agree(T, D, Hq, Hk, Hv):
    """The apply pass after the GEMM runs the 16-byte vector kernel with
    aligned gamma and the scalar-access kernel with unaligned gamma.  Both
    combine the same partial sums in the same order, so they agree bit for
    bit; sampled rows are also checked against the oracle."""
    b = workloads.qkv_projection(T=T, D=D, Hq=Hq, Hk=Hk, Hv=Hv, seed=T + Hk)
    x, w = b.x.to(DEV), b.w.to(DEV)
    gq, gk = b.gamma_q.to(DEV), b.gamma_k.to(DEV)
    fused = qk.qknorm_qkv_projection(x, w, gq, gk, Hq, Hk, Hv, b.eps)
    two = qk.qknorm_qkv_projection(x, w, _unaligned_copy(gq), _unaligned_copy(gk), Hq, Hk, Hv, b.eps)
    plain, _, _ = qk.qknorm_qkv_gemm_stats(x, w, Hq, Hk, Hv)
    torch.cuda.synchronize()
    assert torch.equal(fused, two)
    rows = _sample_rows(T, 12, T + 1)
    proj = check_projection(b, plain, rows)
    check_normalized(b, proj, fused, rows)
    assert qk.device_timeouts() == 0


@pytest.mark.parametrize("T,D,Hq,Hk,Hv", [
    (4096, 64, 4096, 1024, 1024),   # the GQA bench shape's tiling (384 units, a partial last wave of V tiles)
    (4000, 72, 2048, 512, 2304),    # ragged last token block (160 tokens) and k-block
])
def test_projection_every_row(T, D, Hq, Hk, Hv):
    """Every row and every column against the oracle (projection, tile sums
    and the normalized Q and K), the vector apply pass bit for bit against
    the scalar one (unaligned gamma), V equal to the plain projection."""
    b = workloads.qkv_projection(T=T, D=D, Hq=Hq, Hk=Hk, Hv=Hv, seed=T + D + Hv)
    x, w = b.x.to(DEV), b.w.to(DEV)
    gq, gk = b.gamma_q.to(DEV), b.gamma_k.to(DEV)
    plain, qs, ks = qk.qknorm_qkv_gemm_stats(x, w, Hq, Hk, Hv)
    fused = qk.qknorm_qkv_projection(x, w, gq, gk, Hq, Hk, Hv, b.eps)
    two = qk.qknorm_qkv_projection(x, w, _unaligned_copy(gq), _unaligned_copy(gk), Hq, Hk, Hv, b.eps)
    torch.cuda.synchronize()
    assert qk.device_timeouts() == 0
    assert torch.equal(fused, two)
    assert torch.equal(fused[:, Hq + Hk:], plain[:, Hq + Hk:])  # V keeps the projection
    rows = np.arange(T)
    proj = check_projection(b, plain, rows)
    check_tile_sums(proj, qs, rows, 0, Hq // TILE)
    check_tile_sums(proj, ks, rows, Hq, Hk // TILE)
    check_normalized(b, proj, fused, rows)
