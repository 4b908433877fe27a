"""GPU parity: the CUDA path (through the C-ABI) against the CPU oracle on the
same seeded input bytes.

Tolerances (fp32 accumulation on the GPU, double in the oracle):
  * fp32 outputs: max_j |y - o| / max(|o|, 1e-30) <= 1e-5, o the oracle's
    unrounded double value;
  * bf16 outputs: at most 1 unit in the last place between the GPU's bf16 and
    the oracle's correctly rounded bf16, counted over ordered bit patterns;
  * fp32 partial squared sums: relative error <= 1e-5.
Why these hold: the GPU's squared sum of H terms carries a relative error of
roughly (terms per thread + log2(threads)) * 2^-24 (well under 1e-5 for every
shape here), rsqrtf adds at most 2 ulp and the two multiplies one ulp each, so
an fp32 output is within ~1e-6 relative of the exact value; a bf16 output can
then only differ from the correctly rounded one when the exact value lies that
close to a rounding boundary, i.e. by one unit.

Configurations are the five benchmark workloads (full sizes, the launch the
library picks by default, which is what the benchmark times) plus small and
ragged shapes, unaligned buffers, wide rows and every kernel variant.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import attention_normalization_b200 as qk
import oracle
import workloads
from tests.conftest import bf16_ulp_distance, buffer_np, to_np, ulp_distance

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


# --------------------------------------------------------------------------- helpers

def oracle_rows(view: torch.Tensor, gamma: torch.Tensor, eps: float):
    """Oracle on a (possibly strided) CPU view: (rounded y, exact y, sumsq)."""
    T, H = view.shape
    if T == 0:
        return (np.zeros((0, H), dtype=to_np(gamma).dtype), np.zeros((0, H)), np.zeros((0,)))
    flat, stride = buffer_np(view)
    return oracle.rmsnorm_rows(flat, H, to_np(gamma), eps, stride=stride, T=T)


ALL_DTYPES = [torch.float32, torch.bfloat16, torch.float16, torch.float8_e4m3fn]
NARROW_DTYPES = [torch.bfloat16, torch.float16, torch.float8_e4m3fn]


def esz(dtype: torch.dtype) -> int:
    return {torch.float32: 4, torch.bfloat16: 2, torch.float16: 2, torch.float8_e4m3fn: 1}[dtype]


def assert_close(got: torch.Tensor, y_rounded: np.ndarray, y_exact: np.ndarray, what: str):
    got = got.detach().cpu().contiguous()
    if got.dtype != torch.float32:
        d = ulp_distance(to_np(got), y_rounded, got.dtype)
        worst = int(d.max()) if d.size else 0
        assert worst <= 1, (f"{what}: {worst} ulp of {got.dtype} from the oracle "
                            f"(at {np.unravel_index(d.argmax(), d.shape)})")
    else:
        o = y_exact
        rel = np.abs(got.double().numpy() - o) / np.maximum(np.abs(o), 1e-30)
        worst = float(rel.max()) if rel.size else 0.0
        assert worst <= 1e-5, f"{what}: relative error {worst:.3g} > 1e-5"


def upload(batch: workloads.QKBatch):
    """Device copies keeping every layout detail (strides, padding, packing)."""
    if batch.packed is not None:
        base = batch.packed.to(DEV)
        q = base[:, :batch.Hq]
        k = base[:, batch.Hq:batch.Hq + batch.Hk]
        return q, k, base
    qb = batch.meta.get("q_buffer")
    kb = batch.meta.get("k_buffer")
    if qb is not None:
        qd, kd = qb.to(DEV), kb.to(DEV)
        return qd[:batch.T, :batch.Hq], kd[:batch.T, :batch.Hk], (qd, kd)
    return batch.q.to(DEV), batch.k.to(DEV), None


def check_layerwise(batch: workloads.QKBatch, in_place: bool = False, launch=None):
    q, k, keep = upload(batch)
    gq, gk = batch.gamma_q.to(DEV), batch.gamma_k.to(DEV)
    before = keep[0].clone() if isinstance(keep, tuple) else (keep.clone() if keep is not None else None)
    if in_place:
        qo, ko = qk.qknorm_layerwise(q, k, gq, gk, batch.eps, q_out=q, k_out=k, launch=launch)
    else:
        qo, ko = qk.qknorm_layerwise(q, k, gq, gk, batch.eps, launch=launch)
    torch.cuda.synchronize()
    yq, eq, _ = oracle_rows(batch.q, batch.gamma_q, batch.eps)
    yk, ek, _ = oracle_rows(batch.k, batch.gamma_k, batch.eps)
    assert_close(qo, yq, eq, f"{batch.name} Q")
    assert_close(ko, yk, ek, f"{batch.name} K")
    return q, k, qo, ko, keep, before


# --------------------------------------------------------------------------- the five workloads

def test_tiny_fp32_out_of_place_then_in_place_bitwise_equal():
    b = workloads.tiny_fp32()
    _, _, qo, ko, _, _ = check_layerwise(b)
    q2, k2, qi, ki, _, _ = check_layerwise(b, in_place=True)
    assert qi.data_ptr() == q2.data_ptr()
    assert torch.equal(qo, qi) and torch.equal(ko, ki)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16, torch.float8_e4m3fn])
def test_prefill_full_size(dtype):
    b = workloads.prefill_bf16(dtype=dtype)
    check_layerwise(b)


@pytest.mark.parametrize("T", workloads.DECODE_TOKENS)
def test_decode_bf16(T):
    check_layerwise(workloads.decode_bf16(T))


def test_gqa_shard_decomposed_full_size():
    b = workloads.gqa_sharded()
    P, T = b.P, b.T
    qs = [s.to(DEV) for s in b.q_shards]
    ks = [s.to(DEV) for s in b.k_shards]
    wq, wk = b.Hq // P, b.Hk // P
    q_all = torch.empty((P, T), dtype=torch.float32, device=DEV)
    k_all = torch.empty((P, T), dtype=torch.float32, device=DEV)
    for p in range(P):
        qk.qknorm_partial_stats(qs[p], ks[p], q_all[p], k_all[p])
    gq, gk = b.gamma_q.to(DEV), b.gamma_k.to(DEV)
    outs = []
    for p in range(P):
        outs.append(qk.qknorm_combine_apply(qs[p], ks[p], gq[p * wq:(p + 1) * wq].contiguous(),
                                            gk[p * wk:(p + 1) * wk].contiguous(), q_all, k_all,
                                            b.Hq, b.Hk, b.eps))
    torch.cuda.synchronize()
    # Phase A partial sums against the oracle's double partial sums
    for p in range(P):
        oq = oracle.partial_sumsq(to_np(b.q_shards[p]), wq, wq, T)
        ok_ = oracle.partial_sumsq(to_np(b.k_shards[p]), wk, wk, T)
        np.testing.assert_allclose(q_all[p].cpu().double().numpy(), oq, rtol=1e-5, atol=0)
        np.testing.assert_allclose(k_all[p].cpu().double().numpy(), ok_, rtol=1e-5, atol=0)
    # outputs against the oracle over the FULL rows
    yq, eq, _ = oracle_rows(b.q_full, b.gamma_q, b.eps)
    yk, ek, _ = oracle_rows(b.k_full, b.gamma_k, b.eps)
    got_q = torch.cat([o[0] for o in outs], dim=1)
    got_k = torch.cat([o[1] for o in outs], dim=1)
    assert_close(got_q, yq, eq, "gqa Q shards")
    assert_close(got_k, yk, ek, "gqa K shards")
    # ... and against the fused kernel on the unsplit rows (at most one ulp apart:
    # the two forms add the same squares in different orders)
    fq, fk = qk.qknorm_layerwise(b.q_full.to(DEV), b.k_full.to(DEV), gq, gk, b.eps)
    assert int(bf16_ulp_distance(to_np(fq.cpu()), to_np(got_q.cpu())).max()) <= 1
    assert int(bf16_ulp_distance(to_np(fk.cpu()), to_np(got_k.cpu())).max()) <= 1


def _split(full: torch.Tensor, P: int, stride_pad: int = 0):
    """P column shards of `full` in separate device buffers, each with
    `stride_pad` padding elements after its row."""
    w = full.shape[1] // P
    out = []
    for p in range(P):
        buf = torch.full((full.shape[0], w + stride_pad), 7.0, dtype=full.dtype).to(DEV)
        buf[:, :w] = full[:, p * w:(p + 1) * w].to(DEV)
        out.append(buf[:, :w])
    return out


def test_gqa_multi_shard_calls_full_size_equal_the_per_shard_calls():
    """The GQA step through the two multi-shard calls (one launch per phase):
    partial sums and outputs bit-equal to the per-shard calls at this shape
    (same row groups), and against the oracle over the full rows."""
    b = workloads.gqa_sharded()
    P, T = b.P, b.T
    wq, wk = b.Hq // P, b.Hk // P
    qs = [s.to(DEV) for s in b.q_shards]
    ks = [s.to(DEV) for s in b.k_shards]
    gq, gk = b.gamma_q.to(DEV), b.gamma_k.to(DEV)
    gqs = [gq[p * wq:(p + 1) * wq].contiguous() for p in range(P)]
    gks = [gk[p * wk:(p + 1) * wk].contiguous() for p in range(P)]
    q_all, k_all = qk.qknorm_partial_stats_shards(qs, ks)
    qo, ko = qk.qknorm_combine_apply_shards(qs, ks, gqs, gks, q_all, k_all, b.Hq, b.Hk, b.eps)
    ref_q = torch.empty((P, T), dtype=torch.float32, device=DEV)
    ref_k = torch.empty((P, T), dtype=torch.float32, device=DEV)
    for p in range(P):
        qk.qknorm_partial_stats(qs[p], ks[p], ref_q[p], ref_k[p])
    per = [qk.qknorm_combine_apply(qs[p], ks[p], gqs[p], gks[p], ref_q, ref_k, b.Hq, b.Hk, b.eps) for p in range(P)]
    torch.cuda.synchronize()
    assert torch.equal(q_all, ref_q) and torch.equal(k_all, ref_k)
    for p in range(P):
        assert torch.equal(qo[p], per[p][0]) and torch.equal(ko[p], per[p][1])
    yq, eq, _ = oracle_rows(b.q_full, b.gamma_q, b.eps)
    yk, ek, _ = oracle_rows(b.k_full, b.gamma_k, b.eps)
    assert_close(torch.cat([o.cpu() for o in qo], dim=1), yq, eq, "gqa multi-shard Q")
    assert_close(torch.cat([o.cpu() for o in ko], dim=1), yk, ek, "gqa multi-shard K")


@pytest.mark.parametrize("dtype", ALL_DTYPES)
@pytest.mark.parametrize("P,T,Hq,Hk,pad", [
    (1, 100, 1024, 256, 0),
    (2, 37, 2048, 512, 8),      # padded rows
    (4, 1, 5120, 1024, 0),      # one token: few rows, the latency plan
    (8, 300, 4096, 1024, 0),    # eight shards: sixteen row sets
    (3, 129, 768, 384, 0),      # shard rows whose width is not a power of two
    (4, 64, 1000, 200, 0),      # unaligned shard widths: shard by shard, scalar kernels
])
def test_multi_shard_calls_match_the_oracle(dtype, P, T, Hq, Hk, pad):
    b = workloads.random_rows(T, Hq, Hk, dtype, seed=P * 1000 + T, scale=1.5)
    qs, ks = _split(b.q, P, pad), _split(b.k, P, pad)
    wq, wk = Hq // P, Hk // P
    gq, gk = b.gamma_q.to(DEV), b.gamma_k.to(DEV)
    gqs = [gq[p * wq:(p + 1) * wq].contiguous() for p in range(P)]
    gks = [gk[p * wk:(p + 1) * wk].contiguous() for p in range(P)]
    q_all, k_all = qk.qknorm_partial_stats_shards(qs, ks)
    torch.cuda.synchronize()
    for p in range(P):
        oq = oracle.partial_sumsq(to_np(b.q[:, p * wq:(p + 1) * wq]), wq, wq, T)
        ok_ = oracle.partial_sumsq(to_np(b.k[:, p * wk:(p + 1) * wk]), wk, wk, T)
        np.testing.assert_allclose(q_all[p].cpu().double().numpy(), oq, rtol=1e-5, atol=0)
        np.testing.assert_allclose(k_all[p].cpu().double().numpy(), ok_, rtol=1e-5, atol=0)
    # out of place, then in place: bit for bit the same
    qo, ko = qk.qknorm_combine_apply_shards(qs, ks, gqs, gks, q_all, k_all, Hq, Hk, b.eps)
    torch.cuda.synchronize()
    yq, eq, _ = oracle_rows(b.q, b.gamma_q, b.eps)
    yk, ek, _ = oracle_rows(b.k, b.gamma_k, b.eps)
    assert_close(torch.cat([o.cpu() for o in qo], dim=1), yq, eq, "multi-shard Q")
    assert_close(torch.cat([o.cpu() for o in ko], dim=1), yk, ek, "multi-shard K")
    qk.qknorm_combine_apply_shards(qs, ks, gqs, gks, q_all, k_all, Hq, Hk, b.eps, q_out=qs, k_out=ks)
    torch.cuda.synchronize()
    for p in range(P):
        assert torch.equal(qs[p], qo[p]) and torch.equal(ks[p], ko[p])
        if pad:  # padding after each shard row untouched
            base_q = qs[p].as_strided((T, wq + pad), (wq + pad, 1))
            assert torch.all(base_q[:, wq:].float() == 7.0)


@pytest.mark.parametrize("launch", [{"kernel": 0, "vec_per_thread": 2, "threads": 96, "grid": 7},
                                    {"kernel": 0, "vec_per_thread": 4, "threads": 128, "grid": 300},
                                    {"kernel": 0, "vec_per_thread": 1, "threads": 160, "grid": 1184},
                                    {"kernel": 0, "vec_per_thread": 8, "threads": 64, "grid": 50},
                                    {"kernel": 0, "vec_per_thread": 5, "threads": 128, "grid": 592}])
def test_multi_shard_pinned_launches_match_the_oracle(launch):
    """Any valid launch of the multi-shard calls (rows grouped differently,
    any grid) gives the oracle's results."""
    P, T, Hq, Hk = 4, 333, 5120, 1024
    b = workloads.random_rows(T, Hq, Hk, torch.bfloat16, seed=77, scale=1.5)
    qs, ks = _split(b.q, P), _split(b.k, P)
    wq, wk = Hq // P, Hk // P
    gq, gk = b.gamma_q.to(DEV), b.gamma_k.to(DEV)
    gqs = [gq[p * wq:(p + 1) * wq].contiguous() for p in range(P)]
    gks = [gk[p * wk:(p + 1) * wk].contiguous() for p in range(P)]
    q_all, k_all = qk.qknorm_partial_stats_shards(qs, ks, launch=launch)
    qo, ko = qk.qknorm_combine_apply_shards(qs, ks, gqs, gks, q_all, k_all, Hq, Hk, b.eps, launch=launch)
    torch.cuda.synchronize()
    for p in range(P):
        oq = oracle.partial_sumsq(to_np(b.q[:, p * wq:(p + 1) * wq]), wq, wq, T)
        np.testing.assert_allclose(q_all[p].cpu().double().numpy(), oq, rtol=1e-5, atol=0)
    yq, eq, _ = oracle_rows(b.q, b.gamma_q, b.eps)
    yk, ek, _ = oracle_rows(b.k, b.gamma_k, b.eps)
    assert_close(torch.cat([o.cpu() for o in qo], dim=1), yq, eq, f"pinned {launch} Q")
    assert_close(torch.cat([o.cpu() for o in ko], dim=1), yk, ek, f"pinned {launch} K")


def test_multi_shard_calls_reject_overlapping_shards():
    x = torch.zeros((8, 256), dtype=torch.bfloat16, device=DEV)
    g = torch.ones((128,), dtype=torch.bfloat16, device=DEV)
    qa, ka = qk.qknorm_partial_stats_shards([x[:, :128], x[:, 128:]], [x[:, :128], x[:, 128:]])
    out = torch.empty((8, 256), dtype=torch.bfloat16, device=DEV)
    with pytest.raises(qk.QKNormError, match="overlap"):  # shard 1's output on shard 0's input
        qk.qknorm_combine_apply_shards([x[:, :128], x[:, 128:]], [x[:, :128], x[:, 128:]], [g, g], [g, g], qa, ka,
                                       256, 256, q_out=[out[:, :128], x[:, :128]], k_out=[out[:, 128:], x[:, 128:]])


def _e4m3_case(T, H, seed):
    b = workloads.random_rows(T, H, H, torch.float8_e4m3fn, seed=seed, scale=1.5)
    q, k = b.q.clone(), b.k.clone()
    # rows 3, 10, ... hold one smallest subnormal (2^-9) and zeros: with eps = 0
    # their factor is sqrt(H) / 2^-9 = 2^15.5 for H = 8192
    tiny = torch.zeros((H,), dtype=torch.float32)
    tiny[H // 3] = 2.0 ** -9
    for t in range(3, T, 7):
        q[t] = tiny.to(torch.float8_e4m3fn)
        k[t] = (-tiny).to(torch.float8_e4m3fn)
    return b, q, k


@pytest.mark.parametrize("gamma_kind", ["ordinary", "one large", "tiny and zero"])
def test_e4m3_extreme_gamma_and_factors(gamma_kind):
    """E4M3 rows at the edges of the arithmetic: gamma entries far from 1
    (200, where x * gamma exceeds f16's range; 2^-20, below it; exact zeros)
    and, with eps = 0, rows holding a single 2^-9 among 8192 zeros, whose
    factor 2^-9 * sqrt(8192) ~ 2^15.5 scales the lone element to ~90.  Every
    output within one E4M3 unit of the oracle; zero gamma gives exact zeros."""
    T, H = 64, 8192
    b, q, k = _e4m3_case(T, H, seed=91)
    gq, gk = b.gamma_q.clone(), b.gamma_k.clone()
    if gamma_kind == "one large":
        gq[17] = 200.0
    elif gamma_kind == "tiny and zero":
        gq[5] = 2.0 ** -20
        gk[::9] = 0.0
    eps = 0.0
    qo, ko = qk.qknorm_layerwise(q.to(DEV), k.to(DEV), gq.to(DEV), gk.to(DEV), eps)
    torch.cuda.synchronize()
    yq, eq, _ = oracle_rows(q, gq, eps)
    yk, ek, _ = oracle_rows(k, gk, eps)
    assert_close(qo, yq, eq, f"E4M3 Q ({gamma_kind})")
    assert_close(ko, yk, ek, f"E4M3 K ({gamma_kind})")
    if gamma_kind == "tiny and zero":
        assert torch.all(ko.cpu().float()[:, ::9] == 0)
    # the same through combine/apply with one shard
    sq, sk = qk.qknorm_partial_stats(q.to(DEV), k.to(DEV))
    ao, bo = qk.qknorm_combine_apply(q.to(DEV), k.to(DEV), gq.to(DEV), gk.to(DEV), sq[None], sk[None], H, H, eps)
    torch.cuda.synchronize()
    assert_close(ao, yq, eq, f"E4M3 apply Q ({gamma_kind})")
    assert_close(bo, yk, ek, f"E4M3 apply K ({gamma_kind})")


@pytest.mark.parametrize("T", workloads.PACKED_TOKENS)
def test_packed_qkv_in_place_v_untouched(T):
    b = workloads.packed_qkv(T)
    _, _, _, _, base, before = check_layerwise(b, in_place=True)
    v0 = b.Hq + b.Hk
    assert torch.equal(base[:, v0:], before[:, v0:]), "V columns were modified"


# --------------------------------------------------------------------------- edge cases

def aligned_stride(H: int, dtype: torch.dtype, extra_vectors: int = 1) -> int:
    """A row stride whose byte size is a multiple of 16, leaving padding after H."""
    per = 16 // esz(dtype)
    return -(-H // per) * per + extra_vectors * per


@pytest.mark.parametrize("layout", ["contiguous", "padded"])
@pytest.mark.parametrize("dtype", ALL_DTYPES)
@pytest.mark.parametrize("T,Hq,Hk", [(1, 1, 1), (2, 3, 7), (3, 8, 9), (17, 127, 129), (5, 513, 64),
                                      (33, 4096, 1024), (7, 5120, 5120), (300, 1000, 24)])
def test_small_and_ragged_shapes(layout, dtype, T, Hq, Hk):
    """Layout "contiguous": strides equal the widths (unaligned whenever a width
    is not a multiple of the vector).  Layout "padded": strides are 16-byte
    multiples, so widths that are not run the vector kernels' ragged tail."""
    kw = {}
    if layout == "padded":
        kw = dict(q_stride=aligned_stride(Hq, dtype), k_stride=aligned_stride(Hk, dtype))
    check_layerwise(workloads.random_rows(T, Hq, Hk, dtype, seed=T * 131 + Hq + Hk, **kw))


@pytest.mark.parametrize("dtype", ALL_DTYPES)
def test_padding_columns_untouched(dtype):
    Hq, Hk = 203, 43  # ragged: neither is a whole number of 16-byte vectors
    b = workloads.random_rows(9, Hq, Hk, dtype, seed=3, q_stride=aligned_stride(Hq, dtype, 3),
                              k_stride=aligned_stride(Hk, dtype))
    q, k, _ = upload(b)
    assert qk.qknorm_layerwise_plan(q, k, b.gamma_q.to(DEV), b.gamma_k.to(DEV))["kernel"] == 0
    q, k, qo, ko, keep, before = check_layerwise(b, in_place=True)
    qd, kd = keep
    assert torch.all(qd[:, Hq:].float() == -7.0) and torch.all(kd[:, Hk:].float() == -7.0)


@pytest.mark.parametrize("dtype", ALL_DTYPES)
def test_unaligned_buffers_use_the_scalar_kernel(dtype):
    b = workloads.random_rows(13, 301, 77, dtype, seed=4, q_stride=301, k_stride=77)
    q, k, _ = upload(b)
    gq, gk = b.gamma_q.to(DEV), b.gamma_k.to(DEV)
    plan = qk.qknorm_layerwise_plan(q, k, gq, gk)
    assert plan["kernel"] == 2
    check_layerwise(b)
    # shift the start by one element: still correct
    buf = torch.zeros((13 * 301 + 1,), dtype=dtype)
    buf[1:] = b.q.reshape(-1)
    bq = buf[1:].view(13, 301)
    shifted = workloads.QKBatch("shifted", dtype, 13, 301, 77, bq, b.k, b.gamma_q, b.gamma_k)
    qd = buf.to(DEV)[1:].view(13, 301)
    qo, ko = qk.qknorm_layerwise(qd, k, gq, gk, b.eps)
    yq, eq, _ = oracle_rows(shifted.q, b.gamma_q, b.eps)
    assert_close(qo, yq, eq, "shifted Q")


@pytest.mark.parametrize("dtype,H", [(torch.bfloat16, 20000), (torch.float32, 9000), (torch.float16, 20000),
                                     (torch.float8_e4m3fn, 40000)])
def test_rows_too_wide_for_registers(dtype, H):
    b = workloads.random_rows(6, H, 64, dtype, seed=5)
    q, k, _ = upload(b)
    assert qk.qknorm_layerwise_plan(q, k, b.gamma_q.to(DEV), b.gamma_k.to(DEV))["kernel"] == 1
    check_layerwise(b)


def test_prefill_rows_beyond_2gib():
    """Q and K of 2.16 GB each (T = 2^31 / 8192 + 1000 rows of 4096 bf16):
    rows on both sides of the 2^31-byte offset, and the first and last rows,
    against the oracle (64-bit row offsets in every address)."""
    T = (1 << 31) // (4096 * 2) + 1000
    b = workloads.large_rows_on_device(T, 4096, 4096, torch.bfloat16, seed=77, device=DEV)
    gq, gk = b.gamma_q.to(DEV), b.gamma_k.to(DEV)
    qo, ko = qk.qknorm_layerwise(b.q, b.k, gq, gk, b.eps)
    torch.cuda.synchronize()
    edge = (1 << 31) // (4096 * 2)
    rows = torch.tensor([0, 1, edge - 1, edge, edge + 1, T // 2, T - 2, T - 1], device=DEV)
    for x, out, g, name in ((b.q, qo, b.gamma_q, "Q"), (b.k, ko, b.gamma_k, "K")):
        y, e, _ = oracle_rows(x[rows].cpu(), g, b.eps)
        assert_close(out[rows].cpu(), y, e, f"{b.name} {name}")
    del qo, ko, b
    torch.cuda.empty_cache()


def test_zero_rows_give_zero_and_empty_batch_is_a_no_op():
    b = workloads.random_rows(4, 64, 32, torch.bfloat16, seed=6)
    b.q[1].zero_()
    b.meta["q_buffer"][1].zero_()
    q, k, qo, ko, _, _ = check_layerwise(b)
    assert torch.all(qo[1] == 0)
    e = torch.empty((0, 64), dtype=torch.bfloat16, device=DEV)
    g = torch.ones((64,), dtype=torch.bfloat16, device=DEV)
    a, c = qk.qknorm_layerwise(e, e, g, g)
    assert a.shape == (0, 64)


VARIANTS = [
    {"kernel": 0, "vec_per_thread": 1, "threads": 1024, "grid": 7},
    {"kernel": 0, "vec_per_thread": 2, "threads": 256, "grid": 148},
    {"kernel": 0, "vec_per_thread": 4, "threads": 128, "grid": 1},
    {"kernel": 0, "vec_per_thread": 4, "threads": 128, "grid": 1184},
    {"kernel": 0, "vec_per_thread": 8, "threads": 64, "grid": 1000},
    {"kernel": 0, "vec_per_thread": 8, "threads": 256, "grid": 134},
    {"kernel": 1, "vec_per_thread": 0, "threads": 96, "grid": 33},
    {"kernel": 2, "vec_per_thread": 0, "threads": 1024, "grid": 5},
]


def _cover(launch: dict, units: int) -> dict | None:
    """Widen a register launch so that it covers `units` vectors, or None if
    no CTA of its vec_per_thread can."""
    if launch["kernel"] != 0:
        return launch
    nv = launch["vec_per_thread"]
    if nv * launch["threads"] >= units:
        return launch
    limit = 1024 if nv <= 2 else (512 if nv == 4 else 256)
    threads = -(-units // nv)
    threads = -(-threads // 32) * 32
    return None if threads > limit else dict(launch, threads=threads)


@pytest.mark.parametrize("launch", VARIANTS, ids=lambda L: "k{kernel}_nv{vec_per_thread}_t{threads}_g{grid}".format(**L))
@pytest.mark.parametrize("dtype", ALL_DTYPES)
@pytest.mark.parametrize("Hk", [1000, 1003])
def test_every_kernel_variant_matches_the_oracle_and_is_deterministic(launch, dtype, Hk):
    """Hk = 1003 leaves K rows with a ragged last vector (padded, aligned stride)."""
    per = 16 // esz(dtype)
    launch = _cover(launch, -(-4096 // per))
    if launch is None:
        pytest.skip("no CTA of this vec_per_thread covers the fp32 row")
    b = workloads.random_rows(67, 4096, Hk, dtype, seed=7, k_stride=aligned_stride(Hk, dtype))
    _, _, qo, ko, _, _ = check_layerwise(b, launch=launch)
    _, _, qo2, ko2, _, _ = check_layerwise(b, launch=launch)
    assert torch.equal(qo, qo2) and torch.equal(ko, ko2)


@pytest.mark.parametrize("T", [1, 3, 300])
def test_register_kernel_in_place_on_packed_rows_any_grid(T):
    """Q-first items with an even grid: both tensors' rows are covered."""
    b = workloads.packed_qkv(T)
    launch = {"kernel": 0, "vec_per_thread": 4, "threads": 128, "grid": 2 if T > 1 else 1}
    _, _, _, _, base, before = check_layerwise(b, in_place=True, launch=launch)
    assert torch.equal(base[:, b.Hq + b.Hk:], before[:, b.Hq + b.Hk:])


SHARD_LAUNCHES = [
    None,
    {"kernel": 0, "vec_per_thread": 1, "threads": 160, "grid": 50},
    {"kernel": 0, "vec_per_thread": 2, "threads": 96, "grid": 7},
    {"kernel": 0, "vec_per_thread": 4, "threads": 128, "grid": 148},
    {"kernel": 0, "vec_per_thread": 8, "threads": 128, "grid": 3},
    {"kernel": 0, "vec_per_thread": 8, "threads": 32, "grid": 1},
    {"kernel": 1, "vec_per_thread": 0, "threads": 64, "grid": 9},
    {"kernel": 2, "vec_per_thread": 0, "threads": 256, "grid": 11},
]


@pytest.mark.parametrize("launch", SHARD_LAUNCHES, ids=lambda L: "default" if L is None else
                         "k{kernel}_nv{vec_per_thread}_t{threads}_g{grid}".format(**L))
@pytest.mark.parametrize("dtype,Hq,Hk,P", [(torch.bfloat16, 5120, 1024, 4), (torch.float32, 1200, 260, 4),
                                           (torch.bfloat16, 1000, 200, 5), (torch.float16, 5120, 1024, 4),
                                           (torch.float8_e4m3fn, 5120, 1024, 4)])
def test_shard_pipeline_launch_variants(launch, dtype, Hq, Hk, P):
    """partial_stats then combine_apply over P shards, each with a pinned
    launch, against the oracle's full-row normalization."""
    per = 16 // esz(dtype)
    wq, wk = Hq // P, Hk // P
    if launch is not None and launch["kernel"] == 0 and launch["vec_per_thread"] * launch["threads"] < -(-wq // per):
        pytest.skip("launch does not cover a shard row")
    if launch is not None and launch["kernel"] in (0, 1) and ((wq * esz(dtype)) % 16 or (wk * esz(dtype)) % 16):
        pytest.skip("vector kernels need 16-byte aligned shard strides")
    T = 131
    g = torch.Generator().manual_seed(Hq + Hk + P)
    q = (torch.randn((T, Hq), generator=g) * 2).to(dtype)
    k = (torch.randn((T, Hk), generator=g) * 0.5).to(dtype)
    gq = workloads.gamma(Hq, 5, dtype)  # bf16 for E4M3 activations
    gk = workloads.gamma(Hk, 6, dtype)
    qs = [q[:, i * wq:(i + 1) * wq].contiguous().to(DEV) for i in range(P)]
    ks = [k[:, i * wk:(i + 1) * wk].contiguous().to(DEV) for i in range(P)]
    q_all = torch.empty((P, T), dtype=torch.float32, device=DEV)
    k_all = torch.empty((P, T), dtype=torch.float32, device=DEV)
    for i in range(P):
        qk.qknorm_partial_stats(qs[i], ks[i], q_all[i], k_all[i], launch=launch)
    outs = [qk.qknorm_combine_apply(qs[i], ks[i], gq[i * wq:(i + 1) * wq].contiguous().to(DEV),
                                    gk[i * wk:(i + 1) * wk].contiguous().to(DEV), q_all, k_all, Hq, Hk, 1e-6,
                                    launch=launch) for i in range(P)]
    torch.cuda.synchronize()
    for i in range(P):
        np.testing.assert_allclose(q_all[i].cpu().double().numpy(),
                                   oracle.partial_sumsq(to_np(q[:, i * wq:(i + 1) * wq]), wq, wq, T), rtol=1e-5)
        np.testing.assert_allclose(k_all[i].cpu().double().numpy(),
                                   oracle.partial_sumsq(to_np(k[:, i * wk:(i + 1) * wk]), wk, wk, T), rtol=1e-5)
    yq, eq, _ = oracle_rows(q, gq, 1e-6)
    yk, ek, _ = oracle_rows(k, gk, 1e-6)
    assert_close(torch.cat([o[0] for o in outs], dim=1), yq, eq, "shards Q")
    assert_close(torch.cat([o[1] for o in outs], dim=1), yk, ek, "shards K")


def test_fp32_variants_and_apply_with_one_shard_equals_fused():
    b = workloads.tiny_fp32()
    q, k = b.q.to(DEV), b.k.to(DEV)
    gq, gk = b.gamma_q.to(DEV), b.gamma_k.to(DEV)
    sq, sk = qk.qknorm_partial_stats(q, k)
    yq, eq, s_or = oracle_rows(b.q, b.gamma_q, b.eps)
    np.testing.assert_allclose(sq.cpu().double().numpy(), s_or, rtol=1e-5)
    aq, ak = qk.qknorm_combine_apply(q, k, gq, gk, sq[None, :], sk[None, :], b.Hq, b.Hk, b.eps)
    assert_close(aq, yq, eq, "P=1 apply Q")
    fq, fk = qk.qknorm_layerwise(q, k, gq, gk, b.eps)
    # same launch shape, same squared sums: P = 1 apply reproduces the fused result bit for bit
    assert torch.equal(aq, fq) and torch.equal(ak, fk)


def test_runs_on_a_side_stream():
    b = workloads.random_rows(64, 2048, 512, torch.bfloat16, seed=8)
    q, k, _ = upload(b)
    gq, gk = b.gamma_q.to(DEV), b.gamma_k.to(DEV)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        qo, ko = qk.qknorm_layerwise(q, k, gq, gk, b.eps)
    s.synchronize()
    yq, eq, _ = oracle_rows(b.q, b.gamma_q, b.eps)
    assert_close(qo, yq, eq, "side stream Q")


def test_invalid_call_on_gpu_raises_and_launches_nothing():
    x = torch.zeros((4, 64), dtype=torch.bfloat16, device=DEV)
    g = torch.ones((64,), dtype=torch.bfloat16, device=DEV)
    with pytest.raises(qk.QKNormError, match="invalid argument"):
        qk.qknorm_layerwise(x, x, g, g, -1.0)
    big = torch.zeros((4, 128), dtype=torch.bfloat16, device=DEV)
    with pytest.raises(qk.QKNormError, match="overlap"):
        qk.qknorm_layerwise(big[:, :64], big[:, 32:96], g, g, q_out=big[:, :64], k_out=big[:, 32:96])


# --------------------------------------------------------------------------- host pipeline

@pytest.mark.parametrize("T,chunk", [(1, 512), (1000, 512), (1537, 256), (64, 7)])
def test_host_pipeline_matches_the_oracle(T, chunk):
    b = workloads.random_rows(T, 2048, 512, torch.bfloat16, seed=T + chunk)
    hq, hk = b.q.contiguous().pin_memory(), b.k.contiguous().pin_memory()
    qo, ko = qk.qknorm_layerwise_host(hq, hk, b.gamma_q, b.gamma_k, b.eps, chunk_tokens=chunk)
    torch.cuda.current_stream().synchronize()
    assert not qo.is_cuda and not ko.is_cuda
    yq, eq, _ = oracle_rows(b.q, b.gamma_q, b.eps)
    yk, ek, _ = oracle_rows(b.k, b.gamma_k, b.eps)
    assert_close(qo, yq, eq, "host pipeline Q")
    assert_close(ko, yk, ek, "host pipeline K")
    # in place on the host buffers, fp32
    bf = workloads.random_rows(T, 512, 96, torch.float32, seed=T)
    hq2, hk2 = bf.q.contiguous().pin_memory(), bf.k.contiguous().pin_memory()
    qk.qknorm_layerwise_host(hq2, hk2, bf.gamma_q, bf.gamma_k, bf.eps, q_out=hq2, k_out=hk2, chunk_tokens=chunk)
    torch.cuda.current_stream().synchronize()
    yq, eq, _ = oracle_rows(bf.q, bf.gamma_q, bf.eps)
    assert_close(hq2, yq, eq, "host pipeline in place Q")


@pytest.mark.parametrize("T", [3, 1500])
def test_packed_host_pipeline_leaves_v_untouched(T):
    b = workloads.packed_qkv(T)
    host = b.packed.clone().pin_memory()
    qk.qknorm_packed_host(host, 0, b.Hq, b.Hq, b.Hk, b.gamma_q, b.gamma_k, b.eps, chunk_tokens=512)
    torch.cuda.current_stream().synchronize()
    v0 = b.Hq + b.Hk
    assert torch.equal(host[:, v0:], b.packed[:, v0:])
    yq, eq, _ = oracle_rows(b.q, b.gamma_q, b.eps)
    yk, ek, _ = oracle_rows(b.k, b.gamma_k, b.eps)
    assert_close(host[:, :b.Hq], yq, eq, "packed host Q")
    assert_close(host[:, b.Hq:v0], yk, ek, "packed host K")


# --------------------------------------------------------------------------- headwise

def oracle_heads(view: torch.Tensor, n_heads: int, head_dim: int, gamma: torch.Tensor, eps: float):
    T = view.shape[0]
    flat, stride = buffer_np(view)
    return oracle.rmsnorm_heads(flat, n_heads, head_dim, to_np(gamma), eps, stride=stride, T=T)


def check_headwise(q, k, gq, gk, head_dim, eps=1e-6, in_place=False, launch=None, q_dev=None, k_dev=None):
    """q, k: CPU views; q_dev/k_dev: device views with the same layout."""
    qd = q.to(DEV) if q_dev is None else q_dev
    kd = k.to(DEV) if k_dev is None else k_dev
    kw = dict(q_out=qd, k_out=kd) if in_place else {}
    qo, ko = qk.qknorm_headwise(qd, kd, gq.to(DEV), gk.to(DEV), head_dim, eps, launch=launch, **kw)
    torch.cuda.synchronize()
    yq, eq = oracle_heads(q, q.shape[1] // head_dim, head_dim, gq, eps)
    yk, ek = oracle_heads(k, k.shape[1] // head_dim, head_dim, gk, eps)
    assert_close(qo, yq, eq, "headwise Q")
    assert_close(ko, yk, ek, "headwise K")
    return qo, ko


@pytest.mark.parametrize("dtype", ALL_DTYPES)
@pytest.mark.parametrize("T,nq,nk,hd", [(1, 32, 8, 128), (37, 16, 4, 64), (300, 8, 8, 128), (5, 3, 2, 7),
                                        (9, 4, 2, 32), (2, 1, 1, 256), (1000, 40, 8, 128)])
def test_headwise_matches_the_oracle(dtype, T, nq, nk, hd):
    g = torch.Generator().manual_seed(T + nq + nk + hd)
    q = (torch.randn((T, nq * hd), generator=g) * 2).to(dtype)
    k = (torch.randn((T, nk * hd), generator=g) * 0.5).to(dtype)
    gq, gk = workloads.gamma(hd, 1, dtype), workloads.gamma(hd, 2, dtype)
    check_headwise(q, k, gq, gk, hd)


def test_headwise_in_place_on_packed_rows_v_untouched():
    b = workloads.packed_qkv(333)
    base = b.packed.to(DEV)
    before = base.clone()
    hd = 128
    gq, gk = workloads.gamma(hd, 3, torch.bfloat16), workloads.gamma(hd, 4, torch.bfloat16)
    qv, kv = base[:, :b.Hq], base[:, b.Hq:b.Hq + b.Hk]
    check_headwise(b.q, b.k, gq, gk, hd, in_place=True, q_dev=qv, k_dev=kv)
    assert torch.equal(base[:, b.Hq + b.Hk:], before[:, b.Hq + b.Hk:])


@pytest.mark.parametrize("launch", [
    {"kernel": 0, "vec_per_thread": 1, "threads": 128, "grid": 37},
    {"kernel": 0, "vec_per_thread": 2, "threads": 256, "grid": 148},
    {"kernel": 0, "vec_per_thread": 4, "threads": 128, "grid": 5},
    {"kernel": 0, "vec_per_thread": 8, "threads": 64, "grid": 1000},
    {"kernel": 0, "vec_per_thread": 1, "threads": 32, "grid": 1},
    {"kernel": 1, "vec_per_thread": 0, "threads": 64, "grid": 77},
    {"kernel": 2, "vec_per_thread": 0, "threads": 128, "grid": 9},
], ids=lambda L: "k{kernel}_nv{vec_per_thread}_t{threads}_g{grid}".format(**L))
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float8_e4m3fn])
def test_headwise_every_kernel_variant(launch, dtype):
    g = torch.Generator().manual_seed(77)
    T, nq, nk, hd = 131, 12, 4, 128
    q = (torch.randn((T, nq * hd), generator=g)).to(dtype)
    k = (torch.randn((T, nk * hd), generator=g) * 3).to(dtype)
    gq, gk = workloads.gamma(hd, 5, dtype), workloads.gamma(hd, 6, dtype)
    qo, ko = check_headwise(q, k, gq, gk, hd, launch=launch)
    qo2, ko2 = check_headwise(q, k, gq, gk, hd, launch=launch)
    assert torch.equal(qo, qo2) and torch.equal(ko, ko2)


def test_layerwise_narrow_shards_use_sub_warp_groups():
    """Rows of 2 and 4 vectors: several rows per warp, reduced by segments."""
    for H, Hk in ((8, 8), (16, 8), (24, 12), (32, 16), (12, 20)):
        # strides rounded up to whole 16-byte vectors; 12- and 20-wide rows end in a partial vector
        b = workloads.random_rows(77, H, Hk, torch.bfloat16, seed=H, q_stride=-(-H // 8) * 8,
                                  k_stride=-(-Hk // 8) * 8)
        for launch in ({"kernel": 0, "vec_per_thread": 1, "threads": 128, "grid": 3},
                       {"kernel": 0, "vec_per_thread": 2, "threads": 64, "grid": 150}):
            check_layerwise(b, launch=launch)


def test_headwise_full_size_bench_workload():
    """The benchmarked headwise batch (T=4096, 32 Q heads and 8 K heads of 128,
    bf16) with the planner's own launch, every element against the oracle."""
    b = workloads.headwise_bf16()
    hd = b.meta["head_dim"]
    check_headwise(b.q, b.k, b.gamma_q, b.gamma_k, hd, eps=b.eps)


@pytest.mark.parametrize("dtype,bound,floor", [(torch.bfloat16, 2.0 ** -8, 2.0 ** -134),
                                               (torch.float8_e4m3fn, 2.0 ** -3, 2.0 ** -10)])
def test_prefill_error_band_against_fp64_gold(dtype, bound, floor):
    """Fig. 2(b) context: max / mean / RMS absolute error of the GPU output
    against the unrounded double oracle on the prefill batch (the paper reports
    5.0e-2 / 2.1e-3 / 3.4e-3 for BF16 and 5.0e-1 / 2.5e-2 / 3.9e-2 for FP8-E4M3
    on inputs it does not describe).  The error here is the output rounding
    alone, so it stays within half an ulp plus the fp32 work:
    |err| <= bound * |y| + floor, bound = 2^-8 (bf16) / 2^-3 (E4M3), floor =
    half the subnormal spacing (2^-134 / 2^-10)."""
    b = workloads.prefill_bf16(dtype=dtype)
    q, k, _ = upload(b)
    qo, ko = qk.qknorm_layerwise(q, k, b.gamma_q.to(DEV), b.gamma_k.to(DEV), b.eps)
    torch.cuda.synchronize()
    errs = []
    for got, view, g in ((qo, b.q, b.gamma_q), (ko, b.k, b.gamma_k)):
        _, exact, _ = oracle_rows(view, g, b.eps)
        y = got.float().cpu().double().numpy()
        err = np.abs(y - exact)
        assert np.all(err <= bound * np.abs(exact) + floor), "error beyond half an ulp of the type"
        errs.append(err.ravel())
    e = np.concatenate(errs)
    print(f"\nerror band {dtype}: max {e.max():.3e}  mean {e.mean():.3e}  rms {np.sqrt((e * e).mean()):.3e}")
