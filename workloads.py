"""Seeded synthetic inputs for layerwise QK-RMSNorm.

This module draws random numbers and lays them out; it holds none of the
normalization's arithmetic.  Both the CUDA path (tests, benchmark) and the CPU
oracle (tests) take their inputs from here, as the same bytes.

Every generator draws in float32 on the host with a seeded ``torch.Generator``,
applies the stated scaling, and rounds ONCE to the element type
(``Tensor.to(torch.bfloat16)`` rounds to nearest, ties to even).  Tensors are
returned on the CPU; callers copy them to a device themselves.

Seeds: x uses ``seed``; gamma_q ``seed + 100``; gamma_k ``seed + 200``; the
choice of outlier channels ``seed + 300``.  gamma is ``1 + 0.1 * N(0, 1)``
everywhere.

The workloads mirror the models the pages measure (OLMo2/OLMo3-shaped
projections; prefill token counts 64 and 4096 as in the latency figure), with
synthetic activations standing in for real ones.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import torch

EPS = 1e-6
_CHUNK_ROWS = 4096


def _gen(seed: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    return g


def _normal_rows(gen: torch.Generator, T: int, H: int, dtype: torch.dtype,
                 row_scale: torch.Tensor | None = None) -> torch.Tensor:
    """T x H standard normal draws (row by row blocks, so memory stays bounded),
    optionally multiplied by a per-row scale, rounded once to ``dtype``."""
    out = torch.empty((T, H), dtype=dtype)
    for r0 in range(0, T, _CHUNK_ROWS):
        r1 = min(T, r0 + _CHUNK_ROWS)
        blk = torch.randn((r1 - r0, H), generator=gen, dtype=torch.float32)
        if row_scale is not None:
            blk.mul_(row_scale[r0:r1, None])
        out[r0:r1] = blk.to(dtype)
    return out


def gamma(H: int, seed: int, dtype: torch.dtype) -> torch.Tensor:
    """Learnable-scale stand-in: 1 + 0.1 * N(0, 1), rounded once to the gamma
    type that goes with activations of ``dtype`` (bfloat16 for FP8 E4M3)."""
    g = _gen(seed)
    gdt = torch.bfloat16 if dtype == torch.float8_e4m3fn else dtype
    return (1.0 + 0.1 * torch.randn((H,), generator=g, dtype=torch.float32)).to(gdt)


@dataclass
class QKBatch:
    """One batch of projected Q and K rows (all CPU tensors).

    ``q`` and ``k`` are 2-D views ``[T, H]`` whose row stride (in elements) is
    ``q.stride(0)`` / ``k.stride(0)``; for the packed layout both are views
    into ``packed`` (``[T, Hq + Hk + Hv]``) and V sits after K.
    """
    name: str
    dtype: torch.dtype
    T: int
    Hq: int
    Hk: int
    q: torch.Tensor
    k: torch.Tensor
    gamma_q: torch.Tensor
    gamma_k: torch.Tensor
    eps: float = EPS
    packed: torch.Tensor | None = None
    Hv: int = 0
    meta: dict = field(default_factory=dict)

    @property
    def q_stride(self) -> int:
        return self.q.stride(0)

    @property
    def k_stride(self) -> int:
        return self.k.stride(0)


@dataclass
class ShardedBatch:
    """Q and K each split into P contiguous column shards held in separate
    buffers (``q_shards[p]`` is ``[T, Hq / P]``, contiguous).  ``q_full`` and
    ``k_full`` are the unsplit rows, for checking."""
    name: str
    dtype: torch.dtype
    T: int
    Hq: int
    Hk: int
    P: int
    q_full: torch.Tensor
    k_full: torch.Tensor
    q_shards: list
    k_shards: list
    gamma_q: torch.Tensor
    gamma_k: torch.Tensor
    eps: float = EPS


def tiny_fp32(seed: int = 0, T: int = 64, H: int = 512) -> QKBatch:
    """Tiny correctness case: T=64, Hq=Hk=512, fp32, x ~ N(0,1), separate
    contiguous Q and K buffers."""
    g = _gen(seed)
    q = _normal_rows(g, T, H, torch.float32)
    k = _normal_rows(g, T, H, torch.float32)
    return QKBatch("tiny_fp32_T64_H512", torch.float32, T, H, H, q, k,
                   gamma(H, seed + 100, torch.float32), gamma(H, seed + 200, torch.float32))


_DT_NAME = {torch.bfloat16: "bf16", torch.float16: "f16", torch.float32: "f32", torch.float8_e4m3fn: "e4m3"}


def prefill_bf16(seed: int = 1, T: int = 4096, H: int = 4096, dtype: torch.dtype = torch.bfloat16) -> QKBatch:
    """OLMo2-7B-shaped prefill: T=4096, Hq=Hk=4096 (MHA), bf16 (other element
    types on request).  x = N(0,1) * s_t with one scale per token
    s_t = exp(U(ln 0.1, ln 10)), shared by the token's Q and K rows."""
    g = _gen(seed)
    u = torch.rand((T,), generator=g, dtype=torch.float32)
    s = torch.exp(math.log(0.1) + u * (math.log(10.0) - math.log(0.1)))
    q = _normal_rows(g, T, H, dtype, row_scale=s)
    k = _normal_rows(g, T, H, dtype, row_scale=s)
    return QKBatch(f"prefill_{_DT_NAME[dtype]}_T{T}_H{H}", dtype, T, H, H, q, k,
                   gamma(H, seed + 100, dtype), gamma(H, seed + 200, dtype),
                   meta={"row_scale": "LogUniform(0.1, 10) per token"})


DECODE_TOKENS = (1, 8, 32, 128, 256)


def decode_bf16(T: int, seed: int = 2, H: int = 5120) -> QKBatch:
    """Decode-shaped latency case: T in {1, 8, 32, 128, 256}, Hq=Hk=5120, bf16."""
    g = _gen(seed)
    q = _normal_rows(g, T, H, torch.bfloat16)
    k = _normal_rows(g, T, H, torch.bfloat16)
    return QKBatch(f"decode_bf16_T{T}_H{H}", torch.bfloat16, T, H, H, q, k,
                   gamma(H, seed + 100, torch.bfloat16), gamma(H, seed + 200, torch.bfloat16))


def gqa_sharded(seed: int = 3, T: int = 16384, Hq: int = 5120, Hk: int = 1024,
                P: int = 4) -> ShardedBatch:
    """GQA shard-decomposed case: T=16384, Hq=5120, Hk=1024, bf16; Q and K each
    split into P=4 contiguous column shards held in separate buffers."""
    if Hq % P or Hk % P:
        raise ValueError("widths must divide into P equal shards")
    g = _gen(seed)
    q = _normal_rows(g, T, Hq, torch.bfloat16)
    k = _normal_rows(g, T, Hk, torch.bfloat16)
    wq, wk = Hq // P, Hk // P
    q_shards = [q[:, p * wq:(p + 1) * wq].contiguous() for p in range(P)]
    k_shards = [k[:, p * wk:(p + 1) * wk].contiguous() for p in range(P)]
    return ShardedBatch(f"gqa_sharded_T{T}_Hq{Hq}_Hk{Hk}_P{P}", torch.bfloat16, T, Hq, Hk, P,
                        q, k, q_shards, k_shards,
                        gamma(Hq, seed + 100, torch.bfloat16), gamma(Hk, seed + 200, torch.bfloat16))


def headwise_bf16(seed: int = 5, T: int = 4096, q_heads: int = 32, k_heads: int = 8,
                  head_dim: int = 128) -> QKBatch:
    """Headwise QK-Norm case (GQA-shaped: 32 query heads, 8 key heads of 128),
    bf16, x ~ N(0,1) * s_t with s_t ~ LogUniform(0.1, 10) per token; gamma
    [head_dim] per tensor.  ``meta['head_dim']`` holds the head size."""
    g = _gen(seed)
    u = torch.rand((T,), generator=g, dtype=torch.float32)
    s = torch.exp(math.log(0.1) + u * (math.log(10.0) - math.log(0.1)))
    q = _normal_rows(g, T, q_heads * head_dim, torch.bfloat16, row_scale=s)
    k = _normal_rows(g, T, k_heads * head_dim, torch.bfloat16, row_scale=s)
    return QKBatch(f"headwise_bf16_T{T}_q{q_heads}_k{k_heads}_d{head_dim}", torch.bfloat16, T,
                   q_heads * head_dim, k_heads * head_dim, q, k,
                   gamma(head_dim, seed + 100, torch.bfloat16), gamma(head_dim, seed + 200, torch.bfloat16),
                   meta={"head_dim": head_dim, "q_heads": q_heads, "k_heads": k_heads})


@dataclass
class ProjectionBatch:
    """Hidden states and QKV projection weights (CPU tensors, bfloat16).

    ``x`` is ``[T, D]``; ``w`` is ``[Hq + Hk + Hv, D]``, one row per output
    column (Q columns first, then K, then V); ``gamma_q`` ``[Hq]`` and
    ``gamma_k`` ``[Hk]`` are the QK-Norm scales."""
    name: str
    T: int
    D: int
    Hq: int
    Hk: int
    Hv: int
    x: torch.Tensor
    w: torch.Tensor
    gamma_q: torch.Tensor
    gamma_k: torch.Tensor
    eps: float = 1e-6


def qkv_projection(T: int = 4096, D: int = 4096, Hq: int = 4096, Hk: int = 4096, Hv: int = 4096,
                   seed: int = 6) -> ProjectionBatch:
    """Pre-LN hidden states and a QKV projection of OLMo2-7B's shape by
    default (hidden 4096, 32 query / key / value heads of 128).  x ~ N(0,1) * s_t
    with one s_t ~ LogUniform(0.1, 10) per token (the spread of per-token
    scales the prefill workload uses); W ~ N(0, 1/D), the usual fan-in
    scaling, so projected values are of order s_t.  gamma = 1 + 0.1 N(0,1).
    Seeds: x uses ``seed``, W seed + 50, gamma_q seed + 100, gamma_k seed + 200."""
    g = _gen(seed)
    u = torch.rand((T,), generator=g, dtype=torch.float32)
    s = torch.exp(math.log(0.1) + u * (math.log(10.0) - math.log(0.1)))
    x = _normal_rows(g, T, D, torch.bfloat16, row_scale=s)
    gw = _gen(seed + 50)
    N = Hq + Hk + Hv
    w = _normal_rows(gw, N, D, torch.bfloat16, row_scale=torch.full((N,), 1.0 / math.sqrt(D)))
    return ProjectionBatch(f"qkv_projection_bf16_T{T}_D{D}_q{Hq}_k{Hk}_v{Hv}", T, D, Hq, Hk, Hv, x, w,
                           gamma(Hq, seed + 100, torch.bfloat16), gamma(Hk, seed + 200, torch.bfloat16))


PACKED_TOKENS = (1024, 4096, 16384, 65536)


def packed_qkv(T: int, seed: int = 4, Hq: int = 4096, Hk: int = 1024, Hv: int = 1024,
               n_outliers: int = 8, outlier_scale: float = 100.0) -> QKBatch:
    """Packed QKV rows [Q | K | V] (stride Hq+Hk+Hv = 6144), bf16.  x ~ N(0,1)
    except ``n_outliers`` seeded channels per tensor (Q, K and V), scaled by
    ``outlier_scale``.  Q and K are normalized in place; V must stay untouched."""
    W = Hq + Hk + Hv
    go = _gen(seed + 300)
    col_scale = torch.ones((W,), dtype=torch.float32)
    chosen = {}
    for name, c0, width in (("q", 0, Hq), ("k", Hq, Hk), ("v", Hq + Hk, Hv)):
        cols = torch.randperm(width, generator=go)[:n_outliers] + c0
        col_scale[cols] = outlier_scale
        chosen[name] = sorted(int(c) for c in cols)
    g = _gen(seed)
    packed = torch.empty((T, W), dtype=torch.bfloat16)
    for r0 in range(0, T, _CHUNK_ROWS):
        r1 = min(T, r0 + _CHUNK_ROWS)
        blk = torch.randn((r1 - r0, W), generator=g, dtype=torch.float32)
        blk.mul_(col_scale[None, :])
        packed[r0:r1] = blk.to(torch.bfloat16)
    q = packed[:, :Hq]
    k = packed[:, Hq:Hq + Hk]
    return QKBatch(f"packed_qkv_T{T}_Hq{Hq}_Hk{Hk}_Hv{Hv}", torch.bfloat16, T, Hq, Hk, q, k,
                   gamma(Hq, seed + 100, torch.bfloat16), gamma(Hk, seed + 200, torch.bfloat16),
                   packed=packed, Hv=Hv, meta={"outlier_channels": chosen})


def random_rows(T: int, Hq: int, Hk: int, dtype: torch.dtype, seed: int,
                q_stride: int | None = None, k_stride: int | None = None,
                scale: float = 1.0) -> QKBatch:
    """Small random shapes for edge cases: Q and K in separate buffers whose
    row strides may exceed the widths.  Padding columns hold a sentinel so a
    stray write is visible."""
    q_stride = Hq if q_stride is None else q_stride
    k_stride = Hk if k_stride is None else k_stride
    g = _gen(seed)
    qb = torch.full((max(T, 1), q_stride), -7.0, dtype=torch.float32)
    kb = torch.full((max(T, 1), k_stride), -7.0, dtype=torch.float32)
    if T > 0:
        qb[:T, :Hq] = torch.randn((T, Hq), generator=g) * scale
        kb[:T, :Hk] = torch.randn((T, Hk), generator=g) * scale
    qb = qb.to(dtype)[:T] if T > 0 else qb.to(dtype)[:0]
    kb = kb.to(dtype)[:T] if T > 0 else kb.to(dtype)[:0]
    return QKBatch(f"random_T{T}_Hq{Hq}_Hk{Hk}", dtype, T, Hq, Hk,
                   qb[:, :Hq], kb[:, :Hk],
                   gamma(Hq, seed + 100, dtype), gamma(Hk, seed + 200, dtype),
                   meta={"q_buffer": qb, "k_buffer": kb})


def large_rows_on_device(T: int, Hq: int, Hk: int, dtype: torch.dtype, seed: int, device) -> QKBatch:
    """Q and K batches too large to build on the host (several GB), drawn on
    the device: x ~ N(0, 1) from a CUDA generator seeded with ``seed`` (Q
    first, then K), rounded once to ``dtype``; gamma as elsewhere, on the
    host.  The oracle reads back the rows it checks."""
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    q = torch.randn((T, Hq), generator=g, dtype=torch.float32, device=device).to(dtype)
    k = torch.randn((T, Hk), generator=g, dtype=torch.float32, device=device).to(dtype)
    return QKBatch(f"large_T{T}_Hq{Hq}_Hk{Hk}", dtype, T, Hq, Hk, q, k,
                   gamma(Hq, seed + 100, dtype), gamma(Hk, seed + 200, dtype))


def effective_bytes(T: int, Hq: int, Hk: int, esz: int) -> int:
    """Bytes a layerwise QK-Norm call must move: read + write of every Q and K
    element, plus one read of gamma_q and gamma_k."""
    return 2 * esz * (Hq + Hk) * T + esz * (Hq + Hk)
