"""Pins for the CPU oracle, against things other than itself.

The oracle restates RMS-Norm (Background, Equation 1 of "SwiftQK: Fast and
Communication-Efficient Tensor Parallelism for Query-Key Normalization") and its
Phase A shard decomposition in double precision.  Before any GPU result is
compared with it, it is checked here against:

* hand-derived closed forms (``tests/golden/closed_forms.json``);
* a library routine that computes the same definition
  (``torch.nn.functional.rms_norm`` in float64) and torch's own conversions
  between float32 and bfloat16, float16 and float8_e4m3fn (within its range);
* invariants the mathematics fixes (output RMS with gamma = 1, scale
  invariance, one-hot and power-of-two gamma, the shard-sum identity).

Each plausible slip — a dropped eps, a sum instead of a mean, a shard width
used as the divisor, a wrong sign, a stride or gamma index mix-up, truncation
instead of round-to-nearest-even — fails at least one test below.
"""
from __future__ import annotations

import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from tests.conftest import buffer_np, to_np

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "closed_forms.json")


def _golden():
    with open(GOLDEN) as f:
        return json.load(f)


def _parse_value(s):
    if isinstance(s, (int, float)):
        return float(s)
    table = {"inf": math.inf, "-inf": -math.inf, "-0": -0.0}
    if s in table:
        return table[s]
    # small closed-form expressions over powers of two, e.g. "1 + 3*2^-8"
    return float(eval(s.replace("^", "**"), {"__builtins__": {}}, {}))


# --------------------------------------------------------------------------- codec

def test_bf16_decode_matches_field_definition():
    for case in _golden()["bf16_decode"]:
        got = oracle.bf16_decode([int(case["bits"], 16)])[0]
        want = _parse_value(case["value"])
        assert got == want and math.copysign(1, got) == math.copysign(1, want), case


def test_bf16_encode_ties_to_even_fixtures():
    for case in _golden()["bf16_encode_rne"]:
        got = int(oracle.bf16_encode([_parse_value(case["value"])])[0])
        assert got == int(case["bits"], 16), (case, hex(got))


def test_bf16_encode_matches_torch_rounding_of_float32():
    """torch rounds float32 -> bfloat16 to nearest, ties to even.  Every float32
    is exact in double, so the oracle's single rounding must agree bit for bit.
    Exact ties (low 16 bits == 0x8000) are included on purpose."""
    g = torch.Generator().manual_seed(11)
    raw = torch.randint(0, 2**31 - 1, (20000,), generator=g, dtype=torch.int64)
    bits = raw.to(torch.int32)
    ties = (bits & ~0xFFFF) | 0x8000
    all_bits = torch.cat([bits, ties, -bits, -ties])
    f = all_bits.view(torch.float32)
    f = f[torch.isfinite(f)]
    want = f.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = oracle.bf16_encode(f.double().numpy())
    assert np.array_equal(got, want)


def test_bf16_decode_matches_torch_for_every_finite_pattern():
    bits = np.arange(0, 1 << 16, dtype=np.uint32).astype(np.uint16)
    vals = torch.from_numpy(bits.view(np.int16).copy()).view(torch.bfloat16).double().numpy()
    got = oracle.bf16_decode(bits)
    finite = np.isfinite(vals)
    assert np.array_equal(got[finite], vals[finite])
    assert np.array_equal(np.isnan(got), np.isnan(vals))


def test_f16_and_e4m3_fixtures():
    g = _golden()
    for case in g["f16_encode_rne"]:
        got = int(oracle.f16_encode([_parse_value(case["value"])])[0])
        assert got == int(case["bits"], 16), (case, hex(got))
    for case in g["e4m3_decode"]:
        assert oracle.e4m3_decode([int(case["bits"], 16)])[0] == case["value"], case
    for case in g["e4m3_encode_rne_sat"]:
        got = int(oracle.e4m3_encode([_parse_value(case["value"])])[0])
        assert got == int(case["bits"], 16), (case, hex(got))


def test_f16_codec_matches_torch():
    bits = np.arange(0, 1 << 16, dtype=np.uint32).astype(np.uint16)
    vals = torch.from_numpy(bits.view(np.int16).copy()).view(torch.float16).double().numpy()
    got = oracle.f16_decode(bits)
    fin = np.isfinite(vals)
    assert np.array_equal(got[fin], vals[fin]) and np.array_equal(np.isinf(got), np.isinf(vals))
    g = torch.Generator().manual_seed(12)
    f = torch.randn((20000,), generator=g) * torch.exp(torch.randn((20000,), generator=g) * 4)
    ties = (torch.from_numpy(bits[(bits & 0x7C00) != 0x7C00].astype(np.int16)).view(torch.float16).float()
            * (1 + 2.0 ** -11))  # exact halfway points between neighbouring halves
    f = torch.cat([f, ties[torch.isfinite(ties)]])
    want = f.to(torch.float16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(oracle.f16_encode(f.double().numpy()), want)


def test_e4m3_codec_matches_torch_within_range():
    bits = np.arange(256, dtype=np.uint8)
    vals = torch.from_numpy(bits.copy()).view(torch.float8_e4m3fn).double().numpy()
    got = oracle.e4m3_decode(bits)
    fin = np.isfinite(vals)
    assert np.array_equal(got[fin], vals[fin]) and np.array_equal(np.isnan(got), np.isnan(vals))
    g = torch.Generator().manual_seed(13)
    f = torch.randn((20000,), generator=g) * torch.exp(torch.randn((20000,), generator=g) * 3)
    f = f[f.abs() <= 448]
    pos = np.sort(np.unique(np.abs(vals[fin])))  # midpoints between neighbours are exact ties
    mids = torch.from_numpy((pos[:-1] + pos[1:]) / 2).float()
    f = torch.cat([f, mids, -mids])
    want = f.to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(oracle.e4m3_encode(f.double().numpy()), want)


# --------------------------------------------------------------------------- closed forms

def test_rmsnorm_closed_forms():
    for case in _golden()["rmsnorm"]:
        x = np.array(case["x"], dtype=np.float32)[None, :]
        gm = np.array(case["gamma"], dtype=np.float32)
        H = x.shape[1]
        _, y, s = oracle.rmsnorm_rows(x, H, gm, case["eps"])
        assert s[0] == case["sumsq"], case["name"]
        np.testing.assert_allclose(y[0], case["y"], rtol=1e-15, atol=0, err_msg=case["name"])


def test_sharded_closed_form_divides_by_full_width():
    case = _golden()["sharded"][0]
    x = np.array(case["x_full"], dtype=np.float32)
    gm = np.array(case["gamma_full"], dtype=np.float32)
    widths = case["shard_widths"]
    H = int(sum(widths))
    cols = np.cumsum([0] + widths)
    parts = []
    for p, w in enumerate(widths):
        xs = np.ascontiguousarray(x[cols[p]:cols[p + 1]][None, :])
        parts.append(oracle.partial_sumsq(xs, w, w, 1))
    assert [float(v[0]) for v in parts] == case["partial_sumsq"]
    stats = np.stack(parts)
    for p, w in enumerate(widths):
        xs = np.ascontiguousarray(x[cols[p]:cols[p + 1]][None, :])
        gs = np.ascontiguousarray(gm[cols[p]:cols[p + 1]])
        _, y = oracle.combine_apply(xs, w, w, 1, gs, stats, H, case["eps"])
        np.testing.assert_allclose(y[0], case["y_shards"][p], rtol=1e-15, atol=0)


# --------------------------------------------------------------------------- library routine

@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16, torch.float16, torch.float8_e4m3fn])
@pytest.mark.parametrize("T,H,pad", [(1, 1, 0), (3, 7, 5), (17, 64, 3), (9, 513, 0), (4, 4096, 8)])
def test_rmsnorm_matches_torch_rms_norm_float64(dtype, T, H, pad):
    g = torch.Generator().manual_seed(1000 + T * 7 + H)
    stride = H + pad
    buf = (torch.randn((T, stride), generator=g) * 3.0).to(dtype)
    view = buf[:, :H]
    gdt = torch.bfloat16 if dtype == torch.float8_e4m3fn else dtype
    gm = (1.0 + 0.1 * torch.randn((H,), generator=g)).to(gdt)
    eps = 1e-6
    flat, st = buffer_np(view)
    y_rounded, y, s = oracle.rmsnorm_rows(flat, H, to_np(gm), eps, stride=st, T=T)
    ref = torch.nn.functional.rms_norm(view.double(), (H,), weight=gm.double(), eps=eps)
    np.testing.assert_allclose(y, ref.numpy(), rtol=1e-13, atol=1e-300)
    np.testing.assert_allclose(s, (view.double() ** 2).sum(dim=1).numpy(), rtol=1e-13)
    # the stored output is one correct rounding of the double result
    if dtype == torch.float32:
        assert np.array_equal(y_rounded, y.astype(np.float32))
    elif dtype == torch.bfloat16:
        assert np.array_equal(y_rounded, oracle.bf16_encode(y))
    elif dtype == torch.float16:
        assert np.array_equal(y_rounded.view(np.uint16), oracle.f16_encode(y))
    else:
        assert np.array_equal(y_rounded, oracle.e4m3_encode(y))


def test_layerwise_treats_q_and_k_independently():
    g = torch.Generator().manual_seed(5)
    T, Hq, Hk = 6, 40, 24
    q = torch.randn((T, Hq), generator=g)
    k = torch.randn((T, Hk), generator=g) * 10
    gq = 1 + 0.1 * torch.randn((Hq,), generator=g)
    gk = 1 + 0.1 * torch.randn((Hk,), generator=g)
    qo, ko = oracle.qknorm_layerwise(to_np(q), Hq, to_np(gq), Hq, to_np(k), Hk, to_np(gk), Hk, T, 1e-6)
    rq = torch.nn.functional.rms_norm(q.double(), (Hq,), weight=gq.double(), eps=1e-6).float()
    rk = torch.nn.functional.rms_norm(k.double(), (Hk,), weight=gk.double(), eps=1e-6).float()
    np.testing.assert_allclose(qo, rq.numpy(), rtol=2e-7)
    np.testing.assert_allclose(ko, rk.numpy(), rtol=2e-7)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16, torch.float8_e4m3fn])
@pytest.mark.parametrize("T,nh,hd,pad", [(1, 1, 1, 0), (5, 4, 8, 3), (3, 32, 128, 16), (7, 3, 7, 0)])
def test_headwise_matches_torch_rms_norm_over_heads(dtype, T, nh, hd, pad):
    """Headwise RMS-Norm is rms_norm over the last axis of the [T, n_heads,
    head_dim] view, gamma [head_dim] broadcast over heads (a library routine)."""
    g = torch.Generator().manual_seed(31 + T + nh + hd)
    W = nh * hd
    buf = (torch.randn((T, W + pad), generator=g) * 2).to(dtype)
    view = buf[:, :W]
    gdt = torch.bfloat16 if dtype == torch.float8_e4m3fn else dtype
    gm = (1 + 0.1 * torch.randn((hd,), generator=g)).to(gdt)
    flat, st = buffer_np(view)
    y_r, y = oracle.rmsnorm_heads(flat, nh, hd, to_np(gm), 1e-6, stride=st, T=T)
    ref = torch.nn.functional.rms_norm(view.double().reshape(T, nh, hd), (hd,), weight=gm.double(), eps=1e-6)
    np.testing.assert_allclose(y, ref.reshape(T, W).numpy(), rtol=1e-13, atol=1e-300)


def test_headwise_with_one_head_is_layerwise_and_heads_are_independent():
    g = torch.Generator().manual_seed(32)
    T, nh, hd = 4, 6, 16
    x = torch.randn((T, nh * hd), generator=g)
    gm = 1 + 0.1 * torch.randn((hd,), generator=g)
    # one head spanning the row equals the layerwise form
    _, y1 = oracle.rmsnorm_heads(to_np(x), 1, nh * hd, to_np(gm.repeat(nh)), 1e-6, stride=nh * hd, T=T)
    _, yl, _ = oracle.rmsnorm_rows(to_np(x), nh * hd, to_np(gm.repeat(nh)), 1e-6)
    np.testing.assert_allclose(y1, yl, rtol=1e-15)
    # scaling one head leaves every other head's output unchanged (eps = 0: the scaled head is unchanged too)
    x2 = x.clone()
    x2[:, 2 * hd:3 * hd] *= 64.0
    _, ya = oracle.rmsnorm_heads(to_np(x), nh, hd, to_np(gm), 0.0, stride=nh * hd, T=T)
    _, yb = oracle.rmsnorm_heads(to_np(x2), nh, hd, to_np(gm), 0.0, stride=nh * hd, T=T)
    assert np.array_equal(ya, yb)
    # the per-head closed form: a head of constant c normalizes to gamma * c / sqrt(c^2 + eps)
    x3 = torch.zeros((1, nh * hd))
    x3[0, hd:2 * hd] = 0.5
    _, y3 = oracle.rmsnorm_heads(to_np(x3), nh, hd, to_np(torch.ones(hd)), 0.25, stride=nh * hd, T=1)
    np.testing.assert_allclose(y3[0, hd:2 * hd], 0.5 / math.sqrt(0.5), rtol=1e-15)
    assert np.count_nonzero(y3[0, :hd]) == 0 and np.count_nonzero(y3[0, 2 * hd:]) == 0


# --------------------------------------------------------------------------- invariants

@pytest.mark.parametrize("eps_ratio", [0.0, 1e-6, 1.0, 37.0])
def test_output_rms_with_unit_gamma(eps_ratio):
    """gamma = 1: mean_j y_j^2 = m / (m + eps) exactly, m = mean_j x_j^2."""
    g = torch.Generator().manual_seed(21)
    T, H = 8, 300
    x = torch.randn((T, H), generator=g, dtype=torch.float32)
    m = (x.double() ** 2).mean(dim=1).numpy()
    eps = float(eps_ratio * m.mean())
    _, y, _ = oracle.rmsnorm_rows(to_np(x), H, np.ones(H, np.float32), eps)
    got = (y ** 2).mean(axis=1)
    np.testing.assert_allclose(got, m / (m + eps), rtol=1e-13)


def test_scale_invariance_power_of_two():
    """eps = 0 and c = 2^k: every step scales exactly, so y(c x) == y(x) bit for bit.
    With eps small against mean(x^2) the two agree to about eps / mean(x^2)."""
    g = torch.Generator().manual_seed(22)
    T, H = 5, 256
    x = torch.randn((T, H), generator=g, dtype=torch.float32)
    gm = (1 + 0.1 * torch.randn((H,), generator=g)).float()
    _, y0, _ = oracle.rmsnorm_rows(to_np(x), H, to_np(gm), 0.0)
    for c in (2.0 ** -7, 2.0 ** 6):
        _, yc, _ = oracle.rmsnorm_rows(to_np(x * c), H, to_np(gm), 0.0)
        assert np.array_equal(yc, y0)
    for c in (1e-2, 1e2):
        _, yc, _ = oracle.rmsnorm_rows(to_np((x.double() * c).float()), H, to_np(gm), 1e-12)
        np.testing.assert_allclose(yc, y0, rtol=1e-6)


def test_one_hot_gamma_selects_one_column():
    g = torch.Generator().manual_seed(23)
    T, H, col = 4, 33, 17
    x = torch.randn((T, H), generator=g, dtype=torch.float32)
    gm = np.zeros(H, np.float32)
    gm[col] = 1.0
    _, y, s = oracle.rmsnorm_rows(to_np(x), H, gm, 1e-6)
    assert np.count_nonzero(y[:, np.arange(H) != col]) == 0
    r = 1.0 / np.sqrt(s / H + 1e-6)
    np.testing.assert_allclose(y[:, col], x[:, col].double().numpy() * r, rtol=1e-15)


def test_power_of_two_gamma_scales_exactly():
    g = torch.Generator().manual_seed(24)
    T, H = 3, 100
    x = torch.randn((T, H), generator=g, dtype=torch.float32)
    _, y1, _ = oracle.rmsnorm_rows(to_np(x), H, np.ones(H, np.float32), 1e-6)
    _, y8, _ = oracle.rmsnorm_rows(to_np(x), H, np.full(H, 8.0, np.float32), 1e-6)
    assert np.array_equal(y8, 8.0 * y1)


def test_shard_sums_add_to_full_sum_exactly_for_integers():
    """Small integers: every square and partial sum is exact in double, so
    sum_p S_p == S_full with no rounding at all (Phase A identity)."""
    g = torch.Generator().manual_seed(25)
    T, H, P = 7, 96, 4
    x = torch.randint(-50, 51, (T, H), generator=g).float()
    _, _, s_full = oracle.rmsnorm_rows(to_np(x), H, np.ones(H, np.float32), 0.0)
    w = H // P
    parts = [oracle.partial_sumsq(to_np(x[:, p * w:(p + 1) * w]), w, w, T) for p in range(P)]
    assert np.array_equal(np.sum(parts, axis=0), s_full)
    assert np.array_equal(s_full, (x.double() ** 2).sum(dim=1).numpy())


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_shard_pipeline_matches_full_row(dtype):
    """partial_sumsq per shard, then combine_apply per shard, reproduces the
    unsharded normalization (same global semantics, Phase A)."""
    g = torch.Generator().manual_seed(26)
    T, Hq, P = 11, 160, 4
    x = torch.randn((T, Hq), generator=g).to(dtype)
    gm = (1 + 0.1 * torch.randn((Hq,), generator=g)).to(dtype)
    _, y_full, _ = oracle.rmsnorm_rows(to_np(x), Hq, to_np(gm), 1e-6)
    w = Hq // P
    stats = np.stack([oracle.partial_sumsq(to_np(x[:, p * w:(p + 1) * w]), w, w, T) for p in range(P)])
    for p in range(P):
        _, yp = oracle.combine_apply(to_np(x[:, p * w:(p + 1) * w]), w, w, T,
                                     to_np(gm[p * w:(p + 1) * w]), stats, Hq, 1e-6)
        np.testing.assert_allclose(yp, y_full[:, p * w:(p + 1) * w], rtol=1e-14)


def test_strided_rows_read_only_their_columns():
    """Padding columns hold huge values; they must not leak into the result."""
    T, H, stride = 4, 10, 16
    buf = np.full((T, stride), 1e30, dtype=np.float32)
    buf[:, :H] = np.arange(1, H + 1, dtype=np.float32)
    _, y, s = oracle.rmsnorm_rows(buf, H, np.ones(H, np.float32), 0.0, stride=stride, T=T)
    assert np.all(s == 385.0)  # 1^2 + ... + 10^2
    np.testing.assert_allclose(y[0], np.arange(1, H + 1) / math.sqrt(38.5), rtol=1e-15)


def test_empty_batch_and_bad_arguments():
    y, ye, s = oracle.rmsnorm_rows(np.zeros((0, 8), np.float32), 8, np.ones(8, np.float32), 1e-6, T=0)
    assert y.shape == (0, 8) and s.shape == (0,)
    with pytest.raises(ValueError):
        oracle.rmsnorm_rows(np.zeros((2, 8), np.float32), 8, np.ones(8, np.float32), -1.0)
    with pytest.raises(ValueError):
        oracle.rmsnorm_rows(np.zeros((2, 8), np.float32), 8, np.ones(8, np.float32), 1e-6, stride=4, T=2)
    with pytest.raises(ValueError):
        oracle.combine_apply(np.zeros((2, 8), np.float32), 8, 8, 2, np.ones(8, np.float32),
                             np.zeros((1, 2)), 4, 1e-6)  # full width below shard width


# --------------------------------------------------------------------------- projection

@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16, torch.float32])
def test_projection_matches_numpy_matmul(dtype):
    """The projection against a library matmul of the same decoded values
    (float64 BLAS): W is [N][D], so y = x[rows] @ W^T."""
    g = torch.Generator().manual_seed(41)
    T, D, N = 9, 70, 33
    x = torch.randn((T, D), generator=g).to(dtype)
    w = (torch.randn((N, D), generator=g) * 0.1).to(dtype)
    rows = [8, 0, 3, 3, 5]
    y, y_exact = oracle.project_rows(to_np(x), to_np(w), rows)
    ref = x.double().numpy()[rows] @ w.double().numpy().T
    np.testing.assert_allclose(y_exact, ref, rtol=1e-12, atol=1e-12)
    # the stored result is the exact sum rounded once to the element type
    if dtype == torch.float32:
        np.testing.assert_array_equal(y, ref.astype(np.float32))


def test_projection_of_small_integers_is_exact_and_rounds_once():
    """Integer inputs: every dot product is an exact integer (computed here in
    Python integers); below 2^24 it converts to float32 exactly, and torch's
    float32 -> bfloat16 rounding (pinned above) then gives the stored value."""
    rng = np.random.default_rng(42)
    T, D, N = 5, 48, 24
    xi = rng.integers(-60, 61, size=(T, D))
    wi = rng.integers(-60, 61, size=(N, D))
    x = torch.tensor(xi, dtype=torch.bfloat16)
    w = torch.tensor(wi, dtype=torch.bfloat16)
    assert torch.equal(x.double(), torch.tensor(xi, dtype=torch.float64))  # |v| <= 60 is exact in bf16
    y, y_exact = oracle.project_rows(to_np(x), to_np(w), list(range(T)))
    exact = [[sum(int(xi[t, d]) * int(wi[n, d]) for d in range(D)) for n in range(N)] for t in range(T)]
    assert y_exact.tolist() == [[float(v) for v in row] for row in exact]
    expect = torch.tensor(exact, dtype=torch.float32).to(torch.bfloat16)
    assert np.array_equal(y, to_np(expect))


def test_projection_identity_weight_and_strides():
    """W = I returns the selected rows bit for bit; padded row strides are
    honoured on both operands; a one-hot W row selects one input column."""
    g = torch.Generator().manual_seed(43)
    T, D, pad = 6, 16, 8
    xb = torch.randn((T, D + pad), generator=g).to(torch.bfloat16)
    wb = torch.zeros((D, D + 4), dtype=torch.bfloat16)
    wb[:, :D] = torch.eye(D)
    wb[:, D:] = 99.0  # padding columns must not be read
    y, _ = oracle.project_rows(to_np(xb), to_np(wb), [4, 1], D=D, N=D, x_stride=D + pad, w_stride=D + 4)
    assert np.array_equal(y, to_np(xb[[4, 1], :D].contiguous()))
    w1 = torch.zeros((3, D), dtype=torch.bfloat16)
    w1[0, 5] = 1.0
    w1[1, 0] = -2.0
    w1[2, D - 1] = 0.5
    _, ye = oracle.project_rows(to_np(xb), to_np(w1), [2], D=D, x_stride=D + pad)
    xd = xb.double()
    assert ye[0].tolist() == [xd[2, 5].item(), -2.0 * xd[2, 0].item(), 0.5 * xd[2, D - 1].item()]


def test_projection_then_tile_sums_recover_the_row_sum():
    """The projected Q row split into 256-column tiles: the tiles' squared sums
    (Phase A's local step) add up to the full row's squared sum."""
    g = torch.Generator().manual_seed(44)
    T, D, N = 3, 64, 1024
    x = torch.randn((T, D), generator=g).to(torch.bfloat16)
    w = (torch.randn((N, D), generator=g) * 0.125).to(torch.bfloat16)
    y, _ = oracle.project_rows(to_np(x), to_np(w), list(range(T)))
    tiles = [oracle.partial_sumsq(np.ascontiguousarray(y[:, p * 256:(p + 1) * 256]), 256, 256, T)
             for p in range(N // 256)]
    _, _, full = oracle.rmsnorm_rows(y, N, np.full(N, 0x3F80, dtype=np.uint16), 0.0)
    np.testing.assert_allclose(sum(tiles), full, rtol=1e-14)
