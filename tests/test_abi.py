"""The C-ABI without a GPU: the library loads, exports every symbol the headers
declare, and its host-side logic (argument validation, overlap detection,
launch planning) behaves as documented.

Validation runs on the host before any CUDA call, so invalid arguments can be
exercised here with fake addresses: nothing is dereferenced.  Arguments that
pass validation go on to query the device; on a machine without a GPU that
query fails with QKN_ERR_CUDA, which is how "accepted" is observed here.
"""
from __future__ import annotations

import ctypes
import itertools
import os
import re

import pytest
import torch

import attention_normalization_b200 as qk
from attention_normalization_b200 import _clib
from attention_normalization_b200 import build as qbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADERS = [os.path.join(ROOT, "include", h) for h in ("qknorm.h", "qknorm_plan.h")]

OK, INVALID, MISALIGNED, UNSUPPORTED, CUDA = 0, 1, 2, 3, 4  # the status codes of the boundary contract
F32, BF16 = 0, 1


@pytest.fixture(scope="module")
def lib():
    qbuild.build(quiet=True)
    return _clib.load()


def _declared_functions() -> set[str]:
    names = set()
    for h in HEADERS:
        src = open(h).read()
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        for m in re.finditer(r"\b(qknorm_\w+)\s*\(", src):
            names.add(m.group(1))
    return names


def test_every_declared_symbol_is_exported(lib):
    declared = _declared_functions()
    assert declared, "no declarations parsed"
    missing = [n for n in declared if not hasattr(lib, n)]
    assert not missing, f"declared but not exported: {missing}"
    assert declared == set(_clib.PROTOTYPES), "binding prototypes differ from the headers"


def test_version_and_status_strings(lib):
    assert lib.qknorm_version() >= 100
    assert lib.qknorm_status_string(OK) == b"ok"
    assert lib.qknorm_status_string(INVALID) == b"invalid argument"
    assert lib.qknorm_status_string(CUDA) == b"CUDA error"
    assert lib.qknorm_status_string(UNSUPPORTED) == b"unsupported"
    assert lib.qknorm_status_string(MISALIGNED).startswith(b"misaligned")
    assert lib.qknorm_status_string(99) == b"unknown status"


# --------------------------------------------------------------------------- validation

BASE = 1 << 32  # fake, 256-byte aligned addresses: never dereferenced


def layerwise(lib, q_in=BASE, q_out=BASE + (1 << 28), gq=BASE + (2 << 28), qs=512,
              k_in=BASE + (3 << 28), k_out=BASE + (4 << 28), gk=BASE + (5 << 28), ks=512,
              T=64, Hq=512, Hk=512, eps=1e-6, dtype=BF16, plan=True):
    """Calls qknorm_layerwise_plan (validation + planning, no launch)."""
    L = _clib.QknLaunch()
    return lib.qknorm_layerwise_plan(q_in, q_out, gq, qs, k_in, k_out, gk, ks, T, Hq, Hk, eps, dtype,
                                     ctypes.byref(L))


def test_well_formed_call_passes_validation(lib):
    st = layerwise(lib)
    # without a GPU the device query fails; with one, planning succeeds
    assert st in (OK, CUDA)
    if st == CUDA:
        assert lib.qknorm_last_error()


@pytest.mark.parametrize("kw,why", [
    ({"dtype": 7}, "dtype"),
    ({"dtype": 4}, "dtype past E4M3"),
    ({"dtype": -1}, "negative dtype"),
    ({"T": -1}, "T < 0"),
    ({"Hq": 0}, "Hq = 0"),
    ({"Hk": -3}, "Hk < 0"),
    ({"qs": 511}, "q stride below width"),
    ({"ks": 100}, "k stride below width"),
    ({"eps": -1e-6}, "negative eps"),
    ({"eps": float("nan")}, "nan eps"),
    ({"eps": float("inf")}, "inf eps"),
    ({"q_in": 0}, "null q_in"),
    ({"k_out": 0}, "null k_out"),
    ({"gq": 0}, "null gamma_q"),
    ({"q_out": BASE + 16}, "q_out partly overlaps q_in"),
    ({"k_out": BASE + (3 << 28) + 2}, "k_out partly overlaps k_in"),
    ({"k_out": BASE + 64}, "k_out overlaps q_in"),
    ({"q_out": BASE + (3 << 28) + 1024}, "q_out overlaps k_in"),
    ({"k_out": BASE + (1 << 28) + 512}, "q_out and k_out overlap"),
    ({"gq": BASE + (1 << 28) + 4096}, "gamma_q inside q_out"),
    ({"gk": BASE + (1 << 28)}, "gamma_k inside q_out"),
    ({"T": 1 << 61}, "extent overflow"),
])
def test_invalid_arguments_rejected_before_any_launch(lib, kw, why):
    assert layerwise(lib, **kw) == INVALID, why
    assert lib.qknorm_last_error(), why


def test_empty_batch_is_ok_without_touching_the_device(lib):
    T0 = dict(T=0)
    L = _clib.QknLaunch()
    assert lib.qknorm_layerwise(BASE, BASE, BASE + 4096, 512, BASE + 8192, BASE + 8192, BASE + 12288,
                                512, 0, 512, 512, 1e-6, BF16, None) == OK
    assert layerwise(lib, **T0) == OK
    # null pointers are tolerated when there is nothing to do
    assert lib.qknorm_layerwise(0, 0, 0, 512, 0, 0, 0, 512, 0, 512, 512, 1e-6, F32, None) == OK


def test_in_place_and_packed_layouts_pass_validation(lib):
    # in place: out == in
    assert layerwise(lib, q_out=BASE, k_out=BASE + (3 << 28)) in (OK, CUDA)
    # packed [Q | K | V] rows, bf16, stride 6144: K starts 4096 elements into each row
    base, stride = BASE, 6144
    k = base + 4096 * 2
    st = layerwise(lib, q_in=base, q_out=base, qs=stride, k_in=k, k_out=k, ks=stride,
                   T=16384, Hq=4096, Hk=1024)
    assert st in (OK, CUDA)
    # ... but a K width reaching into the next row's Q is rejected
    st = layerwise(lib, q_in=base, q_out=base, qs=stride, k_in=k, k_out=k, ks=stride,
                   T=16384, Hq=4096, Hk=2049)
    assert st == INVALID


def test_partial_stats_validation(lib):
    f = lib.qknorm_partial_stats
    good = [BASE, 1280, 1280, BASE + (1 << 28), BASE + (2 << 28), 256, 256, BASE + (3 << 28), 16384, BF16, None]
    assert f(*good) in (OK, CUDA)
    bad = list(good)
    bad[3] = bad[7]  # both sums into one array
    assert f(*bad) == INVALID
    bad = list(good)
    bad[3] = BASE + 100  # sums written into the Q shard
    assert f(*bad) == INVALID
    bad = list(good)
    bad[2] = 0
    assert f(*bad) == INVALID
    bad = list(good)
    bad[8] = -5
    assert f(*bad) == INVALID
    z = list(good)
    z[8] = 0
    assert f(*z) == OK


def test_combine_apply_validation(lib):
    f = lib.qknorm_combine_apply
    T, P = 1024, 4
    good = [BASE, BASE, BASE + (1 << 28), 1280, 1280, BASE + (2 << 28), 5120,
            BASE + (3 << 28), BASE + (3 << 28), BASE + (4 << 28), 256, 256, BASE + (5 << 28), 1024,
            P, T, 1e-6, BF16, None]
    assert f(*good) in (OK, CUDA)
    for idx, val, why in [(14, 0, "P < 1"), (6, 1000, "full width below shard"), (16, -1.0, "eps"),
                          (5, 0, "null sums"), (1, BASE + (2 << 28), "q_out onto gamma"),
                          (8, BASE + (5 << 28) + 4, "k_out onto k sums")]:
        bad = list(good)
        bad[idx] = val
        assert f(*bad) == INVALID, why


def test_launch_override_validation(lib):
    f = lib.qknorm_layerwise_launch
    args = [BASE, BASE + (1 << 28), BASE + (2 << 28), 4096, BASE + (3 << 28), BASE + (4 << 28),
            BASE + (5 << 28), 4096, 0, 4096, 4096, 1e-6, BF16, None]

    def st(kernel, nv, threads, grid, a=args):
        L = _clib.QknLaunch(kernel, nv, threads, grid)
        return f(*a, ctypes.byref(L))

    assert st(0, 4, 128, 100) == OK  # T = 0: validated, nothing launched
    assert st(0, 4, 96, 100) == INVALID  # 4 * 96 < 512 vectors
    assert st(0, 3, 256, 100) == INVALID  # vec_per_thread
    assert st(0, 5, 128, 100) == INVALID  # 5: the partial-sum and apply passes only
    assert st(0, 8, 512, 100) == INVALID  # above the NV=8 limit
    assert st(0, 4, 100, 100) == INVALID  # not a multiple of 32
    assert st(0, 4, 128, 0) == INVALID  # grid
    assert st(3, 4, 128, 1) == INVALID  # kind
    assert st(1, 0, 1024, 1) == OK
    assert st(2, 0, 64, 1) == OK
    ragged = list(args)
    ragged[3] = ragged[9] = 4100  # stride 8200 B is not 16-aligned: only the scalar kernel
    assert st(0, 8, 128, 10, a=ragged) == INVALID
    assert st(2, 0, 128, 10, a=ragged) == OK
    ragged[3] = 4104  # aligned stride, ragged width: the register kernel takes the tail
    assert st(0, 8, 128, 10, a=ragged) == OK
    unaligned = list(args)
    unaligned[0] += 2
    unaligned[1] += 2
    assert st(0, 4, 128, 1, a=unaligned) == INVALID  # register kernel on unaligned data
    assert st(2, 0, 128, 1, a=unaligned) == OK


def test_shard_launch_override_validation(lib):
    T = 16384
    stats = [BASE, 1280, 1280, BASE + (1 << 28), BASE + (2 << 28), 256, 256, BASE + (3 << 28), T, BF16, None]
    apply = [BASE, BASE, BASE + (1 << 28), 1280, 1280, BASE + (2 << 28), 5120,
             BASE + (3 << 28), BASE + (3 << 28), BASE + (4 << 28), 256, 256, BASE + (5 << 28), 1024,
             4, T, 1e-6, BF16, None]
    for f, args in ((lib.qknorm_partial_stats_launch, stats), (lib.qknorm_combine_apply_launch, apply)):
        zero = list(args)
        zero[8 if f is lib.qknorm_partial_stats_launch else 15] = 0  # T = 0: validated, nothing launched
        assert f(*zero, ctypes.byref(_clib.QknLaunch(0, 2, 96, 10))) == OK
        assert f(*zero, ctypes.byref(_clib.QknLaunch(0, 5, 32, 10))) == OK  # one warp per 160-vector shard row
        assert f(*zero, ctypes.byref(_clib.QknLaunch(0, 1, 96, 10))) == INVALID  # 96 < 160 vectors
        assert f(*zero, ctypes.byref(_clib.QknLaunch(0, 2, 100, 10))) == INVALID
        assert f(*zero, None) == INVALID
        bad = list(args)
        bad[1 if f is lib.qknorm_partial_stats_launch else 3] = 1279  # stride below width
        assert f(*bad, ctypes.byref(_clib.QknLaunch(0, 2, 96, 10))) == INVALID


# --------------------------------------------------------------------------- overlap

def _brute(a, b):
    def bytes_of(r):
        base, w, s, n = r
        return {base + t * s + j for t in range(n) for j in range(w)}
    return bool(bytes_of(a) & bytes_of(b))


def test_regions_overlap_exact_against_brute_force():
    cases = 0
    for wa, sa, na in itertools.product((1, 3, 8), (8, 12), (1, 2, 4)):
        for wb, sb, nb in itertools.product((1, 5), (8, 12), (1, 3)):
            if wa > sa or wb > sb:
                continue
            for off in range(-40, 41, 3):
                a = (1000, wa, sa, na)
                b = (1000 + off, wb, sb, nb)
                got = qk.regions_overlap(a, b)
                want = _brute(a, b)
                if sa == sb or na == 1 or nb == 1:
                    assert got == want, (a, b)
                else:
                    assert got or not want, (a, b)  # conservative: never misses an overlap
                assert qk.regions_overlap(b, a) == got
                cases += 1
    assert cases > 500


def test_regions_overlap_edge_cases():
    assert not qk.regions_overlap((100, 10, 10, 0), (100, 10, 10, 5))  # empty set
    assert not qk.regions_overlap((100, 10, 20, 3), (110, 10, 20, 3))  # interleaved columns
    assert qk.regions_overlap((100, 11, 20, 3), (110, 10, 20, 3))
    # packed QKV, bf16: Q cols [0, 4096), K cols [4096, 5120) of a 6144 stride
    q = (0, 8192, 12288, 65536)
    k = (8192, 2048, 12288, 65536)
    v = (10240, 2048, 12288, 65536)
    assert not qk.regions_overlap(q, k)
    assert not qk.regions_overlap(k, v)
    assert not qk.regions_overlap(q, v)


# --------------------------------------------------------------------------- planning

@pytest.mark.parametrize("rows,units", [(2, 640), (16, 640), (256, 640), (512, 640), (8192, 512),
                                        (128, 128), (65536 * 2, 512), (32768, 160), (4096, 1),
                                        (2, 2048), (1 << 20, 2048), (10, 33), (131072, 16), (8192, 32)])
def test_plan_shape_covers_the_row(rows, units):
    L = qk.plan_shape(rows, units, True, 148)
    assert L["kernel"] == 0
    nv, th = L["vec_per_thread"], L["threads"]
    assert nv in (1, 2, 4, 8)
    assert th % 32 == 0 and 32 <= th <= _clib.load().qknorm_register_max_threads(nv)
    assert nv * th >= units
    if rows > 148 and units < 64:
        assert th == 256 and nv == min(4, 1 << (units - 1).bit_length())  # many narrow rows: many per CTA
    else:
        assert nv * (th - 32) < units  # no whole idle warp


def test_plan_shape_one_byte_elements_hold_half_the_vectors():
    """1-byte elements widen to twice the registers: half the vectors per
    thread for few rows and for narrow rows; many wide rows (gamma re-read per
    row) keep the full count in half the threads."""
    two = qk.plan_shape(8192, 512, True, 148, 2)
    one = qk.plan_shape(8192, 256, True, 148, 1)   # the same rows in 1-byte elements: half the vectors
    assert one["vec_per_thread"] == two["vec_per_thread"] == 4
    assert one["threads"] * 2 == two["threads"]
    for rows, units in ((100, 640), (8192, 16)):   # few rows; narrow rows
        assert qk.plan_shape(rows, units, True, 148, 1)["vec_per_thread"] * 2 == \
            qk.plan_shape(rows, units, True, 148, 2)["vec_per_thread"]
    assert one["vec_per_thread"] * one["threads"] >= 256
    with pytest.raises(qk.QKNormError):
        qk.plan_shape(10, 10, True, 148, 3)


def test_plan_shape_wide_and_unaligned():
    assert qk.plan_shape(100, 2049, True, 148)["kernel"] == 1
    u = qk.plan_shape(100, 4097, False, 148)
    assert u["kernel"] == 2 and u["threads"] == 256
    assert qk.plan_shape(100, 5, False, 148)["threads"] == 32
    with pytest.raises(qk.QKNormError):
        qk.plan_shape(0, 5, True, 148)


def test_plan_shape_latency_mode_uses_more_threads_for_few_rows():
    few = qk.plan_shape(2, 640, True, 148)
    many = qk.plan_shape(8192, 640, True, 148)
    assert few["threads"] > many["threads"]
    assert few["vec_per_thread"] <= 2


@pytest.mark.parametrize("rows", [1, 2, 147, 148, 149, 1000, 8192, 131072, 10 ** 7])
@pytest.mark.parametrize("bps,sms", [(1, 148), (8, 148), (16, 148), (3, 1)])
def test_plan_grid_fills_every_resident_slot(rows, bps, sms):
    g = qk.plan_grid(rows, bps, sms)
    assert g == min(rows, bps * sms)
    trips = -(-rows // g)
    assert trips == -(-rows // (bps * sms))  # no more loop trips than the resident limit forces


def test_plan_grid_degenerate():
    assert qk.plan_grid(0, 8, 148) == 0
    assert qk.plan_grid(10, 0, 0) == 1


# --------------------------------------------------------------------------- binding

def test_binding_refuses_cpu_tensors():
    x = torch.zeros((4, 8), dtype=torch.float32)
    g = torch.ones((8,), dtype=torch.float32)
    with pytest.raises(ValueError, match="CUDA"):
        qk.qknorm_layerwise(x, x, g, g)
    with pytest.raises(ValueError, match="CUDA"):
        qk.qknorm_partial_stats(x, x)


def test_host_pipeline_argument_checks():
    x = torch.zeros((4, 8), dtype=torch.float32)
    g = torch.ones((8,), dtype=torch.float32)
    with pytest.raises(ValueError, match="same number of tokens"):
        qk.qknorm_layerwise_host(x, torch.zeros((5, 8)), g, g)
    with pytest.raises(ValueError, match="chunk_tokens"):
        qk.qknorm_layerwise_host(x, x, g, g, chunk_tokens=0)
    with pytest.raises(ValueError, match="inside the packed row"):
        qk.qknorm_packed_host(torch.zeros((4, 16)), 0, 8, 8, 9, g, g)


def _proj_call(lib, **kw):
    a = dict(x=0x10000, xs=4096, w=0x2000000, ws=4096, qkv=0x8000000, qs=12288, T=4096, D=4096, Hq=4096,
             Hk=4096, Hv=4096, q_sums=0x20000000, k_sums=0x21000000, dtype=BF16)
    a.update(kw)
    return lib.qknorm_qkv_gemm_stats(a["x"], a["xs"], a["w"], a["ws"], a["qkv"], a["qs"], a["T"], a["D"], a["Hq"],
                                     a["Hk"], a["Hv"], a["q_sums"], a["k_sums"], a["dtype"], None)


@pytest.mark.parametrize("kw,want", [
    ({}, CUDA),                                  # well formed: validation passes, the device query fails here
    ({"T": 0}, OK),                              # empty batch: nothing enqueued
    ({"dtype": F32}, UNSUPPORTED),
    ({"dtype": 9}, INVALID),
    ({"Hq": 4000}, UNSUPPORTED),                 # not a whole number of 256-column tiles
    ({"Hv": 100}, UNSUPPORTED),
    ({"Hk": 0}, INVALID),
    ({"D": 0}, INVALID),
    ({"T": -1}, INVALID),
    ({"T": 1 << 31}, INVALID),
    ({"xs": 4000}, INVALID),                     # stride below D
    ({"qs": 12000}, INVALID),                    # stride below N
    ({"xs": 4100}, INVALID),                     # stride not a multiple of 8 elements (TMA rows)
    ({"x": 0x10008}, INVALID),                   # not 16-byte aligned
    ({"w": 0}, INVALID),
    ({"q_sums": 0}, INVALID),
    ({"q_sums": 0x20000002}, INVALID),           # sums not 4-byte aligned
    ({"qkv": 0x10000 + 2 * 4096 * 100}, INVALID),  # output overlaps x
    ({"k_sums": 0x20000000 + 4 * 4096 * 3}, INVALID),  # K sums overlap the Q sums
])
def test_projection_validation(lib, kw, want):
    assert _proj_call(lib, **kw) == want


def test_projection_pipeline_validation(lib):
    T, D, H = 4096, 4096, 4096
    need = lib.qknorm_qkv_projection_workspace_bytes(T, H, H)
    assert need == (H // 256 + H // 256) * T * 4  # the partial sums of Q, then of K
    assert lib.qknorm_qkv_projection_workspace_bytes(T, 100, H) == -1
    assert lib.qknorm_qkv_projection_workspace_bytes(-1, H, H) == -1

    def call(**kw):
        a = dict(gq=0x30000000, gk=0x30100000, eps=1e-6, ws=0x40000000, wsb=need)
        a.update(kw)
        return lib.qknorm_qkv_projection(0x10000, D, 0x2000000, D, 0x8000000, 3 * H, a["gq"], a["gk"], T, D, H, H,
                                         H, a["eps"], a["ws"], a["wsb"], BF16, None)
    assert call() == CUDA
    assert call(wsb=need - 4) == INVALID
    assert call(gq=0) == INVALID
    assert call(eps=-1.0) == INVALID
    assert call(eps=float("nan")) == INVALID
    assert call(ws=0x8000000 + 64) == INVALID        # workspace inside qkv
    assert call(gk=0x8000000) == INVALID             # gamma inside qkv
    assert lib.qknorm_device_timeouts(None) == INVALID


def _tp_call(lib, **kw):
    P = ctypes.c_void_p
    a = dict(R=4, first=0, n=4, T=128, hq=256, Hq=1024, hk=128, Hk=512, qs=256, ks=128, eps=1e-6, dtype=BF16,
             epoch=1, G=0, recv=[0x40000000 + r * 0x100000 for r in range(4)])
    a.update(kw)
    n = a["n"]
    base = lambda off: (P * max(n, 1))(*[0x10000000 + off + j * 0x1000000 for j in range(max(n, 1))])
    recv = (P * len(a["recv"]))(*a["recv"])
    return lib.qknorm_tp_layerwise(a["R"], a["first"], n, base(0), base(0x400000), base(0x800000), a["qs"], a["hq"],
                                   a["Hq"], base(0x900000), base(0xB00000), base(0xD00000), a["ks"], a["hk"], a["Hk"],
                                   a["T"], a["eps"], a["dtype"], recv, a["epoch"], a["G"], 0, None)


@pytest.mark.parametrize("kw,want", [
    ({}, CUDA),                                    # well formed: validation passes, the device query fails here
    ({"T": 0}, OK),
    ({"R": 0}, INVALID),
    ({"R": 9}, INVALID),
    ({"first": 2, "n": 3}, INVALID),               # ranks beyond R
    ({"epoch": 0}, INVALID),                       # reserved
    ({"G": -1}, INVALID),
    ({"dtype": 7}, INVALID),
    ({"eps": -1.0}, INVALID),
    ({"Hq": 100}, INVALID),                        # full width below the shard width
    ({"qs": 200}, INVALID),                        # stride below the shard width
    ({"hq": 252, "qs": 256}, UNSUPPORTED),         # shard width not whole 16-byte vectors
    ({"recv": [0x40000000, 0, 0x40200000, 0x40300000]}, INVALID),
    ({"recv": [0x40000004, 0x40100000, 0x40200000, 0x40300000]}, INVALID),  # not 16-byte aligned
    ({"recv": [0x40000000, 0x40100008, 0x40200000, 0x40300000]}, INVALID),
    ({"recv": [0x40000000, 0x40001000, 0x40200000, 0x40300000]}, INVALID),  # two receive buffers overlap
    ({"recv": [0x40000000, 0x40100000, 0x40200000, 0x11400000]}, INVALID),  # rank 3's buffer on rank 1's q_out
    ({"recv": [0x40000000, 0x40100000, 0x10000000, 0x40300000]}, INVALID),  # rank 2's buffer on rank 0's q_in
    ({"recv": [0x40000000, 0x40100000, 0x40200000, 0x10800000]}, INVALID),  # on rank 0's gamma_q slice
])
def test_tp_validation(lib, kw, want):
    assert _tp_call(lib, **kw) == want


def test_status_codes_in_the_header_are_the_contract():
    """The enumerators' values as include/qknorm.h spells them (0..4, with 2
    reserved for misaligned buffers, which the library never reports)."""
    import re
    text = open(os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "qknorm.h")).read()
    got = {m.group(1): int(m.group(2)) for m in re.finditer(r"\b(QKN_(?:OK|ERR_[A-Z_]+))\s*=\s*(\d+)", text)}
    assert got == {"QKN_OK": 0, "QKN_ERR_INVALID_ARG": 1, "QKN_ERR_MISALIGNED": 2, "QKN_ERR_UNSUPPORTED": 3,
                   "QKN_ERR_CUDA": 4}
    assert (_clib.QKN_OK, _clib.QKN_ERR_INVALID_ARG, _clib.QKN_ERR_MISALIGNED, _clib.QKN_ERR_UNSUPPORTED,
            _clib.QKN_ERR_CUDA) == (0, 1, 2, 3, 4)


def test_tp_recv_bytes(lib):
    assert lib.qknorm_tp_recv_bytes(4, 4096) == 4 * 4096 * 16 + 16  # exchange words, then the abort-word trailer
    assert lib.qknorm_tp_recv_bytes(0, 10) == -1 and lib.qknorm_tp_recv_bytes(9, 10) == -1


def test_tp_scope_validation(lib):
    """qknorm_tp_layerwise_scope: scope 0 or 1 pass validation (the device
    query then fails here), any other scope is refused."""
    P = ctypes.c_void_p
    n = 4
    base = lambda off: (P * n)(*[0x10000000 + off + j * 0x1000000 for j in range(n)])
    recv = (P * 4)(*[0x40000000 + r * 0x100000 for r in range(4)])

    def call(scope):
        return lib.qknorm_tp_layerwise_scope(4, 0, n, base(0), base(0x400000), base(0x800000), 256, 256, 1024,
                                             base(0x900000), base(0xB00000), base(0xD00000), 128, 128, 512, 128,
                                             1e-6, BF16, recv, 1, 0, 0, scope, None)
    assert call(0) == CUDA and call(1) == CUDA
    assert call(2) == INVALID and call(-1) == INVALID


# --------------------------------------------------------------------------- host-buffer entry point

HOST = 0x7F0000000000  # fake host addresses: validation never dereferences them


def _host_call(lib, **kw):
    a = dict(q_in=HOST, q_out=HOST + (1 << 30), k_in=HOST + (2 << 30), k_out=HOST + (3 << 30), gq=BASE,
             gk=BASE + 4096, qs=512, ks=256, T=1000, Hq=512, Hk=256, eps=1e-6, dtype=BF16, ring=BASE + (1 << 20),
             chunk=128, slots=2, ring_bytes=None)
    a.update(kw)
    rb = a["ring_bytes"]
    if rb is None:
        rb = lib.qknorm_layerwise_host_ring_bytes(a["chunk"], a["Hq"], a["Hk"], BF16, a["slots"])
    return lib.qknorm_layerwise_host(a["q_in"], a["q_out"], a["gq"], a["qs"], a["k_in"], a["k_out"], a["gk"], a["ks"],
                                     a["T"], a["Hq"], a["Hk"], a["eps"], a["dtype"], a["ring"], rb, a["chunk"], None,
                                     None, None)


@pytest.mark.parametrize("kw,want", [
    ({}, CUDA),                                        # well formed: validation passes, event creation fails here
    ({"T": 0}, OK),
    ({"T": -1}, INVALID),
    ({"chunk": 0}, INVALID),
    ({"ring": 0}, INVALID),
    ({"ring": BASE + (1 << 20) + 16}, INVALID),        # ring not 256-byte aligned
    ({"ring_bytes": 1000}, INVALID),                   # smaller than one slot
    ({"gq": BASE + (1 << 20) + 256}, INVALID),         # gamma inside the ring
    ({"q_out": HOST + 2}, INVALID),                    # partly overlaps q_in
    ({"q_out": HOST, "k_out": HOST + (2 << 30)}, CUDA),  # in place: allowed
    ({"k_out": HOST + 512}, INVALID),                  # k_out on q_in's rows (q_in rows are 1024 B)
    ({"qs": 500}, INVALID),                            # stride below width
    ({"eps": float("nan")}, INVALID),
    ({"dtype": 7}, INVALID),
    ({"gk": 0}, INVALID),
    # packed [Q | K | V] host rows in place: Q at the base, K at +Hq, shared stride 6144
    ({"q_in": HOST, "q_out": HOST, "k_in": HOST + 8192, "k_out": HOST + 8192, "Hq": 4096, "Hk": 1024, "qs": 6144,
      "ks": 6144}, CUDA),
])
def test_host_entry_point_validation(lib, kw, want):
    assert _host_call(lib, **kw) == want


def test_host_ring_bytes(lib):
    # two 256-byte aligned parts per slot
    assert lib.qknorm_layerwise_host_ring_bytes(512, 4096, 4096, BF16, 3) == 3 * 2 * 512 * 4096 * 2
    assert lib.qknorm_layerwise_host_ring_bytes(3, 8, 8, BF16, 1) == 256 + 256
    assert lib.qknorm_layerwise_host_ring_bytes(1, 4, 4, 3, 8) == 8 * 512  # E4M3
    assert lib.qknorm_layerwise_host_ring_bytes(0, 8, 8, BF16, 1) == -1
    assert lib.qknorm_layerwise_host_ring_bytes(8, 8, 8, BF16, 0) == -1
    assert lib.qknorm_layerwise_host_ring_bytes(8, 8, 8, BF16, 9) == -1
    assert lib.qknorm_layerwise_host_ring_bytes(8, 0, 8, BF16, 1) == -1
    assert lib.qknorm_layerwise_host_ring_bytes(8, 8, 8, 9, 1) == -1


# --------------------------------------------------------------------------- multi-shard calls

def _shards_call(lib, which, **kw):
    P_ = ctypes.c_void_p
    a = dict(P=4, T=256, hq=256, hk=128, qs=256, ks=128, eps=1e-6, dtype=BF16, Hq=1024, Hk=512,
             q_all=0x60000000, k_all=0x61000000, q_out=None, k_out=None)
    a.update(kw)
    n = max(a["P"], 1)
    arr = lambda base, step=0x100000: (P_ * n)(*[base + j * step for j in range(n)])
    q_in, k_in = arr(0x10000000), arr(0x20000000)
    if which == "stats":
        return lib.qknorm_partial_stats_shards(a["P"], q_in, a["qs"], a["hq"], a["q_all"], k_in, a["ks"], a["hk"],
                                               a["k_all"], a["T"], a["dtype"], None)
    q_out = a["q_out"] if a["q_out"] is not None else arr(0x30000000)
    k_out = arr(0x40000000)
    return lib.qknorm_combine_apply_shards(a["P"], q_in, q_out, arr(0x50000000, 0x1000), a["qs"], a["hq"], a["q_all"],
                                           a["Hq"], k_in, k_out, arr(0x50800000, 0x1000), a["ks"], a["hk"],
                                           a["k_all"], a["Hk"], a["T"], a["eps"], a["dtype"], None)


@pytest.mark.parametrize("which", ["stats", "apply"])
@pytest.mark.parametrize("kw,want", [
    ({}, CUDA),                                 # well formed: validation passes, the device query fails here
    ({"T": 0}, OK),
    ({"P": 0}, INVALID),
    ({"P": 9}, INVALID),
    ({"T": -1}, INVALID),
    ({"hq": 0}, INVALID),
    ({"qs": 100}, INVALID),                     # stride below the shard width
    ({"dtype": 7}, INVALID),
    ({"q_all": 0}, INVALID),
])
def test_multi_shard_validation(lib, which, kw, want):
    assert _shards_call(lib, which, **kw) == want


def test_multi_shard_stats_sums_must_not_overlap(lib):
    """The stats call writes the sums: they may not touch a shard or each
    other.  The apply call only reads them, beside inputs it only reads."""
    assert _shards_call(lib, "stats", q_all=0x10000000 + 512) == INVALID   # sums on shard 0's rows
    assert _shards_call(lib, "stats", k_all=0x60000000 + 8) == INVALID     # the two sum arrays overlap
    assert _shards_call(lib, "apply", q_all=0x10000000 + 512) == CUDA


def test_multi_shard_apply_outputs_checked_across_shards(lib):
    P_ = ctypes.c_void_p
    # shard 1's Q output lands on shard 0's Q input
    q_out = (P_ * 4)(0x30000000, 0x10000000, 0x30200000, 0x30300000)
    assert _shards_call(lib, "apply", q_out=q_out) == INVALID
    assert b"shard" in lib.qknorm_last_error()
    assert _shards_call(lib, "apply", Hq=100) == INVALID        # full width below the shard width
    assert _shards_call(lib, "apply", eps=-1.0) == INVALID


def test_multi_shard_launch_override_validation(lib):
    P_ = ctypes.c_void_p
    n = 4
    arr = lambda base, step=0x100000: (P_ * n)(*[base + j * step for j in range(n)])

    def stats(L):
        # Q shard rows of 1024 bf16 = 128 vectors
        return lib.qknorm_partial_stats_shards_launch(4, arr(0x10000000), 1024, 1024, 0x60000000, arr(0x20000000),
                                                      128, 128, 0x61000000, 256, BF16, None,
                                                      ctypes.byref(L) if L else None)
    assert stats(None) == INVALID                                                   # no launch given
    assert stats(_clib.QknLaunch(kernel=0, vec_per_thread=2, threads=100, grid=10)) == INVALID  # not a warp multiple
    assert stats(_clib.QknLaunch(kernel=0, vec_per_thread=2, threads=32, grid=10)) == INVALID   # row not covered
    assert stats(_clib.QknLaunch(kernel=1, vec_per_thread=0, threads=256, grid=10)) == INVALID  # not the register kernel
    assert stats(_clib.QknLaunch(kernel=0, vec_per_thread=2, threads=64, grid=10)) == CUDA      # valid: launch fails here


# --------------------------------------------------------------- GEMM schedule
L2_B200 = 126 * 1024 * 1024


def _group_rule(m_units: int, D: int, N: int, clusters: int, l2: int) -> int:
    """The raster group, restated: all token blocks when X fits in half of L2,
    one when W does, else the G minimising G + ceil(clusters / G)."""
    half = l2 / 2
    if m_units * 256 * D * 2 <= half:
        return m_units
    if N * D * 2 <= half:
        return 1
    return min(range(1, min(m_units, clusters) + 1), key=lambda g: (g + -(-clusters // g), g))


@pytest.mark.parametrize("T,D,Hq,Hk,Hv,clusters,group", [
    (4096, 4096, 4096, 1024, 1024, 74, 16),    # X 33.5 MB fits: one group of all 16 token blocks
    (4096, 4096, 4096, 4096, 4096, 74, 16),
    (16384, 4096, 4096, 1024, 1024, 74, 1),    # X 134 MB does not, W 50 MB does: one block per group
    (16384, 4096, 4096, 4096, 4096, 74, 7),    # neither: G + ceil(74 / G) smallest at 7 (7 + 11)
    (12000, 4096, 4096, 4096, 2048, 74, 7),
    (512, 256, 512, 512, 512, 74, 2),          # fewer units (12) than clusters
    (1, 64, 256, 256, 0, 74, 1),
])
def test_qkv_gemm_schedule(T, D, Hq, Hk, Hv, clusters, group):
    s = qk.qkv_gemm_schedule(T, D, Hq, Hk, Hv, clusters, L2_B200)
    m_units = -(-T // 256)
    N = Hq + Hk + Hv
    units = m_units * (N // 256)
    assert s["units"] == units and s["clusters"] == min(units, clusters)
    assert s["group_units"] == group == _group_rule(m_units, D, N, min(units, clusters), L2_B200)


@pytest.mark.parametrize("args,want", [
    ((0, 64, 256, 256, 0, 74, L2_B200), _clib.QKN_ERR_INVALID_ARG),
    ((1 << 31, 64, 256, 256, 0, 74, L2_B200), _clib.QKN_ERR_INVALID_ARG),
    ((16, 0, 256, 256, 0, 74, L2_B200), _clib.QKN_ERR_INVALID_ARG),
    ((16, 64, 0, 256, 0, 74, L2_B200), _clib.QKN_ERR_INVALID_ARG),
    ((16, 64, 256, 256, -256, 74, L2_B200), _clib.QKN_ERR_INVALID_ARG),
    ((16, 64, 128, 256, 0, 74, L2_B200), _clib.QKN_ERR_UNSUPPORTED),
    ((16, 64, 256, 256, 0, 0, L2_B200), _clib.QKN_ERR_INVALID_ARG),
    ((16, 64, 256, 256, 0, 74, -1), _clib.QKN_ERR_INVALID_ARG),
])
def test_qkv_gemm_schedule_validation(lib, args, want):
    S = _clib.QknGemmSchedule()
    assert lib.qknorm_qkv_gemm_schedule(*args, ctypes.byref(S)) == want
    assert lib.qknorm_qkv_gemm_schedule(16, 64, 256, 256, 0, 74, L2_B200, None) == _clib.QKN_ERR_INVALID_ARG


def test_noalloc_scratch_limit_on_the_host(lib):
    """The allocation-free projection's scratch holds the partial sums of
    T = 32768 tokens at Hq = Hk = 4096 (the header's example) and refuses one
    token more before touching the device."""
    cap = lib.qknorm_qkv_projection_noalloc_max_bytes()
    assert cap == 4 << 20
    assert lib.qknorm_qkv_projection_workspace_bytes(32768, 4096, 4096) == cap
    assert lib.qknorm_qkv_projection_workspace_bytes(32769, 4096, 4096) > cap
    st = lib.qknorm_qkv_projection_noalloc(0x10000, 64, 0x20000000, 64, 0x40000000, 8192, 0x60000000, 0x60010000,
                                           32769, 64, 4096, 4096, 0, 1e-6, _clib.QKN_BF16, None)
    assert st == _clib.QKN_ERR_INVALID_ARG
    assert b"scratch" in lib.qknorm_last_error()
