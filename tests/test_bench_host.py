"""Host-side pieces of the benchmark, on CPU: which committed profile a bench
line takes its DRAM traffic from, how many buffer sets keep L2 cold, the
whole-job throughput, and the peak the roofline divides by."""
from __future__ import annotations

import json
import os

import pytest

import bench

PROFILE = """# ncu summary: a test kernel

workload: {workload}
kernel: test
source_digest: {digest}
dram_bytes_per_launch: {bytes}
{launch}
"""


@pytest.fixture
def fake_root(tmp_path, monkeypatch):
    (tmp_path / "profiles").mkdir()
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    return tmp_path


def _profile(root, name, workload, digest, nbytes, launch=None):
    text = PROFILE.format(workload=workload, digest=digest, bytes=nbytes,
                          launch=f"launch: {launch}" if launch else "")
    (root / "profiles" / name).write_text(text)


def test_traffic_only_from_a_profile_of_the_same_workload_sources_and_launch(fake_root):
    launch = "kernel=0 vec_per_thread=4 threads=128 grid=1184"
    _profile(fake_root, "a.md", "prefill_x", "d1", 111, launch)
    _profile(fake_root, "b.md", "packed_y", "d1", 222)
    assert bench.profiled_traffic("prefill_x", "d1", launch) == 111
    assert bench.profiled_traffic("prefill_x", "d2", launch) is None          # the kernel changed since
    assert bench.profiled_traffic("prefill_x", "d1", "kernel=0 vec_per_thread=2 threads=128 grid=1332") is None
    assert bench.profiled_traffic("prefill_x", "d1", None) == 111             # no plan to compare
    assert bench.profiled_traffic("packed_y", "d1", launch) == 222            # the summary names no launch
    assert bench.profiled_traffic("other", "d1", launch) is None


def test_committed_profiles_name_a_known_kernel_family_and_parse():
    """Every committed summary that carries counters names its workload,
    digest and bytes in the form the bench reads."""
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    seen = 0
    for name in sorted(os.listdir(os.path.join(root, "profiles"))):
        text = open(os.path.join(root, "profiles", name)).read()
        if "source_digest:" not in text:
            continue
        seen += 1
        fields = dict(line.split(":", 1) for line in text.splitlines()
                      if line.split(":", 1)[0] in ("workload", "source_digest", "dram_bytes_per_launch"))
        assert set(fields) == {"workload", "source_digest", "dram_bytes_per_launch"}, name
        assert int(fields["dram_bytes_per_launch"]) > 0, name
        assert len(fields["source_digest"].strip()) == 16, name
    assert seen >= 5


def test_digest_follows_the_kernel_sources(fake_root):
    csrc = fake_root / "attention_normalization_b200" / "csrc"
    csrc.mkdir(parents=True)
    for f in ("qknorm_kernels.cuh", "qknorm_tp.cu", "qknorm_tp.cuh", "qkv_gemm.cu", "qkv_gemm.cuh"):
        (csrc / f).write_text(f"// {f}\n")
    rows, tp = bench.source_digest("rows"), bench.source_digest("tp")
    (csrc / "qknorm_tp.cu").write_text("// changed\n")
    assert bench.source_digest("rows") == rows      # the rows kernel did not change
    assert bench.source_digest("tp") != tp          # the TP kernel did


@pytest.mark.parametrize("set_bytes,l2,want", [
    (134_234_112, 132_120_576, 3),    # prefill: 2 other sets (268 MB) > 2 x L2
    (402_653_184, 132_120_576, 2),    # one other set already exceeds 2 x L2
    (61_440, 132_120_576, bench.MAX_SETS),  # decode T=1: capped
])
def test_rotation_keeps_more_than_twice_l2_between_reuses(set_bytes, l2, want):
    n = bench.rotation_count(set_bytes, l2)
    assert n == want
    if n < bench.MAX_SETS:
        assert (n - 1) * set_bytes > 2 * l2


def test_whole_job_counts_every_rank_at_the_slowest_rank_time():
    r = bench.whole_job(134_234_112, 100, 2.5, 4)   # 100 steps in 2.5 ms on the slowest of 4 ranks
    assert r["ms_per_step"] == pytest.approx(0.025)
    assert r["per_rank_gbs"] == pytest.approx(134_234_112 / 25e-6 / 1e9)
    assert r["value_gbs"] == pytest.approx(4 * r["per_rank_gbs"])


def test_peak_from_the_measured_file_else_the_fallback(fake_root):
    assert bench.load_peaks() == {"hbm_gbs": bench.FALLBACK_HBM_GBS, "source": "fallback"}
    (fake_root / "MEASURED_PEAKS.json").write_text(json.dumps({"hbm_gbs": 6550.1}))
    assert bench.load_peaks() == {"hbm_gbs": 6550.1, "source": "measured"}


def test_launch_text_matches_the_summaries_form():
    assert bench.launch_text({"kernel": 0, "vec_per_thread": 4, "threads": 128, "grid": 1184}) == \
        "kernel=0 vec_per_thread=4 threads=128 grid=1184"
    assert bench.launch_text(None) is None


@pytest.mark.parametrize("kind,tokens", [("prefill", None), ("tiny", None), ("decode", 8), ("packed", 1024),
                                         ("gqa", None), ("headwise", 256), ("tp", None)])
def test_roofline_record_for_every_workload(kind, tokens, fake_root):
    """The roofline object of each workload's line builds on the host (no GPU):
    achieved = effective bytes / the dominant kernel's time, frac against the
    peak; the GQA line adds the decomposed form's double-read floor."""
    wl = bench.Workload(kind, tokens, seed_offset=0)
    peaks = {"hbm_gbs": 6000.0, "source": "test"}
    step_s = 1e-3
    r = bench.roofline_record(wl, step_s, peaks, "d0", None)
    kernel_s = step_s if kind == "gqa" else step_s / wl.launches_per_step
    assert r["achieved"] == pytest.approx(wl.eff_bytes / kernel_s / 1e9, abs=0.05)  # GB/s to one place
    assert r["frac"] == pytest.approx(r["achieved"] / 6000.0, abs=1e-4)  # frac is rounded to 4 places
    assert r["bound"] == "hbm" and r["traffic"] is None
    if kind == "gqa":
        assert "partial_stats_shards" in r["kernel"] and wl.launches_per_step == 2
        assert r["floor_bytes_per_step"] > 1.49 * wl.eff_bytes
    else:
        assert "floor_bytes_per_step" not in r


@pytest.mark.parametrize("kind", ["tiny", "decode"])
def test_reference_arm_line_on_the_host(kind, capsys):
    """The reference arm (the oracle on the host cores) prints one JSON line
    with the contract's keys and the native arm's config, so the two lines
    name the same workload."""
    rc = bench.main(["--impl", "reference", "--workload", kind, "--steps", "1", "--warmup", "3"])
    assert rc == 0
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better", "scaling",
                "vs_baseline", "dtype", "data", "config", "impl", "cpu_baseline", "e2e"):
        assert key in line, key
    assert line["impl"] == "reference" and line["value"] > 0
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["d2h_bytes_per_step"] == 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["value"] == line["value"]
    want = bench.Workload(kind, None, seed_offset=0).config()
    want["parallelism"] = bench.parallelism(1)
    assert line["config"] == want
