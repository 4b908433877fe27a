#!/usr/bin/env python
"""Benchmark of fused layerwise QK-RMSNorm on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl native|reference]
                    [--workload prefill|decode|packed|gqa|tiny|headwise|projection] [--tokens T]

Prints ONE JSON line (rank 0).  A step is one pass of the whole path over one
batch of synthetic input: for the default workload, one ``qknorm_layerwise``
call normalizing the Q and K rows of a T=4096, Hq=Hk=4096 bf16 prefill batch
(OLMo2-7B-shaped).  ``value`` is effective GB/s: the bytes the call must move
(read + write of every Q and K element, plus gamma) divided by the time.

Timing: W untimed warm-up steps, then exactly K steps captured in one CUDA
graph (the C-ABI calls, replayed without host overhead) and timed with CUDA
events on the launching stream, between a barrier and a device synchronize on
both sides; the maximum over ranks is reported.  Consecutive steps rotate over
several input/output sets whose total exceeds twice the L2 size, so no step
finds its inputs in L2.  Under torchrun each rank normalizes its own batch
(tokens are independent: no collective on the data path; weak scaling).

``e2e`` times the same call through the public Python API with pinned host
buffers: each step copies its inputs host->device, normalizes, and copies the
outputs back.  ``cpu_baseline`` times the CPU oracle (double precision, one
thread) on the same workload on this host.  ``--impl reference`` times that
oracle alone, as the reference arm.
"""
from __future__ import annotations

import argparse
import datetime
import glob
import hashlib
import json
import math
import os
import re
import statistics
import sys
import threading
import time

import torch

import workloads

ROOT = os.path.dirname(os.path.abspath(__file__))
METRIC = "fused QK-RMSNorm effective HBM GB/s (% of B200 peak); µs per call"
UNIT = "GB/s"
FALLBACK_HBM_GBS = 6650.0  # used only when the measured peaks file is absent


# --------------------------------------------------------------------------- plumbing

def parse_args(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["native", "reference"], default="native")
    ap.add_argument("--workload", choices=["prefill", "decode", "packed", "gqa", "tiny", "headwise", "projection", "tp"],
                    default="prefill")
    ap.add_argument("--ranks", type=int, default=4, help="tensor-parallel ranks of the tp workload")
    ap.add_argument("--gqa-form", choices=["multi", "per-shard"], default="multi",
                    help="gqa workload: the two multi-shard calls (2 launches) or P calls of each phase (2P)")
    ap.add_argument("--proj", default="4096,4096,4096,4096",
                    help="D,Hq,Hk,Hv of the projection workload (T from --tokens, default 4096)")
    ap.add_argument("--tokens", type=int, default=None, help="T for decode / packed workloads")
    ap.add_argument("--dtype", choices=["bf16", "f16", "e4m3"], default="bf16",
                    help="element type of the prefill workload (gamma is bf16 with e4m3)")
    ap.add_argument("--e2e-steps", type=int, default=50)
    ap.add_argument("--e2e-chunk", type=int, default=512, help="tokens per chunk of the host-buffer pipeline")
    ap.add_argument("--e2e-slots", type=int, default=3, help="device ring slots of the host-buffer pipeline")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=10.0, help="CPU baseline budget")
    a = ap.parse_args(argv)
    if a.warmup < 3:
        ap.error("--warmup must be >= 3")
    if a.steps < 1:
        ap.error("--steps must be >= 1")
    return a


def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


class Ranks:
    """Barrier and max-over-ranks for the timing plumbing (no data-path
    collective).  ``dist`` is torch.distributed or None (one process); NCCL
    needs a CUDA ``device`` for its tensors, gloo takes the CPU."""

    def __init__(self, dist=None, device=None):
        self.dist = dist
        self.device = device if device is not None else torch.device("cpu")

    @property
    def world(self) -> int:
        return self.dist.get_world_size() if self.dist is not None else 1

    def barrier(self):
        if self.dist is not None:
            self.dist.barrier()

    def max(self, x: float) -> float:
        if self.dist is None:
            return x
        t = torch.tensor([x], dtype=torch.float64, device=self.device)
        self.dist.all_reduce(t, op=self.dist.ReduceOp.MAX)
        return float(t.item())


def parallelism(world: int) -> str:
    return f"replicas x{world} (tokens independent, no collective)"


def whole_job(eff_bytes_per_step: int, steps: int, max_ms: float, world: int) -> dict:
    """Whole-job throughput: every rank processed `steps` steps of
    `eff_bytes_per_step`; the job took the slowest rank's time."""
    step_s = max_ms / 1e3 / steps
    return {"value_gbs": world * eff_bytes_per_step / step_s / 1e9, "ms_per_step": max_ms / steps,
            "per_rank_gbs": eff_bytes_per_step / step_s / 1e9}


def load_peaks() -> dict:
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return {"hbm_gbs": float(d["hbm_gbs"]), "source": "measured"}
    except (OSError, KeyError, ValueError):
        return {"hbm_gbs": FALLBACK_HBM_GBS, "source": "fallback"}


KERNEL_SOURCES = {
    "rows": ["qknorm_kernels.cuh"],
    "projection": ["qkv_gemm.cu", "qkv_gemm.cuh"],
    "tp": ["qknorm_tp.cu", "qknorm_tp.cuh", "qknorm_kernels.cuh"],
}


def source_digest(kind: str = "rows") -> str:
    """Digest of one kernel family's device sources: profile counters apply
    only to the kernel they were taken from (the launch shape is checked
    separately, see profiled_traffic)."""
    h = hashlib.sha256()
    files = sorted(os.path.join(ROOT, "attention_normalization_b200", "csrc", f) for f in KERNEL_SOURCES[kind])
    for p in files:
        h.update(os.path.basename(p).encode())
        with open(p, "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def profiled_traffic(workload: str, digest: str, launch: str | None = None):
    """DRAM bytes per launch from a committed ncu summary for this workload, if
    it was taken from the current kernel sources (and, when the summary names
    one, the same launch shape); else None."""
    for p in sorted(glob.glob(os.path.join(ROOT, "profiles", "*.md"))):
        text = open(p).read()
        m_w = re.search(r"^workload:\s*(\S+)", text, re.M)
        m_d = re.search(r"^source_digest:\s*(\S+)", text, re.M)
        m_t = re.search(r"^dram_bytes_per_launch:\s*(\d+)", text, re.M)
        m_l = re.search(r"^launch:\s*(.+)$", text, re.M)
        if not (m_w and m_d and m_t) or m_w.group(1) != workload or m_d.group(1) != digest:
            continue
        if m_l and launch is not None and m_l.group(1).strip() != launch:
            continue
        return int(m_t.group(1))
    return None


def launch_text(plan) -> str | None:
    """A launch plan as the profile summaries record it."""
    if not plan:
        return None
    return "kernel={kernel} vec_per_thread={vec_per_thread} threads={threads} grid={grid}".format(**plan)


class ClockSampler:
    """Samples SM clock and throttle reasons through NVML (read-only) while
    ``active`` is set."""
    REASONS = [(0x4, "sw_power_cap"), (0x8, "hw_slowdown"), (0x20, "sw_thermal_slowdown"),
               (0x40, "hw_thermal_slowdown"), (0x80, "hw_power_brake_slowdown"),
               (0x2, "applications_clocks_setting"), (0x10, "sync_boost")]

    def __init__(self, cuda_index: int, period_s: float = 0.005):
        self.period = period_s
        self.samples = []
        self.error = None
        self.active = threading.Event()
        self.stop_ev = threading.Event()
        self.handle = None
        self.max_mhz = None
        try:
            import pynvml
            self.nv = pynvml
            pynvml.nvmlInit()
            self.handle = self._handle(cuda_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.handle, pynvml.NVML_CLOCK_SM)
        except Exception as e:  # NVML missing: report, do not fail the run
            self.error = f"{type(e).__name__}: {e}"
        self.thread = threading.Thread(target=self._run, daemon=True)

    def _handle(self, cuda_index):
        nv = self.nv
        props = torch.cuda.get_device_properties(cuda_index)
        try:
            bus = "%08X:%02X:%02X.0" % (props.pci_domain_id, props.pci_bus_id, props.pci_device_id)
            return nv.nvmlDeviceGetHandleByPciBusId(bus)
        except Exception:
            pass
        vis = os.environ.get("CUDA_VISIBLE_DEVICES")
        idx = int(vis.split(",")[cuda_index]) if vis and vis.split(",")[0].isdigit() else cuda_index
        return nv.nvmlDeviceGetHandleByIndex(idx)

    def _reasons(self):
        nv = self.nv
        for fn in ("nvmlDeviceGetCurrentClocksEventReasons", "nvmlDeviceGetCurrentClocksThrottleReasons"):
            if hasattr(nv, fn):
                return getattr(nv, fn)(self.handle)
        return 0

    def sample_now(self):
        """One sample, taken on the calling thread (read-only NVML queries)."""
        if self.handle is None:
            return
        try:
            mhz = self.nv.nvmlDeviceGetClockInfo(self.handle, self.nv.NVML_CLOCK_SM)
            self.samples.append((mhz, int(self._reasons())))
        except Exception as e:
            self.error = f"{type(e).__name__}: {e}"

    def _run(self):
        while not self.stop_ev.is_set():
            if self.active.is_set():
                self.sample_now()
            time.sleep(self.period)

    def start(self):
        self.thread.start()

    def summary(self) -> dict:
        self.stop_ev.set()
        self.thread.join(timeout=2)
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0,
                    **({"error": self.error} if self.error else {})}
        mask = 0
        for _, r in self.samples:
            mask |= r
        return {"sm_mhz": statistics.median(m for m, _ in self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": [n for bit, n in self.REASONS if mask & bit], "samples": len(self.samples)}


# --------------------------------------------------------------------------- workloads

class Workload:
    """A benchmark workload: CPU batch, effective bytes per step, and a step
    function over a device-resident set."""

    DTYPES = {"bf16": torch.bfloat16, "f16": torch.float16, "e4m3": torch.float8_e4m3fn}

    def __init__(self, kind: str, tokens: int | None, seed_offset: int, dtype: str = "bf16", ranks: int = 4,
                 gqa_form: str = "multi"):
        self.kind = kind
        self.gqa_form = gqa_form
        if kind == "prefill":
            self.batch = workloads.prefill_bf16(seed=1 + seed_offset, dtype=self.DTYPES[dtype])
        elif kind == "tiny":
            self.batch = workloads.tiny_fp32(seed=0 + seed_offset)
        elif kind == "decode":
            self.batch = workloads.decode_bf16(tokens or 1, seed=2 + seed_offset)
        elif kind == "packed":
            self.batch = workloads.packed_qkv(tokens or 16384, seed=4 + seed_offset)
        elif kind == "gqa":
            self.batch = workloads.gqa_sharded(seed=3 + seed_offset)
        elif kind == "headwise":
            self.batch = workloads.headwise_bf16(seed=5 + seed_offset, T=tokens or 4096)
        elif kind == "tp":
            self.batch = workloads.prefill_bf16(seed=1 + seed_offset)
        self.ranks = ranks
        b = self.batch
        self.esz = {torch.float32: 4, torch.float8_e4m3fn: 1}.get(b.dtype, 2)
        gesz = 4 if b.dtype == torch.float32 else 2
        # bytes the method must move per step: read + write of every Q and K element, plus gamma
        gamma_elems = 2 * b.meta["head_dim"] if kind == "headwise" else b.Hq + b.Hk
        self.eff_bytes = 2 * self.esz * (b.Hq + b.Hk) * b.T + gesz * gamma_elems
        self.name = f"tp_R{ranks}_{b.name}" if kind == "tp" else b.name
        self.launches_per_step = (2 * b.P if gqa_form == "per-shard" else 2) if kind == "gqa" else 1

    def config(self) -> dict:
        b = self.batch
        c = {"workload": self.name, "T": b.T, "Hq": b.Hq, "Hk": b.Hk, "io_dtype": str(b.dtype).replace("torch.", ""),
             "eps": b.eps}
        if self.kind == "packed":
            c.update({"Hv": b.Hv, "row_stride": b.packed.shape[1], "in_place": True})
        if self.kind == "gqa":
            c.update({"P": b.P, "form": "partial_stats x P -> combine_apply x P" if self.gqa_form == "per-shard" else
                      "partial_stats_shards (P shards, one launch) -> combine_apply_shards (P shards, one launch)"})
        if self.kind == "headwise":
            c.update({"head_dim": b.meta["head_dim"], "q_heads": b.meta["q_heads"], "k_heads": b.meta["k_heads"],
                      "form": "qknorm_headwise (one factor per head)"})
        if self.kind == "tp":
            c.update({"R": self.ranks, "form": f"qknorm_tp_layerwise: {self.ranks} tensor-parallel ranks, each with "
                                               "1/R of every Q and K row, exchanging scalar partial sums; all ranks "
                                               "in one cooperative launch on one GPU"})
        return c

    # one device-resident set of buffers
    def make_set(self, dev):
        b = self.batch
        if self.kind == "packed":
            base = b.packed.to(dev)
            return {"base": base, "q": base[:, :b.Hq], "k": base[:, b.Hq:b.Hq + b.Hk],
                    "gq": b.gamma_q.to(dev), "gk": b.gamma_k.to(dev)}
        if self.kind == "gqa":
            P = b.P
            wq, wk = b.Hq // P, b.Hk // P
            gq, gk = b.gamma_q.to(dev), b.gamma_k.to(dev)
            return {"qs": [s.to(dev) for s in b.q_shards], "ks": [s.to(dev) for s in b.k_shards],
                    "qo": [torch.empty_like(s, device=dev) for s in b.q_shards],
                    "ko": [torch.empty_like(s, device=dev) for s in b.k_shards],
                    "gqs": [gq[p * wq:(p + 1) * wq].contiguous() for p in range(P)],
                    "gks": [gk[p * wk:(p + 1) * wk].contiguous() for p in range(P)],
                    "q_all": torch.empty((P, b.T), dtype=torch.float32, device=dev),
                    "k_all": torch.empty((P, b.T), dtype=torch.float32, device=dev)}
        if self.kind == "tp":
            import attention_normalization_b200 as qk
            R = self.ranks
            wq, wk = b.Hq // R, b.Hk // R
            qs = [b.q[:, r * wq:(r + 1) * wq].contiguous().to(dev) for r in range(R)]
            ks = [b.k[:, r * wk:(r + 1) * wk].contiguous().to(dev) for r in range(R)]
            return {"qs": qs, "ks": ks, "qo": [torch.empty_like(t) for t in qs], "ko": [torch.empty_like(t) for t in ks],
                    "gqs": [b.gamma_q[r * wq:(r + 1) * wq].contiguous().to(dev) for r in range(R)],
                    "gks": [b.gamma_k[r * wk:(r + 1) * wk].contiguous().to(dev) for r in range(R)],
                    "ex": qk.TpExchange(R, b.T, dev)}
        q, k = b.q.to(dev), b.k.to(dev)
        return {"q": q, "k": k, "qo": torch.empty_like(q), "ko": torch.empty_like(k),
                "gq": b.gamma_q.to(dev), "gk": b.gamma_k.to(dev)}

    def set_bytes(self) -> int:
        b = self.batch
        if self.kind == "packed":
            return b.packed.numel() * self.esz
        return 2 * self.esz * (b.Hq + b.Hk) * b.T

    def step(self, qk, s):
        b = self.batch
        if self.kind == "packed":
            qk.qknorm_layerwise(s["q"], s["k"], s["gq"], s["gk"], b.eps, q_out=s["q"], k_out=s["k"])
        elif self.kind == "gqa" and self.gqa_form == "per-shard":
            for p in range(b.P):
                qk.qknorm_partial_stats(s["qs"][p], s["ks"][p], s["q_all"][p], s["k_all"][p])
            for p in range(b.P):
                qk.qknorm_combine_apply(s["qs"][p], s["ks"][p], s["gqs"][p], s["gks"][p], s["q_all"], s["k_all"],
                                        b.Hq, b.Hk, b.eps, q_out=s["qo"][p], k_out=s["ko"][p])
        elif self.kind == "gqa":
            qk.qknorm_partial_stats_shards(s["qs"], s["ks"], s["q_all"], s["k_all"])
            qk.qknorm_combine_apply_shards(s["qs"], s["ks"], s["gqs"], s["gks"], s["q_all"], s["k_all"], b.Hq, b.Hk,
                                           b.eps, q_out=s["qo"], k_out=s["ko"])
        elif self.kind == "headwise":
            qk.qknorm_headwise(s["q"], s["k"], s["gq"], s["gk"], b.meta["head_dim"], b.eps,
                               q_out=s["qo"], k_out=s["ko"])
        elif self.kind == "tp":
            # each call takes the exchange's next epoch: a captured graph is replayed once
            qk.qknorm_tp_layerwise(s["qs"], s["ks"], s["gqs"], s["gks"], b.Hq, b.Hk, b.eps, exchange=s["ex"],
                                   q_out=s["qo"], k_out=s["ko"])
        else:
            qk.qknorm_layerwise(s["q"], s["k"], s["gq"], s["gk"], b.eps, q_out=s["qo"], k_out=s["ko"])


def roofline_record(wl: Workload, step_s: float, peaks: dict, digest: str, plan) -> dict:
    """The line's roofline object: the step's effective bytes over the time of
    the kernel that dominates it (the only kernel of the step, or -- for the
    shard-decomposed GQA step -- the whole step), against the measured peak."""
    kernel_s = step_s / wl.launches_per_step if wl.kind != "gqa" else step_s
    if wl.kind == "gqa":
        kernel = "whole step: " + wl.config()["form"]
    elif wl.kind == "tp":
        kernel = "tp_warp_kernel (one token per warp), all ranks in one launch (the only kernel of the step)"
    else:
        kernel = "qknorm rows kernel (the only kernel of the step)"
    r = {"bound": "hbm", "achieved": round(wl.eff_bytes / kernel_s / 1e9, 1), "peak": peaks["hbm_gbs"],
         "unit": "GB/s", "frac": round(wl.eff_bytes / kernel_s / 1e9 / peaks["hbm_gbs"], 4),
         "traffic": profiled_traffic(wl.name, digest, launch_text(plan)),
         "peak_source": f"{peaks['source']} copy bandwidth", "kernel": kernel,
         "algorithmic_bytes_per_launch": wl.eff_bytes if wl.kind != "gqa" else None,
         "source_digest": digest}
    if wl.kind == "gqa":
        # the decomposed form must read every shard twice (partial sums, then
        # apply): its floor is 2 reads + 1 write of Q and K, gamma, and the
        # [P][T] sums written once and read once
        b = wl.batch
        floor = 3 * wl.esz * (b.Hq + b.Hk) * b.T + 2 * (b.Hq + b.Hk) + 2 * 2 * b.P * b.T * 4
        r.update({"floor_bytes_per_step": floor, "floor_achieved": round(floor / step_s / 1e9, 1),
                  "floor_frac": round(floor / step_s / 1e9 / peaks["hbm_gbs"], 4)})
    return r


def graph_upload(graph: "torch.cuda.CUDAGraph", stream) -> bool:
    """Upload an instantiated CUDA graph to the device ahead of its first
    replay (cudaGraphUpload), so a timed replay does not pay the one-time
    upload.  Executes none of the graph's work.  False if unavailable."""
    import ctypes
    try:
        rt = ctypes.CDLL("libcudart.so.12")  # the runtime torch has loaded
        rt.cudaGraphUpload.argtypes = [ctypes.c_void_p, ctypes.c_void_p]
        rt.cudaGraphUpload.restype = ctypes.c_int
        return rt.cudaGraphUpload(ctypes.c_void_p(graph.raw_cuda_graph_exec()),
                                  ctypes.c_void_p(stream.cuda_stream)) == 0
    except (OSError, AttributeError, RuntimeError):
        return False


HOLD_CYCLES = 200_000  # ~100 us at 1.9 GHz


def hold_queue(stream) -> None:
    """Queue a short device spin (torch's sleep kernel, ~100 us) on `stream`
    before a timed region's start event, so that the start event and the
    graph the host submits next are already queued when the GPU reaches
    them: the timed region then holds the K steps' device time, not the
    host's graph submission.  The spin itself ends before the start event."""
    with torch.cuda.stream(stream):
        torch.cuda._sleep(HOLD_CYCLES)


MAX_SETS = 64


def rotation_count(set_bytes: int, l2_bytes: int) -> int:
    """Sets to rotate over so that the other sets touched between two uses of
    one set exceed twice the L2 size (at most MAX_SETS: a small, latency-bound
    workload then runs partly from L2, as it would right after its producer)."""
    return min(MAX_SETS, max(2, math.ceil(2 * l2_bytes / max(1, set_bytes)) + 1))


# --------------------------------------------------------------------------- CPU baseline (the oracle)

def cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def time_oracle_parallel(wl: Workload, budget_s: float) -> dict:
    """The same oracle calls split over the host's cores: one thread per core,
    each normalizing a contiguous block of tokens (the C oracle runs outside
    the Python lock).  Whole calls until the budget is spent."""
    import concurrent.futures

    import numpy as np

    import oracle
    b = wl.batch
    cores = len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else (os.cpu_count() or 1)

    def bits(view):
        t = view.contiguous()
        if t.dtype == torch.bfloat16:
            return t.view(torch.int16).numpy().view(np.uint16)
        if t.dtype == torch.float8_e4m3fn:
            return t.view(torch.uint8).numpy()
        return t.numpy()
    q, k = bits(b.q), bits(b.k)
    gq, gk = bits(b.gamma_q[None, :]).ravel(), bits(b.gamma_k[None, :]).ravel()
    edges = np.linspace(0, b.T, min(cores, b.T) + 1).astype(int)
    blocks = [(lo, hi) for lo, hi in zip(edges[:-1], edges[1:]) if hi > lo]

    def part(lo_hi):
        lo, hi = lo_hi
        oracle.qknorm_layerwise(np.ascontiguousarray(q[lo:hi]), b.Hq, gq, b.Hq, np.ascontiguousarray(k[lo:hi]), b.Hk,
                                gk, b.Hk, hi - lo, b.eps)
    with concurrent.futures.ThreadPoolExecutor(max_workers=len(blocks)) as ex:
        calls, t0 = 0, time.perf_counter()
        while True:
            list(ex.map(part, blocks))
            calls += 1
            el = time.perf_counter() - t0
            if el >= budget_s or calls >= 1000:
                break
    per_call = el / calls
    return {"value": wl.eff_bytes / per_call / 1e9, "unit": UNIT, "cores": len(blocks), "cpu": cpu_model(),
            "sample": f"{calls} whole oracle call(s) of {wl.name} over {len(blocks)} threads, {el:.1f} s",
            "us_per_call": per_call * 1e6}


def time_oracle(wl: Workload, budget_s: float, max_tokens: int | None = None) -> dict:
    """Times the CPU oracle (double precision, one thread) on the workload's
    own inputs: whole calls until the budget is spent, or, with max_tokens, a
    prefix of that many tokens per call."""
    import numpy as np

    import oracle

    b = wl.batch
    T = b.T if max_tokens is None else max(1, min(b.T, max_tokens))

    def np_rows(view):
        view = view[:T]
        t = view.contiguous()
        if t.dtype == torch.bfloat16:
            a = t.view(torch.int16).numpy().view(np.uint16)
        elif t.dtype == torch.float8_e4m3fn:
            a = t.view(torch.uint8).numpy()
        else:
            a = t.numpy()
        return a, view.shape[1]

    if wl.kind == "gqa":
        qf, _ = np_rows(b.q_full)
        kf, _ = np_rows(b.k_full)
    else:
        qf, _ = np_rows(b.q)
        kf, _ = np_rows(b.k)
    gq = np_rows(b.gamma_q[None, :])[0].ravel()
    gk = np_rows(b.gamma_k[None, :])[0].ravel()

    def one_call():
        if wl.kind == "headwise":
            hd = b.meta["head_dim"]
            oracle.rmsnorm_heads(qf, b.Hq // hd, hd, gq, b.eps, stride=b.Hq, T=T)
            oracle.rmsnorm_heads(kf, b.Hk // hd, hd, gk, b.eps, stride=b.Hk, T=T)
        elif wl.kind == "gqa":
            P = b.P
            wq, wk = b.Hq // P, b.Hk // P
            sq = np.stack([oracle.partial_sumsq(np.ascontiguousarray(qf[:, p * wq:(p + 1) * wq]), wq, wq, T)
                           for p in range(P)])
            sk = np.stack([oracle.partial_sumsq(np.ascontiguousarray(kf[:, p * wk:(p + 1) * wk]), wk, wk, T)
                           for p in range(P)])
            for p in range(P):
                oracle.combine_apply(np.ascontiguousarray(qf[:, p * wq:(p + 1) * wq]), wq, wq, T,
                                     gq[p * wq:(p + 1) * wq], sq, b.Hq, b.eps)
                oracle.combine_apply(np.ascontiguousarray(kf[:, p * wk:(p + 1) * wk]), wk, wk, T,
                                     gk[p * wk:(p + 1) * wk], sk, b.Hk, b.eps)
        else:
            oracle.qknorm_layerwise(qf, b.Hq, gq, b.Hq, kf, b.Hk, gk, b.Hk, T, b.eps)

    calls, t0 = 0, time.perf_counter()
    while True:
        one_call()
        calls += 1
        el = time.perf_counter() - t0
        if el >= budget_s or calls >= 1000:
            break
    per_call = el / calls
    eff = wl.eff_bytes * T / b.T
    return {"value": eff / per_call / 1e9, "unit": UNIT, "cores": 1, "kind": "oracle",
            "sample": f"{calls} oracle call(s) on {T} of {b.T} tokens of {wl.name}, {el:.1f} s",
            "us_per_call": per_call * 1e6, "tokens": T, "calls": calls}


# --------------------------------------------------------------------------- native arm

def native(args) -> int:
    rank, world, local = dist_env()
    if world != args.gpus and rank == 0:
        print(f"warning: --gpus {args.gpus} but WORLD_SIZE={world}", file=sys.stderr)
    if not torch.cuda.is_available():
        print(json.dumps({"metric": METRIC, "error": "no CUDA device"}))
        return 1
    torch.cuda.set_device(local)
    dev = torch.device(f"cuda:{local}")
    dist = None
    if world > 1:
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=180), device_id=dev)

    import attention_normalization_b200 as qk
    qk.capi()  # fails loudly if the library is missing

    ranks = Ranks(dist, dev)
    barrier, max_over_ranks = ranks.barrier, ranks.max

    wl = Workload(args.workload, args.tokens, seed_offset=rank * 1000, dtype=args.dtype, ranks=args.ranks,
                  gqa_form=args.gqa_form)
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    R = rotating = rotation_count(wl.set_bytes(), l2)
    sets = [wl.make_set(dev) for _ in range(R)]
    torch.cuda.synchronize()

    # eager warm-up (loads the library's per-device caches), then capture
    for i in range(3):
        wl.step(qk, sets[i % R])
    torch.cuda.synchronize()
    g_warm, g_timed = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_warm, capture_error_mode="thread_local"):
        for i in range(args.warmup):
            wl.step(qk, sets[i % R])
    with torch.cuda.graph(g_timed, capture_error_mode="thread_local"):
        for i in range(args.steps):
            wl.step(qk, sets[(args.warmup + i) % R])
    torch.cuda.synchronize()
    uploaded = graph_upload(g_timed, torch.cuda.current_stream(dev))
    torch.cuda.synchronize()

    sampler = ClockSampler(local)
    sampler.start()
    g_warm.replay()  # W untimed warm-up steps
    stream = torch.cuda.current_stream(dev)
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    barrier()
    torch.cuda.synchronize()
    # the timed region can be far shorter than the sampling period: samples
    # are also taken at its edges and while the replay is in flight
    sampler.sample_now()
    sampler.active.set()
    hold_queue(stream)
    ev0.record(stream)
    g_timed.replay()
    ev1.record(stream)
    sampler.sample_now()
    torch.cuda.synchronize()
    sampler.active.clear()
    sampler.sample_now()
    barrier()
    ms_rank = ev0.elapsed_time(ev1)
    ms = max_over_ranks(ms_rank)
    clocks = sampler.summary()
    del g_warm, g_timed

    # Spread (informational): 20 replays of a short graph, each timed on its
    # own, give per-call p10 / p50 / p90; and the same calls launched eagerly,
    # back to back, for the latency-bound shapes.
    spread = None
    if rank == 0 and wl.kind != "tp":  # tp captures take fresh epochs: not replayed twice
        m = max(1, min(100, args.steps))
        g_short = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g_short, capture_error_mode="thread_local"):
            for i in range(m):
                wl.step(qk, sets[i % R])
        g_short.replay()
        torch.cuda.synchronize()
        per_call = []
        for _ in range(20):
            hold_queue(stream)
            ev0.record(stream)
            g_short.replay()
            ev1.record(stream)
            torch.cuda.synchronize()
            per_call.append(ev0.elapsed_time(ev1) * 1e3 / m / wl.launches_per_step)
        del g_short
        per_call.sort()
        spread = {"us_per_call_p10": round(per_call[2], 3), "us_per_call_p50": round(statistics.median(per_call), 3),
                  "us_per_call_p90": round(per_call[17], 3), "replays": 20, "calls_per_replay": m}
        ev0.record(stream)
        for i in range(m):
            wl.step(qk, sets[i % R])
        ev1.record(stream)
        torch.cuda.synchronize()
        spread["eager_us_per_call"] = round(ev0.elapsed_time(ev1) * 1e3 / m / wl.launches_per_step, 3)

    agg = whole_job(wl.eff_bytes, args.steps, ms, world)
    step_s = agg["ms_per_step"] / 1e3
    value = agg["value_gbs"]
    per_rank_gbs = agg["per_rank_gbs"]
    peaks = load_peaks()
    digest = source_digest("tp" if wl.kind == "tp" else "rows")
    plan = None
    if wl.kind in ("prefill", "tiny", "decode", "packed"):
        s0 = sets[0]
        if wl.kind == "packed":
            plan = qk.qknorm_layerwise_plan(s0["q"], s0["k"], s0["gq"], s0["gk"], q_out=s0["q"], k_out=s0["k"])
        else:
            plan = qk.qknorm_layerwise_plan(s0["q"], s0["k"], s0["gq"], s0["gk"], q_out=s0["qo"], k_out=s0["ko"])

    roofline = roofline_record(wl, step_s, peaks, digest, plan)

    timeouts = qk.device_timeouts()  # any bounded wait that ran out (tensor-parallel exchange)

    # end to end through the public API with pinned host buffers
    e2e = e2e_measure(qk, wl, dev, args, barrier, max_over_ranks)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = time_oracle(wl, args.cpu_seconds)
        if wl.kind in ("prefill", "packed", "tiny", "decode", "tp"):
            cpu["all_cores"] = time_oracle_parallel(wl, args.cpu_seconds)

    if rank == 0:
        cfg = wl.config()
        cfg["parallelism"] = parallelism(world)
        between = (R - 1) * wl.set_bytes()
        measurement = {"l2": f"rotating {R} input/output sets ({R * wl.set_bytes() / 1e6:.1f} MB; "
                             f"{between / 1e6:.1f} MB touched between reuses "
                             + ("> 2 x" if between > 2 * l2 else "< 2 x (L2-warm)") + f" {l2 / 1e6:.0f} MB L2)",
                       "timing": "CUDA graph of K captured C-ABI calls (uploaded before timing: %s), "
                                 "CUDA events on the launching stream, a ~100 us torch sleep kernel queued "
                                 "ahead of the start event (the host's graph submission is not timed)"
                                 % ("yes" if uploaded else "no"),
                       "launch_plan": plan}
        line = {"metric": METRIC, "value": round(value, 1), "unit": UNIT, "n_gpus": world, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": round(ms / args.steps, 6),
                "us_per_call": round(step_s * 1e6 / wl.launches_per_step, 3),
                "pct_of_peak": round(100 * per_rank_gbs / peaks["hbm_gbs"], 2),
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
                "data": "synthetic (seeded; OLMo2-shaped activations, no dataset or weights)",
                "config": cfg, "measurement": measurement, "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e,
                "gpu_launches": args.steps * wl.launches_per_step, "clocks": clocks,
                "spread": spread, "device_timeouts": timeouts, "impl": "native"}
        print(json.dumps(line))
    if dist is not None:
        dist.destroy_process_group()
    return 0


def link_calibration(dev, h2d_bytes: int, d2h_bytes: int, eff_bytes: int, reps: int = 5) -> dict:
    """The host link on its own: pinned copies of one step's bytes, each
    direction alone and both at once on two streams (best of `reps`), and the
    end-to-end value those copies alone would allow."""
    src_h = torch.empty(h2d_bytes, dtype=torch.uint8, pin_memory=True)
    dst_d = torch.empty(h2d_bytes, dtype=torch.uint8, device=dev)
    src_d = torch.empty(d2h_bytes, dtype=torch.uint8, device=dev)
    dst_h = torch.empty(d2h_bytes, dtype=torch.uint8, pin_memory=True)
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)

    def timed(h2d: bool, d2h: bool) -> float:
        best = float("inf")
        for _ in range(reps):
            torch.cuda.synchronize(dev)
            t0 = time.perf_counter()
            if h2d:
                with torch.cuda.stream(s_in):
                    dst_d.copy_(src_h, non_blocking=True)
            if d2h:
                with torch.cuda.stream(s_out):
                    dst_h.copy_(src_d, non_blocking=True)
            torch.cuda.synchronize(dev)
            best = min(best, time.perf_counter() - t0)
        return best
    t_in, t_out, t_both = timed(True, False), timed(False, True), timed(True, True)
    return {"h2d_gbs": round(h2d_bytes / t_in / 1e9, 2), "d2h_gbs": round(d2h_bytes / t_out / 1e9, 2),
            "both_ms": round(t_both * 1e3, 4), "e2e_copy_limit": round(eff_bytes / t_both / 1e9, 2),
            "how": "pinned torch copies of the step's bytes, host clock, best of %d" % reps}


def e2e_measure(qk, wl: Workload, dev, args, barrier, max_over_ranks) -> dict:
    """The same metric end to end through the public API on pinned host
    buffers: per step, the inputs travel host->device, are normalized, and
    the results travel device->host, all inside the timed region."""
    b = wl.batch
    steps = max(1, min(args.e2e_steps, args.steps))
    h_g = [b.gamma_q.clone().pin_memory(), b.gamma_k.clone().pin_memory()]
    gbytes = sum(t.numel() * t.element_size() for t in h_g)
    if wl.kind == "packed":
        h_packed = b.packed.clone().pin_memory()

        def one():
            qk.qknorm_packed_host(h_packed, 0, b.Hq, b.Hq, b.Hk, h_g[0], h_g[1], b.eps, device=dev,
                                  chunk_tokens=args.e2e_chunk, slots=args.e2e_slots)
        qk_bytes = b.T * (b.Hq + b.Hk) * wl.esz
        h2d = qk_bytes + gbytes
        d2h = qk_bytes
        path = (f"C-ABI qknorm_layerwise_host: the Q and K columns of the pinned packed host rows -> device in "
                f"{args.e2e_chunk}-token chunks (pitched copies; V never moves), normalized in place, back into "
                f"the same host columns; {args.e2e_slots}-slot device ring, copies and kernel overlap on three "
                "streams")
    elif wl.kind == "gqa":
        s = wl.make_set(dev)
        h_in = [t.clone().pin_memory() for t in b.q_shards + b.k_shards]
        h_out = [torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for t in s["qo"] + s["ko"]]
        d_g = [torch.empty_like(b.gamma_q, device=dev), torch.empty_like(b.gamma_k, device=dev)]

        def one():
            for h, d in zip(h_in + h_g, s["qs"] + s["ks"] + d_g):
                d.copy_(h, non_blocking=True)
            P = b.P
            wq, wk = b.Hq // P, b.Hk // P
            for p in range(P):
                s["gqs"][p].copy_(d_g[0][p * wq:(p + 1) * wq])
                s["gks"][p].copy_(d_g[1][p * wk:(p + 1) * wk])
            wl.step(qk, s)
            for h, d in zip(h_out, s["qo"] + s["ko"]):
                h.copy_(d, non_blocking=True)
        h2d = sum(t.numel() * t.element_size() for t in h_in) + gbytes
        d2h = sum(t.numel() * t.element_size() for t in h_out)
        path = "per-shard pinned host -> device copies, partial_stats x P + combine_apply x P, device -> host copies"
    elif wl.kind == "tp":
        s = wl.make_set(dev)
        h_in = [t.cpu().pin_memory() for t in s["qs"] + s["ks"]]
        h_out = [torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for t in s["qo"] + s["ko"]]

        def one():
            for h, d in zip(h_in, s["qs"] + s["ks"]):
                d.copy_(h, non_blocking=True)
            wl.step(qk, s)
            for h, d in zip(h_out, s["qo"] + s["ko"]):
                h.copy_(d, non_blocking=True)
        h2d = sum(t.numel() * t.element_size() for t in h_in)
        d2h = sum(t.numel() * t.element_size() for t in h_out)
        path = "per-rank shards pinned host -> device, qknorm_tp_layerwise (all ranks, one launch), device -> host"
    elif wl.kind == "headwise":
        s = wl.make_set(dev)
        h_q, h_k = b.q.contiguous().pin_memory(), b.k.contiguous().pin_memory()
        h_qo = torch.empty(h_q.shape, dtype=h_q.dtype, pin_memory=True)
        h_ko = torch.empty(h_k.shape, dtype=h_k.dtype, pin_memory=True)

        def one():
            s["q"].copy_(h_q, non_blocking=True)
            s["k"].copy_(h_k, non_blocking=True)
            s["gq"].copy_(h_g[0], non_blocking=True)
            s["gk"].copy_(h_g[1], non_blocking=True)
            wl.step(qk, s)
            h_qo.copy_(s["qo"], non_blocking=True)
            h_ko.copy_(s["ko"], non_blocking=True)
        h2d = sum(t.numel() * t.element_size() for t in (h_q, h_k)) + gbytes
        d2h = sum(t.numel() * t.element_size() for t in (h_qo, h_ko))
        path = "pinned host -> device copies, qknorm_headwise, device -> pinned host copies, one stream"
    else:
        h_q, h_k = b.q.contiguous().pin_memory(), b.k.contiguous().pin_memory()
        h_qo = torch.empty(h_q.shape, dtype=h_q.dtype, pin_memory=True)
        h_ko = torch.empty(h_k.shape, dtype=h_k.dtype, pin_memory=True)

        def one():
            qk.qknorm_layerwise_host(h_q, h_k, h_g[0], h_g[1], b.eps, q_out=h_qo, k_out=h_ko, device=dev,
                                     chunk_tokens=args.e2e_chunk, slots=args.e2e_slots)
        h2d = sum(t.numel() * t.element_size() for t in (h_q, h_k)) + gbytes
        d2h = sum(t.numel() * t.element_size() for t in (h_qo, h_ko))
        path = (f"C-ABI qknorm_layerwise_host: pinned host -> device in {args.e2e_chunk}-token chunks, normalized "
                f"on the device, device -> pinned host; {args.e2e_slots}-slot device ring, copies and kernel "
                "overlap on three streams")

    for _ in range(3):
        one()
    stream = torch.cuda.current_stream(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    barrier()
    e0.record(stream)
    for _ in range(steps):
        one()
    e1.record(stream)
    torch.cuda.synchronize()
    barrier()
    ms = max_over_ranks(e0.elapsed_time(e1))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    link = link_calibration(dev, h2d, d2h, wl.eff_bytes)
    return {"value": round(world * wl.eff_bytes / (ms / 1e3 / steps) / 1e9, 2), "unit": UNIT,
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": steps,
            "ms_per_step": round(ms / steps, 4), "path": path, "link": link}


# --------------------------------------------------------------------------- reference arm (the oracle)

def reference(args) -> int:
    rank, world, _ = dist_env()
    if rank != 0:
        return 0  # the CPU oracle runs once, on rank 0
    wl = Workload(args.workload, args.tokens, seed_offset=0, dtype=args.dtype)
    b = wl.batch
    # per-step sample: enough tokens that the whole run stays near a minute
    probe = time_oracle(wl, 0.0, max_tokens=min(b.T, 8))
    per_token_s = probe["us_per_call"] / 1e6 / probe["tokens"]
    budget_s = 60.0
    tokens = int(max(1, min(b.T, budget_s / ((args.steps + args.warmup) * per_token_s))))
    for _ in range(args.warmup):
        time_oracle(wl, 0.0, max_tokens=tokens)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        time_oracle(wl, 0.0, max_tokens=tokens)
    el = time.perf_counter() - t0
    eff = wl.eff_bytes * tokens / b.T
    value = eff / (el / args.steps) / 1e9
    cfg = wl.config()  # the native arm's config, so both lines name the same workload
    cfg["parallelism"] = parallelism(world)
    line = {"metric": METRIC, "value": round(value, 5), "unit": UNIT, "n_gpus": 0, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(el / args.steps * 1e3, 4), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic", "config": cfg,
            "impl": "reference",
            "cpu_baseline": {"value": round(value, 5), "unit": UNIT, "cores": 1, "kind": "oracle",
                             "sample": f"{tokens} of {b.T} tokens of {wl.name} per step, one thread"},
            "e2e": {"value": round(value, 5), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line))
    return 0


# --------------------------------------------------------------------------- QKV projection workload

PROJ_METRIC = "QKV projection + layerwise QK-Norm TFLOP/s (tensor-core roofline); µs per call"
PROJ_UNIT = "TFLOP/s"


def load_tensor_peak() -> dict:
    """Measured dense bf16 tensor throughput (burst: the projection kernel is
    timed on its own, not inside a seconds-long loop)."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return {"tflops": float(d["bf16_tflops"]), "sustained": float(d.get("bf16_tflops_sustained", 0.0)),
                "source": "measured cuBLAS bf16 GEMM (burst)"}
    except (OSError, KeyError, ValueError):
        return {"tflops": 1590.0, "sustained": 1400.0, "source": "fallback bf16 GEMM"}


def _proj_flops(b) -> float:
    return 2.0 * b.T * b.D * (b.Hq + b.Hk + b.Hv)


def time_oracle_projection(b, budget_s: float, rows: int = 1) -> dict:
    """The CPU oracle on `rows` tokens per call (projection of those rows in
    double, then RMS-Norm of their Q and K columns), repeated until the budget
    is spent; reported in the workload's unit (TFLOP/s of projection work)."""
    import numpy as np

    import oracle
    xs = b.x.contiguous().view(torch.int16).numpy().view(np.uint16)
    ws = b.w.contiguous().view(torch.int16).numpy().view(np.uint16)
    gq = b.gamma_q.view(torch.int16).numpy().view(np.uint16)
    gk = b.gamma_k.view(torch.int16).numpy().view(np.uint16)
    calls, t0 = 0, time.perf_counter()
    while True:
        sel = [(calls * rows + i) % b.T for i in range(rows)]
        y, _ = oracle.project_rows(xs, ws, sel)
        oracle.rmsnorm_rows(np.ascontiguousarray(y[:, :b.Hq]), b.Hq, gq, b.eps)
        oracle.rmsnorm_rows(np.ascontiguousarray(y[:, b.Hq:b.Hq + b.Hk]), b.Hk, gk, b.eps)
        calls += 1
        el = time.perf_counter() - t0
        if el >= budget_s:
            break
    per_row = el / (calls * rows)
    flops_per_row = _proj_flops(b) / b.T
    return {"value": round(flops_per_row / per_row / 1e12, 9), "unit": PROJ_UNIT, "cores": 1, "kind": "oracle",
            "sample": f"{calls * rows} token rows of {b.name} ({calls} calls), {el:.1f} s",
            "us_per_token": per_row * 1e6}


def native_projection(args) -> int:
    rank, world, local = dist_env()
    if not torch.cuda.is_available():
        print(json.dumps({"metric": PROJ_METRIC, "error": "no CUDA device"}))
        return 1
    torch.cuda.set_device(local)
    dev = torch.device(f"cuda:{local}")
    dist = None
    if world > 1:
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=180), device_id=dev)
    import attention_normalization_b200 as qk
    qk.capi()
    ranks = Ranks(dist, dev)

    D, Hq, Hk, Hv = (int(v) for v in args.proj.split(","))
    b = workloads.qkv_projection(T=args.tokens or 4096, D=D, Hq=Hq, Hk=Hk, Hv=Hv, seed=6 + rank * 1000)
    N = b.Hq + b.Hk + b.Hv
    flops = _proj_flops(b)
    ws_bytes = qk.qkv_workspace_bytes(b.T, b.Hq, b.Hk)
    set_bytes = 2 * (b.T * b.D + N * b.D + b.T * N) + ws_bytes
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    R = rotation_count(set_bytes, l2)
    gq, gk = b.gamma_q.to(dev), b.gamma_k.to(dev)
    sets = [{"x": b.x.to(dev), "w": b.w.to(dev), "qkv": torch.empty((b.T, N), dtype=torch.bfloat16, device=dev),
             "ws": torch.empty((ws_bytes // 4,), dtype=torch.float32, device=dev),
             "qs": torch.empty((b.Hq // 256, b.T), dtype=torch.float32, device=dev),
             "ks": torch.empty((b.Hk // 256, b.T), dtype=torch.float32, device=dev)} for _ in range(R)]

    def step(s):
        qk.qknorm_qkv_projection(s["x"], s["w"], gq, gk, b.Hq, b.Hk, b.Hv, b.eps, qkv=s["qkv"], workspace=s["ws"])

    def gemm_only(s):
        qk.qknorm_qkv_gemm_stats(s["x"], s["w"], b.Hq, b.Hk, b.Hv, qkv=s["qkv"], q_sums=s["qs"], k_sums=s["ks"])

    def cublas_unfused(s):  # library baseline: cuBLAS GEMM, then the fused layerwise kernel in place
        torch.matmul(s["x"], s["w"].t(), out=s["qkv"])
        q, k = s["qkv"][:, :b.Hq], s["qkv"][:, b.Hq:b.Hq + b.Hk]
        qk.qknorm_layerwise(q, k, gq, gk, b.eps, q_out=q, k_out=k)

    stream = torch.cuda.current_stream(dev)

    def graph_time(fn, steps, warm):
        for i in range(3):
            fn(sets[i % R])
        torch.cuda.synchronize()
        gw, gt = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
        with torch.cuda.graph(gw, capture_error_mode="thread_local"):
            for i in range(warm):
                fn(sets[i % R])
        with torch.cuda.graph(gt, capture_error_mode="thread_local"):
            for i in range(steps):
                fn(sets[(warm + i) % R])
        torch.cuda.synchronize()
        graph_upload(gt, stream)
        gw.replay()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        ranks.barrier()
        torch.cuda.synchronize()
        sampler.active.set()
        hold_queue(stream)
        e0.record(stream)
        gt.replay()
        e1.record(stream)
        torch.cuda.synchronize()
        sampler.active.clear()
        ranks.barrier()
        ms = ranks.max(e0.elapsed_time(e1))
        del gw, gt
        return ms

    sampler = ClockSampler(local)
    sampler.start()
    ms = graph_time(step, args.steps, args.warmup)
    clocks = sampler.summary()
    # Comparison (informational): short graphs of the pipeline, the GEMM with
    # partial sums alone and cuBLAS + qknorm_layerwise, interleaved round by
    # round so that clock and power drift hits all three alike; medians.
    side_steps = max(3, min(args.steps, 20))
    sampler = ClockSampler(local)  # the comparison runs get their own (unreported) sampler
    sampler.start()
    side = {"pipeline": [], "gemm": [], "cublas": []}
    for _ in range(5):
        side["pipeline"].append(graph_time(step, side_steps, 3) / side_steps)
        side["gemm"].append(graph_time(gemm_only, side_steps, 3) / side_steps)
        side["cublas"].append(graph_time(cublas_unfused, side_steps, 3) / side_steps)
    sampler.summary()
    side = {k: statistics.median(v) for k, v in side.items()}
    timeouts = qk.device_timeouts()

    step_s = ms / 1e3 / args.steps
    value = world * flops / step_s / 1e12
    peak = load_tensor_peak()

    # end to end: hidden states in from pinned host memory, the normalized QKV back out
    h_x = b.x.contiguous().pin_memory()
    h_qkv = torch.empty((b.T, N), dtype=torch.bfloat16, pin_memory=True)
    s0 = sets[0]

    def one():
        s0["x"].copy_(h_x, non_blocking=True)
        step(s0)
        h_qkv.copy_(s0["qkv"], non_blocking=True)
    for _ in range(2):
        one()
    e2e_steps = max(1, min(args.e2e_steps, args.steps))
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    ranks.barrier()
    e0.record(stream)
    for _ in range(e2e_steps):
        one()
    e1.record(stream)
    torch.cuda.synchronize()
    ranks.barrier()
    ms_e2e = ranks.max(e0.elapsed_time(e1))
    e2e = {"value": round(world * flops / (ms_e2e / 1e3 / e2e_steps) / 1e12, 2), "unit": PROJ_UNIT,
           "h2d_bytes_per_step": h_x.numel() * 2, "d2h_bytes_per_step": h_qkv.numel() * 2, "steps": e2e_steps,
           "ms_per_step": round(ms_e2e / e2e_steps, 4),
           "path": "pinned host -> device copy of x, qknorm_qkv_projection (weights and gamma resident), "
                   "device -> pinned host copy of qkv, one stream"}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = time_oracle_projection(b, args.cpu_seconds)

    if rank == 0:
        between = (R - 1) * set_bytes
        cfg = {"workload": b.name, "T": b.T, "D": b.D, "Hq": b.Hq, "Hk": b.Hk, "Hv": b.Hv, "io_dtype": "bfloat16",
               "eps": b.eps, "form": "qknorm_qkv_projection: tcgen05 GEMM with per-tile squared sums in the "
                                     "epilogue, then combine + scale of the Q and K columns in place",
               "parallelism": f"replicas x{world} (tokens independent, no collective)",
               "l2": f"rotating {R} sets of x, w, qkv, workspace ({R * set_bytes / 1e6:.1f} MB; "
                     f"{between / 1e6:.1f} MB touched between reuses "
                     + ("> 2 x" if between > 2 * l2 else "< 2 x") + f" {l2 / 1e6:.0f} MB L2)",
               "timing": "CUDA graph of K captured C-ABI calls, CUDA events on the launching stream, a ~100 us "
                         "torch sleep kernel queued ahead of the start event (the host's graph submission is not "
                         "timed)"}
        # the dominant kernel is the GEMM (the apply pass after it moves the Q
        # and K columns once): its own time is the comparison's GEMM-only graph
        kernel_tflops = flops / (side["gemm"] / 1e3) / 1e12
        line = {"metric": PROJ_METRIC, "value": round(value, 1), "unit": PROJ_UNIT, "n_gpus": world,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms / args.steps, 6),
                "us_per_call": round(step_s * 1e6, 2), "higher_is_better": True, "scaling": "weak",
                "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded; OLMo2-7B-shaped projection, "
                                                             "random weights)",
                "config": cfg, "measurement": {"gemm_schedule": qk.qkv_gemm_plan(b.T, b.D, b.Hq, b.Hk, b.Hv)},
                "roofline": {"bound": "tensor", "achieved": round(kernel_tflops, 1), "peak": peak["tflops"],
                             "unit": "TFLOP/s", "frac": round(kernel_tflops / peak["tflops"], 4),
                             "traffic": profiled_traffic(b.name, source_digest("projection")),
                             "peak_source": peak["source"],
                             "kernel": "qkv_gemm_stats_kernel (the dominant kernel; timed alone in the comparison's "
                                       "GEMM-only graphs), then the apply pass over the Q and K columns",
                             "algorithmic_flops_per_launch": flops, "source_digest": source_digest("projection")},
                "comparison_us": {"how": f"medians of 5 interleaved rounds of {side_steps}-call graphs",
                                  "projection_with_qk_norm": round(side["pipeline"] * 1e3, 2),
                                  "gemm_with_partial_sums_only": round(side["gemm"] * 1e3, 2),
                                  "cublas_matmul_plus_qknorm_layerwise": round(side["cublas"] * 1e3, 2)},
                "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": 2 * args.steps, "clocks": clocks,
                "device_timeouts": timeouts, "impl": "native"}
        print(json.dumps(line))
    if dist is not None:
        dist.destroy_process_group()
    return 0


def projection_reference(args) -> int:
    rank, world, _ = dist_env()
    if rank != 0:
        return 0
    D, Hq, Hk, Hv = (int(v) for v in args.proj.split(","))
    b = workloads.qkv_projection(T=args.tokens or 4096, D=D, Hq=Hq, Hk=Hk, Hv=Hv, seed=6)
    for _ in range(args.warmup):
        time_oracle_projection(b, 0.0)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        time_oracle_projection(b, 0.0)
    el = time.perf_counter() - t0
    value = _proj_flops(b) / b.T / (el / args.steps) / 1e12
    line = {"metric": PROJ_METRIC, "value": round(value, 9), "unit": PROJ_UNIT, "n_gpus": 0, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(el / args.steps * 1e3, 4), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": b.name, "sample_tokens_per_step": 1}, "impl": "reference",
            "cpu_baseline": {"value": round(value, 9), "unit": PROJ_UNIT, "cores": 1, "kind": "oracle",
                             "sample": f"1 of {b.T} token rows of {b.name} per step, one thread"},
            "e2e": {"value": round(value, 9), "unit": PROJ_UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line))
    return 0


def main(argv=None) -> int:
    args = parse_args(argv)
    if args.workload == "projection":
        return projection_reference(args) if args.impl == "reference" else native_projection(args)
    if args.impl == "reference":
        return reference(args)
    return native(args)


if __name__ == "__main__":
    sys.exit(main())
