#!/usr/bin/env python
"""Throughput benchmark of the speculative-decoding verify step on B200.

One step = one verify call on each of the four full-size workloads, in this
order (every row of the hot path: stochastic accept/correct/bonus, greedy,
multi-candidate):

  greedy_b64_k4_v128256    greedy,          bf16 [64,5,128256]
  stoch_b64_k4_v128256     stochastic,      bf16 [64,5,128256] + fp32 [64,4,128256]
  stoch_b256_k8_v128256    stochastic,      bf16 [256,9,128256] + bf16 [256,8,128256]
  multi_b16_g8_k4_v32000   multi-candidate, bf16 [16,8,5,32000]

Metric: verified positions per second (positions = B (k+1), or B G (k+1)),
whole job over all GPUs.  The latency-bound single-sequence workload
stoch_b1_k4_v32000_f32 (fp32 [1,5,32000] + [1,4,32000]) is timed on its own,
outside the step, and reported in per_workload as microseconds per call.  Inputs are resident in HBM and 1.45 GB are
streamed per step, more than L2 (126 MB), so no buffer is re-read from L2
across steps.  Usage:

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

With N > 1, launch one process per GPU with torch.distributed.run; every
rank verifies its own batch (weak scaling, no collective on the data path).
`--impl reference` times the CPU oracle (the only reference this method has)
on rank 0.
"""
from __future__ import annotations

import argparse
import datetime
import glob
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

STEP = ["greedy_b64_k4_v128256", "stoch_b64_k4_v128256", "stoch_b256_k8_v128256",
        "multi_b16_g8_k4_v32000"]
LATENCY = ["stoch_b1_k4_v32000_f32"]  # timed alone, outside the step
DOMINANT = "stoch_b256_k8_v128256"
HBM_FALLBACK_GBS = 6650.0
HBM_NOMINAL_GBS = 8000.0  # the ~8 TB/s the metric quotes
NEAR_TIE = 1e-5
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "traffic_stochastic_verify_b256_k8.json")
TREE_MODES = ("tree", "tree_stochastic")


# ------------------------------------------------------------------ helpers

def positions(w: dict) -> int:
    if w["mode"] in TREE_MODES:  # every drafted node is a verified position
        return w["B"] * w["N"]
    return w["B"] * w.get("G", 1) * (w["k"] + 1)


def full_bytes(w: dict) -> int:
    """Bytes of one call when every logit row is read once, rows past the
    first rejection included (the per-call count of the measurement plan),
    plus tokens in and results out."""
    from workloads import ELEM_BYTES

    st = ELEM_BYTES[w["t_dtype"]]
    if w["mode"] in TREE_MODES:  # every node row, parents and tokens, path and tokens out
        B, N, V = w["B"], w["N"], w["V"]
        return B * N * V * st + 8 * B * N + 4 * B + 8 * B * N
    B, k, V = w["B"], w["k"], w["V"]
    if w["mode"] in ("greedy", "threshold"):
        return B * (k + 1) * V * st + 4 * B * k + 4 * B * (k + 2)
    if w["mode"] == "multi":
        G = w["G"]
        return B * G * (k + 1) * V * st + 4 * B * G * k + 4 * B * (k + 3)
    if w["mode"] == "multi_rows":  # each distinct prefix row once, plus the row map
        G = w["G"]
        distinct = sum(len(np.unique(w["row_of"][b])) for b in range(B))
        return distinct * V * st + 4 * B * G * (k + 1) + 4 * B * G * k + 4 * B * (k + 3)
    sd = ELEM_BYTES[w["d_dtype"]]
    return B * (k + 1) * V * st + B * k * V * sd + 4 * B * k + 4 * B * (k + 2)


def needed_bytes(w: dict, outcome: dict | None) -> int | None:
    """Bytes the method must read for the outcome the ORACLE computed: rows
    past the first rejection (or a branch's first mismatch) decide nothing.

    stochastic: row pairs 0..n_b (the rejected pair once), and target row k
                alone when n_b = k;
    greedy:     target rows 0..n_b;
    multi:      rows 0..n_{b,g} of every branch g;
    other modes: the full count.  None without an oracle outcome.
    """
    from workloads import ELEM_BYTES

    if outcome is None:
        return None
    if w["mode"] not in ("stochastic", "greedy", "multi"):
        return full_bytes(w)
    st = ELEM_BYTES[w["t_dtype"]]
    B, k, V = w["B"], w["k"], w["V"]
    if w["mode"] == "greedy":
        rows = int((np.asarray(outcome["accepted_len"]) + 1).sum())
        return rows * V * st + 4 * B * k + 4 * B * (k + 2)
    if w["mode"] == "multi":
        G = w["G"]
        rows = int((np.asarray(outcome["branch_len"]) + 1).sum())
        return rows * V * st + 4 * B * G * k + 4 * B * (k + 3)
    sd = ELEM_BYTES[w["d_dtype"]]
    n = np.asarray(outcome["accepted_len"])
    pairs = int(np.minimum(n + 1, k).sum())
    n_full = int((n == k).sum())
    return pairs * V * (st + sd) + n_full * V * st + 4 * B * k + 4 * B * (k + 2)


def measured_hbm_peak() -> tuple[float, str]:
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except Exception:
        return HBM_FALLBACK_GBS, "fallback"


# The sources that build the dominant kernel and set its launch (chunking,
# ticket map, lag); a traffic record is valid only for these exact bytes.
DOMINANT_SOURCES = ("sv_api.cu", "sv_device.cuh", "sv_internal.h", "sv_kernels.cu")
KERNEL_OF_MODE = {"stochastic": "stochastic_verify_kernel", "greedy": "argmax_verify_kernel",
                  "multi": "argmax_verify_kernel", "multi_rows": "argmax_verify_kernel",
                  "tree": "argmax_verify_kernel", "threshold": "argmax_verify_kernel",
                  "tree_stochastic": "tree_stats_kernel + tree_walk_kernel + tree_sample_kernel"}


def kernel_source_hash() -> str:
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "speculative_decoding_verification_88_b200", "csrc")
    for name in DOMINANT_SOURCES:
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(name.encode())
            h.update(f.read())
    return h.hexdigest()


def recorded_traffic(workload: str, batch_override: bool) -> float | None:
    """DRAM bytes per launch of the dominant kernel from an ncu capture of the
    current kernel sources, or None if the sources changed since or the run
    times another workload or batch than the one the record covers."""
    if workload != "stoch_b256_k8_v128256" or batch_override:
        return None
    try:
        with open(TRAFFIC_FILE) as f:
            rec = json.load(f)
    except Exception:
        return None
    if rec.get("kernel_source_sha256") != kernel_source_hash():
        return None
    return float(rec["dram_bytes_per_launch"])


def call_spread(samples_ms: list) -> dict:
    """Median and 10th / 90th percentiles, in microseconds, of per-call
    times in milliseconds (one event pair per call per graph replay).
    Percentiles interpolate between order statistics."""
    xs = sorted(samples_ms)
    if not xs:
        return {}
    def q(f):
        pos = f * (len(xs) - 1)
        lo = int(pos)
        hi = min(lo + 1, len(xs) - 1)
        return (xs[lo] + (xs[hi] - xs[lo]) * (pos - lo)) * 1e3
    return {"p10": round(q(0.1), 2), "median": round(q(0.5), 2), "p90": round(q(0.9), 2),
            "samples": len(xs)}


class NvmlSampler:
    """SM clock and throttle reasons of one GPU read through NVML every half
    millisecond from a background thread, so that a timed region of a few
    milliseconds holds samples (nvidia-smi samples every 50-100 ms).  Reads
    only; changes no setting."""

    BITS = (("hw_slowdown", "nvmlClocksEventReasonHwSlowdown"),
            ("hw_thermal_slowdown", "nvmlClocksEventReasonHwThermalSlowdown"),
            ("sw_thermal_slowdown", "nvmlClocksEventReasonSwThermalSlowdown"),
            ("sw_power_cap", "nvmlClocksEventReasonSwPowerCap"))

    def __init__(self, gpu_uuid: str):
        self.samples: list[tuple[float, float, int]] = []
        self.ok = False
        self._stop = threading.Event()
        try:
            import pynvml

            self.nv = pynvml
            pynvml.nvmlInit()
            self.h = pynvml.nvmlDeviceGetHandleByUUID(gpu_uuid)
            self.max_mhz = float(pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM))
            self.mask = {name: getattr(pynvml, attr) for name, attr in self.BITS}
            self.thread = threading.Thread(target=self._run, daemon=True)
            self.thread.start()
            self.ok = True
        except Exception:
            self.ok = False

    def _run(self):
        nv = self.nv
        while not self._stop.is_set():
            try:
                sm = float(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
                rs = int(nv.nvmlDeviceGetCurrentClocksEventReasons(self.h))
            except Exception:
                break
            self.samples.append((time.time(), sm, rs))
            time.sleep(0.0005)

    def stop(self, t0: float, t1: float) -> dict | None:
        if not self.ok:
            return None
        self._stop.set()
        self.thread.join(timeout=2)
        sel = [(sm, rs) for ts, sm, rs in self.samples if t0 <= ts <= t1]
        if not sel:
            return None
        reasons = sorted({name for name, bit in self.mask.items()
                          for _, rs in sel if rs & bit})
        return {"sm_mhz": statistics.median(sm for sm, _ in sel), "sm_max_mhz": self.max_mhz,
                "reasons": reasons, "samples": len(sel),
                "window": "timed region (NVML, every 0.5 ms)"}


class ClockSampler:
    """nvidia-smi clock / throttle samples of one GPU while it runs."""

    FIELDS = ("timestamp,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    REASONS = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")

    def __init__(self, gpu_id: str):
        self.lines: list[str] = []
        self.proc = None
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "50", "-i", gpu_id], stdout=subprocess.PIPE,
                stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self, t0: float, t1: float) -> dict | None:
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.thread.join(timeout=2)
        return self.summarise(t0, t1)

    def summarise(self, t0: float, t1: float, margin: float = 0.25) -> dict:
        """Median SM clock, max clock and active throttle reasons of the
        samples taken inside [t0, t1]; a timed region shorter than the
        sampling period may hold none, and then the samples within `margin`
        seconds on either side stand in (reported in "window")."""
        rows = []
        for line in self.lines:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                ts = datetime.datetime.strptime(parts[0], "%Y/%m/%d %H:%M:%S.%f").timestamp()
            except ValueError:
                continue
            rows.append((ts, parts))
        window = "timed region"
        sel = [parts for ts, parts in rows if t0 <= ts <= t1]
        if not sel:
            sel = [parts for ts, parts in rows if t0 - margin <= ts <= t1 + margin]
            window = f"no sample inside the timed region; samples within {margin} s of it"
        sm, smax, reasons = [], [], set()
        for parts in sel:
            try:
                sm.append(float(parts[1]))
                smax.append(float(parts[2]))
            except ValueError:
                pass
            for name, val in zip(self.REASONS, parts[5:9]):
                if val.lower() == "active":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sel), "window": window}


# --------------------------------------------------------------- reference

def run_reference(args, rank: int) -> None:
    """The CPU oracle timed on the host cores: each step verifies one sequence
    of each step workload (rotating through the batch), the four in parallel."""
    if rank != 0:
        return
    import oracle
    import workloads

    oracle.build()
    ws = {n: workloads.make(n) for n in STEP}
    cores = min(len(STEP), os.cpu_count() or 1)

    def one(name, b):
        w = ws[name]
        if w["mode"] == "stochastic":
            oracle.verify_stochastic(w["target"][b:b + 1], w["t_dtype"], w["draft"][b:b + 1],
                                     w["d_dtype"], w["tokens"][b:b + 1], w["temperature"],
                                     w["seed"], seq_offset=b)
        elif w["mode"] == "greedy":
            oracle.verify_greedy(w["target"][b:b + 1], w["t_dtype"], w["tokens"][b:b + 1])
        elif w["mode"] == "multi_rows":
            oracle.verify_multi_rows(w["rows"][b:b + 1], w["t_dtype"], w["row_of"][b:b + 1],
                                     w["tokens"][b:b + 1])
        elif w["mode"] == "tree":
            oracle.verify_tree_greedy(w["node_logits"][b:b + 1], w["t_dtype"],
                                      w["parent"][b:b + 1], w["tokens"][b:b + 1])
        elif w["mode"] == "tree_stochastic":
            oracle.verify_tree_stochastic(w["node_logits"][b:b + 1], w["t_dtype"],
                                          w["parent"][b:b + 1], w["tokens"][b:b + 1],
                                          w["temperature"], w["seed"], seq_offset=b)
        elif w["mode"] == "threshold":
            oracle.verify_threshold(w["target"][b:b + 1], w["t_dtype"], w["tokens"][b:b + 1],
                                    w["temperature"], w["threshold"])
        else:
            oracle.verify_multi(w["target"][b:b + 1], w["t_dtype"], w["tokens"][b:b + 1])

    def step(s):
        ts = [threading.Thread(target=one, args=(n, s % ws[n]["B"])) for n in STEP]
        for t in ts:
            t.start()
        for t in ts:
            t.join()

    for s in range(args.warmup):
        step(s)
    t0 = time.perf_counter()
    for s in range(args.steps):
        step(args.warmup + s)
    dt = time.perf_counter() - t0
    pos = sum(positions(ws[n]) // ws[n]["B"] for n in STEP)  # one sequence of each
    value = pos * args.steps / dt
    sample = (f"one sequence of each of the {len(STEP)} step workload(s) per step "
              f"({', '.join(STEP)}), in parallel threads")
    print(json.dumps({
        "impl": "reference", "metric": "verified positions/s", "value": value,
        "unit": "positions/s", "n_gpus": args.gpus, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": "spec_verify step: " + " + ".join(STEP),
                   "positions_per_step": pos, "sample": sample},
        "cpu_baseline": {"value": value, "unit": "positions/s", "cores": cores,
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "positions/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }))


# --------------------------------------------------------------------- ours

def oracle_call(w: dict, threads: int) -> dict:
    """The CPU oracle on every sequence of one workload."""
    import oracle

    if w["mode"] == "stochastic":
        return oracle.verify_stochastic(w["target"], w["t_dtype"], w["draft"], w["d_dtype"],
                                        w["tokens"], w["temperature"], w["seed"],
                                        threads=threads)
    if w["mode"] == "greedy":
        return oracle.verify_greedy(w["target"], w["t_dtype"], w["tokens"], threads=threads)
    if w["mode"] == "multi_rows":
        return oracle.verify_multi_rows(w["rows"], w["t_dtype"], w["row_of"], w["tokens"],
                                        threads=threads)
    if w["mode"] == "tree":
        return oracle.verify_tree_greedy(w["node_logits"], w["t_dtype"], w["parent"],
                                         w["tokens"], threads=threads)
    if w["mode"] == "tree_stochastic":
        return oracle.verify_tree_stochastic(w["node_logits"], w["t_dtype"], w["parent"],
                                             w["tokens"], w["temperature"], w["seed"],
                                             threads=threads)
    if w["mode"] == "threshold":
        return oracle.verify_threshold(w["target"], w["t_dtype"], w["tokens"], w["temperature"],
                                       w["threshold"], threads=threads)
    return oracle.verify_multi(w["target"], w["t_dtype"], w["tokens"], threads=threads)


def oracle_baseline(ws: dict) -> tuple[dict, dict]:
    """The CPU oracle on one full step (all sequences of the step workloads),
    all host cores; repeated while under 5 s of wall time (at most 3 times).
    Returns the cpu_baseline record and the oracle's outcome per workload
    (first repetition)."""
    import oracle

    oracle.build()
    cores = os.cpu_count() or 1
    reps, t_total, outcome, per_s = 0, 0.0, {}, {}
    while reps < 3 and t_total < 5.0:
        t0 = time.perf_counter()
        for name in STEP:
            t1 = time.perf_counter()
            o = oracle_call(ws[name], cores)
            per_s.setdefault(name, time.perf_counter() - t1)
            outcome.setdefault(name, o)
        t_total += time.perf_counter() - t0
        reps += 1
    pos = sum(positions(ws[n]) for n in STEP) * reps
    return ({"value": pos / t_total, "unit": "positions/s", "cores": cores, "kind": "oracle",
             "sample": f"{reps} full step(s): every sequence of the {len(STEP)} workload(s) "
                       f"({pos // reps} positions per step), {t_total:.1f} s",
             "seconds_per_call": {n: round(v, 4) for n, v in per_s.items()}}, outcome)


def branch_lengths(w: dict) -> np.ndarray:
    """Accepted length of every branch of a multi-candidate workload, from the
    oracle's greedy verify of each branch on its own rows."""
    import oracle

    B, G, k = w["B"], w["G"], w["k"]
    o = oracle.verify_greedy(w["target"].reshape(B * G, k + 1, w["V"]), w["t_dtype"],
                             w["tokens"].reshape(B * G, k), threads=os.cpu_count() or 1)
    return o["accepted_len"].reshape(B, G)


def parity_record(w: dict, gpu: dict, o: dict) -> dict:
    """The GPU's outputs of the timed launch configuration against the oracle:
    exact for greedy and multi-candidate; for stochastic verify exact except
    sequences where an oracle decision was a near tie (an acceptance margin
    |u - p/q| at an examined position, or the top-2 Gumbel-max score gap,
    below 1e-5), which are counted."""
    keys = [k for k in ("best_candidate", "accepted_len", "out_tokens", "path") if k in gpu]
    mism = np.zeros(w["B"], bool)
    for key in keys:
        g, want = gpu[key], o[key]
        mism |= (g != want) if g.ndim == 1 else (g != want).any(axis=1)
    rec = {"sequences": int(w["B"]), "mismatches": int(mism.sum())}
    if w["mode"] == "stochastic":
        k, n = w["k"], o["accepted_len"]
        near = o["gaps"] < NEAR_TIE
        for b in range(w["B"]):
            if k > 0:
                near[b] |= bool((o["margins"][b, : min(int(n[b]), k - 1) + 1] < NEAR_TIE).any())
        rec.update(near_ties=int(near.sum()),
                   mismatches_outside_near_ties=int((mism & ~near).sum()),
                   min_gap=float(o["gaps"].min()),
                   rule="exact except near ties (oracle margin or gap < 1e-5)")
    else:
        rec["rule"] = "bit-exact"
    return rec


def run_ours(args, rank: int, world: int, dist) -> None:
    import torch

    import speculative_decoding_verification_88_b200 as sv
    import workloads
    from speculative_decoding_verification_88_b200 import build as libbuild

    if rank == 0:
        libbuild.build()
    if dist is not None:
        dist.barrier()
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    stream = torch.cuda.current_stream(dev)

    # inputs (seeded, synthetic; each rank its own batch through seq_offset)
    threads = max(1, (os.cpu_count() or 1) // max(1, world))
    over = {"B": args.batch} if args.batch else {}
    lat = [n for n in LATENCY if n not in STEP] if not args.only else []
    ws = {n: workloads.make(n, threads=threads, **over) for n in STEP + lat}
    calls, host, devbuf = {}, {}, {}
    extra = {n: [] for n in STEP + lat}  # further inputs: (pinned host, device) pairs
    for name in STEP + lat:
        w = ws[name]
        key = "rows" if "rows" in w else ("node_logits" if "node_logits" in w else "target")
        t_h = workloads.as_torch(w[key], w["t_dtype"]).pin_memory()
        tok_h = torch.from_numpy(w["tokens"]).pin_memory()
        d_h = workloads.as_torch(w["draft"], w["d_dtype"]).pin_memory() if "draft" in w else None
        t_d, tok_d = t_h.to(dev), tok_h.to(dev)
        d_d = d_h.to(dev) if d_h is not None else None
        wsp = sv.Workspace(dev)
        B = w["B"]
        width = w["N"] if w["mode"] in TREE_MODES else w["k"] + 1
        if w["mode"] in ("multi", "multi_rows"):
            out = {"best_candidate": torch.empty(B, dtype=torch.int32, device=dev)}
        elif w["mode"] in TREE_MODES:
            out = {"path": torch.empty((B, width), dtype=torch.int32, device=dev)}
        else:
            out = {}
        out["accepted_len"] = torch.empty(B, dtype=torch.int32, device=dev)
        out["out_tokens"] = torch.empty((B, width), dtype=torch.int32, device=dev)
        if w["mode"] == "stochastic":
            off = rank * B
            fn = (lambda w=w, t=t_d, d=d_d, tok=tok_d, o=out, wsp=wsp, off=off:
                  sv.stochastic(t, d, tok, w["temperature"], w["seed"], off, out=o, workspace=wsp))
        elif w["mode"] == "greedy":
            fn = lambda t=t_d, tok=tok_d, o=out, wsp=wsp: sv.greedy(t, tok, out=o, workspace=wsp)
        elif w["mode"] == "threshold":
            fn = (lambda w=w, t=t_d, tok=tok_d, o=out, wsp=wsp:
                  sv.threshold(t, tok, w["temperature"], w["threshold"], out=o, workspace=wsp))
        elif w["mode"] == "tree":
            par_h = torch.from_numpy(w["parent"]).pin_memory()
            par = par_h.to(dev)
            extra[name].append((par_h, par))
            fn = (lambda t=t_d, pa=par, tok=tok_d, o=out, wsp=wsp:
                  sv.tree_greedy(t, pa, tok, out=o, workspace=wsp))
        elif w["mode"] == "tree_stochastic":
            par_h = torch.from_numpy(w["parent"]).pin_memory()
            par = par_h.to(dev)
            extra[name].append((par_h, par))
            off = rank * B
            fn = (lambda w=w, t=t_d, pa=par, tok=tok_d, o=out, wsp=wsp, off=off:
                  sv.tree_stochastic(t, pa, tok, w["temperature"], w["seed"], off, out=o,
                                     workspace=wsp))
        elif w["mode"] == "multi_rows":
            rmap_h = torch.from_numpy(w["row_of"]).pin_memory()
            rmap = rmap_h.to(dev)
            extra[name].append((rmap_h, rmap))
            fn = (lambda t=t_d, rm=rmap, tok=tok_d, o=out, wsp=wsp:
                  sv.multi_candidate_rows(t, rm, tok, out=o, workspace=wsp))
        else:
            fn = (lambda t=t_d, tok=tok_d, o=out, wsp=wsp:
                  sv.multi_candidate(t, tok, out=o, workspace=wsp))
        calls[name] = fn
        host[name] = (t_h, d_h, tok_h, {kk: torch.empty_like(v, device="cpu").pin_memory()
                                        for kk, v in out.items()})
        devbuf[name] = (t_d, d_d, tok_d, out)

    # warm-up; the outputs of these calls (the launch configuration timed
    # below) are kept for the parity record
    for _ in range(max(1, args.warmup)):
        for name in STEP + lat:
            calls[name]()
    torch.cuda.synchronize()
    gpu_out = {n: {kk: v.cpu().numpy() for kk, v in devbuf[n][3].items()} for n in STEP + lat}

    # One step as a CUDA graph, the way a serving loop issues it: the four
    # verify launches back to back with no host work between them.  The
    # timed graph holds the launches alone; a second graph of the same calls
    # with external event nodes around each call times the calls inside the
    # step (an event pair costs a call a few microseconds, so it stays out of
    # the timed step).
    ev = {n: (torch.cuda.Event(enable_timing=True, external=True),
              torch.cuda.Event(enable_timing=True, external=True)) for n in STEP}
    gstream = torch.cuda.Stream(dev)
    gstream.wait_stream(stream)
    with torch.cuda.stream(gstream):
        for name in STEP:
            calls[name]()
    gstream.synchronize()
    graph = torch.cuda.CUDAGraph()
    n0 = sv.launch_count()
    with torch.cuda.graph(graph, stream=gstream):
        for name in STEP:
            calls[name]()
    per_replay = sv.launch_count() - n0  # kernels of ours in one replay
    graph_ev = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph_ev, stream=gstream):
        for name in STEP:
            a, b = ev[name]
            a.record()
            calls[name]()
            b.record()
    for _ in range(3):
        graph.replay()
        graph_ev.replay()
    torch.cuda.synchronize()

    # timed region: device-resident inputs, K replays between two events on
    # the launching stream
    K = args.steps
    e_start, e_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    uuid = str(torch.cuda.get_device_properties(dev).uuid)
    gpu_uuid = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
    sampler = ClockSampler(gpu_uuid)
    fast = NvmlSampler(gpu_uuid)
    time.sleep(1.0 if sampler.proc is not None else 0.0)
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    t0 = time.time()
    e_start.record(stream)
    for s in range(K):
        graph.replay()
    e_end.record(stream)
    torch.cuda.synchronize()
    t1 = time.time()
    launches = K * per_replay
    clocks = fast.stop(t0, t1) or sampler.stop(t0, t1)
    if sampler.proc is not None and sampler.proc.poll() is None:
        sampler.stop(t0, t1)
    elapsed_ms = e_start.elapsed_time(e_end)
    if dist is not None:
        t = torch.tensor([elapsed_ms], device=dev, dtype=torch.float64)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        elapsed_ms = float(t.item())
        dist.barrier()
    ms_step = elapsed_ms / K
    pos_step = sum(positions(ws[n]) for n in STEP)
    value = pos_step * world / (ms_step * 1e-3)

    # per-call times inside the step: replays of the graph with event nodes,
    # read one at a time
    samples = {n: [] for n in STEP}
    for _ in range(max(K, 200)):
        graph_ev.replay()
        torch.cuda.synchronize()
        for name in STEP:
            a, b = ev[name]
            samples[name].append(a.elapsed_time(b))
    us_call = {n: statistics.fmean(samples[n]) * 1e3 for n in STEP}

    # latency-bound workloads: one call per graph, replayed back to back
    for name in lat:
        g1 = torch.cuda.CUDAGraph()
        with torch.cuda.stream(gstream):
            calls[name]()
        gstream.synchronize()
        with torch.cuda.graph(g1, stream=gstream):
            calls[name]()
        for _ in range(5):
            g1.replay()
        reps = 500
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        a.record(stream)
        for _ in range(reps):
            g1.replay()
        b.record(stream)
        torch.cuda.synchronize()
        us_call[name] = a.elapsed_time(b) * 1e3 / reps

    # the oracle on the host cores: the CPU baseline, the outcomes that fix
    # the bytes each call must read, and the parity of the GPU's outputs
    cpu, outcome = None, None
    if rank == 0 and world == 1 and not args.skip_cpu_baseline:
        cpu, outcome = oracle_baseline(ws)
        for name in lat:  # timed too, though not part of the step's baseline
            t1 = time.perf_counter()
            outcome[name] = oracle_call(ws[name], os.cpu_count() or 1)
            cpu["seconds_per_call"][name] = round(time.perf_counter() - t1, 4)
        for name in STEP + lat:
            if ws[name]["mode"] == "multi":
                outcome[name]["branch_len"] = branch_lengths(ws[name])

    peak, peak_kind = measured_hbm_peak()
    per = {}
    for name in STEP + lat:
        us = us_call[name]
        full = full_bytes(ws[name])
        need = needed_bytes(ws[name], outcome[name] if outcome else None)
        rec = {"us_per_call": round(us, 2), "positions_per_s": positions(ws[name]) / (us * 1e-6),
               "in_step": name in STEP, "full_read_bytes": full,
               "full_read_gbs": full / (us * 1e-6) / 1e9}
        if name in samples:
            rec["us_spread"] = call_spread(samples[name])
        rec["frac_full_read"] = rec["full_read_gbs"] / peak
        if need is not None:
            rec["needed_bytes"] = need
            rec["needed_gbs"] = need / (us * 1e-6) / 1e9
            rec["frac_needed"] = rec["needed_gbs"] / peak
            rec["frac_needed_of_nominal"] = rec["needed_gbs"] / HBM_NOMINAL_GBS
            rec["parity"] = parity_record(ws[name], gpu_out[name], outcome[name])
        per[name] = rec
    d = per[DOMINANT]
    counted = "needed_gbs" if "needed_gbs" in d else "full_read_gbs"
    roofline = {"bound": "hbm", "achieved": d[counted], "peak": peak, "unit": "GB/s",
                "frac": d[counted] / peak,
                "traffic": recorded_traffic(DOMINANT, bool(args.batch)),
                "bytes_counted": ("needed: the rows the oracle's outcome requires (pairs "
                                  "0..n, target row k only when n = k)"
                                  if counted == "needed_gbs" else
                                  "full read: every logit row once"),
                "achieved_full_read": d["full_read_gbs"],
                "frac_of_nominal_8tbs": d[counted] / HBM_NOMINAL_GBS,
                "kernel": KERNEL_OF_MODE[ws[DOMINANT]["mode"]] + " (" + DOMINANT + ")",
                "peak_source": peak_kind + " (MEASURED_PEAKS.json hbm_gbs)"
                if peak_kind == "measured" else "fallback 6.65 TB/s"}

    # end to end through the public API with host buffers
    e2e = None
    if args.e2e_steps > 0:
        h2d = d2h = 0
        for name in STEP:
            t_h, d_h, tok_h, out_h = host[name]
            h2d += t_h.numel() * t_h.element_size() + tok_h.numel() * 4
            h2d += d_h.numel() * d_h.element_size() if d_h is not None else 0
            h2d += sum(h.numel() * h.element_size() for h, _ in extra[name])
            d2h += sum(v.numel() * 4 for v in out_h.values())

        def e2e_step():
            for name in STEP:
                t_h, d_h, tok_h, out_h = host[name]
                t_d, d_d, tok_d, out = devbuf[name]
                t_d.copy_(t_h, non_blocking=True)
                tok_d.copy_(tok_h, non_blocking=True)
                if d_h is not None:
                    d_d.copy_(d_h, non_blocking=True)
                for h, dv in extra[name]:
                    dv.copy_(h, non_blocking=True)
                calls[name]()
                for kk, v in out.items():
                    out_h[kk].copy_(v, non_blocking=True)

        e2e_step()
        torch.cuda.synchronize()
        if dist is not None:
            dist.barrier()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(args.e2e_steps):
            e2e_step()
        b.record(stream)
        torch.cuda.synchronize()
        e_ms = a.elapsed_time(b) / args.e2e_steps
        if dist is not None:
            t = torch.tensor([e_ms], device=dev, dtype=torch.float64)
            dist.all_reduce(t, op=dist.ReduceOp.MAX)
            e_ms = float(t.item())
        e2e = {"value": pos_step * world / (e_ms * 1e-3), "unit": "positions/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
               "ms_per_step": e_ms}

    if rank == 0:
        total_bytes = sum(per[n].get("needed_bytes", per[n]["full_read_bytes"]) for n in STEP)
        print(json.dumps({
            "metric": "verified positions/s", "value": value, "unit": "positions/s",
            "n_gpus": world, "steps": K, "warmup": args.warmup, "ms_per_step": ms_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "f32", "data": "synthetic (seeded numpy Philox; logits N(0, sigma^2), "
                                    "draft = target + noise, tokens from the draft softmax)",
            "config": {"workload": "spec_verify step: " + " + ".join(STEP),
                       "global_batch": sum(ws[n]["B"] for n in STEP) * world,
                       "positions_per_step": pos_step * world,
                       "bytes_per_step": total_bytes,
                       "step_gbs": total_bytes / (ms_step * 1e-3) / 1e9,
                       "latency_workloads": lat,
                       "latency_note": "timed alone, one call per replayed graph; not in the "
                                       "step or its positions/s",
                       "l2": "inputs larger than L2: 1.45 GB streamed per step, no buffer "
                             "re-read across steps from L2",
                       "parallelism": f"weak: {world} GPU(s), each its own batch, no collective",
                       "timing": "one step captured as a CUDA graph of the launches alone, "
                                 "replayed K times between two events; per-call times from a "
                                 "second graph of the same calls with event nodes around each"},
            "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e,
            "gpu_launches": launches, "clocks": clocks, "per_workload": per,
        }))


def select_workloads(only: str | None) -> None:
    """Restrict the step to one workload (profiling runs)."""
    global STEP, DOMINANT
    if only:
        import workloads

        if only not in workloads.WORKLOADS:
            raise SystemExit(f"--only must be one of {list(workloads.WORKLOADS)}")
        STEP = [only]
        DOMINANT = only


def main():
    ap = argparse.ArgumentParser(description=__doc__,
                                 formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--e2e-steps", type=int, default=10)
    ap.add_argument("--skip-cpu-baseline", action="store_true")
    ap.add_argument("--only", help="profiling: time only this workload of the step")
    ap.add_argument("--batch", type=int, default=0,
                    help="profiling: override the batch size B of the workloads")
    args = ap.parse_args()
    select_workloads(args.only)
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if world != args.gpus:
        ap.error(f"--gpus {args.gpus} but WORLD_SIZE={world}: launch N>1 with "
                 "python -m torch.distributed.run --nproc-per-node N")
    if args.impl == "reference":
        run_reference(args, rank)
        return
    dist = None
    if world > 1:
        import torch
        import torch.distributed as tdist

        local = int(os.environ.get("LOCAL_RANK", "0"))
        torch.cuda.set_device(local)
        tdist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                 device_id=torch.device("cuda", local))
        dist = tdist
    try:
        run_ours(args, rank, world, dist)
    finally:
        if dist is not None:
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
