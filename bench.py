#!/usr/bin/env python
"""Benchmark of the DSpark drafter-head hot path on B200.

One step = one draft block through the whole path: Markov-head drafting of gamma
tokens for every request (dspark_draft_step), confidence + STS + survival product
(dspark_confidence_sts), the prefix scheduler (dspark_schedule_prefix) and strict
prefix-match verification (dspark_verify_prefix).  On one GPU with the Markov head the
step is the single call dspark_step (one launch for B <= 128); with the RNN head, the
lagged schedule or several ranks it is the calls above in sequence.  The metric is
draft tokens per second, B * gamma / step time, summed over ranks.

    python bench.py [--gpus N --steps K --warmup W] [--workload qwen3-8b]
    python bench.py --impl reference ...   # the fp64 CPU oracle on a bounded sample
    python bench.py --stage sts-fit        # fitting the STS temperatures (offline calibration)

With N > 1 (torchrun, one process per GPU) every rank drafts its own B requests
(weak scaling) and the survival scores of all ranks are all-gathered over NCCL
before the scheduler, which then decides verify lengths over the global batch.

Inputs are synthetic and seeded (synth.py).  U alone (311 MB at the default
workload) is larger than L2, and L2 is also flushed between timed steps.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

PARITY_MACS = 3.5e11          # oracle multiply-adds spent on the bench line's parity check
METRIC = "draft tokens/s (Markov head+confidence+schedule+verify); % of HBM/TC roofline"
UNIT = "tokens/s"
CSRC = os.path.join(ROOT, "speculative_decoding_drafter_head_b200", "csrc")
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "markov_draft_traffic.json")


def _peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            m = json.load(f)
        return float(m["hbm_gbs"]), float(m["bf16_tflops"]), "measured"
    except Exception:
        return 6650.0, 1590.0, "fallback"


def _kernel_sha(sources):
    """Hash of a kernel's source files with comments and blank space removed, so that a
    committed DRAM-traffic figure stays attached to the code it was measured on."""
    import re
    src = ""
    for name in sources:
        with open(os.path.join(CSRC, name), encoding="utf-8") as f:
            src += f.read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    src = re.sub(r"//[^\n]*", "", src)
    src = re.sub(r"\s+", " ", src).strip()
    return hashlib.sha256(src.encode()).hexdigest()[:16]


def _traffic_per_launch(workload_name, gamma):
    """DRAM bytes per draft launch from the committed ncu summary, if the kernel is unchanged.

    Each entry names the workload and draft length it stands for and the source files of
    the kernel it was measured on, with their hash; an entry whose files have changed
    since is ignored."""
    try:
        with open(TRAFFIC_FILE) as f:
            t = json.load(f)
        for e in t.get("entries", []):
            if (e.get("workload") == workload_name and int(e.get("gamma", -1)) == gamma
                    and e.get("kernel_sha") == _kernel_sha(e["sources"])):
                return float(e["dram_bytes_per_launch"])
    except Exception:
        pass
    return None


_NVML_SAMPLER = r"""
import sys, time
import pynvml as N
N.nvmlInit()
uuid, index, period = sys.argv[1], int(sys.argv[2]), float(sys.argv[3])
h = None
if uuid:
    try:
        h = N.nvmlDeviceGetHandleByUUID(uuid)
    except Exception:
        h = None
if h is None:
    h = N.nvmlDeviceGetHandleByIndex(index)
mx = N.nvmlDeviceGetMaxClockInfo(h, N.NVML_CLOCK_SM)
print("ready", mx, flush=True)
while True:
    t = time.monotonic_ns()
    sm = N.nvmlDeviceGetClockInfo(h, N.NVML_CLOCK_SM)
    why = N.nvmlDeviceGetCurrentClocksEventReasons(h)
    mw = N.nvmlDeviceGetPowerUsage(h)
    print(t, sm, why, mw, flush=True)
    time.sleep(period)
"""


class ClockSampler:
    """SM clock and clock-event reasons sampled by NVML in a separate process (every
    0.5 ms, so the GIL and the host's synchronize do not hold it up) with timestamps on
    the host's monotonic clock; only the samples taken between begin() and end() -- the
    timed region -- are summarised.  Falls back to nvidia-smi (200 ms) without NVML."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    # NVML clock-event reason bits (nvml.h): sw power cap 0x4, hw slowdown 0x8,
    # sw thermal 0x20, hw thermal 0x40, hw power brake 0x80
    BITS = {"sw_power_cap": 0x4, "hw_slowdown": 0x8 | 0x80, "sw_thermal_slowdown": 0x20,
            "hw_thermal_slowdown": 0x40}

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.lines = []
        self.t0 = self.t1 = None
        self.mode = None
        self.max_mhz = None

    def _nvml_target(self):
        """(uuid, NVML index) of the CUDA device this process drives."""
        uuid = ""
        try:
            import torch
            u = str(torch.cuda.get_device_properties(torch.cuda.current_device()).uuid)
            if u:
                uuid = u if u.startswith("GPU-") else "GPU-" + u
        except Exception:                               # noqa: BLE001
            pass
        index = self.index
        vis = os.environ.get("CUDA_VISIBLE_DEVICES", "")
        ids = [v for v in vis.split(",") if v.strip()]
        if ids and all(v.strip().isdigit() for v in ids) and self.index < len(ids):
            index = int(ids[self.index])
        return uuid, index

    def start(self):
        try:
            uuid, index = self._nvml_target()
            self.proc = subprocess.Popen(
                [sys.executable, "-c", _NVML_SAMPLER, uuid, str(index), "0.0005"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            first = self.proc.stdout.readline().split()
            if len(first) == 2 and first[0] == "ready":
                self.mode, self.max_mhz = "nvml", float(first[1])
            else:
                self.proc.kill()
                self.proc = None
        except Exception:                               # noqa: BLE001
            self.proc = None
        if self.proc is None:
            try:
                self.proc = subprocess.Popen(
                    ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.FIELDS}",
                     "--format=csv,noheader,nounits", "-lms", "200"],
                    stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
                self.mode = "nvidia-smi"
            except Exception:                           # noqa: BLE001
                self.proc = None
                return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.monotonic_ns(), line.strip()))

    def begin(self):
        """Start of the timed region (after the synchronize that opens it)."""
        self.t0 = time.monotonic_ns()

    def end(self):
        """End of the timed region (after the synchronize that closes it)."""
        self.t1 = time.monotonic_ns()

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:                               # noqa: BLE001
            self.proc.kill()
        self.thread.join(timeout=2)
        t0 = self.t0 if self.t0 is not None else 0
        t1 = self.t1 if self.t1 is not None else 2 ** 63
        rows = []                               # (t, sm MHz, max MHz, reasons, watts)
        if self.mode == "nvml":
            for _, ln in self.lines:
                parts = ln.split()
                if len(parts) != 4:
                    continue
                t, sm, why = int(parts[0]), float(parts[1]), int(parts[2])
                rows.append((t, sm, self.max_mhz,
                             {n for n, bit in self.BITS.items() if why & bit},
                             float(parts[3]) / 1e3))
        else:
            names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown",
                     "sw_power_cap"]
            for t, ln in self.lines:
                parts = [p.strip() for p in ln.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    sm, mx, w = float(parts[1]), float(parts[2]), float(parts[3])
                except ValueError:
                    continue
                rows.append((t, sm, mx, {n for n, v in zip(names, parts[5:9])
                                         if v.lower().startswith("active")}, w))
        inside = [r for r in rows if t0 <= r[0] <= t1]
        if not inside:                                  # region shorter than one period:
            after = [r for r in rows if r[0] >= t0]     # the first sample after it began
            inside = after[:1]
        if not inside:
            return None
        reasons = set().union(*(r[3] for r in inside))
        return {"sm_mhz": statistics.median(r[1] for r in inside),
                "sm_min_mhz": min(r[1] for r in inside), "sm_max_mhz": inside[-1][2],
                "reasons": sorted(reasons), "samples": len(inside),
                "power_w": round(statistics.median(r[4] for r in inside), 1),
                "source": self.mode,
                "window_ms": round((t1 - t0) / 1e6, 3) if self.t1 is not None else None}


def workload_config(wl, world=1):
    """The `config` object both arms print (identical keys and values)."""
    return {"workload": wl.name, "B_per_gpu": wl.B, "gamma": wl.gamma, "V": wl.V, "r": wl.r,
            "d": wl.d, "mode": "gumbel" if wl.mode else "greedy", "parallelism": f"dp{world}",
            "l2_flush": True}


def cpu_oracle_step(wl, inp, bs, target_rows, oracle, Whh=None):
    """The oracle's whole path on the listed requests (one bounded sample of a step)."""
    bs = list(bs)
    U = synth.u_requests(wl, bs) if inp.U is None else inp.U[bs]
    h = synth.h_requests(wl, bs) if inp.h is None else inp.h[bs]
    if Whh is None:
        x, _, _ = oracle.draft(U, inp.anchor[bs], inp.W1, inp.W2, mode=wl.mode, tau=wl.tau,
                               seed=wl.seed, b_index=np.array(bs, np.int32))
    else:
        x, _, _ = oracle.draft_rnn(U, inp.anchor[bs], inp.W1, inp.W2, Whh, mode=wl.mode,
                                   tau=wl.tau, seed=wl.seed, b_index=np.array(bs, np.int32))
    conf = oracle.confidence(h, inp.anchor[bs], x, inp.W1, inp.w, inp.b_conf, inp.T)
    sub = wl.with_(B=len(bs))
    L, _, _, _ = oracle.schedule(conf["P32"], synth.tstep_us(sub))
    oracle.verify(x, L, target_rows)
    return x


def run_reference(args, wl):
    """The CPU oracle as the reference arm: bounded samples of the workload per step."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import oracle
    oracle.build()
    inp = synth.make_inputs(wl, with_u=False, with_h=False)
    sample = list(range(min(wl.B, args.ref_sample)))
    inp.U = synth.u_requests(wl, sample)          # inputs are drawn outside the timed steps
    inp.h = synth.h_requests(wl, sample)
    target = synth.targets(wl, np.zeros((len(sample), wl.gamma), np.int32), sample)
    for _ in range(args.warmup):
        cpu_oracle_step(wl, inp, sample, target, oracle)
    t = []
    for _ in range(args.steps):
        t0 = time.perf_counter()
        cpu_oracle_step(wl, inp, sample, target, oracle)
        t.append(time.perf_counter() - t0)
    sec = sum(t)
    value = len(sample) * wl.gamma * args.steps / sec
    cores = oracle.num_threads()
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * sec / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": workload_config(wl, int(os.environ.get("WORLD_SIZE", "1"))),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": f"{len(sample)} of {wl.B} requests per step, whole path"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def cpu_baseline(wl, inp, target, budget_s, Whh=None):
    """Time the oracle's whole step on the host cores for about budget_s seconds.

    The sample grows from one request to the whole batch; when the whole batch takes
    less than the budget, the full step is repeated until the budget is spent.
    """
    import oracle
    oracle.build()
    n = 1
    while True:
        t0 = time.perf_counter()
        cpu_oracle_step(wl, inp, list(range(n)), target[:n], oracle, Whh)
        dt = time.perf_counter() - t0
        if n >= wl.B or dt >= budget_s / 4:
            break
        n = min(wl.B, max(n + 1, int(n * min(8.0, budget_s / 4 / max(dt, 1e-3)))))
    reps, total = 1, dt
    while total < budget_s:
        t0 = time.perf_counter()
        cpu_oracle_step(wl, inp, list(range(n)), target[:n], oracle, Whh)
        total += time.perf_counter() - t0
        reps += 1
    return {"value": reps * n * wl.gamma / total, "unit": UNIT, "cores": oracle.num_threads(),
            "kind": "oracle", "sample": f"{n} of {wl.B} requests x {reps} full steps "
                                        f"(draft, confidence, schedule, verify), {total:.1f} s"}


def parity_report(wl, inp, target, out, oracle, Whh=None, n_rows=None, schedule=True):
    """The GPU outputs of one timed step against the oracle (outside every timed region).

    Drafts: every position of the first n_rows requests against the oracle run
    teacher-forced on the GPU's previous tokens; tokens may differ only where the oracle's
    top-2 gap is below 2e-2 (near ties), the logit at a matching token within 2e-2.
    Confidence: c and P against the oracle fed the GPU's drafts.  Scheduler and verify:
    bit for bit against the oracle fed the GPU's scores and lengths.
    """
    tol = 2e-2
    n = wl.B if n_rows is None else min(n_rows, wl.B)
    bs = list(range(n))
    x, lx = out["x"][:n], out["lx"][:n]
    prev = np.concatenate([inp.anchor[:n, None], x[:, :-1]], axis=1).astype(np.int32)
    U = synth.u_requests(wl, bs) if inp.U is None else inp.U[:n]
    if Whh is None:
        xo, lo, go = oracle.draft(U, inp.anchor[:n], inp.W1, inp.W2, mode=wl.mode, tau=wl.tau,
                                  seed=wl.seed, b_index=np.array(bs, np.int32), forced_prev=prev)
    else:
        xo, lo, go = oracle.draft_rnn(U, inp.anchor[:n], inp.W1, inp.W2, Whh, mode=wl.mode,
                                      tau=wl.tau, seed=wl.seed, b_index=np.array(bs, np.int32),
                                      forced_prev=prev)
    same = x == xo
    rep = {"rows": n, "positions": int(x.size), "compared": int(same.sum()),
           "near_ties": int((~same & (go < tol)).sum()),
           "hard_mismatch": int((~same & (go >= tol)).sum()),
           "max_logit_err": float(np.abs(lx[same] - lo[same]).max()) if same.any() else 0.0}
    h = synth.h_requests(wl, bs) if inp.h is None else inp.h[:n]
    conf = oracle.confidence(h, inp.anchor[:n], x, inp.W1, inp.w, inp.b_conf, inp.T)
    rep["max_c_err"] = float(np.abs(out["c"][:n] - conf["c"]).max())
    if schedule:            # the scores of this step fed this step's scheduler
        rep["max_P_err"] = float(np.abs(out["P"][:n] - conf["P64"]).max())
        L_or, N_or, F_or, _ = oracle.schedule(out["P"], inp.Tstep)
        rep["schedule_bit_exact"] = bool((out["L"] == L_or).all() and out["N"] == N_or and
                                         out["F"] == F_or)
    a_or, b_or = oracle.verify(out["x"], out["L"], target)
    rep["verify_bit_exact"] = bool((out["acc"] == a_or).all() and (out["bonus"] == b_or).all())
    rep["ok"] = bool(rep["hard_mismatch"] == 0 and rep["max_logit_err"] <= tol and
                     rep["max_c_err"] <= tol and rep.get("max_P_err", 0.0) <= tol and
                     rep.get("schedule_bit_exact", True) and rep["verify_bit_exact"])
    return rep


STS_METRIC = "STS fit candidate evaluations/s (blocks x gamma x grid temperatures)"
STS_UNIT = "evaluations/s"


def run_sts_fit(args):
    """Time dspark_sts_fit on the held-out calibration set (65536 blocks, gamma = 16,
    451 temperatures 0.5..5.0, 15 bins); the oracle's fit on a subset is the CPU baseline."""
    import torch
    import speculative_decoding_drafter_head_b200 as ds

    N, gamma = synth.STS_CALIBRATION_N, synth.STS_CALIBRATION_GAMMA
    n_t, n_bins = 451, 15
    z_h, acc_h = synth.calibration_set(N, gamma, 0)
    z, acc = torch.from_numpy(z_h).cuda(), torch.from_numpy(acc_h).cuda()
    ws = torch.empty(ds.sts_fit_workspace_bytes(N, gamma, n_t, n_bins), dtype=torch.uint8,
                     device="cuda")
    idx = torch.empty(gamma, dtype=torch.int32, device="cuda")
    T = torch.empty(gamma, dtype=torch.float32, device="cuda")
    e = torch.empty(gamma, dtype=torch.float64, device="cuda")
    stream = torch.cuda.current_stream()
    for _ in range(args.warmup):
        ds.sts_fit(z, acc, idx, T, e, ws)
    torch.cuda.synchronize()
    assert ds.get_error() == 0
    clocks = ClockSampler(int(os.environ.get("LOCAL_RANK", "0")))
    clocks.start()
    time.sleep(0.05)
    clocks.begin()
    evs = []
    for _ in range(args.steps):
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        ds.sts_fit(z, acc, idx, T, e, ws)
        e1.record(stream)
        evs.append((e0, e1))
    torch.cuda.synchronize()
    clocks.end()
    clk = clocks.stop()
    ms = [a.elapsed_time(b) for a, b in evs]
    evals = float(N) * gamma * n_t
    value = evals * args.steps / (sum(ms) / 1e3)

    # e2e: calibration set copied from pinned host memory, temperatures read back
    z_pin, acc_pin = torch.from_numpy(z_h).pin_memory(), torch.from_numpy(acc_h).pin_memory()
    T_pin = torch.empty(gamma, dtype=torch.float32).pin_memory()
    e2e = []
    for it in range(args.steps + 1):
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        z.copy_(z_pin, non_blocking=True)
        acc.copy_(acc_pin, non_blocking=True)
        ds.sts_fit(z, acc, idx, T, e, ws)
        T_pin.copy_(T, non_blocking=True)
        e1.record(stream)
        if it:
            e2e.append((e0, e1))
    torch.cuda.synchronize()
    e2e_ms = sum(a.elapsed_time(b) for a, b in e2e)

    import oracle
    oracle.build()
    n_cpu = 4096
    t0 = time.perf_counter()
    oracle.sts_fit(z_h[:n_cpu], acc_h[:n_cpu], n_t=n_t, n_bins=n_bins)
    cpu_s = time.perf_counter() - t0
    line = {
        "metric": STS_METRIC, "value": value, "unit": STS_UNIT, "n_gpus": 1, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": statistics.mean(ms), "higher_is_better": True,
        "scaling": "none", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": f"sts-calibration N={N} gamma={gamma} n_t={n_t} bins={n_bins}",
                   "l2_flush": False, "inputs_bytes": int(z_h.nbytes + acc_h.nbytes)},
        "roofline": {"bound": "alu", "kernel": "sts_hist_kernel",
                     "note": "fp64 exp/divide per candidate; fp64 pipe share from ncu"},
        "cpu_baseline": {"value": n_cpu * gamma * n_t / cpu_s, "unit": STS_UNIT,
                         "cores": oracle.num_threads(), "kind": "oracle",
                         "sample": f"oracle fit of the first {n_cpu} of {N} blocks"},
        "e2e": {"value": evals * args.steps / (e2e_ms / 1e3), "unit": STS_UNIT,
                "h2d_bytes_per_step": int(z_h.nbytes + acc_h.nbytes),
                "d2h_bytes_per_step": gamma * 4},
        "gpu_launches": (2 * gamma) * args.steps,
        "clocks": clk,
        "T": [round(float(v), 2) for v in T.cpu()],
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="qwen3-8b", choices=sorted(synth.WORKLOADS))
    ap.add_argument("--gamma", type=int, default=None,
                    help="draft length instead of the workload's own (e.g. a short case to profile)")
    ap.add_argument("--ref-sample", type=int, default=4)
    ap.add_argument("--cpu-budget", type=float, default=12.0)
    ap.add_argument("--eager", action="store_true", help="launch kernels one by one (no CUDA graph)")
    ap.add_argument("--stage", default="path", choices=["path", "sts-fit"],
                    help="path: the per-step hot path; sts-fit: the temperature fit")
    ap.add_argument("--head", default="markov", choices=["markov", "rnn"],
                    help="sequential block: Markov head, or RNN head (Elman reading)")
    ap.add_argument("--schedule", default="sync", choices=["sync", "lagged"],
                    help="sync: schedule on this step's scores; lagged: on the scores of two "
                         "steps earlier, on a side stream that overlaps the draft kernel")
    args = ap.parse_args()
    wl = synth.WORKLOADS[args.workload]
    if args.gamma is not None:
        import re
        wl = wl.with_(gamma=args.gamma, name=re.sub(r"gamma=\d+", f"gamma={args.gamma}", wl.name))
    if args.stage == "sts-fit":
        if int(os.environ.get("RANK", "0")) == 0 and args.impl == "ours":
            run_sts_fit(args)
        return

    if args.impl == "reference":
        run_reference(args, wl)
        return

    import torch
    import torch.distributed as dist
    import speculative_decoding_drafter_head_b200 as ds
    from speculative_decoding_drafter_head_b200 import sharding

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    B, gamma, V = wl.B, wl.gamma, wl.V
    wlg = wl.with_(B=B * world)                 # the global batch across ranks
    b0 = sharding.request_offset(rank, B)
    bs = range(b0, b0 + B)

    # ---------------- inputs (host, seeded) and device copies
    W1h, W2h = synth.w1(wl), synth.w2(wl)
    Uh = synth.u_requests(wlg, bs)
    hh = synth.h_requests(wlg, bs)
    anchor_h = synth.anchors(wlg)[b0:b0 + B].copy()
    wh, Th = synth.conf_w(wl), synth.temperatures(wl)
    Tstep_h = synth.tstep_us(wlg)

    def bf(a):
        return torch.from_numpy(a).view(torch.bfloat16).cuda()

    U, h, W1, W2, w = bf(Uh), bf(hh), bf(W1h), bf(W2h), bf(wh)
    rnn = args.head == "rnn"
    Whh = bf(synth.whh(wl)) if rnn else None

    def draft(**kw):
        if rnn:
            ds.draft_step_rnn(U, anchor, W1, W2, Whh, x, lx, ws, **kw)
        else:
            ds.draft_step(U, anchor, W1, W2, x, lx, ws, **kw)
    anchor = torch.from_numpy(anchor_h).cuda()
    T = torch.from_numpy(Th).cuda()
    Tstep = torch.from_numpy(Tstep_h).cuda()
    ws = torch.empty(ds.workspace_bytes(B * world, gamma, V), dtype=torch.uint8, device="cuda")
    x = torch.empty(B, gamma, dtype=torch.int32, device="cuda")
    lx = torch.empty(B, gamma, dtype=torch.float32, device="cuda")
    c = torch.empty(B, gamma, dtype=torch.float32, device="cuda")
    P = torch.empty(B, gamma, dtype=torch.float32, device="cuda")
    Pg = torch.empty(B * world, gamma, dtype=torch.float32, device="cuda")
    Lg = torch.empty(B * world, dtype=torch.int32, device="cuda")
    Nst = torch.empty(1, dtype=torch.int32, device="cuda")
    obj = torch.empty(1, dtype=torch.float64, device="cuda")
    acc = torch.empty(B, dtype=torch.int32, device="cuda")
    bonus = torch.empty(B, dtype=torch.int32, device="cuda")
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")   # > 126 MB L2
    stream = torch.cuda.current_stream()

    # target tokens: the target model agrees with the drafts w.p. q_k (from a first draft)
    draft(mode=wl.mode, temperature=wl.tau, seed=wl.seed, b_offset=b0)
    torch.cuda.synchronize()
    target_h = synth.targets(wlg, x.cpu().numpy(), bs)
    target = torch.from_numpy(target_h).cuda()

    ev_draft = []
    lagged = args.schedule == "lagged"
    lsched = None
    last_L = [None]
    if lagged:
        from speculative_decoding_drafter_head_b200 import pipeline
        lsched = pipeline.LaggedScheduler(B * world, gamma, Tstep, lag=2)
    step_no = [0]

    # the Markov head drafts and scores in one call (one launch, two for Gumbel-max above
    # 128 requests); the RNN
    # head drafts, then the confidence kernel scores
    fused = not rnn

    def draft_and_score(P_dst):
        if fused:
            ds.draft_confidence_step(U, anchor, W1, W2, h, w, wl.b_conf, T, x, lx, c, P_dst, ws,
                                     mode=wl.mode, temperature=wl.tau, seed=wl.seed, b_offset=b0)
        else:
            draft(mode=wl.mode, temperature=wl.tau, seed=wl.seed, b_offset=b0)

    def score(P_dst):
        if not fused:
            ds.confidence_sts(h, anchor, x, W1, w, wl.b_conf, T, c, P_dst)

    # one process and this step's scores: the whole step is one call (one launch for
    # B <= 128 and B gamma <= 1024, the calls in sequence above)
    one_call = fused and world == 1 and not lagged

    def step(record=None):
        t = step_no[0]
        step_no[0] += 1
        if one_call and record is None:
            ds.step(U, anchor, W1, W2, h, w, wl.b_conf, T, Tstep, target, x, lx, c, P, Lg, Nst,
                    obj, acc, bonus, ws, mode=wl.mode, temperature=wl.tau, seed=wl.seed,
                    b_offset=b0)
            last_L[0] = Lg
            return
        e0 = e1 = None
        P_dst = lsched.scores(t) if lagged and world == 1 else P
        if record is not None:
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record(stream)
        draft_and_score(P_dst)
        if record is not None:
            e1.record(stream)
            record.append((e0, e1))
        if lagged:
            lsched.begin_step(t)                   # overlaps the confidence kernel
            score(P_dst)
            if world > 1:
                sharding.gather_scores(P, out=lsched.scores(t))
            Lt = lsched.lengths(t, workspace=ws)
            Lloc = sharding.local_lengths(Lt, rank, B) if world > 1 else Lt
        else:
            score(P)
            if world > 1:
                sharding.gather_scores(P, out=Pg)
                ds.schedule_prefix(Pg, Tstep, Lg, Nst, obj, ws)
                Lloc = sharding.local_lengths(Lg, rank, B)
            else:
                ds.schedule_prefix(P, Tstep, Lg, Nst, obj, ws)
                Lloc = Lg
        ds.verify_prefix(x, Lloc, target, acc, bonus)
        last_L[0] = Lloc

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    assert ds.get_error() == 0, "device error during warm-up"

    # one step as a CUDA graph (launch gaps removed); eager launches if capture is refused.
    # The lagged schedule rotates through 3 ring slots, so it needs one graph per slot.
    graphs, graph_L = [], []
    if not args.eager:
        try:
            for _ in range(3 if lagged else 1):
                g = torch.cuda.CUDAGraph()
                with torch.cuda.graph(g):
                    step()
                graphs.append(g)
                graph_L.append(last_L[0])
            for g in graphs:
                g.replay()
            torch.cuda.synchronize()
            assert ds.get_error() == 0
        except Exception as exc:                        # noqa: BLE001
            print(f"# CUDA graph capture unavailable, timing eager launches: {exc}",
                  file=sys.stderr)
            torch.cuda.synchronize()
            graphs = []
    graph = graphs[0] if graphs else None
    replay_no = [0]

    def replay():
        j = replay_no[0] % len(graphs)
        graphs[j].replay()
        last_L[0] = graph_L[j]                     # the lengths this step verified with
        replay_no[0] += 1

    run_step = replay if graphs else step

    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.05)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    clocks.begin()
    step_ev = []
    for _ in range(args.steps):
        flush.zero_()                                   # evict L2 between timed steps
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        run_step()
        e1.record(stream)
        step_ev.append((e0, e1))
    torch.cuda.synchronize()
    clocks.end()
    if world > 1:
        dist.barrier()
    clk = clocks.stop()
    step_ms = [a.elapsed_time(b) for a, b in step_ev]
    total_ms = sum(step_ms)
    assert ds.get_error() == 0, "device error during the timed steps"
    # outputs of the last timed step, checked against the oracle after all timing
    snap = None
    if world == 1:
        snap = {"x": x.cpu().numpy(), "lx": lx.cpu().numpy(), "c": c.cpu().numpy(),
                "P": P.cpu().numpy(), "L": last_L[0].cpu().numpy(), "N": int(Nst.item()),
                "F": float(obj.item()), "acc": acc.cpu().numpy(), "bonus": bonus.cpu().numpy()}

    # the draft call alone, for its roofline (same inputs, L2 flushed before each launch),
    # replayed as a CUDA graph so that no host time falls between the events
    g_draft = None
    if not args.eager:
        try:
            g_draft = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g_draft):
                draft_and_score(P)
        except Exception:                                  # noqa: BLE001
            torch.cuda.synchronize()
            g_draft = None
    for _ in range(args.steps):
        flush.zero_()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        if g_draft is not None:
            g_draft.replay()
        else:
            draft_and_score(P)
        e1.record(stream)
        ev_draft.append((e0, e1))
    torch.cuda.synchronize()
    g_draft = None
    draft_ms = [a.elapsed_time(b) for a, b in ev_draft]

    # ---------------- end to end through the public API with host buffers
    pin = lambda a: torch.from_numpy(a).pin_memory()  # noqa: E731
    U_pin, h_pin = pin(Uh).view(torch.bfloat16), pin(hh).view(torch.bfloat16)
    anchor_pin, target_pin = pin(anchor_h), pin(target_h)
    out_x = torch.empty(B, gamma, dtype=torch.int32).pin_memory()
    out_L = torch.empty(B, dtype=torch.int32).pin_memory()
    out_acc = torch.empty(B, dtype=torch.int32).pin_memory()
    out_bonus = torch.empty(B, dtype=torch.int32).pin_memory()
    h2d = sum(t.numel() * t.element_size() for t in (U_pin, h_pin, anchor_pin, target_pin))
    d2h = sum(t.numel() * t.element_size() for t in (out_x, out_L, out_acc, out_bonus))

    def e2e_step():
        U.copy_(U_pin, non_blocking=True)
        h.copy_(h_pin, non_blocking=True)
        anchor.copy_(anchor_pin, non_blocking=True)
        target.copy_(target_pin, non_blocking=True)
        run_step()
        out_x.copy_(x, non_blocking=True)
        out_L.copy_(last_L[0], non_blocking=True)
        out_acc.copy_(acc, non_blocking=True)
        out_bonus.copy_(bonus, non_blocking=True)

    for _ in range(max(1, args.warmup // 2)):
        e2e_step()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    e2e_ev = []
    for _ in range(args.steps):
        flush.zero_()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        e2e_step()
        e1.record(stream)
        e2e_ev.append((e0, e1))
    torch.cuda.synchronize()
    e2e_ms = sum(a.elapsed_time(b) for a, b in e2e_ev)
    assert ds.get_error() == 0, "device error during the end-to-end steps"

    # ---------------- max over ranks
    if world > 1:
        t = torch.tensor([total_ms, e2e_ms, statistics.mean(draft_ms)], dtype=torch.float64,
                         device="cuda")
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        total_ms, e2e_ms, draft_mean = (float(v) for v in t.tolist())
    else:
        draft_mean = statistics.mean(draft_ms)

    tokens = B * world * gamma * args.steps
    value = tokens / (total_ms / 1e3)
    e2e_value = tokens / (e2e_ms / 1e3)

    if rank == 0:
        hbm_gbs, tflops, peak_kind = _peaks()
        # W2 + U_k per position; with the confidence head in the same timed call, h as well
        algo_bytes = gamma * (wl.r * V * 2 + B * V * 2) + (B * gamma * wl.d * 2 if fused else 0)
        achieved = algo_bytes / (draft_mean / 1e3) / 1e9
        flops = gamma * 2.0 * B * wl.r * V
        t_hbm = algo_bytes / (hbm_gbs * 1e9)
        t_tc = flops / (tflops * 1e12)
        roof = {"bound": "hbm" if t_hbm >= t_tc else "tensor", "achieved": achieved,
                "peak": hbm_gbs, "unit": "GB/s", "frac": achieved / hbm_gbs,
                "traffic": None if rnn else _traffic_per_launch(wl.name, gamma),
                "kernel": ("markov_pair_kernel" if B > 128 and not rnn else "markov_draft_kernel")
                + ((" + confidence kernel" if wl.mode == 1 and B > 128 else " + confidence head")
                   if fused else ""),
                "kernel_ms": draft_mean, "algorithmic_bytes": algo_bytes,
                "peak_source": f"{peak_kind} (MEASURED_PEAKS.json hbm_gbs)"
                if peak_kind == "measured" else "fallback 6650 GB/s"}
        cpu = parity = None
        if world == 1:
            inp = synth.Inputs(wl=wl, W1=W1h, W2=W2h, U=Uh, h=hh, anchor=anchor_h, w=wh, T=Th,
                               Tstep=Tstep_h, b_conf=wl.b_conf)
            Whh_h = synth.whh(wl) if rnn else None
            cpu = cpu_baseline(wl, inp, target_h, args.cpu_budget, Whh_h)
            import oracle
            # every request when the oracle can redo the step in a few seconds, else the first
            rows = max(1, min(B, int(PARITY_MACS / (gamma * wl.r * V))))
            parity = parity_report(wl, inp, target_h, snap, oracle, Whh_h, n_rows=rows,
                                   schedule=not lagged)
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": total_ms / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic",
            "config": workload_config(wl, world),
            "roofline": roof,
            "cpu_baseline": cpu,
            "parity": parity,
            "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h},
            "gpu_launches": ((1 if B <= 128 and B * gamma <= 1024 else 3 if B <= 128 or wl.mode == 0
                              else 4) if one_call
                             else (3 if fused and not (wl.mode == 1 and B > 128) else 4))
                            * args.steps,
            "cuda_graph": graph is not None,
            "step_call": "dspark_step" if one_call else "separate calls",
            "schedule": "lagged by 2 steps, side stream" if lagged else "this step's scores",
            "head": args.head,
            "clocks": clk,
            "ms_per_step_median": statistics.median(step_ms),
            "draft_kernel_ms": {"mean": draft_mean, "median": statistics.median(draft_ms),
                                "min": min(draft_ms), "max": max(draft_ms)},
        }
        print(json.dumps(line), flush=True)
    graph = None                                    # release the graphs before the group
    graphs = []
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
