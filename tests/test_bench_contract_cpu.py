"""bench.py's reference arm (the CPU oracle) runs without a GPU: its JSON line carries the
keys the benchmark contract asks for."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_reference_arm_json_line():
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--steps", "1", "--warmup", "1", "--ref-sample", "1",
                          "--workload", "tiny"],
                         capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [l for l in out.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
                "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["value"] > 0 and d["higher_is_better"] is True
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["value"] == d["value"]
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert "workload" in d["config"]
    import bench
    import synth
    assert d["config"] == bench.workload_config(synth.TINY, 1)   # same keys as the GPU arm


def test_parity_report_counts_mismatches(oracle_mod):
    """The bench line's parity summary, fed the oracle's own step, reports no mismatch; a
    token changed at a position with a clear oracle margin counts as a hard mismatch."""
    import numpy as np
    import bench
    import synth
    wl = synth.TINY.with_(V=4000, d=64)
    inp = synth.make_inputs(wl)
    x, l, g = oracle_mod.draft(inp.U, inp.anchor, inp.W1, inp.W2)
    conf = oracle_mod.confidence(inp.h, inp.anchor, x, inp.W1, inp.w, inp.b_conf, inp.T)
    P = conf["P32"]
    L, N, F, _ = oracle_mod.schedule(P, inp.Tstep)
    target = synth.targets(wl, x)
    acc, bonus = oracle_mod.verify(x, L, target)
    out = {"x": x, "lx": l.astype(np.float32), "c": conf["c"].astype(np.float32), "P": P,
           "L": L, "N": N, "F": F, "acc": acc, "bonus": bonus}
    rep = bench.parity_report(wl, inp, target, out, oracle_mod)
    assert rep["ok"] and rep["hard_mismatch"] == 0 and rep["compared"] == x.size
    assert rep["schedule_bit_exact"] and rep["verify_bit_exact"]
    b, k = np.argwhere(g > 0.1)[0]
    bad = dict(out, x=x.copy())
    bad["x"][b, k] = (x[b, k] + 1) % wl.V
    rep = bench.parity_report(wl, inp, target, bad, oracle_mod, schedule=False)
    assert not rep["ok"] and rep["hard_mismatch"] >= 1


def test_clock_sampler_keeps_the_timed_region():
    """Only the NVML samples stamped between begin() and end() are summarised, and the
    clock-event bits map onto the reason names the record uses."""
    import types
    import bench
    s = bench.ClockSampler(0)
    s.mode, s.max_mhz = "nvml", 1965.0
    ms = 1_000_000
    # ten samples 1 ms apart; the one at 3 ms has the sw power cap bit, the one at 8 ms
    # (outside the region) the hw slowdown bit
    s.lines = [(0, f"{i * ms} {1965 - 10 * i} {4 if i == 3 else (8 if i == 8 else 0)} "
                   f"{(600 + i) * 1000}") for i in range(10)]
    s.t0, s.t1 = 2 * ms, 5 * ms
    s.proc = types.SimpleNamespace(terminate=lambda: None, wait=lambda timeout=None: None,
                                   kill=lambda: None)
    s.thread = types.SimpleNamespace(join=lambda timeout=None: None)
    clk = s.stop()
    assert clk["samples"] == 4 and clk["source"] == "nvml"
    assert clk["sm_mhz"] == 1965 - 35 and clk["sm_min_mhz"] == 1965 - 50
    assert clk["reasons"] == ["sw_power_cap"] and clk["window_ms"] == 3.0
    assert clk["power_w"] == 603.5
