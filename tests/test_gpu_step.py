"""dspark_step (the whole per-step path in one call) against the four separate calls.

With B <= 128 and B gamma <= 1024 the scheduler and the verification run in the draft
kernel's tail, with the device code of the scheduler and verify kernels, so every output
must equal that of the separate calls bit for bit; otherwise the call is the separate
launches in sequence.  The separate calls themselves are checked against the oracle elsewhere; here
the scheduler's outputs are also checked against the oracle on the step's own scores.
"""
import numpy as np
import pytest

import synth
from helpers import dev, dev_bf16

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ds():
    import torch
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import speculative_decoding_drafter_head_b200 as m
    m.load()
    assert m.get_error() == 0
    return m


CASES = [
    synth.TINY,
    synth.QWEN3_8B,
    synth.sweep(128),                                       # 2048 scores: separate launches
    synth.Workload("step B=128 gamma=8 V=4104", B=128, gamma=8, V=4104, d=256, w_std=0.2,
                   seed=9),                                 # M = 128, one launch
    synth.Workload("step B=100 V=1032", B=100, gamma=9, V=1032, d=512, w_std=0.2, seed=3),
    synth.Workload("step B=7 V=5000 gumbel", B=7, gamma=12, V=5000, d=256, w_std=0.2,
                   mode=1, tau=0.8, seed=4),
    synth.Workload("step B=1 gamma=64 V=2048", B=1, gamma=64, V=2048, d=256, w_std=0.2, seed=8),
    synth.Workload("step B=300 V=5000", B=300, gamma=4, V=5000, d=256, w_std=0.2, seed=5),
]


@pytest.mark.parametrize("wl", CASES, ids=[w.name for w in CASES])
def test_step_equals_separate_calls(ds, oracle_mod, wl):
    import torch
    inp = synth.make_inputs(wl)
    U, W1, W2 = dev_bf16(inp.U), dev_bf16(inp.W1), dev_bf16(inp.W2)
    h, w = dev_bf16(inp.h), dev_bf16(inp.w)
    anchor, T = dev(inp.anchor), dev(inp.T)
    Tstep = dev(inp.Tstep)
    B, g = wl.B, wl.gamma
    ws = torch.empty(ds.workspace_bytes(B, g, wl.V), dtype=torch.uint8, device="cuda")

    def outs():
        i32 = dict(dtype=torch.int32, device="cuda")
        f32 = dict(dtype=torch.float32, device="cuda")
        return dict(x=torch.full((B, g), -1, **i32), lx=torch.full((B, g), float("nan"), **f32),
                    c=torch.full((B, g), float("nan"), **f32),
                    P=torch.full((B, g), float("nan"), **f32),
                    L=torch.full((B,), -1, **i32), N=torch.full((1,), -1, **i32),
                    obj=torch.full((1,), float("nan"), dtype=torch.float64, device="cuda"),
                    acc=torch.full((B,), -1, **i32), bonus=torch.full((B,), -1, **i32))

    # targets from a first draft, agreeing with it w.p. q_k as in the benchmark
    a = outs()
    ds.draft_confidence_step(U, anchor, W1, W2, h, w, wl.b_conf, T, a["x"], a["lx"], a["c"],
                             a["P"], ws, mode=wl.mode, temperature=wl.tau, seed=wl.seed)
    target_h = synth.targets(wl, a["x"].cpu().numpy(), range(B))
    target = dev(target_h)
    ds.schedule_prefix(a["P"], Tstep, a["L"], a["N"], a["obj"], ws)
    ds.verify_prefix(a["x"], a["L"], target, a["acc"], a["bonus"])

    b = outs()
    for _ in range(2):                                      # twice: the workspace is reused
        ds.step(U, anchor, W1, W2, h, w, wl.b_conf, T, Tstep, target, b["x"], b["lx"], b["c"],
                b["P"], b["L"], b["N"], b["obj"], b["acc"], b["bonus"], ws, mode=wl.mode,
                temperature=wl.tau, seed=wl.seed)
    assert ds.get_error() == 0
    for k in a:
        np.testing.assert_array_equal(b[k].cpu().numpy(), a[k].cpu().numpy(), err_msg=k)

    # the scheduler's answer on the step's own scores, from the oracle
    L_or, N_or, F_or, _ = oracle_mod.schedule(b["P"].cpu().numpy(), inp.Tstep)
    np.testing.assert_array_equal(b["L"].cpu().numpy(), L_or)
    assert int(b["N"].cpu()[0]) == N_or
    assert float(b["obj"].cpu()[0]) == F_or
    a_or, bonus_or = oracle_mod.verify(b["x"].cpu().numpy(), b["L"].cpu().numpy(), target_h)
    np.testing.assert_array_equal(b["acc"].cpu().numpy(), a_or)
    np.testing.assert_array_equal(b["bonus"].cpu().numpy(), bonus_or)
