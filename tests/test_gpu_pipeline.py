"""The lagged scheduling pipeline on the GPU: verify lengths of step t come from the
survival scores of step t - 2, computed on a side stream that overlaps the draft kernel.

Each step drafts from different anchors, so the scores differ from step to step.  The
lengths (and N*, objective) must equal the oracle scheduler's on the scores of the
source step, bit for bit, and verification must equal the oracle's on those lengths.
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


@pytest.mark.parametrize("lag", [2, 1, 0])
def test_lagged_pipeline_matches_oracle(ds, oracle_mod, lag):
    import torch
    from speculative_decoding_drafter_head_b200 import pipeline

    wl = synth.Workload("pipeline B=24 gamma=8 V=32000", B=24, gamma=8, V=32000, d=1024,
                        sps_knee=64, q_first=0.9, q_last=0.6)
    steps = 7
    B, gamma = wl.B, wl.gamma
    U, h = dev_bf16(synth.u_all(wl)), dev_bf16(synth.h_all(wl))
    W1, W2, w = dev_bf16(synth.w1(wl)), dev_bf16(synth.w2(wl)), dev_bf16(synth.conf_w(wl))
    T = dev(synth.temperatures(wl))
    Tstep_h = synth.tstep_us(wl)
    Tstep = dev(Tstep_h)
    ws = torch.empty(ds.workspace_bytes(B, gamma, wl.V), dtype=torch.uint8, device="cuda")
    anchors = [dev(synth.anchors(wl.with_(seed=100 + t))) for t in range(steps)]

    # drafts of every step (deterministic) give the target tokens of every step
    x = torch.empty(B, gamma, dtype=torch.int32, device="cuda")
    lx = torch.empty(B, gamma, dtype=torch.float32, device="cuda")
    targets = []
    for t in range(steps):
        ds.draft_step(U, anchors[t], W1, W2, x, lx, ws)
        targets.append(dev(synth.targets(wl.with_(seed=t), x.cpu().numpy())))

    sched = pipeline.LaggedScheduler(B, gamma, Tstep, lag=lag)
    c = torch.empty(B, gamma, dtype=torch.float32, device="cuda")
    acc = torch.empty(B, dtype=torch.int32, device="cuda")
    bonus = torch.empty(B, dtype=torch.int32, device="cuda")
    rec = []
    for t in range(steps):                      # no host synchronisation inside the loop
        ds.draft_step(U, anchors[t], W1, W2, x, lx, ws)
        sched.begin_step(t)
        ds.confidence_sts(h, anchors[t], x, W1, w, wl.b_conf, T, c, sched.scores(t))
        L = sched.lengths(t, workspace=ws)
        ds.verify_prefix(x, L, targets[t], acc, bonus)
        N, obj = sched.chosen(t)
        rec.append(dict(P=sched.scores(t).clone(), x=x.clone(), L=L.clone(), N=N.clone(),
                        obj=obj.clone(), acc=acc.clone(), bonus=bonus.clone()))
    torch.cuda.synchronize()
    assert ds.get_error() == 0
    n_async = 0
    for t in range(steps):
        src = pipeline.source_step(t, lag)
        n_async += sched.asynchronous(t)
        P_src = rec[src]["P"].cpu().numpy()
        L_or, N_or, F_or, _ = oracle_mod.schedule(P_src, Tstep_h)
        np.testing.assert_array_equal(rec[t]["L"].cpu().numpy(), L_or)
        assert int(rec[t]["N"].item()) == N_or and float(rec[t]["obj"].item()) == F_or
        acc_or, bonus_or = oracle_mod.verify(rec[t]["x"].cpu().numpy(), L_or,
                                             targets[t].cpu().numpy())
        np.testing.assert_array_equal(rec[t]["acc"].cpu().numpy(), acc_or)
        np.testing.assert_array_equal(rec[t]["bonus"].cpu().numpy(), bonus_or)
    assert n_async == (0 if lag == 0 else steps - lag)
    # the scores really change from step to step, so reading the wrong step would show
    assert not np.array_equal(rec[0]["P"].cpu().numpy(), rec[1]["P"].cpu().numpy())
