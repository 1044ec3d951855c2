"""Failure detection in the draft kernel without faulting the GPU.

The grid barrier is told to expect one more arrival than there are CTAs, so its
bounded wait runs out.  The kernel must record DSPARK_TIMEOUT, stop every role,
drain its own copies and MMAs, free TMEM and return; the context stays usable and
the next call gives the same results as before.
"""
import numpy as np
import pytest

import synth
from helpers import dev, dev_bf16

pytestmark = pytest.mark.gpu

TIMEOUT = 6


def _draft(ds, wl, U, W1, W2, anchor):
    import torch
    x = torch.full((wl.B, wl.gamma), -1, dtype=torch.int32, device="cuda")
    lx = torch.zeros((wl.B, wl.gamma), dtype=torch.float32, device="cuda")
    ws = torch.empty(ds.workspace_bytes(wl.B, wl.gamma, wl.V), dtype=torch.uint8, device="cuda")
    ds.draft_step(U, anchor, W1, W2, x, lx, ws)
    return x, lx


def test_grid_barrier_timeout_is_reported_and_context_survives():
    import speculative_decoding_drafter_head_b200 as ds
    wl = synth.Workload("timeout probe B=5 V=4104", B=5, gamma=4, V=4104, d=64, w_std=0.2)
    U, W1, W2 = dev_bf16(synth.u_all(wl)), dev_bf16(synth.w1(wl)), dev_bf16(synth.w2(wl))
    anchor = dev(synth.anchors(wl))
    assert ds.get_error() == 0
    x_ref, lx_ref = _draft(ds, wl, U, W1, W2, anchor)
    assert ds.get_error() == 0
    try:
        ds.set_wait_timeout_ns(200_000_000)
        ds.debug_barrier_extra(1)
        _draft(ds, wl, U, W1, W2, anchor)
        assert ds.get_error() == TIMEOUT
    finally:
        ds.debug_barrier_extra(0)
        ds.set_wait_timeout_ns(2_000_000_000)
    x, lx = _draft(ds, wl, U, W1, W2, anchor)
    assert ds.get_error() == 0
    np.testing.assert_array_equal(x.cpu().numpy(), x_ref.cpu().numpy())
    np.testing.assert_array_equal(lx.cpu().numpy(), lx_ref.cpu().numpy())


def test_rnn_state_barrier_timeout_is_reported_and_context_survives():
    # the RNN instance waits at a second grid barrier (after the state update, before the
    # gather); the first wait of the launch is that one, so it is the one that runs out
    import torch
    import speculative_decoding_drafter_head_b200 as ds
    wl = synth.Workload("rnn timeout probe B=70 V=4104", B=70, gamma=3, V=4104, d=64,
                        w_std=0.2)
    U, W1, W2 = dev_bf16(synth.u_all(wl)), dev_bf16(synth.w1(wl)), dev_bf16(synth.w2(wl))
    Whh = dev_bf16(synth.whh(wl, 0.1))
    anchor = dev(synth.anchors(wl))

    def run():
        x = torch.full((wl.B, wl.gamma), -1, dtype=torch.int32, device="cuda")
        lx = torch.zeros((wl.B, wl.gamma), dtype=torch.float32, device="cuda")
        ws = torch.empty(ds.workspace_bytes(wl.B, wl.gamma, wl.V), dtype=torch.uint8,
                         device="cuda")
        ds.draft_step_rnn(U, anchor, W1, W2, Whh, x, lx, ws)
        return x, lx

    assert ds.get_error() == 0
    x_ref, lx_ref = run()
    assert ds.get_error() == 0
    try:
        ds.set_wait_timeout_ns(200_000_000)
        ds.debug_barrier_extra(1)
        run()
        assert ds.get_error() == TIMEOUT
    finally:
        ds.debug_barrier_extra(0)
        ds.set_wait_timeout_ns(2_000_000_000)
    x, lx = run()
    assert ds.get_error() == 0
    np.testing.assert_array_equal(x.cpu().numpy(), x_ref.cpu().numpy())
    np.testing.assert_array_equal(lx.cpu().numpy(), lx_ref.cpu().numpy())


@pytest.mark.parametrize("case", ["step tail B=5", "pair+confidence B=300", "pair gumbel B=260"])
def test_timeout_in_fused_and_pair_paths(case):
    # the one-launch step (its scheduler tail waits on every CTA's confidence warp), the
    # CTA-pair kernel with its confidence warp, and the pair kernel's Gumbel instance: the
    # grid barrier runs out, the launch reports DSPARK_TIMEOUT and returns, and the next
    # call repeats the clean results
    import torch
    import speculative_decoding_drafter_head_b200 as ds
    B = {"step tail B=5": 5, "pair+confidence B=300": 300, "pair gumbel B=260": 260}[case]
    gumbel = case.startswith("pair gumbel")
    wl = synth.Workload(f"timeout probe {case}", B=B, gamma=3, V=4104, d=64, w_std=0.2,
                        mode=1 if gumbel else 0, tau=0.7 if gumbel else 1.0)
    inp = synth.make_inputs(wl)
    U, W1, W2 = dev_bf16(inp.U), dev_bf16(inp.W1), dev_bf16(inp.W2)
    h, w = dev_bf16(inp.h), dev_bf16(inp.w)
    anchor, T, Tstep = dev(inp.anchor), dev(inp.T), dev(inp.Tstep)
    target = dev(synth.targets(wl, np.zeros((B, wl.gamma), np.int32)))
    ws = torch.empty(ds.workspace_bytes(B, wl.gamma, wl.V), dtype=torch.uint8, device="cuda")

    def run():
        i32 = dict(dtype=torch.int32, device="cuda")
        f32 = dict(dtype=torch.float32, device="cuda")
        o = dict(x=torch.full((B, wl.gamma), -1, **i32), lx=torch.zeros((B, wl.gamma), **f32),
                 c=torch.zeros((B, wl.gamma), **f32), P=torch.zeros((B, wl.gamma), **f32),
                 L=torch.zeros(B, **i32), N=torch.zeros(1, **i32),
                 obj=torch.zeros(1, dtype=torch.float64, device="cuda"),
                 acc=torch.zeros(B, **i32), bonus=torch.zeros(B, **i32))
        if case.startswith("step"):
            ds.step(U, anchor, W1, W2, h, w, wl.b_conf, T, Tstep, target, o["x"], o["lx"], o["c"],
                    o["P"], o["L"], o["N"], o["obj"], o["acc"], o["bonus"], ws)
        elif gumbel:
            ds.draft_step(U, anchor, W1, W2, o["x"], o["lx"], ws, mode=1, temperature=0.7, seed=3)
        else:
            ds.draft_confidence_step(U, anchor, W1, W2, h, w, wl.b_conf, T, o["x"], o["lx"],
                                     o["c"], o["P"], ws)
        return {k: v.cpu().numpy() for k, v in o.items()}

    assert ds.get_error() == 0
    ref = run()
    assert ds.get_error() == 0
    try:
        ds.set_wait_timeout_ns(200_000_000)
        ds.debug_barrier_extra(1)
        run()
        assert ds.get_error() == TIMEOUT
    finally:
        ds.debug_barrier_extra(0)
        ds.set_wait_timeout_ns(2_000_000_000)
    again = run()
    assert ds.get_error() == 0
    for k in ref:
        np.testing.assert_array_equal(again[k], ref[k], err_msg=k)
