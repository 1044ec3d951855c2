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
