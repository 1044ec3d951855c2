"""Asynchronous prefix scheduling from the scores of two steps earlier.

wispaper.ai, "DSpark: Overcoming the Efficiency Wall in LLM Speculative Decoding",
section "Critical Insights & Conclusion", key takeaway on asynchrony: so that scheduling
never stalls the GPU, the verify lengths of step t are decided from the confidence
predictions of step t - 2, which leaves a causal barrier between what is being drafted
and what decides how much of it is verified.
Verification stays a strict prefix match, so any lengths are lossless; the lag only
changes how many drafted tokens are sent to the target.

Here the scheduler kernel of step t reads the survival scores written by the
confidence kernel of step t - lag and runs on a side stream, so it no longer waits for
the confidence kernel of step t.  The draft kernel is a cooperative launch that holds
every SM, so nothing runs beside it; callers fork the side stream right after the draft
launch (``begin_step``), and the scheduler then overlaps the confidence kernel of the
same step.  Before `lag` steps exist, a step schedules on its own scores on the caller's
stream.

Buffers are rings of lag + 1 slots indexed by step: the confidence kernel of step t
writes ``scores(t)``, the scheduler of step t reads ``scores(t - lag)`` and writes the
lengths slot of step t, and verification of step t reads it.  Two events order the
streams, and each step uses them once:
  - fork: at ``begin_step(t)`` the side stream waits for everything already enqueued on
    the caller's stream (all of step t - 1, hence the scores of step t - lag);
  - join: the caller's stream waits for the scheduler of step t before verifying step t.
So scores slot (t - lag) mod (lag + 1), next written by the confidence kernel of step
t + 1, is no longer read by then, and every lengths slot is read by its own step's
verification before the next fork.  Both dependencies live inside one step, so a step
can be captured as one CUDA graph (one graph per ring phase) and replayed.

This module only orders launches of the library's kernels; it computes nothing.
"""
from __future__ import annotations

from . import schedule_prefix, workspace_bytes


def scores_slot(t: int, lag: int) -> int:
    """Ring slot holding the survival scores of step t."""
    return t % (lag + 1)


def source_step(t: int, lag: int) -> int:
    """The step whose scores decide the verify lengths of step t."""
    return t - lag if lag >= 1 and t >= lag else t


class LaggedScheduler:
    """Verify lengths for step t from the survival scores of step t - lag (default 2)."""

    def __init__(self, B: int, gamma: int, Tstep_us, lag: int = 2, device=None):
        import torch
        if lag < 0:
            raise ValueError("lag must be >= 0")
        device = device or Tstep_us.device
        self.B, self.gamma, self.lag = B, gamma, lag
        n = lag + 1
        self.Tstep = Tstep_us
        self.P = torch.empty(n, B, gamma, dtype=torch.float32, device=device)
        self.L = torch.empty(n, B, dtype=torch.int32, device=device)
        self.N = torch.empty(n, 1, dtype=torch.int32, device=device)
        self.obj = torch.empty(n, 1, dtype=torch.float64, device=device)
        # the side stream's own scheduler workspace: it runs concurrently with the draft
        # kernel, which uses the caller's workspace
        self.ws = torch.empty(workspace_bytes(B, gamma, 8), dtype=torch.uint8, device=device)
        self.side = torch.cuda.Stream(device=device)
        self.ev_fork = torch.cuda.Event()
        self.ev_join = torch.cuda.Event()

    def scores(self, t: int):
        """The [B, gamma] fp32 buffer that the confidence kernel of step t writes."""
        return self.P[scores_slot(t, self.lag)]

    def asynchronous(self, t: int) -> bool:
        """Whether step t is scheduled on the side stream (lag >= 1 and t >= lag)."""
        return self.lag >= 1 and t >= self.lag

    def begin_step(self, t: int, stream=None):
        """Launch the scheduler of step t on the side stream (if asynchronous).

        Call it after the draft launch of step t and before ``lengths(t)``."""
        import torch
        if not self.asynchronous(t):
            return
        main = stream or torch.cuda.current_stream()
        s = scores_slot(t - self.lag, self.lag)
        o = scores_slot(t, self.lag)
        self.ev_fork.record(main)
        self.side.wait_event(self.ev_fork)
        schedule_prefix(self.P[s], self.Tstep, self.L[o], self.N[o], self.obj[o], self.ws,
                        stream=self.side)
        self.ev_join.record(self.side)

    def lengths(self, t: int, workspace=None, stream=None):
        """Verify lengths [B] of step t, ordered before what the caller's stream runs next.

        Before `lag` steps exist (and always when lag = 0) this schedules step t on its own
        scores, on the caller's stream, with `workspace` or else the side workspace, which
        is idle then.
        """
        import torch
        main = stream or torch.cuda.current_stream()
        o = scores_slot(t, self.lag)
        if not self.asynchronous(t):
            schedule_prefix(self.P[o], self.Tstep, self.L[o], self.N[o], self.obj[o],
                            self.ws if workspace is None else workspace, stream=main)
        else:
            main.wait_event(self.ev_join)
        return self.L[o]

    def chosen(self, t: int):
        """(N*, objective) tensors of the schedule used at step t."""
        o = scores_slot(t, self.lag)
        return self.N[o], self.obj[o]
