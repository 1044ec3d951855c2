"""The lagged ("2 steps prior") scheduling pipeline's stream ordering, on CPU.

`LaggedScheduler` only orders kernel launches across two CUDA streams with events.
Here the streams and events are simulated: every launch is a queued operation that
reads and writes tagged buffer slots, the two queues execute in random interleavings,
and a wait refers to the event record most recently enqueued before it (CUDA's rule).
Every interleaving must give the scheduler of step t the scores of step t - lag and
the verification of step t the lengths of step t.
"""
import random

import numpy as np
import pytest
import torch

from speculative_decoding_drafter_head_b200 import pipeline


class Sim:
    def __init__(self):
        self.queues = {}
        self.records_enqueued = {}
        self.records_done = {}
        self.slots = {}          # (buffer, slot) -> step tag
        self.log = []


class FakeStream:
    def __init__(self, sim, name):
        self.sim, self.name = sim, name
        sim.queues[name] = []

    def wait_event(self, ev):
        target = self.sim.records_enqueued.get(id(ev), 0)
        self.sim.queues[self.name].append(("wait", id(ev), target))

    def enqueue(self, fn):
        self.sim.queues[self.name].append(("run", fn, None))


class FakeEvent:
    def __init__(self, sim):
        self.sim = sim

    def record(self, stream):
        sim = self.sim
        sim.records_enqueued[id(self)] = sim.records_enqueued.get(id(self), 0) + 1
        key = id(self)

        def done():
            sim.records_done[key] = sim.records_done.get(key, 0) + 1
        stream.enqueue(done)


def run(sim, rng):
    """Execute both queues to completion in a random order that respects the waits."""
    while any(sim.queues.values()):
        ready = []
        for name, q in sim.queues.items():
            if not q:
                continue
            kind, a, target = q[0]
            if kind == "wait" and sim.records_done.get(a, 0) < target:
                continue
            ready.append(name)
        assert ready, "deadlock: every stream waits"
        name = rng.choice(ready)
        kind, a, _ = sim.queues[name].pop(0)
        if kind == "run":
            a()


@pytest.mark.parametrize("lag", [0, 1, 2, 3])
@pytest.mark.parametrize("seed", range(6))
def test_lagged_schedule_reads_the_right_step(monkeypatch, lag, seed):
    sim = Sim()
    main = FakeStream(sim, "main")
    monkeypatch.setattr(torch.cuda, "Stream", lambda device=None: FakeStream(sim, "side"))
    monkeypatch.setattr(torch.cuda, "Event", lambda: FakeEvent(sim))
    monkeypatch.setattr(torch.cuda, "current_stream", lambda: main)

    B, gamma, steps = 3, 4, 12
    sched = pipeline.LaggedScheduler(B, gamma, torch.zeros(B * (gamma + 1) + 1, dtype=torch.float64),
                                     lag=lag, device="cpu")
    n = lag + 1

    def fake_schedule(P, Tstep, L, N, obj, ws, stream=None):
        # which scores slot is read and which lengths slot is written, by storage offset
        ps = (P.data_ptr() - sched.P.data_ptr()) // (B * gamma * 4)
        ls = (L.data_ptr() - sched.L.data_ptr()) // (B * 4)

        def go():
            sim.log.append(("sched", ls, sim.slots.get(("P", ps))))
            sim.slots[("L", ls)] = sim.slots.get(("P", ps))
        stream.enqueue(go)
    monkeypatch.setattr(pipeline, "schedule_prefix", fake_schedule)

    for t in range(steps):
        main.enqueue(lambda: None)                                             # draft
        sched.begin_step(t)
        s = pipeline.scores_slot(t, lag)
        main.enqueue(lambda s=s, t=t: sim.slots.__setitem__(("P", s), t))     # confidence
        L = sched.lengths(t)
        ls = (L.data_ptr() - sched.L.data_ptr()) // (B * 4)
        main.enqueue(lambda ls=ls, t=t: sim.log.append(("verify", t, sim.slots.get(("L", ls)))))
    run(sim, random.Random(seed))

    verified = [(t, src) for kind, t, src in sim.log if kind == "verify"]
    assert [t for t, _ in verified] == list(range(steps))
    for t, src in verified:
        assert src == pipeline.source_step(t, lag), (t, src)
    n_async = sum(1 for t in range(steps) if sched.asynchronous(t))
    assert n_async == (0 if lag == 0 else steps - lag)
    assert len(sched.P) == n


def test_source_step_and_slots():
    assert [pipeline.source_step(t, 2) for t in range(5)] == [0, 1, 0, 1, 2]
    assert [pipeline.source_step(t, 0) for t in range(3)] == [0, 1, 2]
    # a step never writes the scores slot that its own scheduler reads
    for lag in (1, 2, 3):
        for t in range(lag, 20):
            assert pipeline.scores_slot(t, lag) != pipeline.scores_slot(t - lag, lag)
    assert np.all(np.diff([pipeline.scores_slot(t, 2) for t in range(9)]) != 0)
