"""Shared test helpers: device upload of generator arrays and the draft comparison rule."""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np

TOL = 2e-2   # absolute tolerance on logits at the chosen token and on c_k; near-tie gap bound


def dev_bf16(a: np.ndarray):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.uint16)).view(torch.bfloat16).cuda()


def dev(a: np.ndarray, dtype=None):
    import torch
    t = torch.from_numpy(np.ascontiguousarray(a))
    if dtype is not None:
        t = t.to(dtype)
    return t.cuda()


@dataclass
class DraftComparison:
    compared: int = 0          # positions compared token for token
    near_ties: int = 0         # positions where the tokens differ at an oracle near-tie
    hard_mismatch: int = 0     # tokens differ with a clear oracle margin
    max_logit_err: float = 0.0

    def ok(self) -> bool:
        return self.hard_mismatch == 0 and self.max_logit_err <= TOL


# (case name, DraftComparison) of every draft parity check of the session, printed in
# the terminal summary by conftest.py so that near-tie counts appear in a -q run
PARITY_LOG: list = []


def forced_prev(anchor_rows, x_rows) -> np.ndarray:
    """x_{k-1} for every position of the GPU's drafts: the anchor, then x_1..x_{gamma-1}."""
    x_rows = np.asarray(x_rows, dtype=np.int32)
    return np.ascontiguousarray(
        np.concatenate([np.asarray(anchor_rows, np.int32)[:, None], x_rows[:, :-1]], axis=1))


def compare_forced(x_gpu, logit_gpu, x_or, logit_or, gap_or, tol: float = TOL,
                   name: str = "") -> DraftComparison:
    """Every position against the oracle teacher-forced on the GPU's previous tokens.

    The oracle's position k conditions on the GPU's x_{k-1}, so no position is skipped:
    tokens must match except where the oracle's top-2 gap is below tol (counted as a
    near tie), and the logit at a matching token must be within tol.
    """
    x_gpu = np.asarray(x_gpu); x_or = np.asarray(x_or)
    assert x_gpu.shape == x_or.shape
    res = DraftComparison()
    same = x_gpu == x_or
    res.compared = int(same.sum())
    if res.compared:
        err = np.abs(np.asarray(logit_gpu, np.float64)[same] - np.asarray(logit_or)[same])
        res.max_logit_err = float(err.max())
    diff = ~same
    res.near_ties = int((diff & (np.asarray(gap_or) < tol)).sum())
    res.hard_mismatch = int((diff & (np.asarray(gap_or) >= tol)).sum())
    if name:
        PARITY_LOG.append((name, res))
    return res
