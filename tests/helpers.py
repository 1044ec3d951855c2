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
    after_divergence: int = 0  # positions after a near-tie divergence (trajectories differ)
    hard_mismatch: int = 0     # tokens differ with a clear oracle margin
    max_logit_err: float = 0.0

    def ok(self) -> bool:
        return self.hard_mismatch == 0 and self.max_logit_err <= TOL


def compare_drafts(x_gpu, logit_gpu, x_or, logit_or, gap_or, tol: float = TOL) -> DraftComparison:
    """Tokens must match except where the oracle's top-2 gap is below tol.

    Once a request's tokens differ at a near-tie, its later positions condition on
    different previous tokens, so they are counted but not compared.
    """
    x_gpu = np.asarray(x_gpu); x_or = np.asarray(x_or)
    res = DraftComparison()
    for b in range(x_or.shape[0]):
        for k in range(x_or.shape[1]):
            if x_gpu[b, k] == x_or[b, k]:
                res.compared += 1
                err = abs(float(logit_gpu[b, k]) - float(logit_or[b, k]))
                res.max_logit_err = max(res.max_logit_err, err)
                continue
            if gap_or[b, k] < tol:
                res.near_ties += 1
                res.after_divergence += x_or.shape[1] - k - 1
            else:
                res.hard_mismatch += 1
            break
    return res
