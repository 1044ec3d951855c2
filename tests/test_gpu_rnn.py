"""RNN-head drafting (CUDA, through the C ABI) against the oracle's Elman reading.

Same comparison rule as the Markov head: logits at the chosen token within 2e-2,
tokens identical except at oracle near-ties (top-2 gap < 2e-2), every position compared
against the oracle teacher-forced on the GPU's previous tokens (its state then runs
along the GPU's tokens).  The GPU keeps the state in fp32 and the
oracle in fp64; both round the GEMM operand to bf16.
"""
import numpy as np
import pytest

import synth
from helpers import compare_forced, dev, dev_bf16, forced_prev

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
    (synth.Workload("rnn B=5 V=4104", B=5, gamma=6, V=4104, d=64, w_std=0.2), 0.1),
    (synth.Workload("rnn B=64 V=9000", B=64, gamma=8, V=9000, d=64, w_std=0.2, seed=1), 0.08),
    (synth.Workload("rnn B=130 V=2056", B=130, gamma=4, V=2056, d=64, w_std=0.2, seed=2), 0.1),
    (synth.Workload("rnn B=300 V=5000 gumbel", B=300, gamma=3, V=5000, d=64, w_std=0.2,
                    logits="zipf", mode=1, tau=0.7, seed=3), 0.1),
    (synth.Workload("rnn B=9 V=40000 gumbel", B=9, gamma=5, V=40000, d=64, w_std=0.2,
                    mode=1, tau=1.3, seed=5), 0.06),
]


def _run(ds, wl, Whh, U=None):
    import torch
    U = synth.u_all(wl) if U is None else U
    W1, W2, anchor = synth.w1(wl), synth.w2(wl), synth.anchors(wl)
    x = torch.full((wl.B, wl.gamma), -1, dtype=torch.int32, device="cuda")
    lx = torch.full((wl.B, wl.gamma), float("nan"), dtype=torch.float32, device="cuda")
    ws = torch.empty(ds.workspace_bytes(wl.B, wl.gamma, wl.V), dtype=torch.uint8, device="cuda")
    ds.draft_step_rnn(dev_bf16(U), dev(anchor), dev_bf16(W1), dev_bf16(W2), dev_bf16(Whh), x, lx,
                      ws, mode=wl.mode, temperature=wl.tau, seed=wl.seed)
    assert ds.get_error() == 0
    return U, W1, W2, anchor, x.cpu().numpy(), lx.cpu().numpy()


@pytest.mark.parametrize("wl,whh_std", CASES, ids=[c[0].name for c in CASES])
def test_rnn_draft_matches_oracle(ds, oracle_mod, wl, whh_std):
    Whh = synth.whh(wl, whh_std)
    U, W1, W2, anchor, x, lx = _run(ds, wl, Whh)
    x_or, l_or, gap_or = oracle_mod.draft_rnn(U, anchor, W1, W2, Whh, mode=wl.mode, tau=wl.tau,
                                              seed=wl.seed, forced_prev=forced_prev(anchor, x))
    cmp = compare_forced(x, lx, x_or, l_or, gap_or, name=wl.name)
    print(f"{wl.name}: {cmp}")
    assert cmp.ok(), cmp
    assert cmp.compared + cmp.near_ties == wl.B * wl.gamma
    # the recurrence matters here: the Markov head on the same tables drafts differently
    x_mk, _, _ = oracle_mod.draft(U, anchor, W1, W2, mode=wl.mode, tau=wl.tau, seed=wl.seed)
    assert (x_mk != x_or).any()


def test_rnn_qwen3_shaped_sampled_rows(ds, oracle_mod):
    wl = synth.QWEN3_8B.with_(w_std=0.2)
    Whh = synth.whh(wl, 0.06)
    U, W1, W2, anchor, x, lx = _run(ds, wl, Whh)
    bs = [0, 21, 37, 63]
    x_or, l_or, gap_or = oracle_mod.draft_rnn(U[bs], anchor[bs], W1, W2, Whh,
                                              b_index=np.array(bs, np.int32),
                                              forced_prev=forced_prev(anchor[bs], x[bs]))
    cmp = compare_forced(x[bs], lx[bs], x_or, l_or, gap_or, name="rnn qwen3-8b-shaped (4 rows)")
    print(f"qwen3-8b-shaped rnn: {cmp}")
    assert cmp.ok(), cmp
