"""dspark_draft_confidence_step (drafting and the confidence head in one call) against the
separate calls and the oracle.

The drafts must be those of dspark_draft_step bit for bit (same arithmetic, same kernel
code); c and P must agree with dspark_confidence_sts on those drafts to fp32 rounding of
the logit's sum order, and with the oracle within 2e-2.
"""
import numpy as np
import pytest

import synth
from helpers import TOL, dev, dev_bf16

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
    synth.sweep(128),                                       # M = 128, one launch
    synth.Workload("fused B=100 V=1032", B=100, gamma=9, V=1032, d=512, w_std=0.2, seed=3),
    synth.Workload("fused B=7 V=5000 gumbel", B=7, gamma=12, V=5000, d=256, w_std=0.2,
                   mode=1, tau=0.8, seed=4),
    synth.Workload("fused B=300 V=5000", B=300, gamma=4, V=5000, d=256, w_std=0.2, seed=5),
    # the pair kernel's confidence warp: Gumbel instance, and three 256-row passes
    synth.Workload("fused B=260 V=4104 gumbel", B=260, gamma=6, V=4104, d=512, w_std=0.2,
                   mode=1, tau=0.7, seed=6),
    synth.Workload("fused B=640 V=2056", B=640, gamma=5, V=2056, d=256, w_std=0.2, seed=7),
]


@pytest.mark.parametrize("wl", CASES, ids=[w.name for w in CASES])
def test_fused_equals_separate_calls(ds, oracle_mod, wl):
    import torch
    inp = synth.make_inputs(wl)
    U, W1, W2 = dev_bf16(inp.U), dev_bf16(inp.W1), dev_bf16(inp.W2)
    h, w = dev_bf16(inp.h), dev_bf16(inp.w)
    anchor, T = dev(inp.anchor), dev(inp.T)
    B, g = wl.B, wl.gamma

    def outs():
        return (torch.full((B, g), -1, dtype=torch.int32, device="cuda"),
                torch.full((B, g), float("nan"), dtype=torch.float32, device="cuda"),
                torch.full((B, g), float("nan"), dtype=torch.float32, device="cuda"),
                torch.full((B, g), float("nan"), dtype=torch.float32, device="cuda"))

    ws = torch.empty(ds.workspace_bytes(B, g, wl.V), dtype=torch.uint8, device="cuda")
    x1, l1, c1, P1 = outs()
    ds.draft_step(U, anchor, W1, W2, x1, l1, ws, mode=wl.mode, temperature=wl.tau, seed=wl.seed)
    ds.confidence_sts(h, anchor, x1, W1, w, wl.b_conf, T, c1, P1)
    x2, l2, c2, P2 = outs()
    for _ in range(2):                                      # twice: the workspace is reused
        ds.draft_confidence_step(U, anchor, W1, W2, h, w, wl.b_conf, T, x2, l2, c2, P2, ws,
                                 mode=wl.mode, temperature=wl.tau, seed=wl.seed)
    assert ds.get_error() == 0
    np.testing.assert_array_equal(x2.cpu().numpy(), x1.cpu().numpy())
    np.testing.assert_array_equal(l2.cpu().numpy(), l1.cpu().numpy())
    cg, Pg = c2.cpu().numpy(), P2.cpu().numpy()
    assert np.abs(cg - c1.cpu().numpy()).max() <= 1e-5
    assert np.abs(Pg - P1.cpu().numpy()).max() <= 1e-5
    ref = oracle_mod.confidence(inp.h, inp.anchor, x2.cpu().numpy(), inp.W1, inp.w, inp.b_conf,
                                inp.T)
    assert np.abs(cg - ref["c"]).max() <= TOL
    assert np.abs(Pg - ref["P64"]).max() <= TOL
    assert (np.diff(Pg.astype(np.float64), axis=1) <= 0).all()
    # P is the fp32 product of c in position order
    prod = np.cumprod(cg.astype(np.float32), axis=1, dtype=np.float32)
    np.testing.assert_array_equal(Pg, prod)
