"""Parity of the CUDA path (through the C ABI) with the CPU oracle on seeded inputs.

Bit-exact: scheduler lengths / N* / objective and verification outputs fed identical
inputs.  Tolerance 2e-2 absolute: the logit at the chosen token and c_k.  Drafted
tokens must be identical except at positions where the oracle's top-2 gap is below
2e-2 (counted, and printed in the session summary).  Every drafted position is
compared: the oracle is run teacher-forced on the GPU's previous tokens, so a near-tie
divergence does not hide the positions after it.
"""
import numpy as np
import pytest

import synth
from helpers import TOL, compare_forced, dev, dev_bf16, forced_prev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ds():
    import torch
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import speculative_decoding_drafter_head_b200 as m
    m.load()
    assert m.get_error() == 0
    return m


def _ws(ds, B, gamma, V):
    import torch
    return torch.empty(ds.workspace_bytes(B, gamma, V), dtype=torch.uint8, device="cuda")


# ---------------------------------------------------------------------------- verify
@pytest.mark.parametrize("B,gamma,V,agree", [(1, 1, 10, 0.5), (7, 5, 50, 0.9), (1000, 16, 151936, 0.85),
                                             (4096, 24, 1000, 0.97), (33, 64, 7, 0.8)])
def test_verify_bit_exact(ds, oracle_mod, B, gamma, V, agree):
    import torch
    x, L, t = synth.verify_inputs(B, gamma, V, seed=B + gamma, agree=agree)
    L[0] = 0
    L[-1] = gamma
    acc = torch.empty(B, dtype=torch.int32, device="cuda")
    bonus = torch.empty_like(acc)
    ds.verify_prefix(dev(x), dev(L), dev(t), acc, bonus)
    a_or, b_or = oracle_mod.verify(x, L, t)
    np.testing.assert_array_equal(acc.cpu().numpy(), a_or)
    np.testing.assert_array_equal(bonus.cpu().numpy(), b_or)
    assert ds.get_error() == 0


def test_verify_records_bad_length(ds):
    import torch
    x, L, t = synth.verify_inputs(4, 3, 20, seed=1)
    L[2] = 7
    acc = torch.empty(4, dtype=torch.int32, device="cuda")
    bonus = torch.empty_like(acc)
    ds.verify_prefix(dev(x), dev(L), dev(t), acc, bonus)
    assert ds.get_error() == 7
    assert 0 <= int(acc[2]) <= 3


# ---------------------------------------------------------------------------- schedule
def _tstep(kind, B, gamma, rng):
    n = B * (gamma + 1) + 1
    i = np.arange(n, dtype=np.float64)
    if kind == "knee":
        return 20000.0 + 30.0 * np.maximum(0.0, i - max(B, n // 3))
    if kind == "flat":
        return np.full(n, 15000.0)
    if kind == "linear":
        return 1000.0 + 7.0 * i
    if kind == "random":
        return rng.uniform(100.0, 5000.0, n)
    raise ValueError(kind)


SCHED_CASES = [(1, 1), (1, 16), (3, 4), (4, 8), (37, 13), (64, 16), (256, 16), (512, 16),
               (1024, 24), (2048, 32), (1024, 64), (32768, 2)]     # the last two: largest B*gamma, gamma, B


@pytest.mark.parametrize("B,gamma", SCHED_CASES)
def test_schedule_bit_exact(ds, oracle_mod, B, gamma):
    import torch
    rng = np.random.default_rng(B * 100 + gamma)
    ws = _ws(ds, B, gamma, 1000)
    for trial, (tie, zero, negz) in enumerate([(0.0, 0.0, False), (0.3, 0.0, False),
                                               (0.2, 0.3, False), (0.2, 0.5, True)]):
        P = synth.monotone_scores(B, gamma, seed=trial, tie_frac=tie, zero_frac=zero,
                                  neg_zero=negz)
        for kind in ("knee", "flat", "linear", "random"):
            Tstep = _tstep(kind, B, gamma, rng)
            L = torch.empty(B, dtype=torch.int32, device="cuda")
            N = torch.empty(1, dtype=torch.int32, device="cuda")
            F = torch.empty(1, dtype=torch.float64, device="cuda")
            ds.schedule_prefix(dev(P), dev(Tstep), L, N, F, ws)
            L_or, N_or, F_or, _ = oracle_mod.schedule(P, Tstep)
            np.testing.assert_array_equal(L.cpu().numpy(), L_or, err_msg=f"{kind} trial {trial}")
            assert int(N.item()) == N_or
            assert float(F.item()) == F_or      # bit-exact
    assert ds.get_error() == 0


def test_schedule_records_increasing_scores(ds):
    import torch
    P = synth.monotone_scores(8, 4, seed=0)
    P[3, 2] = min(1.0, P[3, 1] + 0.1)
    ws = _ws(ds, 8, 4, 100)
    L = torch.empty(8, dtype=torch.int32, device="cuda")
    N = torch.empty(1, dtype=torch.int32, device="cuda")
    F = torch.empty(1, dtype=torch.float64, device="cuda")
    ds.schedule_prefix(dev(P), dev(np.full(8 * 5 + 1, 100.0)), L, N, F, ws)
    assert ds.get_error() == 4
    assert 0 <= int(N.item()) <= 32 and (L.cpu().numpy() <= 4).all()


# ---------------------------------------------------------------------------- confidence
_CONF_EXTRA = {"large-vocab-part": synth.LARGE_VOCAB.with_(B=96),
               "gamma64": synth.Workload("conf B=5 gamma=64 d=256", B=5, gamma=64, V=1000, d=256)}


@pytest.mark.parametrize("name", ["tiny", "qwen3-8b", "large-vocab-part", "gamma64"])
def test_confidence_within_tolerance(ds, oracle_mod, name):
    import torch
    wl = _CONF_EXTRA.get(name) or synth.WORKLOADS[name]
    W1 = synth.w1(wl)
    h = synth.h_all(wl)
    anchor = synth.anchors(wl)
    x = synth.draft_tokens(wl.B, wl.gamma, wl.V, seed=3)
    w = synth.conf_w(wl)
    T = synth.temperatures(wl)
    c = torch.empty(wl.B, wl.gamma, dtype=torch.float32, device="cuda")
    P = torch.empty_like(c)
    ds.confidence_sts(dev_bf16(h), dev(anchor), dev(x), dev_bf16(W1), dev_bf16(w), wl.b_conf,
                      dev(T), c, P)
    ref = oracle_mod.confidence(h, anchor, x, W1, w, wl.b_conf, T)
    c_g, P_g = c.cpu().numpy(), P.cpu().numpy()
    assert np.abs(c_g - ref["c"]).max() <= TOL
    assert np.abs(P_g - ref["P64"]).max() <= TOL
    assert (np.diff(P_g.astype(np.float64), axis=1) <= 0).all()
    assert ds.get_error() == 0
    print(f"{name}: max |c - c_oracle| = {np.abs(c_g - ref['c']).max():.3e}")


# ---------------------------------------------------------------------------- draft
def _draft_gpu(ds, wl, U_dev, W1_dev, W2_dev, anchor):
    import torch
    x = torch.full((wl.B, wl.gamma), -1, dtype=torch.int32, device="cuda")
    lx = torch.full((wl.B, wl.gamma), float("nan"), dtype=torch.float32, device="cuda")
    ws = _ws(ds, wl.B, wl.gamma, wl.V)
    ds.draft_step(U_dev, dev(anchor), W1_dev, W2_dev, x, lx, ws, mode=wl.mode,
                  temperature=wl.tau, seed=wl.seed)
    st = ds.get_error()
    return x.cpu().numpy(), lx.cpu().numpy(), st


def quadrant_rows(B):
    """One request from every group of 32 rows (each TMEM lane quadrant of every M tile),
    at a varying lane, plus the first and the last request."""
    rows = {0, B - 1}
    for j in range((B + 31) // 32):
        rows.add(min(B - 1, 32 * j + (7 * j + 3) % 32))
    return sorted(rows)


def _check_draft(ds, oracle_mod, wl, sample=None, U_host=None, U_dev=None):
    W1, W2 = synth.w1(wl), synth.w2(wl)
    anchor = synth.anchors(wl)
    if U_dev is None:
        U_host = synth.u_all(wl) if U_host is None else U_host
        U_dev = dev_bf16(U_host)
    x, lx, st = _draft_gpu(ds, wl, U_dev, dev_bf16(W1), dev_bf16(W2), anchor)
    assert st == 0, ds.status_string(st)
    assert ((x >= 0) & (x < wl.V)).all()
    bs = list(range(wl.B)) if sample is None else list(sample)
    U_s = U_host[bs] if U_host is not None else synth.u_requests(wl, bs)
    x_or, l_or, gap_or = oracle_mod.draft(U_s, anchor[bs], W1, W2, mode=wl.mode, tau=wl.tau,
                                          seed=wl.seed, b_index=np.array(bs, np.int32),
                                          forced_prev=forced_prev(anchor[bs], x[bs]))
    cmp = compare_forced(x[bs], lx[bs], x_or, l_or, gap_or, name=f"{wl.name} ({len(bs)} rows)")
    print(f"{wl.name}: {cmp}")
    assert cmp.ok(), cmp
    assert cmp.compared + cmp.near_ties == len(bs) * wl.gamma
    return x, lx


STRESS = [
    synth.Workload("stress B=5 V=4104", B=5, gamma=6, V=4104, d=64, w_std=0.2),
    synth.Workload("stress B=1 V=64", B=1, gamma=9, V=64, d=64, w_std=0.3),
    synth.Workload("stress B=130 V=2056", B=130, gamma=3, V=2056, d=64, w_std=0.2),
    synth.Workload("stress B=128 V=10000", B=128, gamma=4, V=10000, d=64, w_std=0.2),
    synth.Workload("stress B=300 V=5000 gumbel", B=300, gamma=3, V=5000, d=64, w_std=0.2,
                   logits="zipf", mode=1, tau=0.7),
    synth.Workload("stress B=9 V=40000 gumbel", B=9, gamma=5, V=40000, d=64, w_std=0.2,
                   logits="normal", mode=1, tau=1.3, seed=5),
    # M = 64 tiles with 1- and 2-unit CTAs, a ragged vocabulary tail and a full 64-row tile
    synth.Workload("stress B=33 V=9000 gumbel", B=33, gamma=4, V=9000, d=64, w_std=0.2,
                   logits="normal", mode=1, tau=0.9, seed=3),
    synth.Workload("stress B=64 V=4104", B=64, gamma=5, V=4104, d=64, w_std=0.2, seed=2),
    # 5 and 10 units (160 and 320 columns) per CTA: a one-unit remainder tile on every CTA
    synth.Workload("stress B=20 V=23680", B=20, gamma=4, V=23680, d=64, w_std=0.2, seed=7),
    synth.Workload("stress B=48 V=47360 gumbel", B=48, gamma=3, V=47360, d=64, w_std=0.2,
                   mode=1, tau=0.8, seed=8),
    # the largest gamma the kernel takes, one row and a 130-row tile pair
    synth.Workload("stress B=3 gamma=64 V=2048", B=3, gamma=64, V=2048, d=64, w_std=0.3, seed=4),
    synth.Workload("stress B=130 gamma=64 V=1032", B=130, gamma=64, V=1032, d=64, w_std=0.3,
                   seed=6),
    # pair kernel: Gumbel-max over three 256-request blocks (one block per walk, the block
    # after next gathered into the buffer just released), and greedy over four blocks, two
    # per W2 tile, the last one partial (232 rows)
    synth.Workload("stress B=600 V=3000 gumbel", B=600, gamma=3, V=3000, d=64, w_std=0.2,
                   logits="zipf", mode=1, tau=0.7, seed=9),
    synth.Workload("stress B=1000 V=2056", B=1000, gamma=3, V=2056, d=64, w_std=0.2, seed=10),
]


@pytest.mark.parametrize("wl", STRESS, ids=[w.name for w in STRESS])
def test_draft_stress_shapes(ds, oracle_mod, wl):
    _check_draft(ds, oracle_mod, wl)


def test_draft_tiny_workload(ds, oracle_mod):
    _check_draft(ds, oracle_mod, synth.TINY)


def test_draft_qwen3_shaped_all_requests(ds, oracle_mod):
    _check_draft(ds, oracle_mod, synth.QWEN3_8B)


def test_draft_sampled_gumbel_workload(ds, oracle_mod):
    wl = synth.SAMPLED
    _check_draft(ds, oracle_mod, wl, sample=quadrant_rows(wl.B))


@pytest.mark.parametrize("B", synth.SWEEP_BS)
def test_draft_sweep_workloads(ds, oracle_mod, B):
    wl = synth.sweep(B)
    _check_draft(ds, oracle_mod, wl, sample=quadrant_rows(B))


def test_draft_large_vocab_workload(ds, oracle_mod):
    wl = synth.LARGE_VOCAB
    U_dev = synth.u_all_device_zipf(wl)
    _check_draft(ds, oracle_mod, wl, sample=quadrant_rows(wl.B), U_dev=U_dev)
    del U_dev


def test_draft_is_deterministic(ds):
    wl = STRESS[0]
    W1, W2 = dev_bf16(synth.w1(wl)), dev_bf16(synth.w2(wl))
    U = dev_bf16(synth.u_all(wl))
    a = _draft_gpu(ds, wl, U, W1, W2, synth.anchors(wl))
    b = _draft_gpu(ds, wl, U, W1, W2, synth.anchors(wl))
    np.testing.assert_array_equal(a[0], b[0])
    np.testing.assert_array_equal(a[1], b[1])


def test_draft_zero_factors_pick_backbone_argmax(ds):
    wl = synth.Workload("zero W", B=7, gamma=4, V=3000, d=64)
    U = synth.u_all(wl)
    zW1 = np.zeros((wl.V, wl.r), np.uint16)
    zW2 = np.zeros((wl.r, wl.V), np.uint16)
    x, lx, st = _draft_gpu(ds, wl, dev_bf16(U), dev_bf16(zW1), dev_bf16(zW2), synth.anchors(wl))
    assert st == 0
    Uf = synth.bf16_bits_to_f32(U)
    np.testing.assert_array_equal(x, np.argmax(Uf, axis=2))
    np.testing.assert_array_equal(lx, np.max(Uf, axis=2))


def test_draft_records_bad_anchor(ds):
    wl = STRESS[0]
    anchor = synth.anchors(wl)
    anchor[1] = wl.V + 5
    x, lx, st = _draft_gpu(ds, wl, dev_bf16(synth.u_all(wl)), dev_bf16(synth.w1(wl)),
                           dev_bf16(synth.w2(wl)), anchor)
    assert st == 7
    assert ((x >= 0) & (x < wl.V)).all()


# ---------------------------------------------------------------------------- whole path
def test_whole_path_tiny(ds, oracle_mod):
    """Draft -> confidence -> schedule -> verify on the GPU, against the oracle chain."""
    import torch
    wl = synth.TINY
    inp = synth.make_inputs(wl)
    x, lx, st = _draft_gpu(ds, wl, dev_bf16(inp.U), dev_bf16(inp.W1), dev_bf16(inp.W2), inp.anchor)
    assert st == 0
    x_or, l_or, gap_or = oracle_mod.draft(inp.U, inp.anchor, inp.W1, inp.W2)
    xf, lf, gf = oracle_mod.draft(inp.U, inp.anchor, inp.W1, inp.W2,
                                  forced_prev=forced_prev(inp.anchor, x))
    cmp = compare_forced(x, lx, xf, lf, gf, name="whole path tiny")
    assert cmp.ok() and cmp.near_ties == 0, cmp
    np.testing.assert_array_equal(x, x_or)
    c = torch.empty(wl.B, wl.gamma, dtype=torch.float32, device="cuda")
    P = torch.empty_like(c)
    ds.confidence_sts(dev_bf16(inp.h), dev(inp.anchor), dev(x), dev_bf16(inp.W1), dev_bf16(inp.w),
                      inp.b_conf, dev(inp.T), c, P)
    ref = oracle_mod.confidence(inp.h, inp.anchor, x_or, inp.W1, inp.w, inp.b_conf, inp.T)
    assert np.abs(c.cpu().numpy() - ref["c"]).max() <= TOL
    ws = _ws(ds, wl.B, wl.gamma, wl.V)
    L = torch.empty(wl.B, dtype=torch.int32, device="cuda")
    N = torch.empty(1, dtype=torch.int32, device="cuda")
    F = torch.empty(1, dtype=torch.float64, device="cuda")
    ds.schedule_prefix(P, dev(inp.Tstep), L, N, F, ws)
    L_or, N_or, F_or, _ = oracle_mod.schedule(P.cpu().numpy(), inp.Tstep)
    np.testing.assert_array_equal(L.cpu().numpy(), L_or)
    # the flat step-time curve of this workload makes verifying every draft optimal
    assert (L_or == wl.gamma).all()
    target = synth.targets(wl, x_or)
    acc = torch.empty(wl.B, dtype=torch.int32, device="cuda")
    bonus = torch.empty_like(acc)
    ds.verify_prefix(dev(x), L, dev(target), acc, bonus)
    a_or, b_or = oracle_mod.verify(x_or, L_or, target)
    np.testing.assert_array_equal(acc.cpu().numpy(), a_or)
    np.testing.assert_array_equal(bonus.cpu().numpy(), b_or)
    assert ds.get_error() == 0


def test_whole_path_qwen3_shaped(ds, oracle_mod):
    """The bench workload through all four calls; each stage's oracle is fed the GPU's
    output of the stage before (identical inputs), as the bench chains them."""
    import torch
    wl = synth.QWEN3_8B
    inp = synth.make_inputs(wl)
    x, lx, st = _draft_gpu(ds, wl, dev_bf16(inp.U), dev_bf16(inp.W1), dev_bf16(inp.W2), inp.anchor)
    assert st == 0
    xf, lf, gf = oracle_mod.draft(inp.U, inp.anchor, inp.W1, inp.W2,
                                  forced_prev=forced_prev(inp.anchor, x))
    cmp = compare_forced(x, lx, xf, lf, gf, name="whole path qwen3-8b (draft stage)")
    assert cmp.ok(), cmp
    c = torch.empty(wl.B, wl.gamma, dtype=torch.float32, device="cuda")
    P = torch.empty_like(c)
    ds.confidence_sts(dev_bf16(inp.h), dev(inp.anchor), dev(x), dev_bf16(inp.W1),
                      dev_bf16(inp.w), inp.b_conf, dev(inp.T), c, P)
    ref = oracle_mod.confidence(inp.h, inp.anchor, x, inp.W1, inp.w, inp.b_conf, inp.T)
    assert np.abs(c.cpu().numpy() - ref["c"]).max() <= TOL
    assert np.abs(P.cpu().numpy() - ref["P64"]).max() <= TOL
    ws = _ws(ds, wl.B, wl.gamma, wl.V)
    L = torch.empty(wl.B, dtype=torch.int32, device="cuda")
    N = torch.empty(1, dtype=torch.int32, device="cuda")
    F = torch.empty(1, dtype=torch.float64, device="cuda")
    ds.schedule_prefix(P, dev(inp.Tstep), L, N, F, ws)
    L_or, N_or, F_or, _ = oracle_mod.schedule(P.cpu().numpy(), inp.Tstep)
    np.testing.assert_array_equal(L.cpu().numpy(), L_or)
    assert int(N.item()) == N_or and float(F.item()) == F_or
    target = synth.targets(wl, x)
    acc = torch.empty(wl.B, dtype=torch.int32, device="cuda")
    bonus = torch.empty_like(acc)
    ds.verify_prefix(dev(x), L, dev(target), acc, bonus)
    a_or, b_or = oracle_mod.verify(x, L_or, target)
    np.testing.assert_array_equal(acc.cpu().numpy(), a_or)
    np.testing.assert_array_equal(bonus.cpu().numpy(), b_or)
    assert ds.get_error() == 0
