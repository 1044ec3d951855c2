"""Parity of the STS temperature fit (CUDA, through the C ABI) with the CPU oracle.

The fit is an argmin over a grid, taken on each side in its own summation: fp64 in
the oracle, 2^-40 fixed point on the device.  So the device's choice is checked the
way several correct answers are: with the earlier positions frozen at the device's
own choices, the oracle scores every candidate, and the device's candidate must be a
minimum of those scores to within the fixed-point bound; its reported ECE must equal
the oracle's score of it to the same bound.  Where the oracle's own argmin differs,
the two scores must tie within that bound (counted).
"""
import math

import numpy as np
import pytest

import synth
from helpers import dev

pytestmark = pytest.mark.gpu

ECE_TOL = 1e-11      # N * 2^-41 / N from the fixed point, plus fp64 rounding of the sums


@pytest.fixture(scope="module")
def ds():
    import torch
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import speculative_decoding_drafter_head_b200 as m
    m.load()
    assert m.get_error() == 0
    return m


def _gpu_fit(ds, z, acc, **grid):
    import torch
    N, gamma = z.shape
    g = dict(t_min=0.5, t_step=0.01, n_t=451, n_bins=15)
    g.update(grid)
    ws = torch.empty(ds.sts_fit_workspace_bytes(N, gamma, g["n_t"], g["n_bins"]),
                     dtype=torch.uint8, device="cuda")
    idx = torch.full((gamma,), -1, dtype=torch.int32, device="cuda")
    T = torch.zeros(gamma, dtype=torch.float32, device="cuda")
    e = torch.zeros(gamma, dtype=torch.float64, device="cuda")
    ds.sts_fit(dev(z), dev(acc), idx, T, e, ws, **g)
    assert ds.get_error() == 0
    return idx.cpu().numpy(), T.cpu().numpy(), e.cpu().numpy(), g


def _check_against_oracle(oracle_mod, z, acc, idx, T, e, g):
    gamma = z.shape[1]
    assert ((idx >= 0) & (idx < g["n_t"])).all()
    T64 = g["t_min"] + idx * g["t_step"]
    np.testing.assert_array_equal(T, T64.astype(np.float32))
    _, _, G = oracle_mod.sts_fit(z, acc, t_min=g["t_min"], t_step=g["t_step"], n_t=g["n_t"],
                                 n_bins=g["n_bins"], T_fixed=T64, return_grid=True)
    ties = 0
    for k in range(gamma):
        best = G[k].min()
        assert G[k][idx[k]] <= best + ECE_TOL, (k, G[k][idx[k]], best)
        assert abs(e[k] - G[k][idx[k]]) <= ECE_TOL, (k, e[k], G[k][idx[k]])
        if idx[k] != int(np.argmin(G[k])):
            ties += 1
    return ties


@pytest.mark.parametrize("N,gamma,seed", [(4096, 16, 0), (1000, 5, 1), (1, 3, 2), (257, 8, 3)])
def test_sts_fit_matches_oracle(ds, oracle_mod, N, gamma, seed):
    z, acc = synth.calibration_set(N, gamma, seed)
    idx, T, e, g = _gpu_fit(ds, z, acc)
    ties = _check_against_oracle(oracle_mod, z, acc, idx, T, e, g)
    print(f"N={N} gamma={gamma}: T={np.round(T, 2)} near-tie choices {ties}")
    if N >= 1000:
        T_or, _ = oracle_mod.sts_fit(z, acc)
        assert (np.abs(T - T_or) < 1e-6).sum() >= gamma - ties


@pytest.mark.parametrize("grid", [dict(n_t=37, n_bins=7, t_min=0.3, t_step=0.07),
                                  dict(n_t=1201, n_bins=15, t_min=0.25, t_step=0.005),
                                  dict(n_t=100, n_bins=256), dict(n_t=1, n_bins=1),
                                  dict(n_t=5, n_bins=3, t_step=0.0)])
def test_sts_fit_grid_shapes(ds, oracle_mod, grid):
    # ragged grids: fewer candidates than a warp, several CTA rows of candidates
    # (n_t > 512), the largest bin count (smaller CTAs), one candidate, a flat grid
    z, acc = synth.calibration_set(3001, 6, seed=9)
    idx, T, e, g = _gpu_fit(ds, z, acc, **grid)
    _check_against_oracle(oracle_mod, z, acc, idx, T, e, g)
    if grid.get("t_step") == 0.0 or grid["n_t"] == 1:
        assert (idx == 0).all()


def test_sts_fit_exact_calibration(ds):
    # two groups exactly calibrated at T = (2, 3): the ECE is zero there
    za, zb, z2 = 2 * math.log(0.3 / 0.7), 2 * math.log(0.7 / 0.3), 3 * math.log(4.0)
    z = np.zeros((100, 2), np.float32)
    z[:50, 0], z[50:, 0], z[:, 1] = za, zb, z2
    acc = np.zeros(100, np.int32)
    acc[:12] = 2; acc[12:15] = 1; acc[50:78] = 2; acc[78:85] = 1
    idx, T, e, _ = _gpu_fit(ds, z, acc)
    np.testing.assert_array_equal(idx, [150, 250])
    assert (e < 1e-6).all()


def test_sts_fit_full_calibration_set_and_determinism(ds, oracle_mod):
    # the calibration set the benchmark times: 65536 blocks, gamma = 16
    z, acc = synth.calibration_set(synth.STS_CALIBRATION_N, synth.STS_CALIBRATION_GAMMA, 0)
    a = _gpu_fit(ds, z, acc)
    b = _gpu_fit(ds, z, acc)
    for u, v in zip(a[:3], b[:3]):
        np.testing.assert_array_equal(u, v)
    ties = _check_against_oracle(oracle_mod, z, acc, *a)
    assert ties <= 1


def test_sts_fit_feeds_confidence(ds):
    # the fitted temperatures are the fp32 T that dspark_confidence_sts takes
    z, acc = synth.calibration_set(2048, 16, seed=5)
    idx, T, _, _ = _gpu_fit(ds, z, acc)
    assert T.dtype == np.float32 and (T > 0).all()
