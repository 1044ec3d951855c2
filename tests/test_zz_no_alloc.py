"""The scheduler entry point for callers that cannot allocate device memory.

dspark_schedule_prefix_noalloc takes no workspace: it is for callers whose device
memory is fixed at start-up or who must not call cudaMalloc on this path.  Its
scratch is a static array inside the library, so its results must equal those of
the workspace entry point (bit for bit, like every scheduler check here) on
consecutive calls that reuse that array.  This file is collected last on purpose.
"""
import ctypes as C

import numpy as np
import pytest

import synth

pytestmark = pytest.mark.gpu


def _schedule(lib, fn_name, P, Tstep, ws=None):
    import torch
    B, gamma = P.shape
    dP = torch.from_numpy(P).cuda()
    dT = torch.from_numpy(Tstep).cuda()
    L = torch.full((B,), -1, dtype=torch.int32, device="cuda")
    N = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    F = torch.full((1,), -1.0, dtype=torch.float64, device="cuda")
    stream = C.c_void_p(torch.cuda.current_stream().cuda_stream)
    args = [C.c_void_p(dP.data_ptr()), B, gamma, C.c_void_p(dT.data_ptr()),
            C.c_void_p(L.data_ptr()), C.c_void_p(N.data_ptr()), C.c_void_p(F.data_ptr())]
    if ws is not None:
        args += [C.c_void_p(ws.data_ptr()), C.c_size_t(ws.numel())]
    st = getattr(lib, fn_name)(*args, stream)
    assert st == 0, st
    torch.cuda.synchronize()
    return L.cpu().numpy(), int(N.item()), float(F.item())


def test_noalloc_scheduler_matches_workspace_scheduler_on_consecutive_calls(oracle_mod):
    import torch
    import speculative_decoding_drafter_head_b200 as ds
    lib = ds.load()
    f = lib.dspark_schedule_prefix_noalloc
    f.argtypes = [C.c_void_p, C.c_int, C.c_int, C.c_void_p, C.c_void_p, C.c_void_p, C.c_void_p,
                  C.c_void_p]
    f.restype = C.c_int
    # calls in a row that share the static scratch: the largest size first, so that a
    # smaller call runs over leftovers of a larger one; then a case with -0.0 scores
    # (equal to +0.0) and ties, and the largest size again
    cases = [(1024, 24, 0.3, 0.0, False), (64, 16, 0.0, 0.0, False),
             (512, 16, 0.2, 0.5, True), (1024, 24, 0.0, 0.0, False)]
    for B, gamma, tie, zero, negz in cases:
        P = synth.monotone_scores(B, gamma, seed=B, tie_frac=tie, zero_frac=zero, neg_zero=negz)
        n = np.arange(B * (gamma + 1) + 1, dtype=np.float64)
        Tstep = 15000.0 + 20.0 * np.maximum(0.0, n - (B * (gamma + 1)) // 3)
        ws = torch.empty(ds.workspace_bytes(B, gamma, 1000), dtype=torch.uint8, device="cuda")
        ref = _schedule(lib, "dspark_schedule_prefix", P, Tstep, ws)
        got = _schedule(lib, "dspark_schedule_prefix_noalloc", P, Tstep)
        L_or, N_or, F_or, _ = oracle_mod.schedule(P, Tstep)
        np.testing.assert_array_equal(got[0], ref[0])
        assert got[1] == ref[1] and got[2] == ref[2]
        np.testing.assert_array_equal(got[0], L_or)
        assert got[1] == N_or and got[2] == F_or
        assert 0 < ref[1] <= B * gamma
    assert ds.get_error() == 0


def test_noalloc_scheduler_rejects_sizes_beyond_its_scratch():
    import speculative_decoding_drafter_head_b200 as ds
    lib = ds.load()
    f = lib.dspark_schedule_prefix_noalloc
    f.argtypes = [C.c_void_p, C.c_int, C.c_int, C.c_void_p, C.c_void_p, C.c_void_p, C.c_void_p,
                  C.c_void_p]
    fake = C.c_void_p(0x10000)
    assert f(fake, 1025, 24, fake, fake, fake, fake, None) == 2     # 24600 > 24576 scores
    assert f(fake, 4, 65, fake, fake, fake, fake, None) == 2
