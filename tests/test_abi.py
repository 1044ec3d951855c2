"""The C-ABI library loads on a CPU-only host, exports every declared entry point and
rejects bad arguments on the host before touching the device."""
import ctypes as C
import os
import re

import pytest

import speculative_decoding_drafter_head_b200 as ds

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    text = open(os.path.join(ROOT, "include", "dspark.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(dspark_\w+)\s*\(", text)))


def test_library_exports_every_declared_symbol():
    lib = ds.load()
    names = _declared()
    assert "dspark_draft_step" in names and len(names) >= 9
    for name in names:
        assert hasattr(lib, name), name
    assert set(ds.EXPORTED) <= set(names)


def test_status_strings():
    assert ds.status_string(0) == "ok"
    for code in range(1, 9):
        assert ds.status_string(code) != "unknown status"
    assert ds.status_string(99) == "unknown status"


def test_workspace_bytes_covers_both_users():
    n = 64 * 16
    ws = ds.workspace_bytes(64, 16, 151936)
    assert ws >= 256 + n * 8 and ws >= 256 + n * 12
    assert ds.workspace_bytes(0, 16, 100) == 0


_FAKE = C.c_void_p(0x10000)   # never dereferenced: every call below fails its host checks


def test_draft_step_host_checks():
    lib = ds.load()
    f = lib.dspark_draft_step
    args = dict(U=_FAKE, anchor=_FAKE, W1=_FAKE, W2=_FAKE, B=64, gamma=16, V=151936, r=256,
                mode=0, temperature=1.0, seed=0, b_offset=0, x=_FAKE, lx=_FAKE, ws=_FAKE,
                wsb=1 << 30, stream=None)

    def call(**kw):
        a = {**args, **kw}
        return f(a["U"], a["anchor"], a["W1"], a["W2"], a["B"], a["gamma"], a["V"], a["r"],
                 a["mode"], a["temperature"], a["seed"], a["b_offset"], a["x"], a["lx"], a["ws"],
                 a["wsb"], a["stream"])

    assert call(U=None) == 1
    assert call(U=C.c_void_p(0x10008)) == 1          # not 16-byte aligned
    assert call(mode=2) == 1
    assert call(mode=1, temperature=0.0) == 1
    assert call(r=128) == 2
    assert call(V=151937) == 2
    assert call(B=0) == 2 and call(B=1025) == 2
    assert call(gamma=65) == 2
    assert call(wsb=100) == 3


def test_draft_confidence_step_host_checks():
    lib = ds.load()
    f = lib.dspark_draft_confidence_step
    args = dict(U=_FAKE, anchor=_FAKE, W1=_FAKE, W2=_FAKE, h=_FAKE, w=_FAKE, b_conf=1.0, T=_FAKE,
                B=64, gamma=16, V=151936, r=256, d=4096, mode=0, temperature=1.0, seed=0,
                b_offset=0, x=_FAKE, lx=_FAKE, c=_FAKE, P=_FAKE, ws=_FAKE, wsb=1 << 30, stream=None)

    def call(**kw):
        a = {**args, **kw}
        return f(a["U"], a["anchor"], a["W1"], a["W2"], a["h"], a["w"], a["b_conf"], a["T"], a["B"],
                 a["gamma"], a["V"], a["r"], a["d"], a["mode"], a["temperature"], a["seed"],
                 a["b_offset"], a["x"], a["lx"], a["c"], a["P"], a["ws"], a["wsb"], a["stream"])

    assert call(h=None) == 1 and call(P=None) == 1
    assert call(h=C.c_void_p(0x10008)) == 1          # not 16-byte aligned
    assert call(d=1020) == 2
    assert call(U=None) == 1                          # the drafting checks apply as well
    assert call(B=1025) == 2
    assert call(wsb=100) == 3


def test_step_host_checks():
    lib = ds.load()
    f = lib.dspark_step
    args = dict(U=_FAKE, anchor=_FAKE, W1=_FAKE, W2=_FAKE, h=_FAKE, w=_FAKE, b_conf=1.0, T=_FAKE,
                Tstep=_FAKE, target=_FAKE, B=64, gamma=16, V=151936, r=256, d=4096, mode=0,
                temperature=1.0, seed=0, b_offset=0, x=_FAKE, lx=_FAKE, c=_FAKE, P=_FAKE,
                L=_FAKE, N=_FAKE, obj=_FAKE, acc=_FAKE, bonus=_FAKE, ws=_FAKE, wsb=1 << 30,
                stream=None)

    def call(**kw):
        a = {**args, **kw}
        return f(a["U"], a["anchor"], a["W1"], a["W2"], a["h"], a["w"], a["b_conf"], a["T"],
                 a["Tstep"], a["target"], a["B"], a["gamma"], a["V"], a["r"], a["d"], a["mode"],
                 a["temperature"], a["seed"], a["b_offset"], a["x"], a["lx"], a["c"], a["P"],
                 a["L"], a["N"], a["obj"], a["acc"], a["bonus"], a["ws"], a["wsb"], a["stream"])

    assert call(Tstep=None) == 1 and call(bonus=None) == 1 and call(target=None) == 1
    assert call(obj=C.c_void_p(0x10004)) == 1          # fp64 output not 8-byte aligned
    assert call(B=1024, gamma=65) == 2                  # B gamma above the scheduler's limit
    assert call(wsb=100) == 3
    assert call(h=None) == 1 and call(d=1020) == 2      # the confidence checks apply (B <= 128)
    assert call(U=None) == 1                            # and the drafting checks


def test_schedule_and_verify_host_checks():
    lib = ds.load()
    s = lib.dspark_schedule_prefix
    assert s(None, 4, 4, _FAKE, _FAKE, _FAKE, _FAKE, _FAKE, 1 << 20, None) == 1
    assert s(_FAKE, 4, 65, _FAKE, _FAKE, _FAKE, _FAKE, _FAKE, 1 << 20, None) == 2
    assert s(_FAKE, 2048, 64, _FAKE, _FAKE, _FAKE, _FAKE, _FAKE, 1 << 30, None) == 2
    assert s(_FAKE, 4, 4, _FAKE, _FAKE, _FAKE, _FAKE, _FAKE, 16, None) == 3
    v = lib.dspark_verify_prefix
    assert v(None, _FAKE, _FAKE, 4, 4, _FAKE, _FAKE, None) == 1
    assert v(_FAKE, _FAKE, _FAKE, 0, 4, _FAKE, _FAKE, None) == 2
    c = lib.dspark_confidence_sts
    assert c(_FAKE, _FAKE, _FAKE, _FAKE, _FAKE, 1.0, _FAKE, 4, 8, 1020, 256, 100, _FAKE, _FAKE,
             None) == 2
    assert lib.dspark_set_wait_timeout_ns(0) == 1
    assert lib.dspark_debug_barrier_extra(-1) == 1


def test_binding_rejects_cpu_tensors():
    import torch
    with pytest.raises(TypeError):
        ds.verify_prefix(torch.zeros(2, 3, dtype=torch.int32), torch.zeros(2, dtype=torch.int32),
                         torch.zeros(2, 4, dtype=torch.int32), torch.zeros(2, dtype=torch.int32),
                         torch.zeros(2, dtype=torch.int32))


def test_sts_fit_host_checks():
    lib = ds.load()
    f = lib.dspark_sts_fit
    need = ds.sts_fit_workspace_bytes(4096, 16, 451, 15)
    assert need >= 4096 * 16 + 16 * 451 * 15 * 12
    assert ds.sts_fit_workspace_bytes(0, 16, 451, 15) == 0
    args = dict(z=_FAKE, acc=_FAKE, N=4096, gamma=16, t_min=0.5, t_step=0.01, n_t=451, n_bins=15,
                idx=_FAKE, T=_FAKE, e=_FAKE, ws=C.c_void_p(0x10000), wsb=need, stream=None)

    def call(**kw):
        a = {**args, **kw}
        return f(a["z"], a["acc"], a["N"], a["gamma"], a["t_min"], a["t_step"], a["n_t"],
                 a["n_bins"], a["idx"], a["T"], a["e"], a["ws"], a["wsb"], a["stream"])

    assert call(z=None) == 1
    assert call(e=C.c_void_p(0x10004)) == 1            # fp64 output not 8-byte aligned
    assert call(ws=C.c_void_p(0x10080)) == 1           # workspace not 256-byte aligned
    assert call(t_min=0.0) == 1 and call(t_step=-0.01) == 1
    assert call(N=0) == 2 and call(N=1 << 23) == 2     # fixed-point sums need N < 2^23
    assert call(gamma=65) == 2 and call(n_bins=257) == 2 and call(n_t=0) == 2
    assert call(wsb=need - 1) == 3


def test_draft_step_rnn_host_checks():
    lib = ds.load()
    f = _FAKE
    # a null or misaligned recurrence matrix is rejected before anything is enqueued
    assert lib.dspark_draft_step_rnn(f, f, f, f, None, 4, 2, 4096, 256, 0, 1.0, 0, 0, f, f, f,
                                     1 << 20, None) == 1
    assert lib.dspark_draft_step_rnn(f, f, f, f, C.c_void_p(0x10008), 4, 2, 4096, 256, 0, 1.0, 0,
                                     0, f, f, f, 1 << 20, None) == 1
    # the workspace also holds the [B, 256] state: fp32 + bf16 per row
    assert ds.workspace_bytes(1000, 16, 4096) >= 1000 * 256 * 6
