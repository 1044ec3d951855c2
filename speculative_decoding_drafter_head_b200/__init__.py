"""DSpark drafter-head hot path on B200: Python binding of ``libdspark.so``.

The four calls mirror the C ABI in ``include/dspark.h`` one to one and only
marshal arguments: every step runs in the library's CUDA kernels on the caller's
current CUDA stream, over PyTorch-owned device tensors.  There is no fallback:
if the library cannot be loaded, or a tensor is not on a CUDA device, the call
raises.

    draft_step        Markov-head drafting (tcgen05 GEMM + fused add/argmax)
    draft_step_rnn    RNN-head drafting (recurrent state, same fused GEMM)
    draft_confidence_step  drafting and the confidence head in one call
    confidence_sts    confidence head, sequential temperature scaling, survival product
    schedule_prefix   hardware-aware prefix scheduler (global top-N + scan)
    verify_prefix     strict prefix-match verification
    sts_fit           fitting the per-position temperatures (ECE grid search)
"""
from __future__ import annotations

import ctypes as C
import os

from . import _build

__all__ = [
    "DSparkError", "load", "workspace_bytes", "draft_step", "draft_step_rnn",
    "draft_confidence_step", "step", "confidence_sts", "schedule_prefix",
    "verify_prefix", "sts_fit_workspace_bytes", "sts_fit", "get_error", "status_string", "set_wait_timeout_ns", "debug_barrier_extra",
    "STATUS",
]

STATUS = {
    0: "OK", 1: "INVALID_ARG", 2: "UNSUPPORTED_SHAPE", 3: "WORKSPACE_TOO_SMALL",
    4: "NOT_MONOTONE", 5: "CUDA_ERROR", 6: "TIMEOUT", 7: "INVALID_TOKEN",
    8: "BAD_LAUNCH",
}

EXPORTED = (
    "dspark_status_string", "dspark_workspace_bytes", "dspark_draft_step",
    "dspark_confidence_sts", "dspark_schedule_prefix", "dspark_verify_prefix",
    "dspark_get_error", "dspark_set_wait_timeout_ns", "dspark_debug_barrier_extra",
    "dspark_sts_fit_workspace_bytes", "dspark_sts_fit", "dspark_draft_step_rnn",
    "dspark_draft_confidence_step", "dspark_step",
)

_lib = None


class DSparkError(RuntimeError):
    def __init__(self, call: str, status: int):
        self.status = status
        super().__init__(f"{call}: {STATUS.get(status, status)} ({status_string(status)})")


def load(build_if_missing: bool = True):
    """Load libdspark.so (building it first with nvcc if it is missing or stale)."""
    global _lib
    if _lib is not None:
        return _lib
    if build_if_missing and _build.stale():
        _build.build()
    if not os.path.exists(_build.LIB):
        raise RuntimeError(f"libdspark.so not found at {_build.LIB}")
    lib = C.CDLL(_build.LIB)
    p, i, u64, f32, sz = C.c_void_p, C.c_int, C.c_uint64, C.c_float, C.c_size_t
    lib.dspark_status_string.argtypes = [i]
    lib.dspark_status_string.restype = C.c_char_p
    lib.dspark_workspace_bytes.argtypes = [i, i, i, i]
    lib.dspark_workspace_bytes.restype = sz
    lib.dspark_draft_step.argtypes = [p, p, p, p, i, i, i, i, i, f32, u64, i, p, p, p, sz, p]
    lib.dspark_draft_step_rnn.argtypes = [p, p, p, p, p, i, i, i, i, i, f32, u64, i, p, p, p, sz,
                                          p]
    lib.dspark_confidence_sts.argtypes = [p, p, p, p, p, f32, p, i, i, i, i, i, p, p, p]
    lib.dspark_draft_confidence_step.argtypes = [p, p, p, p, p, p, f32, p, i, i, i, i, i, i, f32,
                                                 u64, i, p, p, p, p, p, sz, p]
    lib.dspark_step.argtypes = [p, p, p, p, p, p, f32, p, p, p, i, i, i, i, i, i, f32, u64, i,
                                p, p, p, p, p, p, p, p, p, p, sz, p]
    lib.dspark_schedule_prefix.argtypes = [p, i, i, p, p, p, p, p, sz, p]
    lib.dspark_verify_prefix.argtypes = [p, p, p, i, i, p, p, p]
    lib.dspark_sts_fit_workspace_bytes.argtypes = [i, i, i, i]
    lib.dspark_sts_fit_workspace_bytes.restype = sz
    lib.dspark_sts_fit.argtypes = [p, p, i, i, C.c_double, C.c_double, i, i, p, p, p, p, sz, p]
    lib.dspark_get_error.argtypes = [p, C.POINTER(C.c_int)]
    lib.dspark_set_wait_timeout_ns.argtypes = [u64]
    lib.dspark_debug_barrier_extra.argtypes = [i]
    for name in EXPORTED:
        if name not in ("dspark_status_string", "dspark_workspace_bytes",
                        "dspark_sts_fit_workspace_bytes"):
            getattr(lib, name).restype = i
    _lib = lib
    return lib


def status_string(status: int) -> str:
    return load().dspark_status_string(int(status)).decode()


def _check(call: str, st: int):
    if st != 0:
        raise DSparkError(call, st)


def _stream(stream=None):
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return C.c_void_p(stream.cuda_stream)


def _dev(t, dtype, name):
    import torch
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return C.c_void_p(t.data_ptr())


def workspace_bytes(B: int, gamma: int, V: int, r: int = 256) -> int:
    return int(load().dspark_workspace_bytes(B, gamma, V, r))


def draft_step(U, anchor, W1, W2, x_out, logit_x_out, workspace, mode: int = 0,
               temperature: float = 1.0, seed: int = 0, b_offset: int = 0, stream=None):
    """Draft gamma tokens per request with the Markov head (see dspark_draft_step)."""
    import torch
    B, gamma, V = U.shape
    r = W1.shape[1]
    st = load().dspark_draft_step(
        _dev(U, torch.bfloat16, "U"), _dev(anchor, torch.int32, "anchor"),
        _dev(W1, torch.bfloat16, "W1"), _dev(W2, torch.bfloat16, "W2"), B, gamma, V, r,
        int(mode), float(temperature), int(seed) & (2**64 - 1), int(b_offset),
        _dev(x_out, torch.int32, "x_out"), _dev(logit_x_out, torch.float32, "logit_x_out"),
        _dev(workspace, torch.uint8, "workspace"), workspace.numel(), _stream(stream))
    _check("dspark_draft_step", st)


def draft_step_rnn(U, anchor, W1, W2, Whh, x_out, logit_x_out, workspace, mode: int = 0,
                   temperature: float = 1.0, seed: int = 0, b_offset: int = 0, stream=None):
    """Draft gamma tokens per request with the RNN head (see dspark_draft_step_rnn)."""
    import torch
    B, gamma, V = U.shape
    r = W1.shape[1]
    st = load().dspark_draft_step_rnn(
        _dev(U, torch.bfloat16, "U"), _dev(anchor, torch.int32, "anchor"),
        _dev(W1, torch.bfloat16, "W1"), _dev(W2, torch.bfloat16, "W2"),
        _dev(Whh, torch.bfloat16, "Whh"), B, gamma, V, r, int(mode), float(temperature),
        int(seed) & (2**64 - 1), int(b_offset), _dev(x_out, torch.int32, "x_out"),
        _dev(logit_x_out, torch.float32, "logit_x_out"),
        _dev(workspace, torch.uint8, "workspace"), workspace.numel(), _stream(stream))
    _check("dspark_draft_step_rnn", st)


def draft_confidence_step(U, anchor, W1, W2, h, w, b_conf: float, T, x_out, logit_x_out, c_out,
                          P_out, workspace, mode: int = 0, temperature: float = 1.0, seed: int = 0,
                          b_offset: int = 0, stream=None):
    """Drafting and the confidence head in one call (see dspark_draft_confidence_step)."""
    import torch
    B, gamma, V = U.shape
    r = W1.shape[1]
    d = h.shape[2]
    st = load().dspark_draft_confidence_step(
        _dev(U, torch.bfloat16, "U"), _dev(anchor, torch.int32, "anchor"),
        _dev(W1, torch.bfloat16, "W1"), _dev(W2, torch.bfloat16, "W2"),
        _dev(h, torch.bfloat16, "h"), _dev(w, torch.bfloat16, "w"), float(b_conf),
        _dev(T, torch.float32, "T"), B, gamma, V, r, d, int(mode), float(temperature),
        int(seed) & (2**64 - 1), int(b_offset), _dev(x_out, torch.int32, "x_out"),
        _dev(logit_x_out, torch.float32, "logit_x_out"), _dev(c_out, torch.float32, "c_out"),
        _dev(P_out, torch.float32, "P_out"), _dev(workspace, torch.uint8, "workspace"),
        workspace.numel(), _stream(stream))
    _check("dspark_draft_confidence_step", st)


def step(U, anchor, W1, W2, h, w, b_conf: float, T, Tstep_us, target, x_out, logit_x_out,
         c_out, P_out, L_out, N_out, objective_out, accepted_out, bonus_out, workspace,
         mode: int = 0, temperature: float = 1.0, seed: int = 0, b_offset: int = 0,
         stream=None):
    """The whole per-step path in one call (see dspark_step)."""
    import torch
    B, gamma, V = U.shape
    r = W1.shape[1]
    d = h.shape[2]
    st = load().dspark_step(
        _dev(U, torch.bfloat16, "U"), _dev(anchor, torch.int32, "anchor"),
        _dev(W1, torch.bfloat16, "W1"), _dev(W2, torch.bfloat16, "W2"),
        _dev(h, torch.bfloat16, "h"), _dev(w, torch.bfloat16, "w"), float(b_conf),
        _dev(T, torch.float32, "T"), _dev(Tstep_us, torch.float64, "Tstep_us"),
        _dev(target, torch.int32, "target"), B, gamma, V, r, d, int(mode), float(temperature),
        int(seed) & (2**64 - 1), int(b_offset), _dev(x_out, torch.int32, "x_out"),
        _dev(logit_x_out, torch.float32, "logit_x_out"), _dev(c_out, torch.float32, "c_out"),
        _dev(P_out, torch.float32, "P_out"), _dev(L_out, torch.int32, "L_out"),
        _dev(N_out, torch.int32, "N_out"), _dev(objective_out, torch.float64, "objective_out"),
        _dev(accepted_out, torch.int32, "accepted_out"), _dev(bonus_out, torch.int32, "bonus_out"),
        _dev(workspace, torch.uint8, "workspace"), workspace.numel(), _stream(stream))
    _check("dspark_step", st)


def confidence_sts(h, anchor, x, W1, w, b_conf: float, T, c_out, P_out, stream=None):
    """Confidence, STS and prefix survival (see dspark_confidence_sts)."""
    import torch
    B, gamma, d = h.shape
    V, r = W1.shape
    st = load().dspark_confidence_sts(
        _dev(h, torch.bfloat16, "h"), _dev(anchor, torch.int32, "anchor"),
        _dev(x, torch.int32, "x"), _dev(W1, torch.bfloat16, "W1"), _dev(w, torch.bfloat16, "w"),
        float(b_conf), _dev(T, torch.float32, "T"), B, gamma, d, r, V,
        _dev(c_out, torch.float32, "c_out"), _dev(P_out, torch.float32, "P_out"), _stream(stream))
    _check("dspark_confidence_sts", st)


def schedule_prefix(P, Tstep_us, L_out, N_out, objective_out, workspace, stream=None):
    """Prefix scheduler (see dspark_schedule_prefix)."""
    import torch
    B, gamma = P.shape
    st = load().dspark_schedule_prefix(
        _dev(P, torch.float32, "P"), B, gamma, _dev(Tstep_us, torch.float64, "Tstep_us"),
        _dev(L_out, torch.int32, "L_out"), _dev(N_out, torch.int32, "N_out"),
        _dev(objective_out, torch.float64, "objective_out"),
        _dev(workspace, torch.uint8, "workspace"), workspace.numel(), _stream(stream))
    _check("dspark_schedule_prefix", st)


def verify_prefix(x, L, target, accepted_out, bonus_out, stream=None):
    """Strict prefix-match verification (see dspark_verify_prefix)."""
    import torch
    B, gamma = x.shape
    st = load().dspark_verify_prefix(
        _dev(x, torch.int32, "x"), _dev(L, torch.int32, "L"), _dev(target, torch.int32, "target"),
        B, gamma, _dev(accepted_out, torch.int32, "accepted_out"),
        _dev(bonus_out, torch.int32, "bonus_out"), _stream(stream))
    _check("dspark_verify_prefix", st)


def sts_fit_workspace_bytes(N: int, gamma: int, n_t: int, n_bins: int) -> int:
    return int(load().dspark_sts_fit_workspace_bytes(N, gamma, n_t, n_bins))


def sts_fit(z, accepted, index_out, T_out, ece_out, workspace, t_min: float = 0.5,
            t_step: float = 0.01, n_t: int = 451, n_bins: int = 15, stream=None):
    """Fit the per-position STS temperatures on a calibration set (see dspark_sts_fit)."""
    import torch
    N, gamma = z.shape
    st = load().dspark_sts_fit(
        _dev(z, torch.float32, "z"), _dev(accepted, torch.int32, "accepted"), N, gamma,
        float(t_min), float(t_step), int(n_t), int(n_bins),
        _dev(index_out, torch.int32, "index_out"), _dev(T_out, torch.float32, "T_out"),
        _dev(ece_out, torch.float64, "ece_out"), _dev(workspace, torch.uint8, "workspace"),
        workspace.numel(), _stream(stream))
    _check("dspark_sts_fit", st)


def get_error(stream=None) -> int:
    """Synchronise the stream and return (and clear) the device error word."""
    out = C.c_int(0)
    _check("dspark_get_error", load().dspark_get_error(_stream(stream), C.byref(out)))
    return int(out.value)


def set_wait_timeout_ns(ns: int):
    _check("dspark_set_wait_timeout_ns", load().dspark_set_wait_timeout_ns(int(ns)))


def debug_barrier_extra(extra: int):
    _check("dspark_debug_barrier_extra", load().dspark_debug_barrier_extra(int(extra)))
