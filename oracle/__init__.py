"""CPU oracle of the DSpark drafter-head path (fp64, plain loops).

TEST INFRASTRUCTURE: only ``tests/``, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline leg import this package.  The CUDA library and its
Python binding never import it, and it imports nothing from them.

``build()`` compiles ``dspark_oracle.c`` with gcc into ``liboracle.so`` next
to it; the functions below marshal numpy arrays into the C entry points.
"""
from __future__ import annotations

import ctypes as C
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "dspark_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (OpenMP, no FMA contraction)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O3", "-std=c11", "-fopenmp", "-ffp-contract=off",
                               "-fno-fast-math", "-shared", "-fPIC", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        lib = C.CDLL(_LIB)
        p = C.c_void_p
        lib.oracle_num_threads.restype = C.c_int
        lib.oracle_philox4x32_10.argtypes = [p, p, p]
        lib.oracle_uniform_from_word.argtypes = [C.c_uint32]
        lib.oracle_uniform_from_word.restype = C.c_double
        lib.oracle_gumbel.argtypes = [C.c_uint64, C.c_int, C.c_int, C.c_int]
        lib.oracle_gumbel.restype = C.c_double
        lib.oracle_draft.argtypes = [p, p, p, p, C.c_int, C.c_int, C.c_int, C.c_int, C.c_int,
                                     C.c_double, C.c_uint64, p, p, p, p, p, C.c_int]
        lib.oracle_draft.restype = C.c_int
        lib.oracle_draft_rnn.argtypes = [p, p, p, p, p, C.c_int, C.c_int, C.c_int, C.c_int,
                                         C.c_int, C.c_double, C.c_uint64, p, p, p, p, p, C.c_int]
        lib.oracle_draft_rnn.restype = C.c_int
        lib.oracle_confidence.argtypes = [p, p, p, p, p, C.c_double, p, C.c_int, C.c_int,
                                          C.c_int, C.c_int, C.c_int, p, p, p, p, C.c_int]
        lib.oracle_confidence.restype = C.c_int
        lib.oracle_schedule.argtypes = [p, C.c_int, C.c_int, p, p, p, p, p]
        lib.oracle_schedule.restype = C.c_int
        lib.oracle_verify.argtypes = [p, p, p, C.c_int, C.c_int, p, p]
        lib.oracle_verify.restype = C.c_int
        lib.oracle_ece.argtypes = [p, p, C.c_int, C.c_int, C.c_int]
        lib.oracle_ece.restype = C.c_double
        lib.oracle_sts_fit.argtypes = [p, p, C.c_int, C.c_int, C.c_double, C.c_double, C.c_int,
                                       C.c_int, p, p, p, p, C.c_int]
        lib.oracle_sts_fit.restype = C.c_int
        _lib = lib
    return _lib


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(C.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def num_threads() -> int:
    return int(_load().oracle_num_threads())


def philox4x32_10(ctr, key) -> np.ndarray:
    ctr = _c(ctr, np.uint32)
    key = _c(key, np.uint32)
    out = np.zeros(4, dtype=np.uint32)
    _load().oracle_philox4x32_10(_ptr(ctr), _ptr(key), _ptr(out))
    return out


def uniform_from_word(w: int) -> float:
    return float(_load().oracle_uniform_from_word(int(w) & 0xFFFFFFFF))


def gumbel(seed: int, b: int, k: int, v: int) -> float:
    return float(_load().oracle_gumbel(int(seed), int(b), int(k), int(v)))


def _forced(forced_prev, nb, gamma):
    if forced_prev is None:
        return None, None
    fp = _c(forced_prev, np.int32)
    assert fp.shape == (nb, gamma)
    return fp, _ptr(fp)


def draft(U, anchor, W1, W2, mode: int = 0, tau: float = 1.0, seed: int = 0, b_index=None,
          nthreads: int = 0, forced_prev=None):
    """Markov-head drafting; returns (x [nb, gamma] int32, logit [nb, gamma] f64, gap f64).

    forced_prev [nb, gamma] (optional): teacher-forced use, position k conditions on
    x_{k-1} = forced_prev[:, k-1] rather than on the token this call picked at k - 1.
    """
    U = _c(U, np.uint16)
    nb, gamma, V = U.shape
    W1 = _c(W1, np.uint16)
    W2 = _c(W2, np.uint16)
    r = W1.shape[1]
    assert W1.shape == (V, r) and W2.shape == (r, V)
    anchor = _c(anchor, np.int32)
    assert anchor.shape == (nb,)
    bi = _c(np.arange(nb) if b_index is None else b_index, np.int32)
    x = np.zeros((nb, gamma), dtype=np.int32)
    logit = np.zeros((nb, gamma), dtype=np.float64)
    gap = np.zeros((nb, gamma), dtype=np.float64)
    fp, fp_ptr = _forced(forced_prev, nb, gamma)
    st = _load().oracle_draft(_ptr(U), _ptr(anchor), _ptr(W1), _ptr(W2), nb, gamma, V, r,
                              int(mode), float(tau), int(seed) & (2**64 - 1), _ptr(bi), _ptr(x),
                              _ptr(logit), _ptr(gap), fp_ptr, int(nthreads))
    if st != 0:
        raise ValueError(f"oracle_draft rejected its arguments (status {st})")
    return x, logit, gap


def draft_rnn(U, anchor, W1, W2, Whh, mode: int = 0, tau: float = 1.0, seed: int = 0,
              b_index=None, nthreads: int = 0, forced_prev=None):
    """RNN-head drafting (Elman reading); returns (x, logit, gap) as draft()."""
    U = _c(U, np.uint16)
    nb, gamma, V = U.shape
    W1 = _c(W1, np.uint16)
    W2 = _c(W2, np.uint16)
    Whh = _c(Whh, np.uint16)
    r = W1.shape[1]
    assert W1.shape == (V, r) and W2.shape == (r, V) and Whh.shape == (r, r)
    anchor = _c(anchor, np.int32)
    bi = _c(np.arange(nb) if b_index is None else b_index, np.int32)
    x = np.zeros((nb, gamma), dtype=np.int32)
    logit = np.zeros((nb, gamma), dtype=np.float64)
    gap = np.zeros((nb, gamma), dtype=np.float64)
    fp, fp_ptr = _forced(forced_prev, nb, gamma)
    st = _load().oracle_draft_rnn(_ptr(U), _ptr(anchor), _ptr(W1), _ptr(W2), _ptr(Whh), nb,
                                  gamma, V, r, int(mode), float(tau), int(seed) & (2**64 - 1),
                                  _ptr(bi), _ptr(x), _ptr(logit), _ptr(gap), fp_ptr,
                                  int(nthreads))
    if st != 0:
        raise ValueError(f"oracle_draft_rnn rejected its arguments (status {st})")
    return x, logit, gap


def confidence(h, anchor, x, W1, w, b_conf: float, T, nthreads: int = 0):
    """Confidence/STS/survival; returns dict z, c, P64 (f64) and P32 (f32), each [B, gamma]."""
    h = _c(h, np.uint16)
    B, gamma, d = h.shape
    W1 = _c(W1, np.uint16)
    V, r = W1.shape
    w = _c(w, np.uint16)
    assert w.shape == (d + r,)
    anchor = _c(anchor, np.int32)
    x = _c(x, np.int32)
    T = _c(T, np.float32)
    assert x.shape == (B, gamma) and T.shape == (gamma,)
    z = np.zeros((B, gamma)); c = np.zeros((B, gamma)); P64 = np.zeros((B, gamma))
    P32 = np.zeros((B, gamma), dtype=np.float32)
    st = _load().oracle_confidence(_ptr(h), _ptr(anchor), _ptr(x), _ptr(W1), _ptr(w),
                                   float(b_conf), _ptr(T), B, gamma, d, r, V, _ptr(z), _ptr(c),
                                   _ptr(P64), _ptr(P32), int(nthreads))
    if st != 0:
        raise ValueError(f"oracle_confidence rejected its arguments (status {st})")
    return {"z": z, "c": c, "P64": P64, "P32": P32}


def schedule(P, Tstep):
    """Prefix scheduler; returns (L [B] int32, N*, F(N*), F_all [B gamma + 1])."""
    P = _c(P, np.float32)
    B, gamma = P.shape
    Tstep = _c(Tstep, np.float64)
    assert Tstep.shape[0] >= B * (gamma + 1) + 1
    L = np.zeros(B, dtype=np.int32)
    N = np.zeros(1, dtype=np.int32)
    F = np.zeros(1, dtype=np.float64)
    F_all = np.zeros(B * gamma + 1, dtype=np.float64)
    st = _load().oracle_schedule(_ptr(P), B, gamma, _ptr(Tstep), _ptr(L), _ptr(N), _ptr(F),
                                 _ptr(F_all))
    if st != 0:
        raise ValueError(f"oracle_schedule rejected its arguments (status {st})")
    return L, int(N[0]), float(F[0]), F_all


def verify(x, L, target):
    """Strict prefix-match verification; returns (accepted [B], bonus [B]) int32."""
    x = _c(x, np.int32)
    B, gamma = x.shape
    L = _c(L, np.int32)
    target = _c(target, np.int32)
    assert target.shape == (B, gamma + 1) and L.shape == (B,)
    acc = np.zeros(B, dtype=np.int32)
    bonus = np.zeros(B, dtype=np.int32)
    st = _load().oracle_verify(_ptr(x), _ptr(L), _ptr(target), B, gamma, _ptr(acc), _ptr(bonus))
    if st != 0:
        raise ValueError(f"oracle_verify rejected its arguments (status {st})")
    return acc, bonus


def ece(P, accepted, k: int, n_bins: int = 15) -> float:
    """Expected calibration error of survival scores P [N] for position k (1-based)."""
    P = _c(P, np.float64)
    acc = _c(accepted, np.int32)
    return float(_load().oracle_ece(_ptr(P), _ptr(acc), P.shape[0], int(k), int(n_bins)))


def sts_fit(z, accepted, t_min: float = 0.5, t_step: float = 0.01, n_t: int = 451,
            n_bins: int = 15, T_fixed=None, return_grid: bool = False, nthreads: int = 0):
    """Sequential temperature scaling fit; returns (T [gamma], ece [gamma]) in fp64.

    With T_fixed [gamma], each position is frozen at T_fixed[k] rather than at its
    own choice before the next position is fitted.  With return_grid, a third
    value holds every candidate's ECE [gamma, n_t].
    """
    z = _c(z, np.float32)
    N, gamma = z.shape
    acc = _c(accepted, np.int32)
    assert acc.shape == (N,)
    fixed = None if T_fixed is None else _c(T_fixed, np.float64)
    assert fixed is None or fixed.shape == (gamma,)
    T = np.zeros(gamma)
    e = np.zeros(gamma)
    grid = np.zeros((gamma, n_t)) if return_grid else None
    st = _load().oracle_sts_fit(_ptr(z), _ptr(acc), N, gamma, float(t_min), float(t_step),
                                int(n_t), int(n_bins), None if fixed is None else _ptr(fixed),
                                _ptr(T), _ptr(e), None if grid is None else _ptr(grid),
                                int(nthreads))
    if st != 0:
        raise ValueError(f"oracle_sts_fit rejected its arguments (status {st})")
    return (T, e, grid) if return_grid else (T, e)
