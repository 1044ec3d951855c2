"""Seeded synthetic inputs for the DSpark drafter-head path.

This module is shared by the CPU oracle's tests, the GPU parity tests and the
benchmark.  It draws random tensors with the shapes and value distributions of
the synthetic workloads and holds none of the method's arithmetic: no logits,
no bias contraction, no argmax, no sigmoid, no product, no scheduling.

Every tensor comes from its own numpy PCG64 stream, keyed by
``SeedSequence([seed, tag])`` or, for per-request tensors, by
``SeedSequence([seed, tag, b])`` so that any subset of requests can be drawn
without drawing the others.  Floating-point values are drawn in fp32, scaled in
fp32 and rounded to bf16 with round-to-nearest-even on the fp32 bit pattern.
bf16 tensors are carried as ``uint16`` bit patterns.

Workload shapes follow the DSpark pages: the Markov head's rank r = 256 and its
two factors W1 [V, r] and W2 [r, V] (gdymind.com "DSpark", section 4, "Markov
head"); gamma drafted positions whose first one is predicted from the anchor
(same section, "Parallel stage"); per-position acceptance that decays from 0.88
to 0.78 (seventnews.com article, "Two bottlenecks DeepSeek identified").
"""
from __future__ import annotations

import math
import os
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass, replace
from typing import Optional, Sequence

import numpy as np

# stream tags (one per tensor kind)
TAG_W1, TAG_W2, TAG_U, TAG_H, TAG_ANCHOR, TAG_W, TAG_T, TAG_TARGET, TAG_ZIPF = range(1, 10)
TAG_SCORES, TAG_VERIFY, TAG_TSTEP, TAG_CALIB, TAG_WHH = 10, 11, 12, 13, 14

_THREADS = max(1, min(16, os.cpu_count() or 1))


# ----------------------------------------------------------------------------
# bf16 bit helpers
# ----------------------------------------------------------------------------
def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round fp32 values to bf16 (round to nearest, ties to even); returns uint16 bits."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    u = a.view(np.uint32)
    rounding = np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))
    return ((u + rounding) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(h: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns to fp32."""
    h = np.ascontiguousarray(h, dtype=np.uint16)
    return (h.astype(np.uint32) << np.uint32(16)).view(np.float32)


def _rng(*key: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence(list(key))))


def _normal_bf16(rng: np.random.Generator, n: int, std: float) -> np.ndarray:
    a = rng.standard_normal(n, dtype=np.float32)
    a *= np.float32(std)
    return f32_to_bf16_bits(a)


# ----------------------------------------------------------------------------
# workload description
# ----------------------------------------------------------------------------
@dataclass(frozen=True)
class Workload:
    """One synthetic workload: shapes, distributions and the steps-per-second curve."""

    name: str
    B: int
    gamma: int
    V: int
    r: int = 256
    d: int = 4096
    logits: str = "normal"          # "normal": N(0, 2^2) + 6 on one token; "zipf": -1.1 ln(rank)
    mode: int = 0                   # 0 greedy argmax, 1 Gumbel-max
    tau: float = 1.0                # Gumbel temperature (divides the logit)
    w_std: float = 0.02             # std of W1 and W2 entries
    q_first: float = 0.85           # target agreement at position 1
    q_last: float = 0.85            # target agreement at position gamma (linear in between)
    sps_base_us: float = 20000.0    # step time on the flat part of the curve
    sps_knee: int = 512             # tokens per step where the flat part ends
    sps_slope_us: float = 30.0      # extra step time per token above the knee
    seed: int = 0
    b_conf: float = 1.0

    def q(self) -> np.ndarray:
        """Per-position target agreement, linear from q_first to q_last."""
        if self.gamma == 1:
            return np.array([self.q_first])
        k = np.arange(self.gamma, dtype=np.float64)
        return self.q_first + (self.q_last - self.q_first) * k / (self.gamma - 1)

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


TINY = Workload("tiny B=4 gamma=8 V=32000 d=1024", B=4, gamma=8, V=32000, d=1024)
QWEN3_8B = Workload("qwen3-8b-shaped B=64 gamma=16 V=151936 d=4096", B=64, gamma=16, V=151936,
                    q_first=0.88, q_last=0.78)
SAMPLED = Workload("sampled B=256 gamma=16 V=129280 d=4096 gumbel tau=0.7", B=256, gamma=16,
                   V=129280, logits="zipf", mode=1, tau=0.7)
SWEEP_BS = (1, 8, 32, 128, 512)


def sweep(B: int) -> Workload:
    return Workload(f"sweep B={B} gamma=16 V=151936 d=4096", B=B, gamma=16, V=151936,
                    q_first=0.88, q_last=0.78, sps_base_us=15000.0, sps_knee=1024,
                    sps_slope_us=20.0)


LARGE_VOCAB = Workload("large-vocab B=1024 gamma=24 V=262144 d=3840", B=1024, gamma=24,
                       V=262144, d=3840, logits="zipf", q_first=0.9, q_last=0.6,
                       sps_base_us=15000.0, sps_knee=4096, sps_slope_us=20.0)

WORKLOADS = {"tiny": TINY, "qwen3-8b": QWEN3_8B, "sampled": SAMPLED,
             "large-vocab": LARGE_VOCAB}
for _b in SWEEP_BS:
    WORKLOADS[f"sweep-{_b}"] = sweep(_b)


# ----------------------------------------------------------------------------
# generators
# ----------------------------------------------------------------------------
def w1(wl: Workload) -> np.ndarray:
    """Markov embedding table W1 [V, r] (bf16 bits), N(0, w_std^2)."""
    return _normal_bf16(_rng(wl.seed, TAG_W1), wl.V * wl.r, wl.w_std).reshape(wl.V, wl.r)


def w2(wl: Workload) -> np.ndarray:
    """Markov logits projection W2 [r, V] (bf16 bits), N(0, w_std^2)."""
    return _normal_bf16(_rng(wl.seed, TAG_W2), wl.r * wl.V, wl.w_std).reshape(wl.r, wl.V)


def whh(wl: Workload, std: float = 0.04) -> np.ndarray:
    """RNN-head recurrence Whh [r, r] (bf16 bits), N(0, std^2); 0.04 sqrt(256) = 0.64 keeps
    the recurrence contractive under tanh."""
    return _normal_bf16(_rng(wl.seed, TAG_WHH), wl.r * wl.r, std).reshape(wl.r, wl.r)


def anchors(wl: Workload) -> np.ndarray:
    """Anchor tokens x_0 [B] (int32), uniform over the vocabulary."""
    return _rng(wl.seed, TAG_ANCHOR).integers(0, wl.V, size=wl.B).astype(np.int32)


def conf_w(wl: Workload) -> np.ndarray:
    """Confidence projection w [d + r] (bf16 bits), N(0, 1/(d + r))."""
    return _normal_bf16(_rng(wl.seed, TAG_W), wl.d + wl.r, math.sqrt(1.0 / (wl.d + wl.r)))


def temperatures(wl: Workload) -> np.ndarray:
    """STS temperatures T [gamma] (fp32), uniform on [1, 3]."""
    return _rng(wl.seed, TAG_T).uniform(1.0, 3.0, size=wl.gamma).astype(np.float32)


def tstep_us(wl: Workload, n_max: Optional[int] = None) -> np.ndarray:
    """Step time in microseconds for n = 0 .. n_max tokens verified in one target pass.

    Flat at sps_base_us up to sps_knee tokens, then sps_slope_us more per token.
    The default table covers n = 0 .. B (gamma + 1).
    """
    if n_max is None:
        n_max = wl.B * (wl.gamma + 1)
    n = np.arange(n_max + 1, dtype=np.float64)
    return wl.sps_base_us + wl.sps_slope_us * np.maximum(0.0, n - wl.sps_knee)


def _zipf_table(wl: Workload) -> np.ndarray:
    rank = np.arange(1, wl.V + 1, dtype=np.float64)
    return f32_to_bf16_bits((-1.1 * np.log(rank)).astype(np.float32))


def zipf_params(wl: Workload, b: int) -> tuple[np.ndarray, np.ndarray]:
    """Per-position rank permutation v -> ((a v + c) mod V) + 1 for request b.

    a is drawn uniform on [1, V) until it is coprime to V; c is uniform on [0, V).
    """
    rng = _rng(wl.seed, TAG_ZIPF, b)
    a = np.empty(wl.gamma, dtype=np.int64)
    c = np.empty(wl.gamma, dtype=np.int64)
    for k in range(wl.gamma):
        while True:
            ak = int(rng.integers(1, wl.V))
            if math.gcd(ak, wl.V) == 1:
                break
        a[k] = ak
        c[k] = int(rng.integers(0, wl.V))
    return a, c


def u_request(wl: Workload, b: int, table: Optional[np.ndarray] = None) -> np.ndarray:
    """Base logits U[b] [gamma, V] (bf16 bits) of one request."""
    if wl.logits == "normal":
        rng = _rng(wl.seed, TAG_U, b)
        a = rng.standard_normal(wl.gamma * wl.V, dtype=np.float32)
        a *= np.float32(2.0)
        planted = rng.integers(0, wl.V, size=wl.gamma)
        a = a.reshape(wl.gamma, wl.V)
        a[np.arange(wl.gamma), planted] += np.float32(6.0)
        return f32_to_bf16_bits(a).reshape(wl.gamma, wl.V)
    if wl.logits == "zipf":
        if table is None:
            table = _zipf_table(wl)
        a, c = zipf_params(wl, b)
        v = np.arange(wl.V, dtype=np.int64)
        idx = (a[:, None] * v[None, :] + c[:, None]) % wl.V
        return table[idx]
    raise ValueError(wl.logits)


def u_requests(wl: Workload, bs: Sequence[int]) -> np.ndarray:
    """Base logits for the listed requests, stacked [len(bs), gamma, V]."""
    table = _zipf_table(wl) if wl.logits == "zipf" else None
    out = np.empty((len(bs), wl.gamma, wl.V), dtype=np.uint16)

    def job(i):
        out[i] = u_request(wl, int(bs[i]), table)

    with ThreadPoolExecutor(_THREADS) as ex:
        list(ex.map(job, range(len(bs))))
    return out


def u_all(wl: Workload) -> np.ndarray:
    """Base logits U [B, gamma, V] (bf16 bits)."""
    return u_requests(wl, range(wl.B))


def u_all_device_zipf(wl: Workload, device: str = "cuda"):
    """Zipf base logits U [B, gamma, V] built directly in device memory (torch bf16).

    Same bytes as ``u_all``: the bf16 value table is made on the host and the
    per-position rank permutation is pure integer arithmetic, done request by
    request on the device to avoid a host copy of a multi-GB tensor.
    """
    import torch
    assert wl.logits == "zipf"
    table = torch.from_numpy(_zipf_table(wl).view(np.int16)).to(device)
    out = torch.empty((wl.B, wl.gamma, wl.V), dtype=torch.int16, device=device)
    v = torch.arange(wl.V, dtype=torch.int64, device=device)
    for b in range(wl.B):
        a, c = zipf_params(wl, b)
        at = torch.from_numpy(a).to(device)
        ct = torch.from_numpy(c).to(device)
        out[b] = table[(at[:, None] * v[None, :] + ct[:, None]) % wl.V]
    return out.view(torch.bfloat16)


def h_requests(wl: Workload, bs: Sequence[int]) -> np.ndarray:
    """Backbone hidden states for the listed requests [len(bs), gamma, d] (bf16 bits), N(0, 1)."""
    out = np.empty((len(bs), wl.gamma, wl.d), dtype=np.uint16)

    def job(i):
        out[i] = _normal_bf16(_rng(wl.seed, TAG_H, int(bs[i])), wl.gamma * wl.d, 1.0).reshape(
            wl.gamma, wl.d)

    with ThreadPoolExecutor(_THREADS) as ex:
        list(ex.map(job, range(len(bs))))
    return out


def h_all(wl: Workload) -> np.ndarray:
    return h_requests(wl, range(wl.B))


def targets(wl: Workload, drafts: np.ndarray, bs: Optional[Sequence[int]] = None) -> np.ndarray:
    """Target-model tokens [nb, gamma + 1] (int32) for the given drafted tokens [nb, gamma].

    Position k agrees with the draft with probability q_k, otherwise it is uniform
    over the other V - 1 tokens; the last column (position gamma + 1) is uniform.
    """
    drafts = np.asarray(drafts, dtype=np.int64)
    nb = drafts.shape[0]
    if bs is None:
        bs = range(nb)
    q = wl.q()
    out = np.empty((nb, wl.gamma + 1), dtype=np.int32)
    for i, b in enumerate(bs):
        rng = _rng(wl.seed, TAG_TARGET, int(b))
        agree = rng.random(wl.gamma) < q
        other = rng.integers(0, wl.V - 1, size=wl.gamma)
        other = other + (other >= drafts[i])
        out[i, :wl.gamma] = np.where(agree, drafts[i], other)
        out[i, wl.gamma] = rng.integers(0, wl.V)
    return out


# ----------------------------------------------------------------------------
# inputs for the scheduler and verify stages on their own
# ----------------------------------------------------------------------------
def monotone_scores(B: int, gamma: int, seed: int, tie_frac: float = 0.0,
                    zero_frac: float = 0.0, neg_zero: bool = False) -> np.ndarray:
    """Scores P [B, gamma] (fp32) in [0, 1] that never increase along a row.

    Values are uniform draws sorted in decreasing order within each row.  With
    tie_frac > 0 some entries repeat their left neighbour and some values are
    copied across rows, so that equal scores occur within and across requests;
    zero_frac sets a tail of some rows to exactly 0; with neg_zero, about half of
    those zeros are written as -0.0 (equal to +0.0 as a number, sign bit set).
    """
    rng = _rng(seed, TAG_SCORES, B, gamma)
    P = np.sort(rng.random((B, gamma)).astype(np.float32), axis=1)[:, ::-1].copy()
    if tie_frac > 0:
        rep = rng.random((B, gamma)) < tie_frac
        for b in range(B):
            for k in range(1, gamma):
                if rep[b, k]:
                    P[b, k] = P[b, k - 1]
        # copy whole rows onto others so that equal values appear across requests
        ncopy = int(tie_frac * B)
        for _ in range(ncopy):
            s, t = rng.integers(0, B, size=2)
            P[t] = P[s]
    if zero_frac > 0:
        for b in range(B):
            if rng.random() < zero_frac:
                cut = int(rng.integers(0, gamma + 1))
                P[b, cut:] = 0.0
        if neg_zero:
            flip = (P == 0.0) & (rng.random((B, gamma)) < 0.5)
            P[flip] = np.float32(-0.0)
    return np.ascontiguousarray(P, dtype=np.float32)


def verify_inputs(B: int, gamma: int, V: int, seed: int, agree: float = 0.8):
    """Drafts x [B, gamma], lengths L [B] in 0..gamma and target tokens [B, gamma + 1]."""
    rng = _rng(seed, TAG_VERIFY, B, gamma)
    x = rng.integers(0, V, size=(B, gamma)).astype(np.int32)
    L = rng.integers(0, gamma + 1, size=B).astype(np.int32)
    same = rng.random((B, gamma)) < agree
    other = rng.integers(0, V, size=(B, gamma)).astype(np.int32)
    t = np.where(same, x, other).astype(np.int32)
    last = rng.integers(0, V, size=(B, 1)).astype(np.int32)
    return x, L, np.ascontiguousarray(np.concatenate([t, last], axis=1))


# held-out calibration set for fitting the temperatures: 65536 blocks of gamma = 16
STS_CALIBRATION_N = 65536
STS_CALIBRATION_GAMMA = 16


def calibration_set(N: int, gamma: int, seed: int, q_first: float = 0.88,
                    q_last: float = 0.78, spread: float = 2.0, scale: float = 3.4):
    """Held-out blocks for fitting the per-position temperatures: raw confidence
    logits z [N, gamma] (fp32) and accepted lengths [N] (int32, 0..gamma).

    z[n, k] ~ N(m_k, spread^2) with m_k chosen so that the mean acceptance at
    position k is near the linear decay q_first -> q_last.  The label process is
    a probit link, the normal CDF Phi, so that it is not the logistic model being
    fitted: draft k of block n is accepted with probability Phi(z[n, k] / scale) given that
    drafts 1..k-1 were accepted, and the accepted length counts the accepted
    drafts before the first rejection.  A small scale makes the raw logits
    under-confident, a large one over-confident; the default 3.4 puts the fitted
    temperatures near 2 (the logistic and normal CDFs match at a factor of ~1.7).
    """
    from scipy import special as _sp
    rng = _rng(seed, TAG_CALIB, N, gamma)
    if gamma == 1:
        q = np.array([q_first])
    else:
        q = q_first + (q_last - q_first) * np.arange(gamma) / (gamma - 1)
    # E[Phi(Z / scale)] with Z ~ N(m, spread^2) is Phi(m / sqrt(scale^2 + spread^2))
    m = _sp.ndtri(q) * math.sqrt(scale * scale + spread * spread)
    z = (m[None, :] + spread * rng.standard_normal((N, gamma))).astype(np.float32)
    u = rng.random((N, gamma))
    ok = u < _sp.ndtr(z.astype(np.float64) / scale)
    acc = np.where(ok.all(axis=1), gamma, np.argmin(ok, axis=1)).astype(np.int32)
    return np.ascontiguousarray(z), acc


def draft_tokens(B: int, gamma: int, V: int, seed: int) -> np.ndarray:
    """Arbitrary token ids [B, gamma] (int32) standing in for drafted tokens."""
    return _rng(seed, TAG_VERIFY, B, gamma, 7).integers(0, V, size=(B, gamma)).astype(np.int32)


@dataclass
class Inputs:
    """All model-side inputs of one workload, as host arrays."""

    wl: Workload
    W1: np.ndarray
    W2: np.ndarray
    U: np.ndarray
    h: np.ndarray
    anchor: np.ndarray
    w: np.ndarray
    T: np.ndarray
    Tstep: np.ndarray
    b_conf: float = 1.0


def make_inputs(wl: Workload, with_u: bool = True, with_h: bool = True) -> Inputs:
    return Inputs(wl=wl, W1=w1(wl), W2=w2(wl), U=u_all(wl) if with_u else None,
                  h=h_all(wl) if with_h else None, anchor=anchors(wl), w=conf_w(wl),
                  T=temperatures(wl), Tstep=tstep_us(wl), b_conf=wl.b_conf)
