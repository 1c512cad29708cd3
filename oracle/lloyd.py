"""Weighted Lloyd-Max learner of per-output-channel mappings and thresholds.

TEST INFRASTRUCTURE ONLY (see the package docstring). Source: "LowRA" article
(cloud.tencent.com.cn), 第五部分 映射与阈值学习器: for every output channel (row of W0)
and bit width, the mapping (representative values) and thresholds (bin edges) that
minimise the channel's mean squared error are found by a weighted Lloyd-Max iteration
over the group-normalised values (§4.1 normalisation), each value weighted by its
group's absmax. Thresholds start from the NormalFloat thresholds for 2 and 4 bits and
at 0.0 for 1 bit; each iteration recomputes the mapping as the weighted centre of the
values assigned to each bin and the thresholds as the midpoints of consecutive mapping
values; the learner stops at the iteration cap or when the MSE stops decreasing and
outputs the mapping and thresholds it computed last.

Readings of what the page leaves open (parity of the GPU learner against this oracle
is pinned by the tests; the readings themselves are conventions):
  * values and weights: x = fp32(w / g), g the 64-group absmax, x = 0 for an all-zero
    group (the per-channel quantizer's normalisation); the weight of x is g;
  * assignment: bin = #{k : x > t_k}, the quantizer's rule (a value on an edge goes to
    the lower bin);
  * bin sums in float64: S0_k = sum g, S1_k = sum g*x (each product of two fp32 values
    is exact in float64); centre m_k = fp32(S1_k / S0_k), and a bin with S0_k = 0 keeps
    its previous value; the values before the first iteration are -1, the midpoints of
    consecutive initial thresholds, and +1;
  * thresholds t_k = fp32((m_k + m_{k+1}) / 2) (the float64 sum and halving are exact,
    one rounding);
  * the MSE of an iteration is the weighted error of its assignment with its new
    centres, E = (S2 - sum_k (2 m_k S1_k - m_k^2 S0_k)) / S0 with S2 = sum (g*x)*x and
    S0 = sum g over the row (float64, terms evaluated left to right); from the second
    iteration on, an E not below the previous one stops the learner after that
    iteration (whose tables are the output);
  * NormalFloat thresholds for b bits: the midpoints (rounded to fp32) of the b-bit
    NormalFloat levels, built as NF4 is (2^(b-1)+1 positive and 2^(b-1) negative
    standard-normal quantiles at evenly spaced probabilities from p_max(b) to 0.5,
    union without the duplicate 0, divided by the largest), with
    p_max(b) = 1 - (1/(2*2^b) + 1/(2*(2^b - 1))) / 2, which is NF4's for b = 4;
  * the threshold averaging the page mentions for its own implementation (one clause,
    undefined further) is not applied;
  * reported error of a channel: mean over the row of (w - fp32(m[c] * g))^2 in float64,
    c from the output thresholds, i.e. the error of the quantization those tables give.
"""
from __future__ import annotations

from statistics import NormalDist

import numpy as np

from . import chanq

GROUP = chanq.GROUP


def nf_levels(bits: int) -> np.ndarray:
    """The 2^bits NormalFloat levels (fp32, ascending) for bits >= 2."""
    n = 1 << bits
    half = n // 2
    p_max = 1.0 - 0.5 * (1.0 / (2.0 * n) + 1.0 / (2.0 * (n - 1)))
    nd = NormalDist()
    pos = [nd.inv_cdf(float(p)) for p in np.linspace(p_max, 0.5, half + 1)]
    neg = [-nd.inv_cdf(float(p)) for p in np.linspace(p_max, 0.5, half)]
    vals = [v for v in pos if v != 0.0] + [v for v in neg if v != 0.0] + [0.0]
    vals = np.array(sorted(vals), dtype=np.float64)
    assert vals.size == n
    return (vals / nd.inv_cdf(p_max)).astype(np.float32)


def midpoints(levels: np.ndarray) -> np.ndarray:
    """fp32((m_k + m_{k+1}) / 2) for consecutive fp32 levels."""
    m = np.asarray(levels, dtype=np.float32).astype(np.float64)
    return ((m[:-1] + m[1:]) * 0.5).astype(np.float32)


def initial_thresholds(bits: int) -> np.ndarray:
    """0.0 for 1 bit; the NormalFloat midpoints for 2 and 4 bits."""
    if bits == 1:
        return np.zeros(1, dtype=np.float32)
    return midpoints(nf_levels(bits))


def normalise_row(w_row: np.ndarray):
    """(x fp32 [K], g fp32 [K/64]) with x = fp32(w / g), 0 in an all-zero group."""
    w = np.asarray(w_row, dtype=np.float32)
    g = np.abs(w.reshape(-1, GROUP)).max(axis=1).astype(np.float32)
    gr = np.repeat(g, GROUP)
    with np.errstate(divide="ignore", invalid="ignore"):
        x = np.where(gr > 0, w / np.where(gr > 0, gr, np.float32(1)), np.float32(0)).astype(np.float32)
    return x, g


def assign(x: np.ndarray, t: np.ndarray) -> np.ndarray:
    """bin = number of thresholds strictly below x."""
    return (np.asarray(x, np.float32)[:, None] > np.asarray(t, np.float32)[None, :]).sum(axis=1)


def learn_row(w_row: np.ndarray, bits: int, t0: np.ndarray, iters: int):
    """(mapping fp32 [2^b], thresholds fp32 [2^b - 1], error float64, iterations run,
    per-iteration E list) for one channel."""
    L = 1 << bits
    x, g = normalise_row(w_row)
    x64 = x.astype(np.float64)
    wt = np.repeat(g, GROUP).astype(np.float64)
    gx = wt * x64                              # exact
    S0tot = float(np.sum(wt))
    S2tot = float(np.sum(gx * x64))
    t = np.asarray(t0, dtype=np.float32).copy()
    m = np.empty(L, dtype=np.float32)
    m[0], m[-1] = np.float32(-1.0), np.float32(1.0)
    if L > 2:
        m[1:-1] = midpoints(t)
    hist = []
    done = 0
    for it in range(iters):
        c = assign(x, t)
        S0 = np.bincount(c, weights=wt, minlength=L)
        S1 = np.bincount(c, weights=gx, minlength=L)
        mnew = m.copy()
        nz = S0 > 0
        mnew[nz] = (S1[nz] / S0[nz]).astype(np.float32)
        m = mnew
        acc = 0.0
        for k in range(L):
            mk = float(m[k])
            acc += (2.0 * mk) * float(S1[k]) - (mk * mk) * float(S0[k])
        E = (S2tot - acc) / S0tot if S0tot > 0 else 0.0
        t = midpoints(m)
        done = it + 1
        hist.append(E)
        if it > 0 and E >= hist[-2]:
            break
    c = assign(x, t)
    deq = (m[c] * np.repeat(g, GROUP)).astype(np.float32)
    err = float(np.mean((np.asarray(w_row, np.float32).astype(np.float64) - deq.astype(np.float64)) ** 2))
    return m, t, err, done, hist


def learn(W: np.ndarray, bits: int, t0: np.ndarray, iters: int):
    """All rows: (maps fp32 [N, 2^b], thresholds fp32 [N, 2^b - 1], errors float64 [N])."""
    W = np.asarray(W, dtype=np.float32)
    N = W.shape[0]
    maps = np.empty((N, 1 << bits), dtype=np.float32)
    thr = np.empty((N, (1 << bits) - 1), dtype=np.float32)
    err = np.empty(N, dtype=np.float64)
    for i in range(N):
        maps[i], thr[i], err[i], _, _ = learn_row(W[i], bits, t0, iters)
    return maps, thr, err
