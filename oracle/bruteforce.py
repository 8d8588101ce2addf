"""Brute-force checker for tiny layers (test infrastructure only).

An independent second statement of the AWQ per-layer search used to pin the
oracle.  It shares nothing with ``awq_oracle.c``:

* binary32 steps are real binary32 operations on ``numpy.float32`` scalars
  (the C oracle instead rounds binary64 results);
* binary16 rounding is CPython's IEEE half packing (``struct`` format ``'e'``)
  (the C oracle has its own bit-level rounding);
* the output-error loss is exact rational arithmetic (``fractions.Fraction``)
  over explicit triple loops (the oracle uses a binary64 matrix product).

Pure-Python loops: only for N <= 8, K <= 256, T <= 16.

Sources: [AWQ-note] = "AWQ: Activation-Aware Weight Quantization For On-Device
LLM Compression AND Acceleration", section "Measures" (statistic a = mean |x|,
candidates a^alpha, error of the output); [QAS-QA] = "Как работает
quantization-aware scaling в AWQ для защиты важных весов?", §5-§6 and §9
(scale, group round-to-nearest, MSE of the layer output).
"""
from __future__ import annotations

import math
import struct
from fractions import Fraction

import numpy as np

f32 = np.float32


def to_f16(x: float) -> float:
    """Nearest binary16 value (ties to even) via CPython's half packing."""
    return struct.unpack("<e", struct.pack("<e", float(x)))[0]


def mean_abs(column) -> np.float32:
    """a = RN32(RN64(sum |x| / T)); the binary16 sum is exact in binary64."""
    tot = Fraction(0)
    for v in column:
        tot += Fraction(abs(float(v)))
    return f32(float(tot) / len(column))


def stored_zero(z: int) -> float:
    """zero = round(-min/scale) as kept in the fp16 zeros: saturated to the
    largest finite binary16 magnitude, then the nearest binary16 (above 2048
    not every integer is one).  The codes and W_hat use this stored value."""
    z = min(max(z, -65504), 65504)
    return to_f16(z) + 0.0          # + 0.0: a zero point of -0 is stored as +0


def quantize_group(w, s, bits, sym=False, keep=None):
    """One group: w (binary16 values as floats), s (float32).  Returns q, sh, z, what.

    sym: the symmetric absmax quantizer (step max|w'| / (2^(bits-1) - 1), zero
    at the middle code 2^(bits-1)).  keep: per-column flags of channels held
    in fp16 -- left out of the range, returned unchanged."""
    qmax = (1 << bits) - 1
    keep = [False] * len(w) if keep is None else [bool(v) for v in keep]
    wp = [f32(f32(w[k]) * s[k]) for k in range(len(w))]
    ranged = [wp[k] for k in range(len(w)) if not keep[k]] or [f32(0.0)]
    mn = min(ranged)
    mx = max(ranged)
    if sym:
        half = (1 << (bits - 1)) - 1
        scale = f32(max(-mn, mx) / f32(half))
    else:
        scale = f32(f32(mx - mn) / f32(qmax))
    scale = min(max(float(scale), 2.0 ** -24), 65504.0)
    sh = to_f16(scale)
    r = f32(f32(1.0) / f32(sh))
    if sym:
        z = 1 << (bits - 1)
    else:
        z = stored_zero(round(-float(mn) * float(r)))   # exact product (24 x 24 bits); round(): ties to even
    q, what = [], []
    for k in range(len(w)):
        t = float(wp[k]) * float(r)         # exact product
        qk = int(min(max(round(t) + z, 0), qmax))
        rs = f32(f32(1.0) / s[k])
        deq = f32(f32(qk - z) * f32(sh))
        what.append(float(w[k]) if keep[k] else to_f16(float(f32(deq * rs))))
        q.append(qk)
    return q, sh, z, what


def quantize(W, s, bits, group, sym=False, keep=None):
    N, K = len(W), len(W[0])
    Q = [[0] * K for _ in range(N)]
    WH = [[0.0] * K for _ in range(N)]
    SH = [[0.0] * (K // group) for _ in range(N)]
    Z = [[0] * (K // group) for _ in range(N)]
    for n in range(N):
        for gi in range(K // group):
            sl = slice(gi * group, (gi + 1) * group)
            q, sh, z, what = quantize_group(W[n][sl], s[sl], bits, sym,
                                            None if keep is None else keep[sl])
            Q[n][sl] = q
            WH[n][sl] = what
            SH[n][gi] = sh
            Z[n][gi] = z
    return Q, SH, Z, WH


def exact_loss(W, WH, X):
    """sum_n sum_t (sum_k (what - w)_nk x_tk)^2, exactly."""
    tot = Fraction(0)
    for n in range(len(W)):
        d = [Fraction(WH[n][k]) - Fraction(W[n][k]) for k in range(len(W[n]))]
        for t in range(len(X)):
            e = Fraction(0)
            for k, dk in enumerate(d):
                if dk:
                    e += dk * Fraction(X[t][k])
            tot += e * e
    return tot


def search(W16: np.ndarray, X16: np.ndarray, bits: int, group: int, alphas, sym=False):
    """Enumerate every alpha independently.  Returns dict(a, losses, best, q, sh, z)."""
    W = [[float(v) for v in row] for row in W16.astype(np.float64)]
    X = [[float(v) for v in row] for row in X16.astype(np.float64)]
    N, K, T = len(W), len(W[0]), len(X)
    a = [mean_abs([X[t][k] for t in range(T)]) for k in range(K)]
    losses = []
    per_alpha = []
    for al in alphas:
        s = [f32(math.pow(max(float(aj), 2.0 ** -126), float(f32(al)))) for aj in a]
        Q, SH, Z, WH = quantize(W, s, bits, group, sym)
        losses.append(exact_loss(W, WH, X) / (N * T))
        per_alpha.append((Q, SH, Z, WH, s))
    best = min(range(len(losses)), key=lambda i: (losses[i], i))
    return dict(a=np.array(a, dtype=np.float32), losses=[float(v) for v in losses],
                exact_losses=losses, best=best, per_alpha=per_alpha)


def masked_loss(W16: np.ndarray, X16: np.ndarray, s, bits: int, group: int, keep, sym=False):
    """Exact MSE of the layer with the channels flagged in `keep` held in fp16."""
    W = [[float(v) for v in row] for row in W16.astype(np.float64)]
    X = [[float(v) for v in row] for row in X16.astype(np.float64)]
    s = [f32(v) for v in s]
    _, _, _, WH = quantize(W, s, bits, group, sym, list(keep))
    return float(exact_loss(W, WH, X) / (len(W) * len(X))), WH
