"""AWQ oracle (test infrastructure only).

A plain, slow, obviously-correct CPU statement of the activation-aware scale
search for one linear layer.  Only the test-suite, ``__graft_entry__.smoke()``
and the ``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import
this package.  It shares no code with the CUDA library and never imports it.

The per-element quantizer lives in ``awq_oracle.c`` (binary64 arithmetic, every
binary32 decision emulated as a binary64 operation rounded to binary32).  The
output-error loss uses one library primitive, a binary64 matrix product.

Sources (web pages; cited by title and section):
  [QAS-QA]   "Как работает quantization-aware scaling в AWQ для защиты важных весов?"
  [AWQ-note] "AWQ: Activation-Aware Weight Quantization For On-Device LLM
             Compression AND Acceleration"
  [Notes-52] "52 · AWQ, GPTQ và SmoothQuant"
  [GPTQ-AWQ] "GPTQ与AWQ"
  [AWQ-wiki] "AWQ" encyclopedia page (French)

Parity status: every function here is pinned by a CPU test (worked examples of
[AWQ-note] "Measures" and [Notes-52] §3, closed forms, invariants, and an
independent brute force).  Nothing here is "parity unpinned".
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from pathlib import Path

import numpy as np

_HERE = Path(__file__).resolve().parent
_SRC = _HERE / "awq_oracle.c"
_LIB_PATH = _HERE / "liboracle.so"
_lib = None

DEFAULT_ALPHAS = np.array([np.float32(i / 20.0) for i in range(20)], dtype=np.float32)


def build(force: bool = False) -> Path:
    """Compile awq_oracle.c into liboracle.so with contraction and fast-math off."""
    if force or not _LIB_PATH.exists() or _LIB_PATH.stat().st_mtime < _SRC.stat().st_mtime:
        tmp = _LIB_PATH.with_suffix(f".so.tmp{os.getpid()}")
        cmd = ["gcc", "-O2", "-ffp-contract=off", "-fno-fast-math", "-fopenmp", "-fPIC",
               "-shared", "-std=c11", "-Wall", "-o", str(tmp), str(_SRC), "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is not None:
        return _lib
    build()
    lib = ctypes.CDLL(str(_LIB_PATH))
    P = ctypes.c_void_p
    i64 = ctypes.c_int64
    lib.awq_oracle_h2d.restype = ctypes.c_double
    lib.awq_oracle_h2d.argtypes = [ctypes.c_uint16]
    lib.awq_oracle_rn16.restype = ctypes.c_uint16
    lib.awq_oracle_rn16.argtypes = [ctypes.c_double]
    lib.awq_oracle_act_stats.argtypes = [P, i64, i64, i64, P]
    lib.awq_oracle_scales.argtypes = [P, i64, ctypes.c_float, P]
    lib.awq_oracle_quantize.argtypes = [P, i64, i64, P, ctypes.c_int, ctypes.c_int, ctypes.c_int, P,
                                        ctypes.c_int, P, P, P, P]
    lib.awq_oracle_topk.argtypes = [P, i64, i64, P]
    lib.awq_oracle_gptq.argtypes = [P, i64, i64, P, P, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                    ctypes.c_double, i64, P, P, P, P, P]
    lib.awq_oracle_pack_codes.argtypes = [P, i64, i64, ctypes.c_int, P]
    lib.awq_oracle_argmin.restype = ctypes.c_int
    lib.awq_oracle_argmin.argtypes = [P, ctypes.c_int]
    lib.awq_oracle_round_to_step.restype = ctypes.c_double
    lib.awq_oracle_round_to_step.argtypes = [ctypes.c_double, ctypes.c_double]
    lib.awq_oracle_absmax_step.restype = ctypes.c_double
    lib.awq_oracle_absmax_step.argtypes = [P, ctypes.c_int, ctypes.c_int]
    _lib = lib
    return lib


def _ptr(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(ctypes.c_void_p)


def _as_f16(a) -> np.ndarray:
    a = np.ascontiguousarray(a)
    assert a.dtype == np.float16, a.dtype
    return a


# --------------------------------------------------------------------------
# binary16 helpers
# --------------------------------------------------------------------------

def rn16_bits(x: float) -> int:
    """IEEE binary16 round-to-nearest-even of a binary64 value (bit pattern)."""
    return int(_load().awq_oracle_rn16(float(x)))


def h2d(bits: int) -> float:
    """Exact value of a binary16 bit pattern."""
    return float(_load().awq_oracle_h2d(int(bits)))


# --------------------------------------------------------------------------
# Step a1 -- [AWQ-note] "Measures"; [GPTQ-AWQ] "量化方法" (X.abs().mean(dim=0))
# --------------------------------------------------------------------------

def act_stats(X: np.ndarray) -> np.ndarray:
    """a_j = RN32(mean_t |X[t, j]|) over the T calibration tokens (rows of X)."""
    X = _as_f16(X)
    T, K = X.shape
    a = np.empty(K, dtype=np.float32)
    _load().awq_oracle_act_stats(_ptr(X.view(np.uint16)), T, K, K, _ptr(a))
    return a


# --------------------------------------------------------------------------
# Step a2 -- [AWQ-note] "Measures": for each candidate alpha compute a^alpha
# --------------------------------------------------------------------------

def scales(a: np.ndarray, alpha: float) -> np.ndarray:
    a = np.ascontiguousarray(a, dtype=np.float32)
    s = np.empty_like(a)
    _load().awq_oracle_scales(_ptr(a), a.size, np.float32(alpha), _ptr(s))
    return s


# --------------------------------------------------------------------------
# Steps a3/a4 -- [QAS-QA] §5, §9; [AWQ-wiki] "Fondements techniques"
# --------------------------------------------------------------------------

def quantize(W: np.ndarray, s: np.ndarray, bits: int, group: int, no_round: bool = False,
             zero_point: bool = True, mask=None):
    """Group-wise RTN of W*diag(s), dequantized and divided by s.

    zero_point=True: asymmetric (min/max, a zero-point code); False: symmetric
    absmax with the zero fixed at the middle code 2^(bits-1).  mask: channels
    kept in fp16 (excluded from their group's range, W_hat = W there).

    Returns dict(q=[N,K] uint8 codes, sh=[N,K/g] fp16 scales, z=[N,K/g] float32
    zero points, what=[N,K] fp16 dequantized-and-unscaled weights)."""
    W = _as_f16(W)
    N, K = W.shape
    assert K % group == 0 and group <= 256
    s = np.ascontiguousarray(s, dtype=np.float32)
    assert s.shape == (K,)
    m = None if mask is None else np.ascontiguousarray(mask, dtype=np.uint8)
    assert m is None or m.shape == (K,)
    G = K // group
    q = np.empty((N, K), dtype=np.uint8)
    sh = np.empty((N, G), dtype=np.uint16)
    z = np.empty((N, G), dtype=np.float32)
    what = np.empty((N, K), dtype=np.uint16)
    _load().awq_oracle_quantize(_ptr(W.view(np.uint16)), N, K, _ptr(s), int(bits), int(group),
                                int(bool(zero_point)), None if m is None else _ptr(m),
                                int(bool(no_round)), _ptr(q), _ptr(sh), _ptr(z), _ptr(what))
    return dict(q=q, sh=sh.view(np.float16), z=z, what=what.view(np.float16))


# --------------------------------------------------------------------------
# Steps a5/a6 -- [AWQ-note] "Measures": Δy = (Ŵ − W) x; [QAS-QA] §6: MSE between
# the outputs of the original and the quantized layer on calibration data.
# --------------------------------------------------------------------------

def output_error_sum(W: np.ndarray, What: np.ndarray, X: np.ndarray) -> np.ndarray:
    """Per-row sum over tokens of ((Ŵ − W) Xᵀ)², in binary64 (one matmul)."""
    dW = What.astype(np.float64) - W.astype(np.float64)       # exact
    E = dW @ X.astype(np.float64).T                            # [N, T]
    return np.einsum("nt,nt->n", E, E)


def search(W: np.ndarray, X: np.ndarray, a: np.ndarray, bits: int, group: int,
           alphas=DEFAULT_ALPHAS, rows=None, no_round: bool = False, zero_point: bool = True):
    """The per-layer grid search.

    For each alpha_i: s = a^alpha_i, Ŵ = Q(W diag(s)) diag(s)^-1, and the loss
    MSE_i = ||(Ŵ − W) Xᵀ||² / (N T).  With ``rows`` given, only those rows of W
    are scored and the per-row sums are returned alongside (the same per-row
    sums that make up the full loss, so a row sample of a large layer can be
    compared).

    Returns dict(losses=[n_alpha] float64 MSE over the scored rows,
                 row_sums=[n_alpha, len(rows)] float64, best=int)."""
    s_table = np.stack([scales(a, float(al)) for al in alphas])
    return search_scales(W, X, s_table, bits, group, rows=rows, no_round=no_round, zero_point=zero_point)


def search_scales(W: np.ndarray, X: np.ndarray, s_table, bits: int, group: int, rows=None,
                  no_round: bool = False, zero_point: bool = True, mask=None):
    """The same loss for caller-given scale vectors s_table[i] (the baselines:
    s = 1 is plain RTN, s = 2 on the salient channels the fixed-scale variant)
    and, with ``mask``, the channels kept in fp16 contribute no error."""
    W = _as_f16(W)
    X = _as_f16(X)
    T = X.shape[0]
    s_table = np.atleast_2d(np.asarray(s_table, dtype=np.float32))
    Ws = W if rows is None else np.ascontiguousarray(W[np.asarray(rows)])
    nr = Ws.shape[0]
    losses = np.empty(len(s_table), dtype=np.float64)
    row_sums = np.empty((len(s_table), nr), dtype=np.float64)
    for i, s in enumerate(s_table):
        what = quantize(Ws, s, bits, group, no_round=no_round, zero_point=zero_point, mask=mask)["what"]
        rs = output_error_sum(Ws, what, X)
        row_sums[i] = rs
        losses[i] = rs.sum() / (nr * T)
    best = argmin(losses)
    return dict(losses=losses, row_sums=row_sums, best=best)


def topk_mask(stat, k: int) -> np.ndarray:
    """mask[j] = 1 for the k channels with the largest statistic (ties: lower
    index first; NaN ranks last)."""
    v = np.ascontiguousarray(stat, dtype=np.float32)
    m = np.empty(v.size, dtype=np.uint8)
    _load().awq_oracle_topk(_ptr(v), v.size, int(k), _ptr(m))
    return m


def argmin(losses) -> int:
    """First index of the smallest loss; NaN counts as +inf."""
    v = np.ascontiguousarray(losses, dtype=np.float64)
    return int(_load().awq_oracle_argmin(_ptr(v), v.size))


# --------------------------------------------------------------------------
# Step a8 -- [AWQ-note] "Measures": save quantized weights + metadata
# --------------------------------------------------------------------------

def pack_codes(q: np.ndarray, bits: int) -> np.ndarray:
    q = np.ascontiguousarray(q, dtype=np.uint8)
    N, K = q.shape
    per = 16 if bits == 2 else 8
    codes = np.empty((N, K // per), dtype=np.uint32)
    _load().awq_oracle_pack_codes(_ptr(q), N, K, int(bits), _ptr(codes))
    return codes


def pack(W: np.ndarray, a: np.ndarray, bits: int, group: int, alphas, losses, rows=None,
         zero_point: bool = True):
    """Argmin over the grid, then codes / fp16 scales / fp16 zeros / s_best."""
    best = argmin(losses)
    out = pack_scales(W, scales(a, float(alphas[best])), bits, group, rows=rows, zero_point=zero_point)
    out["best"] = best
    return out


def pack_scales(W: np.ndarray, s, bits: int, group: int, rows=None, zero_point: bool = True):
    """Codes / fp16 scales / fp16 zeros of W quantized with a given s."""
    W = _as_f16(W)
    s = np.ascontiguousarray(s, dtype=np.float32)
    Ws = W if rows is None else np.ascontiguousarray(W[np.asarray(rows)])
    qz = quantize(Ws, s, bits, group, zero_point=zero_point)
    return dict(s_best=s, codes=pack_codes(qz["q"], bits), q=qz["q"],
                scales=qz["sh"], zeros=qz["z"].astype(np.float16), what=qz["what"])


# --------------------------------------------------------------------------
# Worked-example primitives -- [AWQ-note] "Measures"; [Notes-52] §3
# --------------------------------------------------------------------------

def round_to_step(w: float, step: float) -> float:
    return float(_load().awq_oracle_round_to_step(float(w), float(step)))


def absmax_step(w, bits: int) -> float:
    w = np.ascontiguousarray(w, dtype=np.float64)
    return float(_load().awq_oracle_absmax_step(_ptr(w), w.size, int(bits)))


# --------------------------------------------------------------------------
# Consumer of the packed format: the quantized linear layer
# ([AWQ-note] "Tiny Chat": dequantize inside the kernel, never writing fp16
# weights back; [QAS-QA] §5: the activation is divided by s).
# --------------------------------------------------------------------------

def unpack_codes(codes: np.ndarray, K: int, bits: int) -> np.ndarray:
    """Codes [N, K] from the packed words (least-significant first)."""
    c = 2 if bits == 2 else 4
    per = 32 // c
    words = np.ascontiguousarray(codes).view(np.uint32).astype(np.uint64)
    q = np.empty((words.shape[0], K), dtype=np.int64)
    for i in range(per):
        q[:, i::per] = (words >> np.uint64(c * i)) & np.uint64((1 << c) - 1)
    return q


def qlinear(codes, scales, zeros, s_best, X, bits: int, group: int) -> np.ndarray:
    """Y[t, n] = sum_k x'[t, k] * (q[n, k] - z[n, k/g]) * sh[n, k/g] in binary64, where
    x'[t, k] = RN32(x[t, k] * RN32(1 / s_k)) is the input divided by s (folded into
    the input, as the layer's 1/s is in a deployed model)."""
    X = np.asarray(X)
    K = X.shape[1]
    q = unpack_codes(codes, K, bits).astype(np.float64)
    sh = np.repeat(np.asarray(scales).astype(np.float64), group, axis=1)
    z = np.repeat(np.asarray(zeros).astype(np.float64), group, axis=1)
    Wq = (q - z) * sh                                            # exact
    rs = (np.float32(1.0) / np.asarray(s_best, dtype=np.float32)).astype(np.float32)
    xs = (X.astype(np.float32) * rs[None, :]).astype(np.float32)  # one binary32 rounding
    return xs.astype(np.float64) @ Wq.T


# --------------------------------------------------------------------------
# AWQ followed by GPTQ error compensation -- [AWQ-note] "Measures" (AWQ+GPTQ
# at INT2); [Notes-52] §4 (round a column, push its error into the columns not
# yet quantized, using second-order statistics of the real input);
# [GPTQ-AWQ] "GPTQ" (column-wise sweep, Cholesky factor prepared once).
# --------------------------------------------------------------------------

def gptq_hessian(X: np.ndarray, s=None) -> np.ndarray:
    """H = 2 X'^T X' in binary64 (one library matrix product), with the input
    divided by s as the layer sees it after scaling: x' = RN32(x RN32(1/s))."""
    X = _as_f16(X)
    K = X.shape[1]
    s = np.ones(K, np.float32) if s is None else np.ascontiguousarray(s, dtype=np.float32)
    rs = (np.float32(1.0) / s).astype(np.float32)
    Xs = (X.astype(np.float32) * rs[None, :]).astype(np.float32).astype(np.float64)
    return 2.0 * (Xs.T @ Xs)


def gptq_factor(H: np.ndarray, damp: float = 0.01) -> np.ndarray:
    """U, the upper Cholesky factor of the damped inverse Hessian:
    Hd = H + damp * mean(diag H) * I,  Hd^-1 = U^T U  (library inverse and
    Cholesky, binary64)."""
    H = np.asarray(H, dtype=np.float64)
    Hd = H + damp * np.mean(np.diag(H)) * np.eye(H.shape[0])
    return np.linalg.cholesky(np.linalg.inv(Hd)).T


def gptq(W: np.ndarray, s, U, bits: int, group: int, zero_point: bool = True, rows=None,
         fixed_step: float = 0.0, stop_after: int = -1):
    """The GPTQ sweep over the scaled rows RN32(W s) with the binary32 factor U
    (see awq_oracle_gptq).  Returns dict(q, sh, z, what, w) like quantize(),
    w being the final scaled binary32 weights (dequantized values for the
    columns done)."""
    W = _as_f16(W)
    Ws = W if rows is None else np.ascontiguousarray(W[np.asarray(rows)])
    N, K = Ws.shape
    s = np.ascontiguousarray(s, dtype=np.float32)
    U32 = np.ascontiguousarray(U, dtype=np.float32)
    assert U32.shape == (K, K)
    G = K // group
    q = np.zeros((N, K), dtype=np.uint8)
    sh = np.zeros((N, G), dtype=np.uint16)
    z = np.zeros((N, G), dtype=np.float32)
    what = np.zeros((N, K), dtype=np.uint16)
    w = np.empty((N, K), dtype=np.float32)
    _load().awq_oracle_gptq(_ptr(Ws.view(np.uint16)), N, K, _ptr(s), _ptr(U32), int(bits), int(group),
                            int(bool(zero_point)), float(fixed_step), int(stop_after), _ptr(q), _ptr(sh),
                            _ptr(z), _ptr(what), _ptr(w))
    return dict(q=q, sh=sh.view(np.float16), z=z, what=what.view(np.float16), w=w)


def output_error(W: np.ndarray, What: np.ndarray, X: np.ndarray, rows=None) -> dict:
    """MSE of the layer output for a given W_hat (any quantizer's), binary64."""
    W = _as_f16(W)
    Ws = W if rows is None else np.ascontiguousarray(W[np.asarray(rows)])
    rs = output_error_sum(Ws, What, _as_f16(X))
    return dict(loss=rs.sum() / (Ws.shape[0] * X.shape[0]), row_sums=rs)
