"""Pins of the CPU oracle to facts outside itself.

Each test checks the oracle against something it cannot agree with by
construction: the worked examples printed on the pages (tests/golden), closed
forms, invariants of the method, an independent library (numpy's binary16),
and an independent brute force (oracle/bruteforce.py).  A plausible slip in the
oracle -- a dropped term, a wrong sign or index, a transposed operand, a
division where a multiplication belongs, the wrong rounding -- fails at least
one of them.
"""
import json
import math
import os
import struct
from fractions import Fraction

import numpy as np
import pytest

from awq_activation_aware_b200 import synth
from oracle import bruteforce

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _gold(name):
    with open(os.path.join(GOLD, name)) as f:
        return json.load(f)


# ---------------------------------------------------------------------------
# binary16 rounding vs numpy (independent implementation)
# ---------------------------------------------------------------------------

def test_rn16_matches_numpy(oracle_mod):
    rng = np.random.default_rng(1234)
    vals = np.concatenate([
        rng.standard_normal(3000) * 10.0 ** rng.integers(-9, 5, 3000),
        np.array([0.0, -0.0, 65504.0, 65519.99, 65520.0, -65520.0, 1e9, 2.0 ** -24, 2.0 ** -25,
                  3 * 2.0 ** -25, 2.0 ** -26, 2.0 ** -14, 2.0 ** -14 - 2.0 ** -25,
                  1.0 + 2.0 ** -11, 1.0 + 3 * 2.0 ** -11, 2049.0, 2051.0]),
    ])
    for v in vals:
        with np.errstate(over="ignore"):
            ref = np.array([v]).astype(np.float16).view(np.uint16)[0]
        got = oracle_mod.rn16_bits(v)
        assert got == ref, (v, hex(got), hex(ref))
    for b in [0, 1, 0x3FF, 0x400, 0x3C00, 0x7BFF, 0x8001, 0xFBFF, 0x7C00]:
        assert oracle_mod.h2d(b) == float(np.array([b], dtype=np.uint16).view(np.float16)[0])


# ---------------------------------------------------------------------------
# Worked example of "AWQ: Activation-Aware Weight Quantization For On-Device
# LLM Compression AND Acceleration", section "Measures"
# ---------------------------------------------------------------------------

def test_awq_note_example_primitives(oracle_mod):
    g = _gold("awq_note_int3_example.json")
    w = g["W"]
    # symmetric absmax step for INT3: max|w| / (2^(b-1) - 1)
    assert oracle_mod.absmax_step(w, g["bits"]) == pytest.approx(g["step"], rel=1e-15)
    assert oracle_mod.absmax_step(g["overscaled_W"], g["bits"]) == pytest.approx(
        g["overscaled_step"], rel=1e-15)
    # the non-negative levels of the step-1/3 grid
    levels = sorted({oracle_mod.round_to_step(v, g["step"]) for v in np.linspace(0, 1, 101)})
    assert levels == pytest.approx(g["levels_nonnegative"], abs=1e-15)
    x2 = g["activation_second"]
    assert w[1] * x2 == pytest.approx(g["true_contribution"])
    rtn = oracle_mod.round_to_step(w[1], g["step"]) * x2
    scaled = oracle_mod.round_to_step(w[1] * g["s"], g["step"]) / g["s"] * x2
    tol = 0.5 * 10.0 ** -g["printed_decimals"]
    assert rtn == pytest.approx(g["rtn_output"], abs=tol)
    assert scaled == pytest.approx(g["scaled_output"], abs=tol)


def test_awq_note_example_through_group_quantizer(oracle_mod):
    """The same example through the oracle's asymmetric group quantizer.

    A group [1.0, 0.2, 0, 0] at w_bit = 2 has min 0 and max 1, so scale = 1/3
    (stored in fp16) and the levels are the page's 0, 1/3, 2/3, 1.  Scaling the
    second input channel by 2 keeps the group maximum and halves the effective
    error; scaling it to 2.0 makes the step 2/3."""
    g = _gold("awq_note_int3_example.json")
    W = np.array([[1.0, 0.2, 0.0, 0.0]], dtype=np.float16)
    ones = np.ones(4, dtype=np.float32)
    # the page prints 3 decimals; the quantizer stores the step 1/3 in fp16 and
    # rounds Ŵ to fp16: two roundings of at most 2^-11 relative each
    def tol(v):
        return 0.5 * 10.0 ** -g["printed_decimals"] + abs(v) * 2 * 2.0 ** -11
    r0 = oracle_mod.quantize(W, ones, bits=2, group=4)
    assert float(r0["sh"][0, 0]) == pytest.approx(g["step"], rel=2 ** -11)
    assert float(r0["z"][0, 0]) == 0.0
    assert float(r0["what"][0, 1]) * g["activation_second"] == pytest.approx(g["rtn_output"], abs=tol(g["rtn_output"]))
    s = np.array([1.0, g["s"], 1.0, 1.0], dtype=np.float32)
    r1 = oracle_mod.quantize(W, s, bits=2, group=4)
    assert float(r1["sh"][0, 0]) == float(r0["sh"][0, 0])           # group max unchanged
    assert float(r1["what"][0, 1]) * g["activation_second"] == pytest.approx(g["scaled_output"], abs=tol(g["scaled_output"]))
    s2 = np.array([1.0, g["overscaled_W"][1] / float(W[0, 1]), 1.0, 1.0], dtype=np.float32)
    r2 = oracle_mod.quantize(W, s2, bits=2, group=4)
    assert float(r2["sh"][0, 0]) == pytest.approx(g["overscaled_step"], rel=2 ** -10)


def test_notes52_example_through_group_quantizer(oracle_mod):
    """"52 · AWQ, GPTQ và SmoothQuant" §3: step 0.125; 0.19 -> 0.25, and
    0.38 -> 0.375 -> 0.1875 after halving.  Group [1.875, 0.19, 0, 0] at
    w_bit = 4 has scale exactly 1.875 / 15 = 0.125."""
    g = _gold("notes52_step0125_example.json")
    W = np.array([[1.875, g["w"], 0.0, 0.0]], dtype=np.float16)
    r0 = oracle_mod.quantize(W, np.ones(4, dtype=np.float32), bits=4, group=4)
    assert float(r0["sh"][0, 0]) == g["step"]
    assert float(r0["what"][0, 1]) == g["rtn"]
    assert abs(g["rtn"] - g["w"]) / g["w"] * 100 == pytest.approx(g["rtn_rel_err_pct"], abs=0.5)
    s = np.array([1.0, g["s"], 1.0, 1.0], dtype=np.float32)
    r1 = oracle_mod.quantize(W, s, bits=4, group=4)
    assert int(r1["q"][0, 1]) * g["step"] == g["scaled_rtn"]
    assert float(r1["what"][0, 1]) == g["unscaled"]
    assert abs(g["unscaled"] - g["w"]) / g["w"] * 100 == pytest.approx(g["unscaled_rel_err_pct"], abs=0.5)


# ---------------------------------------------------------------------------
# Closed forms and invariants
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("bits,group", [(4, 128), (3, 128), (2, 64)])
def test_round_trip_exact_codes(oracle_mod, bits, group):
    """W built from chosen codes/scales/zeros (each group holds codes 0 and
    qmax, scales powers of two) is recovered exactly at alpha = 0, and Ŵ = W --
    also for zero points outside [0, qmax], i.e. groups that do not span zero."""
    rng = np.random.default_rng(bits * 100 + group)
    N, K = 6, 2 * group
    qmax = (1 << bits) - 1
    G = K // group
    q = rng.integers(0, qmax + 1, size=(N, K))
    for n in range(N):
        for gi in range(G):
            pos = rng.choice(group, 2, replace=False) + gi * group
            q[n, pos[0]], q[n, pos[1]] = 0, qmax
    z = rng.integers(0, qmax + 1, size=(N, G))
    z[:, 0] = rng.integers(-3 * qmax, 4 * qmax + 1, size=N)   # groups that do not span zero too
    sh = 2.0 ** rng.integers(-9, -3, size=(N, G))
    W = np.empty((N, K))
    for n in range(N):
        for gi in range(G):
            sl = slice(gi * group, (gi + 1) * group)
            W[n, sl] = (q[n, sl] - z[n, gi]) * sh[n, gi]
    W16 = W.astype(np.float16)
    assert np.array_equal(W16.astype(np.float64), W)
    r = oracle_mod.quantize(W16, np.ones(K, dtype=np.float32), bits, group)
    assert np.array_equal(r["q"], q)
    assert np.array_equal(r["z"], z.astype(np.float32))
    assert np.array_equal(r["sh"].astype(np.float64), sh)
    assert np.array_equal(r["what"], W16)


def test_one_signed_group_golden(oracle_mod):
    """A group that does not span zero, worked by hand from the affine formula
    zero = round(-min/scale), q = clamp(round(w/scale) + zero, 0, qmax)
    (tests/golden/one_signed_group_int4.json): the zero point leaves the code
    range ([1, 2] gives zero -15) and the codes still cover 0..15.  A zero
    point clamped to the codes would saturate every code instead."""
    g = _gold("one_signed_group_int4.json")
    for W_vals, part in ((g["W"], g), (g["mirrored"]["W"], g["mirrored"])):
        W = np.array([W_vals], dtype=np.float16)
        s = np.array(g["s"], dtype=np.float32)
        r = oracle_mod.quantize(W, s, bits=g["bits"], group=g["group"])
        assert float(r["sh"][0, 0]) == g["working"]["sh"]
        assert hex(int(r["sh"].view(np.uint16)[0, 0])) == g["working"]["sh_fp16_bits"]
        assert float(r["z"][0, 0]) == part["zero"]
        assert r["q"][0].tolist() == part["q"]
        assert r["what"][0].astype(np.float64).tolist() == part["W_hat"]
        Q, SH, Z, WH = bruteforce.quantize([list(map(float, W_vals))], [np.float32(v) for v in s],
                                           g["bits"], g["group"])
        assert Q == [part["q"]] and Z == [[part["zero"]]] and WH == [part["W_hat"]]
    assert g["zero_clamped_to_codes"]["W_hat"] != g["W_hat"]


def test_large_zero_points_against_bruteforce(oracle_mod):
    """Groups far from zero push |zero| past 2048, where not every integer is a
    binary16 value, and past 65504, where the fp16 zeros saturate: the oracle
    and the independent restatement agree bit for bit, the stored zero is a
    binary16 value, and the stored scale and zero reproduce W_hat."""
    rows = [
        [64.0, 64.5, 64.25, 64.0625, 64.125, 64.375, 64.4375, 64.3125],      # |zero| < 2048
        [128.0, 128.5, 128.25, 128.125, 128.375, 128.0, 128.5, 128.25],     # 2048 < |zero| < 4096
        [-1000.0, -999.5, -999.0, -998.5, -1000.0, -999.0, -999.5, -998.5],
        [3.0, 3.0, 3.0, 3.0, 3.0, 3.0, 3.0, 3.0],                           # constant: zero saturates
        [0.25, 0.25, 0.25, 0.25, 0.25, 0.25, 0.25, 0.25],
    ]
    W = np.array(rows, dtype=np.float16)
    assert np.array_equal(W.astype(np.float64), np.array(rows))
    for bits in (2, 3, 4):
        s = np.ones(8, dtype=np.float32)
        r = oracle_mod.quantize(W, s, bits, 8)
        Q, SH, Z, WH = bruteforce.quantize(rows, [np.float32(1.0)] * 8, bits, 8)
        assert r["q"].tolist() == Q
        assert r["z"].tolist() == Z
        assert r["sh"].astype(np.float64).tolist() == SH
        assert r["what"].astype(np.float64).tolist() == WH
        z = r["z"][:, 0].astype(np.float64)
        assert np.array_equal(z.astype(np.float16).astype(np.float64), z)
        assert np.abs(z).max() == 65504.0 and np.any(np.abs(z) > 2048)
        sh = r["sh"].astype(np.float32)
        deq = ((r["q"].astype(np.float32) - r["z"].astype(np.float32)) * sh).astype(np.float32)
        assert np.array_equal(deq.astype(np.float16), r["what"])


def test_zero_point_of_a_group_starting_at_zero_is_plus_zero(oracle_mod):
    """A group whose minimum is exactly +0 has zero point rint(-0 * r) = -0; the
    fp16 zeros store it as +0 (bits 0x0000), like any other zero, and the brute
    force's stored value is +0 too."""
    W = np.array([[0.0, 1.0, 2.0, 3.0, 0.5, 1.5, 2.5, 3.5]], dtype=np.float16)
    s = np.ones(8, dtype=np.float32)
    pk = oracle_mod.pack_scales(W, s, 4, 8)
    assert int(pk["zeros"].view(np.uint16)[0, 0]) == 0x0000
    _, _, Z, _ = bruteforce.quantize([list(map(float, W[0]))], [np.float32(1.0)] * 8, 4, 8)
    assert Z[0][0] == 0 and math.copysign(1.0, Z[0][0]) == 1.0


def test_ties_round_to_even(oracle_mod):
    # scale = 15/15 = 1; the values k + 1/2 land exactly on ties
    W = np.array([[0.0, 15.0, 0.5, 1.5, 2.5, 3.5, 10.5, 11.5]], dtype=np.float16)
    r = oracle_mod.quantize(W, np.ones(8, dtype=np.float32), bits=4, group=8)
    assert float(r["sh"][0, 0]) == 1.0 and float(r["z"][0, 0]) == 0.0
    assert r["q"][0].tolist() == [0, 15, 0, 2, 2, 4, 10, 12]


def test_scales_closed_forms(oracle_mod):
    """s = RN32(a^alpha) ([AWQ-note] "Measures": a^alpha per candidate alpha)
    at the exponents with closed forms: alpha = 1 gives a itself, alpha = 0
    gives 1, and alpha = 1/2 gives the binary32 value nearest the exact square
    root (chosen here by comparing squares of rationals, without pow); a dead
    channel (a = 0) is lifted to FLT_MIN first."""
    rng = np.random.default_rng(65)
    a = np.concatenate([(10.0 ** rng.uniform(-6, 4, 400)).astype(np.float32),
                        np.array([0.0, 1.0, 4.0, 2.0, 1e-30, 3.0e38], np.float32)])
    fmin = np.float32(2.0 ** -126)
    assert np.array_equal(oracle_mod.scales(a, 1.0), np.maximum(a, fmin))
    assert np.all(oracle_mod.scales(a, 0.0) == 1.0)
    half = oracle_mod.scales(a, 0.5)
    for ai, si in zip(np.maximum(a, fmin), half):
        A = Fraction(float(ai))
        y = np.float32(math.sqrt(float(ai)))
        cands = [np.nextafter(y, np.float32(0)), y, np.nextafter(y, np.float32(np.inf))]
        best = y
        for c in cands:                     # nearest: |sqrt(A) - c| smallest, via squares of midpoints
            lo, hi = min(c, best), max(c, best)
            if lo == hi:
                continue
            mid = (Fraction(float(lo)) + Fraction(float(hi))) / 2
            nearer_lo = A < mid * mid
            best = lo if nearer_lo else hi
        assert si == best, (ai, si, best)


def test_alpha_zero_is_plain_rtn(oracle_mod):
    """alpha = 0 gives s = 1 exactly, so the search's first candidate is plain
    group RTN; the brute force's RTN (binary32 hardware ops) must agree bit
    for bit."""
    W, X, _ = synth.generate(synth.make_config(4, 256, 8, bits=4, group=128, seed=7))
    a = oracle_mod.act_stats(X)
    s = oracle_mod.scales(a, 0.0)
    assert np.all(s == 1.0)
    r = oracle_mod.quantize(W, s, 4, 128)
    Wl = [[float(v) for v in row] for row in W.astype(np.float64)]
    Q, SH, Z, WH = bruteforce.quantize(Wl, [np.float32(1.0)] * 256, 4, 128)
    assert r["q"].tolist() == Q
    assert r["z"].tolist() == Z
    assert r["sh"].astype(np.float64).tolist() == SH
    assert r["what"].astype(np.float64).tolist() == WH


def test_scaling_is_identity_without_rounding(oracle_mod):
    """Y = (W D)(D^-1 x): without the rounding step, scale-quantize-unscale
    returns W up to binary32/binary16 rounding, so the loss is ~0."""
    cfg = synth.make_config(16, 256, 64, bits=4, group=128, seed=3)
    W, X, _ = synth.generate(cfg)
    a = oracle_mod.act_stats(X)
    alphas = synth.default_alphas()
    ident = oracle_mod.search(W, X, a, 4, 128, alphas, no_round=True)["losses"]
    real = oracle_mod.search(W, X, a, 4, 128, alphas)["losses"]
    assert np.all(ident <= 1e-6 * real.min())
    for al in alphas:
        what = oracle_mod.quantize(W, oracle_mod.scales(a, float(al)), 4, 128, no_round=True)["what"]
        # at most one fp16 ulp away from W
        ulp = np.spacing(np.abs(W).astype(np.float16)).astype(np.float64)
        assert np.all(np.abs(what.astype(np.float64) - W.astype(np.float64)) <= ulp)


def test_power_of_two_scale_invariance(oracle_mod):
    """s -> 2^k s multiplies every binary32/binary16 intermediate by 2^k and
    divides it back out, so codes and Ŵ are bit-identical."""
    cfg = synth.make_config(8, 256, 16, bits=4, group=128, seed=11)
    W, X, _ = synth.generate(cfg)
    s = oracle_mod.scales(oracle_mod.act_stats(X), 0.5)
    r0 = oracle_mod.quantize(W, s, 4, 128)
    for k in (-3, 1, 4):
        r1 = oracle_mod.quantize(W, (s * np.float32(2.0 ** k)).astype(np.float32), 4, 128)
        assert np.array_equal(r0["q"], r1["q"])
        assert np.array_equal(r0["z"], r1["z"])
        assert np.array_equal(r0["what"], r1["what"])


def test_loss_identity_activations(oracle_mod):
    """X = I_K (T = K): the output error is the Frobenius norm of Ŵ - W."""
    rng = np.random.default_rng(5)
    W = (rng.standard_normal((3, 64)) * 0.02).astype(np.float16)
    What = (W.astype(np.float64) + rng.integers(-3, 4, W.shape) * 2.0 ** -12).astype(np.float16)
    X = np.eye(64, dtype=np.float16)
    got = oracle_mod.output_error_sum(W, What, X)
    d = What.astype(np.float64) - W.astype(np.float64)
    for n in range(3):
        assert got[n] == pytest.approx(sum(v * v for v in d[n]), rel=1e-13)


def test_loss_rank_one_activations(oracle_mod):
    """Every token equal to x: row error = T (ΔW_n · x)^2."""
    rng = np.random.default_rng(6)
    W = (rng.standard_normal((4, 128)) * 0.02).astype(np.float16)
    What = (W.astype(np.float64) * 1.01).astype(np.float16)
    x = rng.standard_normal(128).astype(np.float16)
    T = 9
    X = np.tile(x, (T, 1))
    got = oracle_mod.output_error_sum(W, What, X)
    for n in range(4):
        dot = sum((float(What[n, k]) - float(W[n, k])) * float(x[k]) for k in range(128))
        assert got[n] == pytest.approx(T * dot * dot, rel=1e-12)


def test_act_stats_exact_mean(oracle_mod):
    rng = np.random.default_rng(9)
    X = (rng.standard_normal((37, 24)) * 10.0 ** rng.integers(-6, 2, (37, 24))).astype(np.float16)
    X[:, 5] = 0
    a = oracle_mod.act_stats(X)
    for j in range(24):
        tot = sum(Fraction(abs(float(v))) for v in X[:, j])
        assert a[j] == np.float32(float(tot) / 37)
    assert a[5] == 0.0


def test_pack_codes_bit_layout(oracle_mod):
    rng = np.random.default_rng(2)
    for bits in (2, 3, 4):
        q = rng.integers(0, 1 << bits, size=(3, 64)).astype(np.uint8)
        codes = oracle_mod.pack_codes(q, bits)
        c = 2 if bits == 2 else 4
        per = 32 // c
        for n in range(3):
            for k in range(64):
                word = int(codes[n, k // per])
                assert (word >> (c * (k % per))) & ((1 << c) - 1) == q[n, k]


def test_argmin_rules(oracle_mod):
    assert oracle_mod.argmin([3.0, 1.0, 1.0, 2.0]) == 1
    assert oracle_mod.argmin([float("nan"), 5.0, float("nan"), 4.0]) == 3
    assert oracle_mod.argmin([float("nan"), float("nan")]) == 0
    assert oracle_mod.argmin([float("inf"), 7.0]) == 1


# ---------------------------------------------------------------------------
# Brute force on tiny layers
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("N,K,T,bits,group,seed", [
    (3, 128, 8, 4, 128, 21),
    (2, 128, 6, 3, 64, 22),
    (4, 64, 5, 2, 64, 23),
    (2, 256, 4, 4, 128, 24),
])
def test_bruteforce_search(oracle_mod, N, K, T, bits, group, seed):
    cfg = synth.make_config(N, K, T, bits=bits, group=group, seed=seed, outlier_frac=0.03)
    W, X, _ = synth.generate(cfg)
    alphas = synth.default_alphas()
    bf = bruteforce.search(W, X, bits, group, alphas)
    a = oracle_mod.act_stats(X)
    assert np.array_equal(a, bf["a"])
    orc = oracle_mod.search(W, X, a, bits, group, alphas)
    np.testing.assert_allclose(orc["losses"], bf["losses"], rtol=1e-12, atol=0)
    assert orc["best"] == bf["best"]
    for i in (0, bf["best"], len(alphas) - 1):
        Q, SH, Z, WH, s = bf["per_alpha"][i]
        r = oracle_mod.quantize(W, oracle_mod.scales(a, float(alphas[i])), bits, group)
        assert r["q"].tolist() == Q
        assert r["z"].tolist() == Z
        assert r["what"].astype(np.float64).tolist() == WH
        assert oracle_mod.scales(a, float(alphas[i])).tolist() == [float(v) for v in s]


# ---------------------------------------------------------------------------
# Premise of the method (sanity, not a value pin)
# ---------------------------------------------------------------------------

def test_premise_activation_aware_beats_rtn(oracle_mod):
    """With ~1% outlier channels the best alpha beats plain RTN (alpha = 0), and
    the error is not monotone in alpha (it falls, then rises again: the note
    "52 · AWQ, GPTQ và SmoothQuant" §3 observes error falling up to a point)."""
    cfg = synth.make_config(64, 512, 128, bits=4, group=128, seed=0, lo=20.0, hi=20.0)
    W, X, _ = synth.generate(cfg)
    a = oracle_mod.act_stats(X)
    r = oracle_mod.search(W, X, a, 4, 128, synth.default_alphas())
    L = r["losses"]
    assert r["best"] > 0 and L[r["best"]] < L[0]
    assert not np.all(np.diff(L) >= 0)


# ---------------------------------------------------------------------------
# The consumer of the packed format (quantized linear layer)
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("bits,group", [(4, 128), (3, 128), (2, 64)])
def test_qlinear_identity_input_gives_dequantized_weights(oracle_mod, bits, group):
    """x = e_t (T = K) and s = 1: Y[t, n] = (q[n, t] - z) sh exactly, read back
    from the packed words."""
    W, X, _ = synth.generate(synth.make_config(12, 128, 8, bits=bits, group=group, seed=61))
    s = np.ones(128, dtype=np.float32)
    r = oracle_mod.quantize(W, s, bits, group)
    codes = oracle_mod.pack_codes(r["q"], bits)
    Y = oracle_mod.qlinear(codes, r["sh"], r["z"].astype(np.float16), s, np.eye(128, dtype=np.float16),
                           bits, group)
    G = np.arange(128) // group
    expect = (r["q"].astype(np.float64) - r["z"][:, G]) * r["sh"].astype(np.float64)[:, G]
    assert np.array_equal(Y, expect.T)


def test_qlinear_matches_dequantized_matmul(oracle_mod):
    """With s folded into the input, Y equals X W_hat^T up to W_hat's fp16 rounding."""
    W, X, _ = synth.generate(synth.make_config(48, 256, 16, seed=62))
    a = oracle_mod.act_stats(X)
    al = synth.default_alphas()
    pk = oracle_mod.pack(W, a, 4, 128, al, oracle_mod.search(W, X, a, 4, 128, al)["losses"])
    Y = oracle_mod.qlinear(pk["codes"], pk["scales"], pk["zeros"], pk["s_best"], X, 4, 128)
    Yh = X.astype(np.float64) @ pk["what"].astype(np.float64).T
    assert np.linalg.norm(Y - Yh) / np.linalg.norm(Yh) < 2.0 ** -11


def test_qlinear_against_exact_rationals(oracle_mod):
    """Tiny case in exact arithmetic: r = RN32(1/s) and x' = RN32(x r) formed
    from exact rationals with an explicit round-to-nearest-even, the sum
    sum_k x' (q - z) sh kept exact.  s is not a power of two, so a division in
    place of the reciprocal, or an x' left in binary64, moves Y off the exact
    value by far more than the binary64 summation can."""
    rng = np.random.default_rng(63)
    N, K, T, bits, group = 3, 64, 2, 4, 32
    q = rng.integers(0, 16, (N, K)).astype(np.uint8)
    sh = (rng.uniform(0.001, 0.02, (N, K // group))).astype(np.float16)
    z = rng.integers(-20, 36, (N, K // group)).astype(np.float16)
    s = rng.uniform(0.3, 7.0, K).astype(np.float32)
    X = (rng.standard_normal((T, K)) * 3).astype(np.float16)
    codes = oracle_mod.pack_codes(q, bits)
    Y = oracle_mod.qlinear(codes, sh, z, s, X, bits, group)
    for t in range(T):
        for n in range(N):
            exact, absum = Fraction(0), Fraction(0)
            for k in range(K):
                r = _rn32_exact(Fraction(1) / Fraction(float(s[k])))
                xp = _rn32_exact(Fraction(float(X[t, k])) * Fraction(float(r)))
                term = Fraction(float(xp)) * (int(q[n, k]) - Fraction(float(z[n, k // group]))) \
                    * Fraction(float(sh[n, k // group]))
                exact += term
                absum += abs(term)
            assert abs(Fraction(float(Y[t, n])) - exact) <= Fraction(1, 10**12) * absum, (t, n)


# ---------------------------------------------------------------------------
# Quantizer variants and baselines: the symmetric absmax quantizer, channels
# held in fp16, caller-given scale vectors, top-k channel selection
# ---------------------------------------------------------------------------

def test_awq_note_example_through_symmetric_quantizer(oracle_mod):
    """[AWQ-note] "Measures": the INT3 grid of step max|w| / (2^(b-1) - 1) is the
    symmetric quantizer at w_bit = 3.  Group [1.0, 0.2, 0, 0]: step 1/3 (fp16),
    middle code 4, W_hat[1] x 10 = 3.333; s = 2 on that channel keeps the group
    maximum and gives 1.667; scaling it to 2.0 makes the step 2/3."""
    g = _gold("awq_note_int3_example.json")
    W = np.array([[1.0, 0.2, 0.0, 0.0]], dtype=np.float16)
    def tol(v):
        return 0.5 * 10.0 ** -g["printed_decimals"] + abs(v) * 2 * 2.0 ** -11
    r0 = oracle_mod.quantize(W, np.ones(4, dtype=np.float32), bits=g["bits"], group=4, zero_point=False)
    assert float(r0["sh"][0, 0]) == pytest.approx(g["step"], rel=2 ** -11)
    assert float(r0["z"][0, 0]) == 4.0
    assert list(r0["q"][0]) == [7, 5, 4, 4]
    assert float(r0["what"][0, 1]) * g["activation_second"] == pytest.approx(g["rtn_output"], abs=tol(g["rtn_output"]))
    s = np.array([1.0, g["s"], 1.0, 1.0], dtype=np.float32)
    r1 = oracle_mod.quantize(W, s, bits=g["bits"], group=4, zero_point=False)
    assert float(r1["sh"][0, 0]) == float(r0["sh"][0, 0])
    assert float(r1["what"][0, 1]) * g["activation_second"] == pytest.approx(g["scaled_output"], abs=tol(g["scaled_output"]))
    s2 = np.array([1.0, g["overscaled_W"][1] / float(W[0, 1]), 1.0, 1.0], dtype=np.float32)
    r2 = oracle_mod.quantize(W, s2, bits=g["bits"], group=4, zero_point=False)
    assert float(r2["sh"][0, 0]) == pytest.approx(g["overscaled_step"], rel=2 ** -10)


@pytest.mark.parametrize("bits", [2, 3, 4])
def test_symmetric_quantizer_is_odd(oracle_mod, bits):
    """Q(-W) = -Q(W) (rint ties to even is odd), zero at 2^(bits-1), codes in
    [1, 2^bits - 1] whenever the fp16 scale is not clamped."""
    W, X, _ = synth.generate(synth.make_config(16, 256, 4, bits=bits, seed=71))
    a = oracle_mod.act_stats(X)
    s = oracle_mod.scales(a, 0.5)
    r = oracle_mod.quantize(W, s, bits, 128, zero_point=False)
    rn = oracle_mod.quantize(-W, s, bits, 128, zero_point=False)
    assert np.array_equal(rn["what"], -r["what"])          # as values: a zero level is +0 on both sides
    assert np.all(r["z"] == 2 ** (bits - 1))
    assert r["q"].min() >= 1 and r["q"].max() <= 2 ** bits - 1


@pytest.mark.parametrize("bits,group,sym", [(4, 16, False), (4, 16, True), (3, 8, True), (2, 8, False)])
def test_variants_against_bruteforce(oracle_mod, bits, group, sym):
    """The C oracle's symmetric quantizer and fp16-kept channels against the
    independent binary32-scalar restatement, codes / scales / zeros / W_hat bit
    for bit and the loss exactly (rational arithmetic)."""
    from oracle import bruteforce as bf
    rng = np.random.default_rng(bits * 100 + group)
    W = (rng.standard_normal((5, 32)) * 0.05).astype(np.float16)
    X = rng.standard_normal((6, 32)).astype(np.float16)
    X[:, [3, 17]] *= np.float16(30)
    s = (rng.random(32) * 3 + 0.25).astype(np.float32)
    keep = np.zeros(32, dtype=np.uint8)
    keep[[3, 9, 17]] = 1
    keep[group:2 * group] = 1                       # a whole group held in fp16
    r = oracle_mod.quantize(W, s, bits, group, zero_point=not sym, mask=keep)
    Q, SH, Z, WH = bf.quantize([[float(v) for v in row] for row in W.astype(np.float64)],
                               [np.float32(v) for v in s], bits, group, sym, list(keep))
    assert np.array_equal(r["q"], np.array(Q, dtype=np.uint8))
    assert np.array_equal(r["sh"].astype(np.float64), np.array(SH))
    assert np.array_equal(r["z"].astype(np.float64), np.array(Z, dtype=np.float64))
    assert np.array_equal(r["what"].astype(np.float64), np.array(WH))
    assert np.array_equal(r["what"][:, keep == 1], W[:, keep == 1])
    exact, _ = bf.masked_loss(W, X, s, bits, group, keep, sym)
    got = oracle_mod.search_scales(W, X, s[None], bits, group, zero_point=not sym, mask=keep)["losses"][0]
    assert got == pytest.approx(exact, rel=1e-12)


def test_mask_extremes(oracle_mod):
    """Every channel held in fp16: W_hat = W and zero loss.  No channel held:
    the plain quantizer."""
    W, X, _ = synth.generate(synth.make_config(8, 256, 16, seed=72))
    s = np.ones(256, dtype=np.float32)
    r = oracle_mod.quantize(W, s, 4, 128, mask=np.ones(256, dtype=np.uint8))
    assert np.array_equal(r["what"].view(np.uint16), W.view(np.uint16))
    assert oracle_mod.search_scales(W, X, s[None], 4, 128, mask=np.ones(256, np.uint8))["losses"][0] == 0.0
    r0 = oracle_mod.quantize(W, s, 4, 128, mask=np.zeros(256, dtype=np.uint8))
    r1 = oracle_mod.quantize(W, s, 4, 128)
    assert np.array_equal(r0["what"].view(np.uint16), r1["what"].view(np.uint16))


def test_topk_matches_sorted_order(oracle_mod):
    """Top-k by value, ties to the lower index, NaN last -- against Python's sort."""
    rng = np.random.default_rng(73)
    v = rng.integers(0, 20, 300).astype(np.float32)       # many ties
    v[[5, 50, 299]] = np.nan
    for k in [0, 1, 3, 17, 150, 297, 298, 300]:
        order = sorted(range(v.size), key=lambda j: (bool(np.isnan(v[j])), -(0 if np.isnan(v[j]) else v[j]), j))
        expect = np.zeros(v.size, dtype=np.uint8)
        expect[order[:k]] = 1
        assert np.array_equal(oracle_mod.topk_mask(v, k), expect), k


def test_given_scales_reduce_to_the_grid(oracle_mod):
    """s = 1 is plain RTN, the alpha = 0 point of the grid; the grid's s
    vectors passed as a table give the grid's losses."""
    W, X, _ = synth.generate(synth.make_config(16, 256, 32, seed=74))
    a = oracle_mod.act_stats(X)
    al = np.array([0.0, 0.25, 0.5], dtype=np.float32)
    grid = oracle_mod.search(W, X, a, 4, 128, al)["losses"]
    table = np.stack([oracle_mod.scales(a, float(x)) for x in al])
    assert np.array_equal(oracle_mod.search_scales(W, X, table, 4, 128)["losses"], grid)
    assert oracle_mod.search_scales(W, X, np.ones((1, 256), np.float32), 4, 128)["losses"][0] == grid[0]


def test_baselines_premise(oracle_mod):
    """[AWQ-note] "Measures": keeping the 1% of channels with the largest
    activations in fp16 helps far more than choosing them by weight magnitude;
    scaling those channels by a fixed 2 helps, and the searched s helps more.
    On a synthetic layer with 1% outlier input channels:"""
    cfg = synth.make_config(256, 512, 256, seed=5)
    W, X, idx = synth.generate(cfg)
    a = oracle_mod.act_stats(X)
    k = round(cfg.K / 100)
    m_act = oracle_mod.topk_mask(a, k)
    m_w = oracle_mod.topk_mask(oracle_mod.act_stats(W), k)       # mean |w| per input channel
    assert np.all(m_act[idx] == 1)                                  # the outliers are found
    one = np.ones((1, cfg.K), np.float32)
    rtn = oracle_mod.search_scales(W, X, one, 4, 128)["losses"][0]
    fp16_act = oracle_mod.search_scales(W, X, one, 4, 128, mask=m_act)["losses"][0]
    fp16_w = oracle_mod.search_scales(W, X, one, 4, 128, mask=m_w)["losses"][0]
    s2 = np.where(m_act == 1, 2.0, 1.0).astype(np.float32)[None]
    fixed2 = oracle_mod.search_scales(W, X, s2, 4, 128)["losses"][0]
    awq = oracle_mod.search(W, X, a, 4, 128, synth.default_alphas())["losses"].min()
    assert fp16_act < 0.1 * rtn
    assert fp16_w > 0.9 * rtn
    assert awq < fixed2 < 0.5 * rtn


# ---------------------------------------------------------------------------
# AWQ followed by GPTQ error compensation
# ---------------------------------------------------------------------------

def test_notes52_gptq_toy(oracle_mod):
    """"52 · AWQ, GPTQ và SmoothQuant" §4: rounding 0.34, 0.33, 0.33 to step
    0.25 gives 0.75; rounding column by column and pushing each error into the
    rest gives exactly 1.00 (input 1 on each weight)."""
    g = _gold("notes52_gptq_toy.json")
    W = np.array([g["W"]], dtype=np.float16)
    X = np.array([g["inputs"]], dtype=np.float16)
    one = np.ones(3, np.float32)
    rtn = np.round(W.astype(np.float64) / g["step"]) * g["step"]
    assert float((rtn * X).sum()) == g["rtn_output"]
    U = oracle_mod.gptq_factor(oracle_mod.gptq_hessian(X, one))
    r = oracle_mod.gptq(W, one, U, 4, 3, fixed_step=g["step"])
    assert float((r["w"].astype(np.float64) * X).sum()) == g["error_feedback_output"]
    assert np.all(np.isin(r["w"], [0.0, 0.25, 0.5]))           # every weight on the grid


def test_gptq_with_uncorrelated_inputs_is_rtn(oracle_mod):
    """With orthogonal input channels H is diagonal, so U is and no error moves:
    the sweep reproduces the plain quantizer bit for bit."""
    rng = np.random.default_rng(101)
    W = (rng.standard_normal((6, 128)) * 0.05).astype(np.float16)
    X = np.zeros((128, 128), np.float16)
    X[np.arange(128), np.arange(128)] = rng.uniform(0.5, 4.0, 128).astype(np.float16)
    s = rng.uniform(0.5, 2.0, 128).astype(np.float32)
    U = oracle_mod.gptq_factor(oracle_mod.gptq_hessian(X, s))
    assert np.count_nonzero(np.triu(U, 1)) == 0
    for zp in (True, False):
        r = oracle_mod.gptq(W, s, U, 4, 64, zero_point=zp)
        ref = oracle_mod.quantize(W, s, 4, 64, zero_point=zp)
        assert np.array_equal(r["q"], ref["q"])
        assert np.array_equal(r["what"].view(np.uint16), ref["what"].view(np.uint16))


def test_gptq_hessian_is_the_output_error_quadratic(oracle_mod):
    """H is the curvature of the output error GPTQ compensates ([Notes-52] §4:
    second-order statistics of the real input): with D = W_hat - W, the summed
    squared output error sum_n ||D_n X^T||^2 equals (1/2) sum_n D_n H D_n^T.
    The left side comes from output_error (a product with X^T, no Gram matrix),
    so a transposed operand or a lost factor 2 in H fails here."""
    rng = np.random.default_rng(103)
    N, K, T = 5, 24, 37
    W = (rng.standard_normal((N, K)) * 0.1).astype(np.float16)
    step = (rng.integers(-3, 4, (N, K)) * 2.0 ** -8).astype(np.float32)
    What = (W.astype(np.float32) + step).astype(np.float16)
    X = (rng.standard_normal((T, K)) + rng.standard_normal((T, 1))).astype(np.float16)
    lhs = oracle_mod.output_error(W, What, X)["loss"] * N * T
    H = oracle_mod.gptq_hessian(X)
    Dd = What.astype(np.float64) - W.astype(np.float64)            # exact: two fp16 values
    assert np.count_nonzero(Dd) > N * K // 2
    rhs = 0.5 * np.einsum("nk,kj,nj->", Dd, H, Dd)
    assert lhs == pytest.approx(rhs, rel=1e-12)
    assert H.shape == (K, K) and np.array_equal(H, H.T)


def test_gptq_hessian_scales_with_the_input(oracle_mod):
    """x' = x / s: with powers of two for s every x' is exact, so
    H(s) = diag(1/s) H(1) diag(1/s) holds bit for bit."""
    rng = np.random.default_rng(104)
    K, T = 16, 50
    X = rng.standard_normal((T, K)).astype(np.float16)
    s = (2.0 ** rng.integers(-3, 4, K)).astype(np.float32)
    H1 = oracle_mod.gptq_hessian(X)
    Hs = oracle_mod.gptq_hessian(X, s)
    r = 1.0 / s.astype(np.float64)
    assert np.array_equal(Hs, H1 * r[:, None] * r[None, :])


def test_gptq_step_is_the_least_squares_correction(oracle_mod):
    """After the first column is rounded, the change the sweep makes to the
    remaining weights is the one that minimises the (damped) output error with
    that column fixed: dw_rest = -Hd_rr^-1 Hd_r0 dw_0 (normal equations, solved
    by the library)."""
    rng = np.random.default_rng(102)
    K = 16
    W = (rng.standard_normal((3, K)) * 0.1).astype(np.float16)
    X = (rng.standard_normal((40, K)) + rng.standard_normal((40, 1))).astype(np.float16)   # correlated
    one = np.ones(K, np.float32)
    H = oracle_mod.gptq_hessian(X, one)
    Hd = H + 0.01 * np.mean(np.diag(H)) * np.eye(K)
    U = oracle_mod.gptq_factor(H)
    r = oracle_mod.gptq(W, one, U, 4, 16, stop_after=1)
    w0 = W.astype(np.float64)
    d0 = r["w"][:, 0].astype(np.float64) - w0[:, 0]
    expect = w0[:, 1:] - np.outer(d0, np.linalg.solve(Hd[1:, 1:], Hd[1:, 0]))
    np.testing.assert_allclose(r["w"][:, 1:], expect, rtol=1e-5, atol=1e-6)


def _rn32_exact(x):
    """Nearest binary32 (ties to even) of an exact rational, without double rounding."""
    from fractions import Fraction
    f = np.float32(float(x))
    lo, hi = (f, np.nextafter(f, np.float32(np.inf))) if Fraction(float(f)) <= x else \
             (np.nextafter(f, np.float32(-np.inf)), f)
    dl, dh = x - Fraction(float(lo)), Fraction(float(hi)) - x
    if dl < dh or (dl == dh and (lo.view(np.uint32) & 1) == 0):
        return lo
    return hi


def test_gptq_sweep_against_scalar_restatement(oracle_mod):
    """The C sweep against a scalar restatement with exact rational FMAs
    (asymmetric groups, 2 groups of 8, 3 rows)."""
    from fractions import Fraction
    rng = np.random.default_rng(103)
    K, g, bits = 16, 8, 3
    qmax = (1 << bits) - 1
    W = (rng.standard_normal((3, K)) * 0.1).astype(np.float16)
    X = (rng.standard_normal((30, K)) + 0.5 * rng.standard_normal((30, 1))).astype(np.float16)
    s = rng.uniform(0.5, 2.0, K).astype(np.float32)
    U = oracle_mod.gptq_factor(oracle_mod.gptq_hessian(X, s)).astype(np.float32)
    got = oracle_mod.gptq(W, s, U, bits, g)
    from oracle import bruteforce as bf
    for n in range(3):
        w = [np.float32(np.float32(W[n, k]) * s[k]) for k in range(K)]
        for k in range(K):
            if k % g == 0:
                mn, mx = min(w[k:k + g]), max(w[k:k + g])
                scale = np.float32(np.float32(mx - mn) / np.float32(qmax))
                sh = bf.to_f16(min(max(float(scale), 2.0 ** -24), 65504.0))
                r = np.float32(np.float32(1.0) / np.float32(sh))
                z = bf.stored_zero(round(-float(mn) * float(r)))
            qk = min(max(round(float(w[k]) * float(r)) + z, 0), qmax)
            wq = np.float32(np.float32(qk - z) * np.float32(sh))
            e = np.float32(np.float32(w[k] - wq) / U[k, k])
            for j in range(k + 1, K):
                w[j] = _rn32_exact(Fraction(float(w[j])) - Fraction(float(e)) * Fraction(float(U[k, j])))
            assert got["q"][n, k] == qk, (n, k)
            w[k] = wq
        assert np.array_equal(got["w"][n], np.array(w, np.float32))


@pytest.mark.parametrize("bits,group", [(2, 64), (3, 128), (4, 128)])
def test_awq_gptq_premise(oracle_mod, bits, group):
    """[AWQ-note] "Measures": AWQ's scaling and GPTQ's error compensation are
    complementary -- AWQ+GPTQ below either alone (a synthetic layer with 1%
    outlier channels; at INT2 plain GPTQ can do worse than RTN there)."""
    cfg = synth.make_config(256, 512, 512, bits=bits, group=group, seed=11)
    W, X, _ = synth.generate(cfg)
    a = oracle_mod.act_stats(X)
    al = synth.default_alphas()
    res = oracle_mod.search(W, X, a, bits, group, al)
    s_best = oracle_mod.scales(a, float(al[res["best"]]))
    one = np.ones(cfg.K, np.float32)
    gptq = oracle_mod.gptq(W, one, oracle_mod.gptq_factor(oracle_mod.gptq_hessian(X, one)), bits, group)
    both = oracle_mod.gptq(W, s_best, oracle_mod.gptq_factor(oracle_mod.gptq_hessian(X, s_best)), bits, group)
    l_gptq = oracle_mod.output_error(W, gptq["what"], X)["loss"]
    l_both = oracle_mod.output_error(W, both["what"], X)["loss"]
    assert l_both < res["losses"].min()
    assert l_both < l_gptq
    if bits > 2:
        assert l_gptq < res["losses"][0]
