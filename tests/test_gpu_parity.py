"""CUDA path vs the CPU oracle, element by element, on seeded inputs.

Acceptance:
  * activation statistics, s tables, W_hat, codes, scales and zeros: bit-exact
    (integer results, and binary32/binary16 values whose every rounding step is
    pinned by the quantizer's definition);
  * per-alpha losses and per-row sums: relative 1e-3 (the tensor core
    accumulates in binary32 over Delta W rounded to fp16; the oracle is binary64);
  * chosen alpha: identical unless the oracle's two best losses lie within 1e-3;
  * the layer output error recomputed from the packed codes: relative 1e-3.
"""
import numpy as np
import pytest
import torch

import oracle
from awq_activation_aware_b200 import synth

pytestmark = pytest.mark.gpu

LOSS_RTOL = 1e-3


@pytest.fixture(scope="module")
def awq():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import awq_activation_aware_b200 as m
    m.set_wait_timeout_ms(2000)
    return m


def dev(x):
    return torch.from_numpy(np.ascontiguousarray(x)).cuda()


def host(t):
    return t.detach().cpu().numpy()


def gen(N, K, T, bits=4, group=128, seed=0, **kw):
    cfg = synth.make_config(N, K, T, bits=bits, group=group, seed=seed, **kw)
    W, X, _ = synth.generate(cfg)
    return W, X


def unpack_codes(codes, N, K, bits):
    c = 2 if bits == 2 else 4
    per = 32 // c
    words = codes.view(np.uint32).reshape(N, K // per).astype(np.uint64)
    q = np.empty((N, K), dtype=np.uint8)
    for i in range(per):
        q[:, i::per] = ((words >> (c * i)) & ((1 << c) - 1)).astype(np.uint8)
    return q


def dequantize(q, scales, zeros, s_best, group):
    """Consumer-side reconstruction w_hat = RN16(RN32(RN32((q - z) sh) RN32(1/s)))."""
    N, K = q.shape
    sh = np.repeat(scales.astype(np.float32), group, axis=1)
    z = np.repeat(zeros.astype(np.float32), group, axis=1)
    deq = (q.astype(np.float32) - z) * sh                       # exact
    rs = (np.float32(1.0) / s_best.astype(np.float32)).astype(np.float32)
    return (deq * rs[None, :]).astype(np.float32).astype(np.float16)


def assert_alpha_choice(best_gpu, losses_oracle):
    best_o = oracle.argmin(losses_oracle)
    if best_gpu != best_o:
        order = np.argsort(losses_oracle, kind="stable")
        l1, l2 = losses_oracle[order[0]], losses_oracle[order[1]]
        assert abs(l2 - l1) <= LOSS_RTOL * l1, (best_gpu, best_o, losses_oracle)
        assert best_gpu in (order[0], order[1])


# ---------------------------------------------------------------------------
# a1: activation statistics
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("T,K,ldx", [(512, 512, 512), (1000, 136, 136), (37, 64, 96), (1, 8, 8),
                                     (4096, 4096, 4096), (3000, 1032, 1040)])
def test_act_stats_bit_exact(awq, T, K, ldx):
    rng = np.random.default_rng(T * 7 + K)
    X = np.zeros((T, ldx), dtype=np.float16)
    X[:, :K] = (rng.standard_normal((T, K)) * 10.0 ** rng.integers(-7, 2, (T, K))).astype(np.float16)
    Xd = dev(X)[:, :K]
    a = host(awq.act_stats(Xd))
    awq.get_status()
    ref = oracle.act_stats(np.ascontiguousarray(X[:, :K]))
    assert np.array_equal(a, ref)


# ---------------------------------------------------------------------------
# a2: s = a^alpha
# ---------------------------------------------------------------------------
def test_alpha_scales_bit_exact(awq):
    W, X = gen(8, 1024, 300, seed=5)
    a = oracle.act_stats(X)
    a[3] = 0.0                                   # a dead channel is lifted to FLT_MIN
    alphas = synth.default_alphas()
    s = host(awq.alpha_scales(dev(a), dev(alphas)))
    for i, al in enumerate(alphas):
        assert np.array_equal(s[i], oracle.scales(a, float(al))), i
    assert np.all(s[0] == 1.0)


def test_bad_alpha_reported(awq):
    a = torch.ones(64, device="cuda")
    awq.alpha_scales(a, torch.tensor([0.5, 1.5], device="cuda"))
    with pytest.raises(awq.AWQError) as e:
        awq.get_status()
    assert e.value.code == 1
    awq.get_status()                             # the flag is cleared


def test_bounded_wait_reports_timeout_and_context_survives(awq):
    """A wait that can never complete ends by itself, is reported as
    AWQ_ERR_TIMEOUT, and the context still runs the search correctly."""
    awq.get_status()
    awq.set_wait_timeout_ms(100)
    try:
        awq.selftest_bounded_wait()
        with pytest.raises(awq.AWQError) as e:
            awq.get_status()
        assert e.value.code == 4                 # AWQ_ERR_TIMEOUT
        awq.get_status()                         # cleared
    finally:
        awq.set_wait_timeout_ms(2000)
    W, X = gen(128, 256, 300, seed=41)
    a = oracle.act_stats(X)
    alphas = synth.default_alphas()
    got = host(awq.search_layer(dev(W), dev(X), dev(a), dev(alphas), 4, 128))
    awq.get_status()
    np.testing.assert_allclose(got, oracle.search(W, X, a, 4, 128, alphas)["losses"], rtol=LOSS_RTOL)


# ---------------------------------------------------------------------------
# a3/a4: W_hat bit-exact for every alpha, and on degenerate groups
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("bits,group", [(4, 128), (3, 128), (2, 64), (4, 64), (2, 128)])
def test_quant_dequant_bit_exact(awq, bits, group):
    W, X = gen(96, 512, 64, bits=bits, group=group, seed=bits * 10 + group)
    W[0, :] = 0                                  # all-zero row
    W[1, :group] = np.float16(0.013)             # constant group
    W[2, :] = np.abs(W[2, :]) + np.float16(0.5)  # all-positive row: zero point clamps to 0
    W[3, :] = -np.abs(W[3, :]) - np.float16(0.5) # all-negative row: zero point clamps to qmax
    W[4, 5] = np.float16(60000.0)                # huge outlier weight
    a = oracle.act_stats(X)
    Wd = dev(W)
    for al in (0.0, 0.25, 0.5, 0.95):
        s = oracle.scales(a, al)
        got = host(awq.quant_dequant(Wd, dev(s), bits, group))
        ref = oracle.quantize(W, s, bits, group)["what"]
        assert np.array_equal(got.view(np.uint16), ref.view(np.uint16)), al


def test_quant_dequant_every_alpha_large(awq):
    """All 20 alphas on a 1024 x 1024 layer: about one element in four thousand
    has w'*r exactly on a half-integer, where a fused multiply-add (or any
    other rounding slip) would flip the code."""
    W, X = gen(1024, 1024, 256, seed=77)
    a = oracle.act_stats(X)
    Wd = dev(W)
    ties = 0
    for al in synth.default_alphas():
        s = oracle.scales(a, float(al))
        got = host(awq.quant_dequant(Wd, dev(s), 4, 128))
        ref = oracle.quantize(W, s, 4, 128)
        assert np.array_equal(got.view(np.uint16), ref["what"].view(np.uint16)), float(al)
        if float(al) == 0.0:
            sh = np.repeat(ref["sh"].astype(np.float32), 128, axis=1)
            t = (W.astype(np.float32) * (np.float32(1) / sh).astype(np.float32)).astype(np.float32)
            ties = int(np.sum(t - np.floor(t) == 0.5))
    assert ties > 0          # the case really exercises exact ties


# ---------------------------------------------------------------------------
# a2-a6: the search
# ---------------------------------------------------------------------------
SEARCH_CASES = [
    # N, K, T, bits, group, seed   (tiles of 128 rows x 512 tokens; ragged tails)
    (256, 512, 512, 4, 128, 0),
    (200, 256, 700, 4, 128, 1),
    (130, 384, 100, 3, 128, 2),
    (64, 192, 1030, 2, 64, 3),
    (1, 128, 1, 4, 128, 4),
    (384, 1024, 257, 4, 64, 5),
]


@pytest.mark.parametrize("N,K,T,bits,group,seed", SEARCH_CASES)
def test_search_losses(awq, N, K, T, bits, group, seed):
    W, X = gen(N, K, T, bits=bits, group=group, seed=seed, outlier_frac=0.02)
    alphas = synth.default_alphas()
    a = oracle.act_stats(X)
    losses, rows = awq.search_layer(dev(W), dev(X), dev(a), dev(alphas), bits, group, row_losses=True)
    awq.get_status()
    losses, rows = host(losses), host(rows)
    ref = oracle.search(W, X, a, bits, group, alphas)
    np.testing.assert_allclose(losses, ref["losses"], rtol=LOSS_RTOL, atol=0)
    np.testing.assert_allclose(rows, ref["row_sums"], rtol=LOSS_RTOL, atol=1e-12)
    assert_alpha_choice(oracle.argmin(losses.astype(np.float64)), ref["losses"])


def test_search_degenerate_groups(awq):
    """Rows whose groups need the code clamp (one-signed rows, a constant
    group, a huge weight), so the producer's clamp path runs."""
    W, X = gen(160, 512, 600, seed=12, outlier_frac=0.02)
    W[0, :] = 0
    W[1, :128] = np.float16(0.013)
    W[2, :] = np.abs(W[2, :]) + np.float16(0.5)
    W[3, :] = -np.abs(W[3, :]) - np.float16(0.5)
    W[4, 5] = np.float16(60000.0)
    W[130, :] = np.abs(W[130, :]) + np.float16(0.25)
    alphas = synth.default_alphas()
    a = oracle.act_stats(X)
    losses, rows = awq.search_layer(dev(W), dev(X), dev(a), dev(alphas), 4, 128, row_losses=True)
    awq.get_status()
    ref = oracle.search(W, X, a, 4, 128, alphas)
    np.testing.assert_allclose(host(losses), ref["losses"], rtol=LOSS_RTOL)
    np.testing.assert_allclose(host(rows), ref["row_sums"], rtol=LOSS_RTOL, atol=1e-12)


def test_search_with_strided_x_and_one_alpha(awq):
    W, X = gen(128, 256, 600, seed=9)
    Xpad = np.zeros((600, 264), dtype=np.float16)
    Xpad[:, :256] = X
    Xd = dev(Xpad)[:, :256]
    a = oracle.act_stats(X)
    alphas = np.array([0.5], dtype=np.float32)
    got = host(awq.search_layer(dev(W), Xd, dev(a), dev(alphas), 4, 128))
    ref = oracle.search(W, X, a, 4, 128, alphas)["losses"]
    np.testing.assert_allclose(got, ref, rtol=LOSS_RTOL)


def test_search_repeatable_and_workspace_reuse(awq):
    W, X = gen(256, 512, 512, seed=10)
    alphas = dev(synth.default_alphas())
    Wd, Xd = dev(W), dev(X)
    a = awq.act_stats(Xd)
    ws = torch.full((awq.search_workspace_bytes(256, 512, 512),), 0xFF, dtype=torch.uint8, device="cuda")
    l1 = host(awq.search_layer(Wd, Xd, a, alphas, workspace=ws))
    l2 = host(awq.search_layer(Wd, Xd, a, alphas, workspace=ws))
    assert np.array_equal(l1, l2)


# ---------------------------------------------------------------------------
# a7-a8: argmin + pack
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("N,K,bits,group", [(160, 512, 4, 128), (64, 256, 3, 128), (96, 256, 2, 64),
                                            (32, 128, 2, 128), (48, 192, 4, 64)])
def test_pack_bit_exact(awq, N, K, bits, group):
    W, X = gen(N, K, 64, bits=bits, group=group, seed=N + K)
    a = oracle.act_stats(X)
    alphas = synth.default_alphas()
    rng = np.random.default_rng(N)
    losses = rng.random(20).astype(np.float32)   # same losses on both sides
    losses[7] = np.nan
    res = awq.pack(dev(W), dev(a), dev(alphas), dev(losses), bits, group)
    ref = oracle.pack(W, a, bits, group, alphas, losses.astype(np.float64))
    assert int(host(res["best_idx"])[0]) == ref["best"]
    assert np.array_equal(host(res["s_best"]), ref["s_best"])
    assert np.array_equal(host(res["codes"]).view(np.uint32), ref["codes"])
    assert np.array_equal(host(res["scales"]).view(np.uint16), ref["scales"].view(np.uint16))
    assert np.array_equal(host(res["zeros"]).view(np.uint16), ref["zeros"].view(np.uint16))


# ---------------------------------------------------------------------------
# The whole path on the 512 x 512, T = 512 layer (oracle in full)
# ---------------------------------------------------------------------------
def test_whole_path_layer512(awq):
    cfg = synth.CONFIGS["layer512"]
    W, X, _ = synth.generate(cfg)
    alphas = synth.default_alphas()
    out = awq.quantize_layer(dev(W), dev(X), dev(alphas), cfg.bits, cfg.group)
    awq.get_status()
    a = oracle.act_stats(X)
    assert np.array_equal(host(out["a"]), a)
    ref = oracle.search(W, X, a, cfg.bits, cfg.group, alphas)
    losses = host(out["losses"])
    np.testing.assert_allclose(losses, ref["losses"], rtol=LOSS_RTOL)
    best = int(host(out["best_idx"])[0])
    assert_alpha_choice(best, ref["losses"])
    pk = oracle.pack(W, a, cfg.bits, cfg.group, alphas, losses.astype(np.float64))
    assert pk["best"] == best
    assert np.array_equal(host(out["codes"]).view(np.uint32), pk["codes"])
    assert np.array_equal(host(out["scales"]).view(np.uint16), pk["scales"].view(np.uint16))
    assert np.array_equal(host(out["zeros"]).view(np.uint16), pk["zeros"].view(np.uint16))
    # final layer output error from the unpacked codes
    q = unpack_codes(host(out["codes"]), cfg.N, cfg.K, cfg.bits)
    what = dequantize(q, host(out["scales"]), host(out["zeros"]), host(out["s_best"]), cfg.group)
    err = oracle.output_error_sum(W, what, X).sum() / (cfg.N * cfg.T)
    assert err == pytest.approx(ref["losses"][best], rel=LOSS_RTOL)
    assert ref["losses"][best] < ref["losses"][0]          # better than plain RTN


# ---------------------------------------------------------------------------
# Layers sharing one input: one s for all, loss = sum of their output errors
# ---------------------------------------------------------------------------
def test_shared_input_joint_search(awq):
    K, T = 256, 600
    W1, X = gen(200, K, T, seed=51, outlier_frac=0.03)
    W2, _ = gen(136, K, T, seed=52, outlier_frac=0.03)
    alphas = synth.default_alphas()
    res = awq.quantize_shared_input([dev(W1), dev(W2)], dev(X), dev(alphas), 4, 128)
    awq.get_status()
    a = oracle.act_stats(X)
    Wst = np.concatenate([W1, W2], axis=0)
    ref = oracle.search(Wst, X, a, 4, 128, alphas)
    joint = host(res[0]["losses"]).astype(np.float64)
    np.testing.assert_allclose(joint, ref["losses"], rtol=LOSS_RTOL)
    # the joint loss is the row-weighted mean of the layers' own losses
    l1 = oracle.search(W1, X, a, 4, 128, alphas)["losses"]
    l2 = oracle.search(W2, X, a, 4, 128, alphas)["losses"]
    np.testing.assert_allclose(ref["losses"], (200 * l1 + 136 * l2) / 336, rtol=1e-12)
    best = int(host(res[0]["best_idx"])[0])
    assert_alpha_choice(best, ref["losses"])
    pk = oracle.pack(Wst, a, 4, 128, alphas, joint)
    assert pk["best"] == best
    codes = np.concatenate([host(r["codes"]) for r in res]).view(np.uint32)
    assert np.array_equal(codes, pk["codes"])
    assert np.array_equal(np.concatenate([host(r["scales"]) for r in res]).view(np.uint16),
                          pk["scales"].view(np.uint16))
    assert np.array_equal(host(res[1]["zeros"]).view(np.uint16), pk["zeros"][200:].view(np.uint16))


# ---------------------------------------------------------------------------
# The quantized linear layer (consumer of the packed format)
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("N,K,T,bits,group", [(1000, 1024, 1, 4, 128), (256, 512, 3, 3, 128),
                                              (300, 512, 4, 2, 64), (64, 4096, 7, 4, 128),
                                              (136, 640, 2, 2, 128), (520, 256, 9, 4, 64),
                                              (4096, 3072, 1, 4, 128), (2048, 8192, 2, 4, 128),
                                              (1000, 4096, 3, 2, 64)])
def test_qlinear(awq, N, K, T, bits, group):
    W, X = gen(N, K, T, bits=bits, group=group, seed=N + T, outlier_frac=0.02)
    a = oracle.act_stats(X)
    alphas = synth.default_alphas()
    losses = np.linspace(1.0, 0.5, 20).astype(np.float32)      # chooses alpha = 0.95
    pk = oracle.pack(W, a, bits, group, alphas, losses.astype(np.float64))
    Y = host(awq.qlinear(dev(pk["codes"].view(np.int32)), dev(pk["scales"]), dev(pk["zeros"]), dev(pk["s_best"]),
                         dev(X), bits, group))
    awq.get_status()
    ref = oracle.qlinear(pk["codes"], pk["scales"], pk["zeros"], pk["s_best"], X, bits, group)
    # binary32 accumulation: bound by the sum of |terms|
    q = oracle.unpack_codes(pk["codes"], K, bits).astype(np.float64)
    Gi = np.arange(K) // group
    wq = np.abs((q - pk["zeros"].astype(np.float64)[:, Gi]) * pk["scales"].astype(np.float64)[:, Gi])
    xs = np.abs(X.astype(np.float32) * (np.float32(1) / pk["s_best"]).astype(np.float32)).astype(np.float64)
    bound = xs @ wq.T
    assert np.all(np.abs(Y - ref) <= 2e-6 * bound + 1e-30)
    # row blocks split across thread blocks are summed in a fixed order
    Y2 = host(awq.qlinear(dev(pk["codes"].view(np.int32)), dev(pk["scales"]), dev(pk["zeros"]),
                          dev(pk["s_best"]), dev(X), bits, group))
    assert np.array_equal(Y, Y2)
