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


def plant_groups(W, group):
    """Rows whose groups exercise every branch of the zero point and the code
    clamp: an all-zero row, a constant group near zero, one-signed rows (zero
    points below 0 and above qmax), a group far from zero (|zero| > 2048, not
    every integer an fp16 value), a constant group far from zero (the fp16
    zero saturates at 65504), and a huge single weight."""
    plants = [
        lambda r: r.fill(0),
        lambda r: r.__setitem__(slice(0, group), np.float16(0.013)),
        lambda r: r.__setitem__(slice(None), np.abs(r) + np.float16(0.5)),
        lambda r: r.__setitem__(slice(None), -np.abs(r) - np.float16(0.5)),
        lambda r: r.__setitem__(5, np.float16(60000.0)),
        lambda r: r.__setitem__(slice(0, group), np.float16(128.0) + np.abs(r[:group]) * np.float16(8.0)),
        lambda r: r.__setitem__(slice(group, 2 * group), np.float16(3.0)),
    ]
    for n, plant in enumerate(plants[:W.shape[0]]):
        plant(W[n])
    return W


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
    plant_groups(W, group)
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
    """Rows whose groups need the code clamp or have zero points outside
    [0, qmax] (one-signed rows, constant groups, a group far from zero, a huge
    weight), so the producer's clamp path runs."""
    W, X = gen(160, 512, 600, seed=12, outlier_frac=0.02)
    plant_groups(W, 128)
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


@pytest.mark.parametrize("N,cut", [(600, 256), (1000, 768)])
def test_search_layer_part_sums_to_the_layer(awq, N, cut):
    """A layer split into two row parts (as across two GPUs): the parts'
    losses, normalised by the layer's row count, add up to the layer's losses,
    and packing each part with the summed losses gives the layer's codes,
    scales and zeros for those rows."""
    from awq_activation_aware_b200 import sharded
    W, X = gen(N, 512, 700, seed=N + cut, outlier_frac=0.02)
    a = oracle.act_stats(X)
    alphas = synth.default_alphas()
    Ad, Xd = dev(a), dev(X)
    whole = host(awq.search_layer(dev(W), Xd, Ad, dev(alphas), 4, 128))
    parts = [np.ascontiguousarray(W[:cut]), np.ascontiguousarray(W[cut:])]
    summed = sum(host(awq.search_layer(dev(Wp), Xd, Ad, dev(alphas), 4, 128, rows_total=N)).astype(np.float64)
                 for Wp in parts)
    awq.get_status()
    np.testing.assert_allclose(summed, whole, rtol=1e-5)
    np.testing.assert_allclose(summed, oracle.search(W, X, a, 4, 128, alphas)["losses"], rtol=LOSS_RTOL)
    ref = awq.pack(dev(W), Ad, dev(alphas), dev(summed.astype(np.float32)), 4, 128)
    got = [awq.pack(dev(Wp), Ad, dev(alphas), dev(summed.astype(np.float32)), 4, 128) for Wp in parts]
    for k in ("codes", "scales", "zeros"):
        assert np.array_equal(np.concatenate([host(g[k]) for g in got]), host(ref[k])), k
    assert sharded.shard_rows(N, 2, 0)[1] % sharded.ROW_UNIT == 0


# ---------------------------------------------------------------------------
# a7-a8: argmin + pack
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("N,K,bits,group", [(160, 512, 4, 128), (64, 256, 3, 128), (96, 256, 2, 64),
                                            (32, 128, 2, 128), (48, 192, 4, 64)])
def test_pack_bit_exact(awq, N, K, bits, group):
    W, X = gen(N, K, 64, bits=bits, group=group, seed=N + K)
    plant_groups(W, group)
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
                                              (1000, 4096, 3, 2, 64),
                                              # 5 to 20 tokens (several passes), G a multiple of 8 or not,
                                              # K not a multiple of 256
                                              (4096, 3072, 5, 4, 128), (2048, 8192, 6, 4, 128),
                                              (3000, 4352, 12, 3, 64), (136, 640, 4, 4, 128),
                                              (200, 384, 3, 3, 64),
                                              (1536, 2048, 16, 4, 128), (700, 1280, 20, 4, 64)])
@pytest.mark.parametrize("tc", [False, True, None], ids=["cuda_cores", "tensor_cores", "dispatch"])
def test_qlinear(awq, N, K, T, bits, group, tc):
    W, X = gen(N, K, T, bits=bits, group=group, seed=N + T, outlier_frac=0.02)
    plant_groups(W, group)
    a = oracle.act_stats(X)
    alphas = synth.default_alphas()
    losses = np.linspace(1.0, 0.5, 20).astype(np.float32)      # chooses alpha = 0.95
    pk = oracle.pack(W, a, bits, group, alphas, losses.astype(np.float64))
    Y = host(awq.qlinear(dev(pk["codes"].view(np.int32)), dev(pk["scales"]), dev(pk["zeros"]), dev(pk["s_best"]),
                         dev(X), bits, group, tensor_cores=tc))
    awq.get_status()
    ref = oracle.qlinear(pk["codes"], pk["scales"], pk["zeros"], pk["s_best"], X, bits, group)
    # binary32 accumulation: bound by the sum of |terms|
    q = oracle.unpack_codes(pk["codes"], K, bits).astype(np.float64)
    Gi = np.arange(K) // group
    wq = np.abs((q - pk["zeros"].astype(np.float64)[:, Gi]) * pk["scales"].astype(np.float64)[:, Gi])
    xs = np.abs(X.astype(np.float32) * (np.float32(1) / pk["s_best"]).astype(np.float32)).astype(np.float64)
    bound = xs @ wq.T
    assert np.all(np.abs(Y - ref) <= 2e-6 * bound + 1e-30)
    # row blocks (and K chunks) split across thread blocks are summed in a fixed order
    Y2 = host(awq.qlinear(dev(pk["codes"].view(np.int32)), dev(pk["scales"]), dev(pk["zeros"]),
                          dev(pk["s_best"]), dev(X), bits, group, tensor_cores=tc))
    assert np.array_equal(Y, Y2)


@pytest.mark.gpu
@pytest.mark.parametrize("T", [1, 2, 4, 11, 16])
def test_qlinear_dispatch_runs_the_named_kernel(awq, T):
    # The two kernels sum in different orders, so their outputs differ in the
    # last bits; the dispatched result is bit-identical to the kernel that
    # awq_qlinear_path names and (on these inputs) differs from the other one.
    N, K, bits, group = 2048, 3072, 4, 128
    W, X = gen(N, K, T, bits=bits, group=group, seed=7 + T, outlier_frac=0.02)
    a = oracle.act_stats(X)
    alphas = synth.default_alphas()
    losses = np.linspace(1.0, 0.5, 20).astype(np.float64)
    pk = oracle.pack(W, a, bits, group, alphas, losses)
    args = (dev(pk["codes"].view(np.int32)), dev(pk["scales"]), dev(pk["zeros"]), dev(pk["s_best"]), dev(X), bits, group)
    y_auto = host(awq.qlinear(*args))
    y_cc = host(awq.qlinear(*args, tensor_cores=False))
    y_tc = host(awq.qlinear(*args, tensor_cores=True))
    awq.get_status()
    named, other = (y_tc, y_cc) if awq.qlinear_path(T) == "tensor_cores" else (y_cc, y_tc)
    assert np.array_equal(y_auto, named)
    assert not np.array_equal(y_auto, other)


# ---------------------------------------------------------------------------
# Quantizer variants and baselines: symmetric groups, channels held in fp16,
# caller-given scale vectors, top-k channel selection
# ---------------------------------------------------------------------------
def _mask(K, seed, group):
    rng = np.random.default_rng(seed)
    m = np.zeros(K, dtype=np.uint8)
    m[rng.choice(K, max(1, K // 60), replace=False)] = 1
    m[group:2 * group] = 1                            # one whole group held in fp16
    return m


@pytest.mark.parametrize("bits,group", [(4, 128), (3, 128), (2, 64), (4, 64)])
@pytest.mark.parametrize("sym", [False, True])
@pytest.mark.parametrize("masked", [False, True])
def test_quant_dequant_variants_bitexact(awq, bits, group, sym, masked):
    W, X = gen(300, 1024, 64, bits=bits, group=group, seed=81 + bits)
    a = oracle.act_stats(X)
    s = oracle.scales(a, 0.45)
    m = _mask(1024, bits, group) if masked else None
    ref = oracle.quantize(W, s, bits, group, zero_point=not sym, mask=m)["what"]
    got = host(awq.quant_dequant(dev(W), dev(s), bits, group, zero_point=not sym,
                                 mask=None if m is None else dev(m)))
    awq.get_status()
    assert np.array_equal(got.view(np.uint16), ref.view(np.uint16))


@pytest.mark.parametrize("N,K,T,bits,group,sym,masked", [
    (300, 1024, 700, 4, 128, False, True), (256, 512, 512, 4, 128, True, False),
    (520, 768, 300, 3, 64, True, True), (136, 640, 1030, 2, 128, False, False),
])
def test_search_scales_matches_oracle(awq, N, K, T, bits, group, sym, masked):
    W, X = gen(N, K, T, bits=bits, group=group, seed=N + K)
    a = oracle.act_stats(X)
    k = max(1, round(K / 100))
    m_act = oracle.topk_mask(a, k)
    table = np.stack([np.ones(K, np.float32), np.where(m_act == 1, 2.0, 1.0).astype(np.float32),
                      oracle.scales(a, 0.5)])
    m = _mask(K, N, group) if masked else None
    ref = oracle.search_scales(W, X, table, bits, group, zero_point=not sym, mask=m)
    losses, rows = awq.search_scales(dev(W), dev(X), dev(table), bits, group, zero_point=not sym,
                                     mask=None if m is None else dev(m), row_losses=True)
    awq.get_status()
    np.testing.assert_allclose(host(losses).astype(np.float64), ref["losses"], rtol=LOSS_RTOL)
    np.testing.assert_allclose(host(rows).astype(np.float64), ref["row_sums"], rtol=LOSS_RTOL, atol=1e-30)


def test_search_scales_equals_grid_search(awq):
    """The grid's own s vectors, passed as a table, give the grid's losses bit for bit."""
    W, X = gen(256, 512, 512, seed=91)
    Wd, Xd = dev(W), dev(X)
    a = awq.act_stats(Xd)
    al = awq.default_alphas()
    grid = awq.search_layer(Wd, Xd, a, al)
    table = awq.alpha_scales(a, al)
    given = awq.search_scales(Wd, Xd, table)
    awq.get_status()
    assert torch.equal(grid, given)


@pytest.mark.parametrize("bits,group", [(4, 128), (3, 64), (2, 64)])
def test_symmetric_whole_path(awq, bits, group):
    """Grid search and packing with the symmetric quantizer against the oracle."""
    W, X = gen(320, 512, 600, bits=bits, group=group, seed=92 + bits)
    alphas = synth.default_alphas()
    res = awq.quantize_layer(dev(W), dev(X), bits=bits, group=group, zero_point=False)
    awq.get_status()
    a = oracle.act_stats(X)
    ref = oracle.search(W, X, a, bits, group, alphas, zero_point=False)
    np.testing.assert_allclose(host(res["losses"]).astype(np.float64), ref["losses"], rtol=LOSS_RTOL)
    best = int(host(res["best_idx"])[0])
    assert_alpha_choice(best, ref["losses"])
    losses_used = ref["losses"].copy()
    losses_used[best] = -1.0                           # pack what the GPU chose
    pk = oracle.pack(W, a, bits, group, alphas, losses_used, zero_point=False)
    assert np.array_equal(host(res["codes"]).view(np.uint32), pk["codes"])
    assert np.array_equal(host(res["scales"]).view(np.uint16), pk["scales"].view(np.uint16))
    assert np.all(host(res["zeros"]) == 2 ** (bits - 1))


@pytest.mark.parametrize("sym", [False, True])
def test_pack_scales_bitexact(awq, sym):
    W, X = gen(200, 768, 8, bits=3, group=128, seed=93)
    s = np.where(oracle.topk_mask(oracle.act_stats(X), 8) == 1, 2.0, 1.0).astype(np.float32)
    out = awq.pack_scales(dev(W), dev(s), 3, 128, zero_point=not sym)
    awq.get_status()
    pk = oracle.pack_scales(W, s, 3, 128, zero_point=not sym)
    assert np.array_equal(host(out["codes"]).view(np.uint32), pk["codes"])
    assert np.array_equal(host(out["scales"]).view(np.uint16), pk["scales"].view(np.uint16))
    assert np.array_equal(host(out["zeros"]).view(np.uint16), pk["zeros"].view(np.uint16))


@pytest.mark.parametrize("K,k", [(1, 1), (300, 0), (300, 3), (4096, 41), (11008, 110), (5000, 5000)])
def test_channel_topk_bitexact(awq, K, k):
    rng = np.random.default_rng(K + k)
    v = rng.integers(0, 50, K).astype(np.float32)          # many ties
    if K > 10:
        v[[1, K // 2, K - 1]] = np.nan
    got = host(awq.channel_topk(dev(v), k))
    awq.get_status()
    assert np.array_equal(got, oracle.topk_mask(v, k))
    assert int(got.sum()) == k


def test_salient_scales(awq):
    m = (np.arange(1000) % 7 == 0).astype(np.uint8)
    s = host(awq.salient_scales(dev(m), 2.0))
    assert np.array_equal(s, np.where(m == 1, 2.0, 1.0).astype(np.float32))


def test_bad_given_scale_is_reported(awq):
    W, X = gen(256, 256, 64, seed=94)
    table = np.ones((2, 256), np.float32)
    table[1, 17] = 0.0
    awq.search_scales(dev(W), dev(X), dev(table))
    with pytest.raises(awq.AWQError):
        awq.get_status()
    awq.get_status()                                   # the flag is cleared


def test_baselines_match_oracle_and_premise(awq):
    """The pages' comparisons on a synthetic layer with 1% outlier channels:
    fp16 protection by activation << RTN, by weight magnitude ~ RTN, and
    AWQ's searched s better than the fixed 2x; each loss against the oracle."""
    cfg = synth.make_config(512, 1024, 1024, seed=95)
    W, X, idx = synth.generate(cfg)
    r = awq.baselines(dev(W), dev(X), 4, 128)
    awq.get_status()
    a = oracle.act_stats(X)
    m_act = oracle.topk_mask(a, r["k"])
    m_w = oracle.topk_mask(oracle.act_stats(W), r["k"])
    assert np.array_equal(host(r["mask_act"]), m_act) and np.array_equal(host(r["mask_weight"]), m_w)
    one = np.ones((1, cfg.K), np.float32)
    ref = dict(rtn=oracle.search_scales(W, X, one, 4, 128)["losses"][0],
               fixed_2x=oracle.search_scales(W, X, np.where(m_act == 1, 2.0, 1.0)[None].astype(np.float32),
                                             4, 128)["losses"][0],
               fp16_act=oracle.search_scales(W, X, one, 4, 128, mask=m_act)["losses"][0],
               fp16_weight=oracle.search_scales(W, X, one, 4, 128, mask=m_w)["losses"][0])
    for key, v in ref.items():
        assert float(host(r[key])) == pytest.approx(v, rel=LOSS_RTOL), key
    awq_best = float(host(r["awq_grid"]).min())
    assert ref["fp16_act"] < 0.1 * ref["rtn"]
    assert ref["fp16_weight"] > 0.9 * ref["rtn"]
    assert awq_best < ref["fixed_2x"] < 0.5 * ref["rtn"]


def test_qlinear_on_symmetric_pack(awq):
    """The decode path reads symmetric packs unchanged (the zero is stored)."""
    W, X = gen(700, 1024, 3, bits=4, group=128, seed=96, outlier_frac=0.02)
    a = oracle.act_stats(X)
    pk = oracle.pack(W, a, 4, 128, synth.default_alphas(), np.linspace(1.0, 0.5, 20), zero_point=False)
    Y = host(awq.qlinear(dev(pk["codes"].view(np.int32)), dev(pk["scales"]), dev(pk["zeros"]),
                         dev(pk["s_best"]), dev(X), 4, 128))
    awq.get_status()
    ref = oracle.qlinear(pk["codes"], pk["scales"], pk["zeros"], pk["s_best"], X, 4, 128)
    np.testing.assert_allclose(Y, ref, rtol=1e-4, atol=1e-4 * np.abs(ref).max())


def test_binding_rejects_non_contiguous_arrays(awq):
    """Every array but X is read densely packed: a strided view is refused on
    the host before anything is launched; X may have strided rows."""
    W, X = gen(256, 256, 64, seed=141)
    Xd = dev(X)
    a = awq.act_stats(Xd)
    al = dev(synth.default_alphas())
    a_strided = torch.stack([a, a], dim=1)[:, 0]                   # stride 2
    assert not a_strided.is_contiguous()
    with pytest.raises(ValueError):
        awq.alpha_scales(a_strided, al)
    with pytest.raises(ValueError):
        awq.alpha_scales(a, torch.stack([al, al], dim=1)[:, 0])
    W_strided = dev(np.concatenate([W, W], axis=1))[:, :256]       # rows 512 apart
    with pytest.raises(ValueError):
        awq.search_layer(W_strided, Xd, a, al)
    X_strided = dev(np.concatenate([X, X], axis=1))[:, :256]       # strided rows: accepted
    assert torch.equal(awq.act_stats(X_strided), a)
    awq.get_status()


def test_saved_layer_reloads_for_decode(awq, tmp_path):
    """A layer quantized on the GPU, saved and loaded back ([QAS-QA] §9:
    save_quantized, then inference from the 4-bit model): the reloaded tensors
    are bit-identical, and the decode from them gives the same Y."""
    from awq_activation_aware_b200 import persist
    W, X = gen(384, 512, 96, seed=131)
    al = dev(synth.default_alphas())
    res = awq.quantize_layer(dev(W), dev(X), al, 4, 128)
    awq.get_status()
    p = tmp_path / "layer.pt"
    persist.save_quantized(p, res, 4, 128, alphas=al)
    back = persist.load_quantized(p, device="cuda")
    for k in ("codes", "scales", "zeros", "s_best", "best_idx", "losses", "a"):
        assert torch.equal(back[k].view(torch.uint8), res[k].view(torch.uint8)), k
    Xt = dev(X[:4])
    Y0 = awq.qlinear(res["codes"], res["scales"], res["zeros"], res["s_best"], Xt, 4, 128)
    Y1 = awq.qlinear(back["codes"], back["scales"], back["zeros"], back["s_best"], Xt,
                     back["bits"], back["group_size"])
    awq.get_status()
    assert torch.equal(Y0, Y1)


# ---------------------------------------------------------------------------
# AWQ followed by GPTQ error compensation
# ---------------------------------------------------------------------------
def test_output_error_equals_the_search_loss(awq):
    """The loss of a given W_hat through the search kernel: for W_hat from the
    quantizer at s, the same number as the search at s (the same Delta W up to
    sign, contracted in the same order), and the oracle's within 1e-3."""
    W, X = gen(300, 512, 700, seed=111)
    a = oracle.act_stats(X)
    s = oracle.scales(a, 0.5)
    Wd, Xd = dev(W), dev(X)
    What = awq.quant_dequant(Wd, dev(s))
    loss, rows = awq.output_error(Wd, What, Xd, row_losses=True)
    grid, grows = awq.search_scales(Wd, Xd, dev(s[None]), row_losses=True)
    awq.get_status()
    assert float(loss) == float(grid[0])
    assert torch.equal(rows, grows[0])
    ref = oracle.output_error(W, host(What), X)
    assert float(loss) == pytest.approx(ref["loss"], rel=LOSS_RTOL)
    np.testing.assert_allclose(host(rows).astype(np.float64), ref["row_sums"], rtol=LOSS_RTOL)


@pytest.mark.parametrize("T,K", [(512, 256), (700, 512), (64, 1024), (129, 320), (4096, 384)])
@pytest.mark.parametrize("tc", [False, True], ids=["cuda_cores", "tensor_cores"])
def test_gptq_hessian_matches_oracle(awq, T, K, tc):
    """binary32 accumulation (in token order on the CUDA cores, of exact piece
    products on the tensor cores) against the binary64 product:
    |H - H_oracle| <= T 2^-24 (2 |X'|^T |X'|) (the standard summation bound)."""
    W, X = gen(8, K, T, seed=112)
    s = oracle.scales(oracle.act_stats(X), 0.4)
    H = host(awq.gptq_hessian(dev(X), dev(s), tensor_cores=tc)).astype(np.float64)
    awq.get_status()
    ref = oracle.gptq_hessian(X, s)
    rs = (np.float32(1.0) / s).astype(np.float32)
    Xa = np.abs((X.astype(np.float32) * rs[None]).astype(np.float32)).astype(np.float64)
    bound = T * 2.0 ** -24 * 2.0 * (Xa.T @ Xa)
    assert np.all(np.abs(H - ref) <= bound)
    assert np.array_equal(H, H.T)


@pytest.mark.parametrize("K", [128, 512, 1024])
def test_gptq_factor_matches_oracle(awq, K):
    """U from the same binary32 H: U^T U inverts the damped H, and U agrees
    with the oracle's binary64 factor to the accuracy binary32 Cholesky
    allows for this conditioning (relative Frobenius error <= 64 K 2^-24 cond)."""
    W, X = gen(8, K, 2 * K, seed=113)
    H32 = oracle.gptq_hessian(X, np.ones(K, np.float32)).astype(np.float32)
    U = host(awq.gptq_factor(dev(H32), 0.01)).astype(np.float64)
    awq.get_status()
    H = H32.astype(np.float64)
    Hd = H + np.float32(0.01 * np.float32(np.mean(np.diag(H)))) * np.eye(K)
    ref = oracle.gptq_factor(H, 0.01)
    assert np.count_nonzero(np.tril(U, -1)) == 0
    cond = np.linalg.cond(Hd)
    err = np.linalg.norm(U - ref) / np.linalg.norm(ref)
    assert err <= 64 * K * 2.0 ** -24 * cond, (err, cond)
    resid = np.abs(U.T @ U @ Hd - np.eye(K)).max()
    assert resid <= 64 * K * 2.0 ** -24 * cond, (resid, cond)


@pytest.mark.parametrize("N,K,bits,group,sym", [(300, 512, 4, 128, False), (136, 1024, 2, 64, False),
                                                (257, 768, 3, 128, True), (64, 256, 2, 64, True),
                                                (12, 4096, 4, 128, False), (5, 8192, 2, 64, True)])
def test_gptq_sweep_bitexact(awq, N, K, bits, group, sym):
    """The sweep against the oracle's, both fed the oracle's binary32 U: codes,
    scales, zeros and W_hat bit for bit (K = 4096 and 8192 take the 2-column
    batches, whose first column is not on a 16-byte boundary every time)."""
    W, X = gen(N, K, min(2 * K, 1024), bits=bits, group=group, seed=N + K + 114)
    plant_groups(W, group)
    a = oracle.act_stats(X)
    s = oracle.scales(a, 0.5)
    U32 = oracle.gptq_factor(oracle.gptq_hessian(X, s)).astype(np.float32)
    out = awq.gptq_quantize(dev(W), dev(s), dev(U32), bits, group, zero_point=not sym)
    awq.get_status()
    ref = oracle.gptq(W, s, U32, bits, group, zero_point=not sym)
    assert np.array_equal(host(out["codes"]).view(np.uint32), oracle.pack_codes(ref["q"], bits))
    assert np.array_equal(host(out["scales"]).view(np.uint16), ref["sh"].view(np.uint16))
    assert np.array_equal(host(out["zeros"]).astype(np.float32), ref["z"])
    assert np.array_equal(host(out["W_hat"]).view(np.uint16), ref["what"].view(np.uint16))


@pytest.mark.parametrize("bits,group", [(2, 64), (3, 128)])
def test_awq_gptq_whole_path(awq, bits, group):
    """AWQ's search, then GPTQ on the scaled layer, all on the GPU: the result
    beats AWQ alone (the pages' premise), and its loss is the oracle's for the
    GPU's own W_hat; the oracle's end-to-end run lands within 5% (its Hessian
    and factor are binary64, so a few codes may differ)."""
    cfg = synth.make_config(256, 512, 512, bits=bits, group=group, seed=11)
    W, X, _ = synth.generate(cfg)
    r = awq.awq_gptq(dev(W), dev(X), bits, group)
    awq.get_status()
    loss = float(r["loss"])
    assert loss < float(host(r["awq_losses"]).min())
    assert loss == pytest.approx(oracle.output_error(W, host(r["W_hat"]), X)["loss"], rel=LOSS_RTOL)
    s_best = host(r["s_best"])
    ref = oracle.gptq(W, s_best, oracle.gptq_factor(oracle.gptq_hessian(X, s_best)), bits, group)
    assert loss == pytest.approx(oracle.output_error(W, ref["what"], X)["loss"], rel=0.05)
