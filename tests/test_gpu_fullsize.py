"""Parity at the benchmark's full layer sizes, in the launch configuration
bench.py times (the whole path: statistics -> search -> pack).

The oracle cannot score every row of a 4096 x 4096 (or 28672 x 8192) layer in
test time, so it scores a seeded sample of rows -- first, last, middle, the
last row block, and random ones -- and the GPU's per-row loss sums for those
rows are compared (relative 1e-3), together with their codes, scales and zeros
(bit-exact), the full statistics vector and s at the chosen alpha (bit-exact).
Properties that hold at any size are checked on every row: the per-alpha loss
equals the sum of the per-row sums over N*T, and every code is in range.
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
    m.set_wait_timeout_ms(4000)
    return m


def sample_rows(N, seed, extra=8):
    rng = np.random.default_rng(seed)
    rows = {0, 1, N // 2, N - 1, max(0, (N // 256) * 256 - 1), min(N - 1, (N // 256) * 256)}
    rows |= set(int(r) for r in rng.choice(N, extra, replace=False))
    return np.array(sorted(rows))


def unpack_codes(codes, bits):
    c = 2 if bits == 2 else 4
    per = 32 // c
    words = codes.view(np.uint32).astype(np.uint64)
    q = np.empty((words.shape[0], words.shape[1] * per), dtype=np.uint8)
    for i in range(per):
        q[:, i::per] = ((words >> (c * i)) & ((1 << c) - 1)).astype(np.uint8)
    return q


@pytest.mark.parametrize("name", ["attn4096", "attn4096_int3", "attn4096_int2", "mlp_gate11008",
                                  "mlp_gateup22016", "mlp_down4096", "mlp_up28672"])
def test_fullsize_layer(awq, name):
    cfg = synth.CONFIGS[name]
    W, X, _ = synth.generate(cfg)
    alphas = synth.default_alphas()
    Wd = torch.from_numpy(W).cuda()
    Xd = torch.from_numpy(X).cuda()
    al = torch.from_numpy(alphas).cuda()
    a = awq.act_stats(Xd)
    losses, row_sums = awq.search_layer(Wd, Xd, a, al, cfg.bits, cfg.group, row_losses=True)
    out = awq.pack(Wd, a, al, losses, cfg.bits, cfg.group)
    awq.get_status()
    a_h = a.cpu().numpy()
    losses_h = losses.cpu().numpy().astype(np.float64)
    row_sums_h = row_sums.cpu().numpy().astype(np.float64)

    # statistics over all of X, bit-exact
    assert np.array_equal(a_h, oracle.act_stats(X))
    # per-alpha loss = sum of per-row sums / (N T), on every row
    np.testing.assert_allclose(losses_h, row_sums_h.sum(axis=1) / (cfg.N * cfg.T), rtol=1e-5)
    # sampled rows against the oracle
    rows = sample_rows(cfg.N, cfg.seed)
    ref = oracle.search(W, X, a_h, cfg.bits, cfg.group, alphas, rows=rows)
    np.testing.assert_allclose(row_sums_h[:, rows], ref["row_sums"], rtol=LOSS_RTOL)
    # the chosen alpha and the packed output for the sampled rows
    best = int(out["best_idx"].cpu()[0])
    assert best == oracle.argmin(losses_h)
    pk = oracle.pack(W, a_h, cfg.bits, cfg.group, alphas, losses_h, rows=rows)
    assert pk["best"] == best
    assert np.array_equal(out["s_best"].cpu().numpy(), pk["s_best"])
    codes = out["codes"].cpu().numpy()
    assert np.array_equal(codes[rows].view(np.uint32), pk["codes"])
    assert np.array_equal(out["scales"].cpu().numpy()[rows].view(np.uint16), pk["scales"].view(np.uint16))
    assert np.array_equal(out["zeros"].cpu().numpy()[rows].view(np.uint16), pk["zeros"].view(np.uint16))
    # every code of every row is a valid code; every zero point is an integer in range
    qmax = (1 << cfg.bits) - 1
    assert unpack_codes(codes, cfg.bits).max() <= qmax
    z = out["zeros"].cpu().numpy().astype(np.float32)
    assert np.all((z >= 0) & (z <= qmax) & (z == np.round(z)))
    # the premise on LLM-shaped layers: the best alpha beats plain RTN
    assert losses_h[best] < losses_h[0]


_layers = {}


def layer(name):
    """The seeded layer of a benchmark config, generated once per test session."""
    if name not in _layers:
        _layers[name] = synth.generate(synth.CONFIGS[name])
    return _layers[name]


@pytest.mark.parametrize("name", ["attn4096", "mlp_up28672"])
@pytest.mark.parametrize("T", [1, 2, 4, 16])
@pytest.mark.parametrize("tc", [False, True], ids=["cuda_cores", "tensor_cores"])
def test_fullsize_qlinear(awq, name, T, tc):
    """The decode layer at the benchmark's sizes and decode token counts, on sampled
    rows.  The expected rows come from the oracle's own pack of those rows."""
    cfg = synth.CONFIGS[name]
    W, X, _ = layer(name)
    alphas = synth.default_alphas()
    losses = np.linspace(1.0, 0.5, len(alphas))                  # chooses the last alpha
    Wd = torch.from_numpy(W).cuda()
    a = awq.act_stats(torch.from_numpy(X).cuda())
    a_h = a.cpu().numpy()
    out = awq.pack(Wd, a, torch.from_numpy(alphas).cuda(), torch.from_numpy(losses.astype(np.float32)).cuda(),
                   cfg.bits, cfg.group)
    Xt = np.ascontiguousarray(X[:T])
    Y = awq.qlinear(out["codes"], out["scales"], out["zeros"], out["s_best"], torch.from_numpy(Xt).cuda(),
                    cfg.bits, cfg.group, tensor_cores=tc).cpu().numpy()
    awq.get_status()
    del Wd
    rows = sample_rows(cfg.N, cfg.seed + T)
    pk = oracle.pack(W, a_h, cfg.bits, cfg.group, alphas, losses, rows=rows)
    ref = oracle.qlinear(pk["codes"], pk["scales"], pk["zeros"], pk["s_best"], Xt, cfg.bits, cfg.group)
    # binary32 accumulation against the binary64 sum: bound by the sum of |terms|
    q = oracle.unpack_codes(pk["codes"], cfg.K, cfg.bits).astype(np.float64)
    gi = np.arange(cfg.K) // cfg.group
    wq = np.abs((q - pk["zeros"].astype(np.float64)[:, gi]) * pk["scales"].astype(np.float64)[:, gi])
    xs = np.abs(Xt.astype(np.float32) * (np.float32(1) / pk["s_best"]).astype(np.float32)).astype(np.float64)
    bound = xs @ wq.T
    assert Y.shape == (T, cfg.N)
    assert np.all(np.abs(Y[:, rows] - ref) <= 2e-6 * bound + 1e-30)
    assert np.all(np.isfinite(Y))


@pytest.mark.parametrize("name", ["attn4096", "mlp_up28672"])
@pytest.mark.parametrize("T", [4, 16])
def test_fullsize_tensor_core_decode_repeats(awq, name, T):
    """Twenty more calls of the tensor-core decode at full size give the first
    call's output bit for bit (its parity is checked by test_fullsize_qlinear):
    a race in the kernel's hand-offs would show as a changed element."""
    cfg = synth.CONFIGS[name]
    W, X, _ = layer(name)
    alphas = synth.default_alphas()
    losses = np.linspace(1.0, 0.5, len(alphas))
    Wd = torch.from_numpy(W).cuda()
    a = awq.act_stats(torch.from_numpy(X).cuda())
    out = awq.pack(Wd, a, torch.from_numpy(alphas).cuda(), torch.from_numpy(losses.astype(np.float32)).cuda(),
                   cfg.bits, cfg.group)
    del Wd
    Xt = torch.from_numpy(np.ascontiguousarray(X[:T])).cuda()
    first = awq.qlinear(out["codes"], out["scales"], out["zeros"], out["s_best"], Xt, cfg.bits, cfg.group,
                        tensor_cores=True).cpu().numpy()
    for _ in range(20):
        Y = awq.qlinear(out["codes"], out["scales"], out["zeros"], out["s_best"], Xt, cfg.bits, cfg.group,
                        tensor_cores=True).cpu().numpy()
        assert np.array_equal(Y, first)
    awq.get_status()
