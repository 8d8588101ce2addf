"""The allocation-free search entry point, awq_search_layer_noalloc.

Some callers cannot allocate device memory when they run the search (plugin
code inside another runtime's execution step, programs that reserved their
whole memory budget up front, latency-critical paths); this entry point uses a
scratch array built into the library instead of a caller workspace.  Its
results must match awq_search_layer's, call after call, although the shared
array keeps whatever the previous call left in it.

This file is collected last on purpose, and it also passes when run alone in
a fresh process.
"""
import ctypes

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

RTOL = 1e-3          # the loss tolerance used by every search test


def _noalloc_fn():
    import awq_activation_aware_b200 as awq
    fn = awq.lib().awq_search_layer_noalloc
    P, i64 = ctypes.c_void_p, ctypes.c_int64
    fn.argtypes = [P, i64, i64, P, i64, i64, P, awq.QCfg, P, ctypes.c_int32, P, P, P]
    fn.restype = ctypes.c_int
    return fn


def _p(t):
    return ctypes.c_void_p(t.data_ptr())


@pytest.fixture(scope="module")
def awq():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import awq_activation_aware_b200 as m
    m.set_wait_timeout_ms(2000)
    return m


def _layer(seed, N, K, T):
    from awq_activation_aware_b200 import synth
    W, X, _ = synth.generate(synth.make_config(N, K, T, bits=4, group=128, seed=seed, outlier_frac=0.02))
    return torch.from_numpy(W).cuda(), torch.from_numpy(X).cuda()


def test_noalloc_matches_workspace_entry_point(awq):
    fn = _noalloc_fn()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    alphas = awq.default_alphas()
    # two different layers, each searched twice in a row through the static scratch
    for seed, (N, K, T) in ((31, (300, 512, 700)), (32, (128, 256, 1100))):
        W, X = _layer(seed, N, K, T)
        a = awq.act_stats(X)
        ref, ref_rows = awq.search_layer(W, X, a, alphas, 4, 128, row_losses=True)
        ref, ref_rows = ref.cpu().numpy(), ref_rows.cpu().numpy()
        for _ in range(2):
            losses = torch.full((alphas.numel(),), float("nan"), device="cuda")
            rows = torch.full((alphas.numel(), N), float("nan"), device="cuda")
            rc = fn(_p(W), N, K, _p(X), T, X.stride(0), _p(a), awq.QCfg(4, 128, 1), _p(alphas),
                    alphas.numel(), _p(losses), _p(rows), stream)
            assert rc == 0, awq.STATUS.get(rc, rc)
            awq.get_status()
            np.testing.assert_allclose(losses.cpu().numpy(), ref, rtol=RTOL, atol=0)
            np.testing.assert_allclose(rows.cpu().numpy(), ref_rows, rtol=RTOL, atol=1e-12)


def test_noalloc_rejects_layers_beyond_its_scratch(awq):
    fn = _noalloc_fn()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    N, K, T = 8192, 8192, 4096          # needs ~88 MiB of scratch, more than the 32 MiB built in
    assert awq.search_workspace_bytes(N, K, T, 4, 128, 20) > 32 << 20
    dummy = torch.empty(64, dtype=torch.float32, device="cuda")
    rc = fn(_p(dummy), N, K, _p(dummy), T, K, _p(dummy), awq.QCfg(4, 128, 1), _p(dummy), 20,
            _p(dummy), None, stream)
    assert rc == 5                      # AWQ_ERR_WORKSPACE, nothing launched
    awq.get_status()
