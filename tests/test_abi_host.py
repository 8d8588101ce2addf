"""The C-ABI library on the host: it loads, exports every entry point that
include/awq.h declares, sizes its workspace, and rejects bad arguments before
touching the GPU (so these run without one)."""
import ctypes
import re
from pathlib import Path

import pytest

import awq_activation_aware_b200 as awq
from awq_activation_aware_b200 import QCfg

ROOT = Path(__file__).resolve().parents[1]

BOGUS = ctypes.c_void_p(0x10000)        # aligned, never dereferenced: validation fails first
MISALIGNED = ctypes.c_void_p(0x10008)


def declared_symbols():
    names = set()
    for h in (ROOT / "include").glob("*.h"):
        names |= set(re.findall(r"AWQ_API\s+[\w\s\*]+?\b(awq_\w+)\s*\(", h.read_text()))
    return names


def test_library_builds_and_loads():
    from awq_activation_aware_b200 import build
    build.build()
    assert awq.LIB_PATH.exists()
    assert awq.lib() is not None


def test_exports_every_declared_symbol():
    names = declared_symbols()
    assert names >= {"awq_act_stats", "awq_search_layer", "awq_pack"}
    L = awq.lib()
    for n in sorted(names):
        assert hasattr(L, n), n


def test_status_strings():
    L = awq.lib()
    for code, name in awq.STATUS.items():
        assert L.awq_status_string(code).decode() == name


def test_workspace_size():
    ws = awq.search_workspace_bytes(4096, 4096, 4096, 4, 128, 20)
    # s and 1/s tables, 8-byte group parameters, fp32 partials per 512-token block
    expect = 2 * 20 * 4096 * 4 + 20 * 32 * 4096 * 8 + 20 * 8 * 4096 * 4
    assert expect <= ws <= expect + 4 * 256
    assert awq.search_workspace_bytes(100, 100, 10, 4, 128, 20) == 0      # K not a multiple of g
    assert awq.search_workspace_bytes(64, 128, 10, 5, 128, 20) == 0       # bits 5 unsupported


def _search(**kw):
    args = dict(W=BOGUS, N=256, K=512, X=BOGUS, T=512, ldx=512, a=BOGUS, q=QCfg(4, 128, 1), alphas=BOGUS,
                n_alpha=20, losses=BOGUS, row_losses=None, ws=BOGUS, ws_bytes=1 << 40, stream=None)
    args.update(kw)
    return awq.lib().awq_search_layer(*args.values())


@pytest.mark.parametrize("bad", [
    dict(W=None), dict(X=None), dict(a=None), dict(alphas=None), dict(losses=None),
    dict(W=MISALIGNED), dict(row_losses=MISALIGNED),
    dict(N=0), dict(T=0), dict(K=100), dict(K=96), dict(ldx=500), dict(ldx=516),
    dict(q=QCfg(5, 128, 1)), dict(q=QCfg(4, 32, 1)), dict(q=QCfg(4, 128, 2)), dict(q=QCfg(4, 128, 1), K=192),
    dict(n_alpha=0), dict(n_alpha=65), dict(N=1 << 31),
])
def test_search_rejects_bad_arguments(bad):
    assert _search(**bad) == 1   # AWQ_ERR_INVALID_ARG


def test_search_rejects_small_workspace():
    assert _search(ws_bytes=1024) == 5               # AWQ_ERR_WORKSPACE
    assert _search(ws=None) == 5
    assert _search(ws=ctypes.c_void_p(0x10010)) == 5  # not 256-byte aligned


def test_other_entry_points_reject_bad_arguments():
    L = awq.lib()
    assert L.awq_act_stats(None, 16, 64, 64, BOGUS, None) == 1
    assert L.awq_act_stats(BOGUS, 16, 60, 64, BOGUS, None) == 1      # K % 8
    assert L.awq_act_stats(BOGUS, 0, 64, 64, BOGUS, None) == 1
    assert L.awq_alpha_scales(BOGUS, 64, BOGUS, 0, BOGUS, None) == 1
    assert L.awq_quant_dequant(BOGUS, 4, 100, BOGUS, QCfg(4, 128, 1), BOGUS, None) == 1
    assert L.awq_pack(BOGUS, 4, 128, BOGUS, QCfg(3, 64, 1), BOGUS, BOGUS, 20, BOGUS, BOGUS, MISALIGNED,
                      BOGUS, BOGUS, None) == 1
    assert L.awq_pack(BOGUS, 4, 128, BOGUS, QCfg(3, 64, 1), BOGUS, BOGUS, 99, BOGUS, BOGUS, BOGUS,
                      BOGUS, BOGUS, None) == 1


def test_binding_requires_cuda_tensors():
    import torch
    with pytest.raises(TypeError):
        awq.act_stats(torch.zeros((4, 64), dtype=torch.float16))


def _search_scales(**kw):
    args = dict(W=BOGUS, N=256, K=512, X=BOGUS, T=512, ldx=512, q=QCfg(4, 128, 0), s_table=BOGUS, n_s=2,
                mask=None, losses=BOGUS, row_losses=None, ws=BOGUS, ws_bytes=1 << 40, stream=None)
    args.update(kw)
    return awq.lib().awq_search_scales(*args.values())


@pytest.mark.parametrize("bad", [
    dict(W=None), dict(X=None), dict(s_table=None), dict(losses=None), dict(s_table=MISALIGNED),
    dict(mask=MISALIGNED), dict(n_s=0), dict(n_s=65), dict(K=96), dict(ldx=500), dict(q=QCfg(4, 128, 3)),
    dict(T=0),
])
def test_search_scales_rejects_bad_arguments(bad):
    assert _search_scales(**bad) == 1


def test_search_scales_workspace():
    L = awq.lib()
    q = QCfg(4, 128, 1)
    plain = L.awq_search_scales_workspace_bytes(4096, 4096, 4096, q, 3, 0)
    masked = L.awq_search_scales_workspace_bytes(4096, 4096, 4096, q, 3, 1)
    assert plain == L.awq_search_workspace_bytes(4096, 4096, 4096, q, 3)
    assert masked - plain == 2 * 4096 * 4096                # X with the kept channels zeroed
    small = L.awq_search_scales_workspace_bytes(256, 512, 512, QCfg(4, 128, 0), 2, 0)
    assert _search_scales(ws_bytes=small, mask=BOGUS) == 5  # a mask needs the larger workspace


def test_variant_entry_points_reject_bad_arguments():
    L = awq.lib()
    assert L.awq_quant_dequant_masked(BOGUS, 4, 128, BOGUS, QCfg(4, 128, 5), BOGUS, BOGUS, None) == 1
    assert L.awq_quant_dequant_masked(None, 4, 128, BOGUS, QCfg(4, 128, 0), BOGUS, BOGUS, None) == 1
    assert L.awq_channel_topk(BOGUS, 64, 65, BOGUS, None) == 1          # k > K
    assert L.awq_channel_topk(BOGUS, 64, -1, BOGUS, None) == 1
    assert L.awq_channel_topk(None, 64, 1, BOGUS, None) == 1
    assert L.awq_salient_scales(BOGUS, 64, ctypes.c_float(0.0), BOGUS, None) == 1
    assert L.awq_salient_scales(BOGUS, 64, ctypes.c_float(float("inf")), BOGUS, None) == 1
    assert L.awq_pack_scales(BOGUS, 4, 100, BOGUS, QCfg(4, 128, 0), BOGUS, BOGUS, BOGUS, None) == 1
    assert L.awq_pack_scales(BOGUS, 4, 128, BOGUS, QCfg(4, 128, 0), MISALIGNED, BOGUS, BOGUS, None) == 1


def test_gptq_entry_points_reject_bad_arguments():
    L = awq.lib()
    assert L.awq_gptq_hessian(BOGUS, 16, 96, 96, BOGUS, BOGUS, None) == 1           # K % 64
    assert L.awq_gptq_hessian(BOGUS, 16, 16384, 16384, BOGUS, BOGUS, None) == 1     # K > 8192
    assert L.awq_gptq_hessian(MISALIGNED, 16, 128, 128, BOGUS, BOGUS, None) == 1
    # the tensor-core form: pieces of x' as bf16 [3][K][T rounded up to 64]
    assert L.awq_gptq_hessian_workspace_bytes(100, 128) == 2 * 3 * 128 * 128
    assert L.awq_gptq_hessian_workspace_bytes(16, 96) == 0
    assert L.awq_gptq_hessian_workspace_bytes(16, 16384) == 0
    wh = L.awq_gptq_hessian_workspace_bytes(16, 128)
    assert L.awq_gptq_hessian_tc(BOGUS, 16, 96, 96, BOGUS, BOGUS, BOGUS, wh, None) == 1        # K % 64
    assert L.awq_gptq_hessian_tc(MISALIGNED, 16, 128, 128, BOGUS, BOGUS, BOGUS, wh, None) == 1
    assert L.awq_gptq_hessian_tc(BOGUS, 16, 128, 128, BOGUS, BOGUS, BOGUS, wh - 1, None) == 5   # workspace
    assert L.awq_gptq_hessian_tc(BOGUS, 16, 128, 128, BOGUS, BOGUS, MISALIGNED, wh, None) == 5  # ws alignment
    assert L.awq_gptq_factor_workspace_bytes(16384) == 0
    assert L.awq_gptq_factor_workspace_bytes(4096) >= 4 * 4096 * 4096
    ws = L.awq_gptq_factor_workspace_bytes(128)
    assert L.awq_gptq_factor(BOGUS, 128, ctypes.c_float(-1.0), BOGUS, BOGUS, ws, None) == 1
    assert L.awq_gptq_factor(BOGUS, 128, ctypes.c_float(0.01), BOGUS, BOGUS, ws - 1, None) == 5
    assert L.awq_gptq_quantize(BOGUS, 4, 192, BOGUS, BOGUS, QCfg(4, 128, 1), BOGUS, BOGUS, BOGUS, BOGUS, None) == 1
    assert L.awq_gptq_quantize(BOGUS, 4, 128, BOGUS, None, QCfg(4, 128, 1), BOGUS, BOGUS, BOGUS, BOGUS, None) == 1
    assert L.awq_output_error_workspace_bytes(10, 100, 10) == 0
    n = L.awq_output_error_workspace_bytes(256, 512, 512)
    assert L.awq_output_error(BOGUS, BOGUS, 256, 512, BOGUS, 512, 500, BOGUS, None, BOGUS, n, None) == 1   # ldx < K
    assert L.awq_output_error(BOGUS, BOGUS, 256, 512, BOGUS, 512, 512, BOGUS, None, BOGUS, n - 1, None) == 5


def test_qlinear_dispatch_query():
    # awq_qlinear runs the CUDA-core kernel for one token and the tensor-core
    # kernel from two tokens on (host logic, no GPU needed)
    assert awq.qlinear_path(1) == "cuda_cores"
    for T in (2, 3, 5, 16, 17, 4096):
        assert awq.qlinear_path(T) == "tensor_cores"


@pytest.mark.parametrize("fn", ["awq_qlinear", "awq_qlinear_cc", "awq_qlinear_tc"])
def test_qlinear_entry_points_reject_bad_arguments(fn):
    """Every decode entry point validates before touching the device."""
    L = awq.lib()
    f = getattr(L, fn)

    def call(**kw):
        a = dict(codes=BOGUS, scales=BOGUS, zeros=BOGUS, s_best=BOGUS, N=512, K=1024, q=QCfg(4, 128, 1),
                 X=BOGUS, T=4, ldx=1024, Y=BOGUS, ws=BOGUS, ws_bytes=1 << 40, stream=None)
        a.update(kw)
        return f(*a.values())

    bad_arg = [dict(codes=None), dict(scales=None), dict(zeros=None), dict(s_best=None), dict(X=None),
               dict(Y=None), dict(codes=MISALIGNED), dict(X=MISALIGNED), dict(Y=MISALIGNED),
               dict(N=0), dict(T=0), dict(K=1000), dict(K=32), dict(ldx=1000), dict(ldx=1028),
               dict(q=QCfg(5, 128, 1)), dict(q=QCfg(4, 96, 1)), dict(K=1024 + 64, q=QCfg(4, 128, 1))]
    for kw in bad_arg:
        assert call(**kw) == 1, kw                          # AWQ_ERR_INVALID_ARG
    need = awq.lib().awq_qlinear_workspace_bytes(4, 1024, 512)
    assert need > 0
    assert call(ws=None) == 5                               # AWQ_ERR_WORKSPACE
    assert call(ws_bytes=need - 1) == 5
    assert call(ws=ctypes.c_void_p(0x10010)) == 5           # not 256-byte aligned


def test_row_part_and_noalloc_entry_points_reject_bad_arguments():
    L = awq.lib()
    L.awq_search_layer_part.restype = ctypes.c_int
    P, i64, i32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32

    def part(**kw):
        a = dict(W=BOGUS, N=256, rows_total=512, K=512, X=BOGUS, T=512, ldx=512, a=BOGUS, q=QCfg(4, 128, 1),
                 alphas=BOGUS, n_alpha=20, losses=BOGUS, row_losses=None, ws=BOGUS, ws_bytes=1 << 40, stream=None)
        a.update(kw)
        return L.awq_search_layer_part(*a.values())

    for kw in (dict(rows_total=255), dict(rows_total=(1 << 31)), dict(W=None), dict(losses=None),
               dict(W=MISALIGNED), dict(row_losses=MISALIGNED), dict(K=500), dict(ldx=510),
               dict(n_alpha=0), dict(n_alpha=65), dict(q=QCfg(4, 64, 2))):
        assert part(**kw) == 1, kw
    assert part(ws=None) == 5
    assert part(ws_bytes=16) == 5

    f = L.awq_search_layer_noalloc
    f.argtypes = [P, i64, i64, P, i64, i64, P, QCfg, P, i32, P, P, P]
    f.restype = ctypes.c_int
    # no workspace size exists for these shapes: rejected before the device is touched
    assert f(BOGUS, 256, 500, BOGUS, 512, 512, BOGUS, QCfg(4, 128, 1), BOGUS, 20, BOGUS, None, None) == 1
    assert f(BOGUS, 256, 512, BOGUS, 512, 512, BOGUS, QCfg(4, 128, 1), BOGUS, 0, BOGUS, None, None) == 1
    # a layer whose workspace exceeds the built-in scratch
    assert awq.search_workspace_bytes(8192, 8192, 8192, 4, 128, 20) > 32 << 20
    assert f(BOGUS, 8192, 8192, BOGUS, 8192, 8192, BOGUS, QCfg(4, 128, 1), BOGUS, 20, BOGUS, None, None) == 5
