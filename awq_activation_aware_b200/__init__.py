"""B200-native AWQ per-layer scale search: Python binding of ``libawq.so``.

Every function here only marshals arguments (tensor pointers, sizes, the
current CUDA stream) into the C ABI declared in ``include/awq.h``; all of the
work runs in the library's sm_100a kernels.  There is no CPU fallback: if the
library is missing or the device is not a B200-class (sm_100) GPU, calls raise.

PyTorch is used for device memory and streams only.
"""
from __future__ import annotations

import ctypes
from pathlib import Path

import torch

__all__ = [
    "AWQError", "lib", "act_stats", "alpha_scales", "quant_dequant", "search_workspace_bytes",
    "search_layer", "pack", "quantize_layer", "get_status", "set_wait_timeout_ms", "default_alphas",
    "profile_next_search", "quantize_shared_input", "selftest_bounded_wait", "qlinear",
    "search_scales", "channel_topk", "pack_scales", "salient_scales", "baselines", "output_error",
    "gptq_hessian", "gptq_factor", "gptq_quantize", "gptq_layer", "awq_gptq", "LIB_PATH",
]

_PKG = Path(__file__).resolve().parent
LIB_PATH = _PKG / "libawq.so"

STATUS = {0: "AWQ_OK", 1: "AWQ_ERR_INVALID_ARG", 2: "AWQ_ERR_UNSUPPORTED", 3: "AWQ_ERR_CUDA",
          4: "AWQ_ERR_TIMEOUT", 5: "AWQ_ERR_WORKSPACE"}


class AWQError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = int(code)
        super().__init__(f"{where}: {STATUS.get(self.code, self.code)}")


class QCfg(ctypes.Structure):
    _fields_ = [("bits", ctypes.c_int32), ("group_size", ctypes.c_int32), ("zero_point", ctypes.c_int32)]


_lib = None


def lib():
    """The loaded C library (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not LIB_PATH.exists():
        raise RuntimeError(f"{LIB_PATH} is missing: build it with `python -m awq_activation_aware_b200.build`")
    L = ctypes.CDLL(str(LIB_PATH))
    P, i64, i32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32
    L.awq_act_stats.argtypes = [P, i64, i64, i64, P, P]
    L.awq_alpha_scales.argtypes = [P, i64, P, i32, P, P]
    L.awq_quant_dequant.argtypes = [P, i64, i64, P, QCfg, P, P]
    L.awq_quant_dequant_masked.argtypes = [P, i64, i64, P, QCfg, P, P, P]
    L.awq_search_scales_workspace_bytes.argtypes = [i64, i64, i64, QCfg, i32, i32]
    L.awq_search_scales_workspace_bytes.restype = ctypes.c_size_t
    L.awq_search_scales.argtypes = [P, i64, i64, P, i64, i64, QCfg, P, i32, P, P, P, P, ctypes.c_size_t, P]
    L.awq_channel_topk.argtypes = [P, i64, i64, P, P]
    L.awq_pack_scales.argtypes = [P, i64, i64, P, QCfg, P, P, P, P]
    L.awq_salient_scales.argtypes = [P, i64, ctypes.c_float, P, P]
    L.awq_output_error_workspace_bytes.argtypes = [i64, i64, i64]
    L.awq_output_error_workspace_bytes.restype = ctypes.c_size_t
    L.awq_output_error.argtypes = [P, P, i64, i64, P, i64, i64, P, P, P, ctypes.c_size_t, P]
    L.awq_gptq_hessian.argtypes = [P, i64, i64, i64, P, P, P]
    L.awq_gptq_hessian_workspace_bytes.argtypes = [i64, i64]
    L.awq_gptq_hessian_workspace_bytes.restype = ctypes.c_size_t
    L.awq_gptq_hessian_tc.argtypes = [P, i64, i64, i64, P, P, P, ctypes.c_size_t, P]
    L.awq_gptq_factor_workspace_bytes.argtypes = [i64]
    L.awq_gptq_factor_workspace_bytes.restype = ctypes.c_size_t
    L.awq_gptq_factor.argtypes = [P, i64, ctypes.c_float, P, P, ctypes.c_size_t, P]
    L.awq_gptq_quantize.argtypes = [P, i64, i64, P, P, QCfg, P, P, P, P, P]
    L.awq_search_workspace_bytes.argtypes = [i64, i64, i64, QCfg, i32]
    L.awq_search_workspace_bytes.restype = ctypes.c_size_t
    L.awq_search_layer.argtypes = [P, i64, i64, P, i64, i64, P, QCfg, P, i32, P, P, P, ctypes.c_size_t, P]
    L.awq_search_layer_part.argtypes = [P, i64, i64, i64, P, i64, i64, P, QCfg, P, i32, P, P, P, ctypes.c_size_t, P]
    L.awq_pack.argtypes = [P, i64, i64, P, QCfg, P, P, i32, P, P, P, P, P, P]
    L.awq_get_status.argtypes = [P]
    L.awq_set_wait_timeout_ms.argtypes = [ctypes.c_uint32]
    L.awq_set_wait_timeout_ms.restype = None
    L.awq_qlinear_workspace_bytes.argtypes = [i64, i64, i64]
    L.awq_qlinear_workspace_bytes.restype = ctypes.c_size_t
    L.awq_qlinear.argtypes = [P, P, P, P, i64, i64, QCfg, P, i64, i64, P, P, ctypes.c_size_t, P]
    L.awq_qlinear_tc.argtypes = [P, P, P, P, i64, i64, QCfg, P, i64, i64, P, P, ctypes.c_size_t, P]
    L.awq_qlinear_cc.argtypes = [P, P, P, P, i64, i64, QCfg, P, i64, i64, P, P, ctypes.c_size_t, P]
    L.awq_qlinear_path.argtypes = [i64]
    L.awq_qlinear_path.restype = ctypes.c_int32
    L.awq_qlinear.restype = ctypes.c_int
    L.awq_selftest_bounded_wait.argtypes = [P]
    L.awq_selftest_bounded_wait.restype = ctypes.c_int
    L.awq_profile_next_search.argtypes = [P, P]
    L.awq_profile_next_search.restype = None
    L.awq_status_string.argtypes = [ctypes.c_int]
    L.awq_status_string.restype = ctypes.c_char_p
    for fn in ("awq_act_stats", "awq_alpha_scales", "awq_quant_dequant", "awq_search_layer", "awq_pack",
               "awq_get_status", "awq_quant_dequant_masked", "awq_search_scales", "awq_channel_topk",
               "awq_pack_scales", "awq_salient_scales", "awq_output_error", "awq_gptq_hessian",
               "awq_gptq_hessian_tc", "awq_gptq_factor",
               "awq_gptq_quantize", "awq_qlinear_tc", "awq_qlinear_cc"):
        getattr(L, fn).restype = ctypes.c_int
    _lib = L
    return L


def _check(code: int, where: str):
    if code != 0:
        raise AWQError(code, where)


def _stream(stream=None):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _dev(t: torch.Tensor, dtype, name, row_strided: bool = False):
    """The device pointer of t.  The library reads every array densely packed,
    except X, whose rows may sit ldx elements apart (row_strided: the caller
    has checked the rows with _rowmajor and passes X.stride(0) as ldx)."""
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not row_strided and not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _rowmajor(t: torch.Tensor, name):
    if t.dim() != 2 or t.stride(1) != 1:
        raise ValueError(f"{name} must be a 2-D tensor with contiguous rows")


def default_alphas(n: int = 20, device="cuda") -> torch.Tensor:
    """The grid alpha_i = RN32(i / n), i = 0..n-1."""
    return torch.tensor([i / n for i in range(n)], dtype=torch.float32, device=device)


def _qcfg(bits, group, zero_point=True):
    return QCfg(int(bits), int(group), 1 if zero_point else 0)


def act_stats(X: torch.Tensor, stream=None) -> torch.Tensor:
    """a_j = mean_t |X[t, j]| for fp16 X[T, K] (rows may be strided)."""
    _rowmajor(X, "X")
    T, K = X.shape
    a = torch.empty(K, dtype=torch.float32, device=X.device)
    _check(lib().awq_act_stats(_dev(X, torch.float16, "X", row_strided=True), T, K, X.stride(0), _dev(a, torch.float32, "a"),
                               _stream(stream)), "awq_act_stats")
    return a


def alpha_scales(a: torch.Tensor, alphas: torch.Tensor, stream=None) -> torch.Tensor:
    """s[i, j] = a_j ** alpha_i (binary64 pow rounded to binary32)."""
    n = alphas.numel()
    s = torch.empty((n, a.numel()), dtype=torch.float32, device=a.device)
    _check(lib().awq_alpha_scales(_dev(a, torch.float32, "a"), a.numel(), _dev(alphas, torch.float32, "alphas"),
                                  n, _dev(s, torch.float32, "s"), _stream(stream)), "awq_alpha_scales")
    return s


def quant_dequant(W: torch.Tensor, s: torch.Tensor, bits: int = 4, group: int = 128, stream=None,
                  zero_point: bool = True, mask: torch.Tensor | None = None):
    """W_hat = Q(W diag(s)) diag(s)^-1 in fp16 (the per-element function of the search).

    mask (uint8 [K]): channels kept in fp16 (out of their group's range, W_hat = W)."""
    W = W.contiguous()
    N, K = W.shape
    out = torch.empty_like(W)
    args = (_dev(W, torch.float16, "W"), N, K, _dev(s, torch.float32, "s"), _qcfg(bits, group, zero_point))
    if mask is None:
        _check(lib().awq_quant_dequant(*args, _dev(out, torch.float16, "W_hat"), _stream(stream)),
               "awq_quant_dequant")
    else:
        _check(lib().awq_quant_dequant_masked(*args, _dev(mask, torch.uint8, "mask"),
                                              _dev(out, torch.float16, "W_hat"), _stream(stream)),
               "awq_quant_dequant_masked")
    return out


def search_workspace_bytes(N, K, T, bits=4, group=128, n_alpha=20, zero_point=True) -> int:
    return int(lib().awq_search_workspace_bytes(N, K, T, _qcfg(bits, group, zero_point), n_alpha))


def search_layer(W: torch.Tensor, X: torch.Tensor, a: torch.Tensor, alphas: torch.Tensor, bits: int = 4,
                 group: int = 128, workspace: torch.Tensor | None = None, row_losses: bool = False,
                 losses_out: torch.Tensor | None = None, stream=None, zero_point: bool = True,
                 rows_total: int | None = None):
    """Per-alpha MSE of the layer output, ||(W_hat_alpha - W) X^T||^2 / (N T).

    Returns ``losses`` (float32 [n_alpha]) or ``(losses, row_losses)`` with
    row_losses float32 [n_alpha, N] holding unnormalised per-row sums.  With
    ``rows_total``, W is one part of a layer of that many rows and the losses
    are normalised by rows_total T (awq_search_layer_part): the parts' losses
    add up to the layer's."""
    _rowmajor(X, "X")
    if not W.is_contiguous():
        raise ValueError("W must be contiguous")
    N, K = W.shape
    T = X.shape[0]
    n = alphas.numel()
    need = search_workspace_bytes(N, K, T, bits, group, n, zero_point)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=W.device)
    losses = losses_out if losses_out is not None else torch.empty(n, dtype=torch.float32, device=W.device)
    rl = torch.empty((n, N), dtype=torch.float32, device=W.device) if row_losses else None
    rest = (_dev(X, torch.float16, "X", row_strided=True), T, X.stride(0), _dev(a, torch.float32, "a"), _qcfg(bits, group, zero_point),
            _dev(alphas, torch.float32, "alphas"), n, _dev(losses, torch.float32, "losses"),
            _dev(rl, torch.float32, "row_losses") if rl is not None else None,
            ctypes.c_void_p(workspace.data_ptr()), workspace.numel(), _stream(stream))
    if rows_total is None:
        _check(lib().awq_search_layer(_dev(W, torch.float16, "W"), N, K, *rest), "awq_search_layer")
    else:
        _check(lib().awq_search_layer_part(_dev(W, torch.float16, "W"), N, int(rows_total), K, *rest),
               "awq_search_layer_part")
    return (losses, rl) if row_losses else losses


def pack(W: torch.Tensor, a: torch.Tensor, alphas: torch.Tensor, losses: torch.Tensor, bits: int = 4,
         group: int = 128, out: dict | None = None, stream=None, zero_point: bool = True) -> dict:
    """Argmin over the grid, then packed codes, fp16 scales/zeros and s at the best alpha."""
    N, K = W.shape
    dev = W.device
    per = 16 if bits == 2 else 8
    o = out if out is not None else dict(
        best_idx=torch.empty(1, dtype=torch.int32, device=dev),
        s_best=torch.empty(K, dtype=torch.float32, device=dev),
        codes=torch.empty((N, K // per), dtype=torch.int32, device=dev),
        scales=torch.empty((N, K // group), dtype=torch.float16, device=dev),
        zeros=torch.empty((N, K // group), dtype=torch.float16, device=dev))
    _check(lib().awq_pack(
        _dev(W, torch.float16, "W"), N, K, _dev(a, torch.float32, "a"), _qcfg(bits, group, zero_point),
        _dev(alphas, torch.float32, "alphas"), _dev(losses, torch.float32, "losses"), alphas.numel(),
        _dev(o["best_idx"], torch.int32, "best_idx"), _dev(o["s_best"], torch.float32, "s_best"),
        _dev(o["codes"], torch.int32, "codes"), _dev(o["scales"], torch.float16, "scales"),
        _dev(o["zeros"], torch.float16, "zeros"), _stream(stream)), "awq_pack")
    return o


def quantize_layer(W: torch.Tensor, X: torch.Tensor, alphas: torch.Tensor | None = None, bits: int = 4,
                   group: int = 128, workspace: torch.Tensor | None = None, stream=None,
                   zero_point: bool = True) -> dict:
    """The whole path for one layer: statistics, grid search, argmin, packing.

    W and X may live in host memory (pinned for asynchronous copies); they are
    then copied to the current device first and the results copied back."""
    host = not W.is_cuda
    dev = torch.device("cuda", torch.cuda.current_device())
    Wd = W.to(dev, non_blocking=True) if host else W
    Xd = X.to(dev, non_blocking=True) if host else X
    al = default_alphas(device=dev) if alphas is None else alphas.to(dev)
    a = act_stats(Xd, stream)
    losses = search_layer(Wd, Xd, a, al, bits, group, workspace=workspace, stream=stream, zero_point=zero_point)
    res = pack(Wd, a, al, losses, bits, group, stream=stream, zero_point=zero_point)
    res["losses"] = losses
    res["a"] = a
    if host:
        res = {k: v.to("cpu", non_blocking=True) for k, v in res.items()}
        torch.cuda.current_stream().synchronize()
    return res


def qlinear(codes: torch.Tensor, scales: torch.Tensor, zeros: torch.Tensor, s_best: torch.Tensor,
            X: torch.Tensor, bits: int = 4, group: int = 128, workspace: torch.Tensor | None = None,
            out: torch.Tensor | None = None, stream=None, tensor_cores: bool | None = None) -> torch.Tensor:
    """Y = X W_hat^T straight from the packed codes (the layer's input X is fp16 [T, K];
    1/s_best is folded into it).  Returns float32 [T, N].  tensor_cores None calls
    awq_qlinear (which picks the kernel by T), True awq_qlinear_tc (tcgen05), False
    awq_qlinear_cc (CUDA cores)."""
    _rowmajor(X, "X")
    N = codes.shape[0]
    T, K = X.shape
    need = int(lib().awq_qlinear_workspace_bytes(T, K, N))
    ws = workspace if workspace is not None else torch.empty(need, dtype=torch.uint8, device=X.device)
    Y = out if out is not None else torch.empty((T, N), dtype=torch.float32, device=X.device)
    name = {None: "awq_qlinear", True: "awq_qlinear_tc", False: "awq_qlinear_cc"}[tensor_cores]
    fn = getattr(lib(), name)
    _check(fn(_dev(codes, torch.int32, "codes"), _dev(scales, torch.float16, "scales"),
              _dev(zeros, torch.float16, "zeros"), _dev(s_best, torch.float32, "s_best"), N, K,
              _qcfg(bits, group), _dev(X, torch.float16, "X", row_strided=True), T, X.stride(0),
              _dev(Y, torch.float32, "Y"), ctypes.c_void_p(ws.data_ptr()), ws.numel(),
              _stream(stream)), name)
    return Y


def qlinear_path(T: int) -> str:
    """The kernel qlinear(tensor_cores=None) runs for T tokens: "cuda_cores" or "tensor_cores"."""
    return "tensor_cores" if lib().awq_qlinear_path(int(T)) == 1 else "cuda_cores"


def quantize_shared_input(Ws, X: torch.Tensor, alphas: torch.Tensor | None = None, bits: int = 4,
                          group: int = 128, stream=None, zero_point: bool = True) -> list:
    """Layers that read the same input (an MLP's gate and up projections, an
    attention block's Q/K/V) must share one s, because 1/s is folded into that
    one input.  Their weights are stacked row-wise and searched as one layer,
    so the loss is the sum of their output errors and one alpha is chosen for
    all of them; the packed output is split back per layer.

    Returns one dict per layer (codes, scales, zeros) plus the shared
    best_idx, s_best, losses and a."""
    rows = [w.shape[0] for w in Ws]
    W = torch.cat([w.contiguous() for w in Ws], dim=0)
    res = quantize_layer(W, X, alphas, bits, group, stream=stream, zero_point=zero_point)
    out, r0 = [], 0
    for n in rows:
        d = {k: res[k][r0:r0 + n] for k in ("codes", "scales", "zeros")}
        d.update({k: res[k] for k in ("best_idx", "s_best", "losses", "a")})
        out.append(d)
        r0 += n
    return out


def search_scales(W: torch.Tensor, X: torch.Tensor, s_table: torch.Tensor, bits: int = 4, group: int = 128,
                  zero_point: bool = True, mask: torch.Tensor | None = None, workspace: torch.Tensor | None = None,
                  row_losses: bool = False, stream=None):
    """MSE of the layer output for caller-given scale vectors s_table [n, K]
    (float32, positive), with the channels in ``mask`` (uint8 [K]) held in fp16."""
    _rowmajor(X, "X")
    if not W.is_contiguous() or not s_table.is_contiguous():
        raise ValueError("W and s_table must be contiguous")
    N, K = W.shape
    T = X.shape[0]
    st = s_table.reshape(-1, K)
    n = st.shape[0]
    q = _qcfg(bits, group, zero_point)
    need = int(lib().awq_search_scales_workspace_bytes(N, K, T, q, n, 0 if mask is None else 1))
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=W.device)
    losses = torch.empty(n, dtype=torch.float32, device=W.device)
    rl = torch.empty((n, N), dtype=torch.float32, device=W.device) if row_losses else None
    _check(lib().awq_search_scales(
        _dev(W, torch.float16, "W"), N, K, _dev(X, torch.float16, "X", row_strided=True), T, X.stride(0), q,
        _dev(st, torch.float32, "s_table"), n, None if mask is None else _dev(mask, torch.uint8, "mask"),
        _dev(losses, torch.float32, "losses"), _dev(rl, torch.float32, "row_losses") if rl is not None else None,
        ctypes.c_void_p(workspace.data_ptr()), workspace.numel(), _stream(stream)), "awq_search_scales")
    return (losses, rl) if row_losses else losses


def channel_topk(stat: torch.Tensor, k: int, stream=None) -> torch.Tensor:
    """uint8 [K] mask of the k channels with the largest statistic (ties: lower index)."""
    K = stat.numel()
    m = torch.empty(K, dtype=torch.uint8, device=stat.device)
    _check(lib().awq_channel_topk(_dev(stat, torch.float32, "stat"), K, int(k), _dev(m, torch.uint8, "mask"),
                                  _stream(stream)), "awq_channel_topk")
    return m


def salient_scales(mask: torch.Tensor, factor: float, stream=None) -> torch.Tensor:
    """s[k] = factor where mask[k] != 0, else 1 (the fixed-scale variant; factor 1 gives RTN)."""
    K = mask.numel()
    s = torch.empty(K, dtype=torch.float32, device=mask.device)
    _check(lib().awq_salient_scales(_dev(mask, torch.uint8, "mask"), K, float(factor), _dev(s, torch.float32, "s"),
                                    _stream(stream)), "awq_salient_scales")
    return s


def pack_scales(W: torch.Tensor, s: torch.Tensor, bits: int = 4, group: int = 128, zero_point: bool = True,
                stream=None) -> dict:
    """Codes, fp16 scales and zeros of W quantized with a given s."""
    N, K = W.shape
    dev = W.device
    per = 16 if bits == 2 else 8
    o = dict(codes=torch.empty((N, K // per), dtype=torch.int32, device=dev),
             scales=torch.empty((N, K // group), dtype=torch.float16, device=dev),
             zeros=torch.empty((N, K // group), dtype=torch.float16, device=dev), s_best=s)
    _check(lib().awq_pack_scales(_dev(W, torch.float16, "W"), N, K, _dev(s, torch.float32, "s"),
                                 _qcfg(bits, group, zero_point), _dev(o["codes"], torch.int32, "codes"),
                                 _dev(o["scales"], torch.float16, "scales"), _dev(o["zeros"], torch.float16, "zeros"),
                                 _stream(stream)), "awq_pack_scales")
    return o


def baselines(W: torch.Tensor, X: torch.Tensor, bits: int = 4, group: int = 128, alphas: torch.Tensor | None = None,
              frac: float = 0.01, zero_point: bool = True, stream=None) -> dict:
    """The comparisons of the AWQ pages on one layer, as output-error losses
    (float32 device scalars): plain RTN, the fixed 2x scale on the salient
    channels, fp16 protection of those channels chosen by activation and by
    weight magnitude, and the AWQ grid search.  k = round(frac K) channels."""
    K = W.shape[1]
    k = max(1, int(round(frac * K)))
    al = default_alphas(device=W.device) if alphas is None else alphas
    a = act_stats(X, stream)
    m_act = channel_topk(a, k, stream)
    m_w = channel_topk(act_stats(W, stream), k, stream)          # mean |w| per input channel
    table = torch.stack([salient_scales(m_act, 1.0, stream), salient_scales(m_act, 2.0, stream)])
    fixed = search_scales(W, X, table, bits, group, zero_point, stream=stream)
    ones = table[0:1].contiguous()
    fp16_act = search_scales(W, X, ones, bits, group, zero_point, mask=m_act, stream=stream)
    fp16_w = search_scales(W, X, ones, bits, group, zero_point, mask=m_w, stream=stream)
    grid = search_layer(W, X, a, al, bits, group, stream=stream, zero_point=zero_point)
    return dict(rtn=fixed[0], fixed_2x=fixed[1], fp16_act=fp16_act[0], fp16_weight=fp16_w[0], awq_grid=grid,
                mask_act=m_act, mask_weight=m_w, k=k)


def output_error(W: torch.Tensor, W_hat: torch.Tensor, X: torch.Tensor, row_losses: bool = False, stream=None):
    """||(W_hat - W) X^T||^2 / (N T) for any quantized weights W_hat (fp16 [N, K])."""
    _rowmajor(X, "X")
    N, K = W.shape
    T = X.shape[0]
    ws = torch.empty(int(lib().awq_output_error_workspace_bytes(N, K, T)), dtype=torch.uint8, device=W.device)
    loss = torch.empty(1, dtype=torch.float32, device=W.device)
    rl = torch.empty((1, N), dtype=torch.float32, device=W.device) if row_losses else None
    _check(lib().awq_output_error(_dev(W.contiguous(), torch.float16, "W"), _dev(W_hat.contiguous(), torch.float16, "W_hat"),
                                  N, K, _dev(X, torch.float16, "X", row_strided=True), T, X.stride(0), _dev(loss, torch.float32, "loss"),
                                  _dev(rl, torch.float32, "row_losses") if rl is not None else None,
                                  ctypes.c_void_p(ws.data_ptr()), ws.numel(), _stream(stream)), "awq_output_error")
    return (loss[0], rl[0]) if row_losses else loss[0]


def gptq_hessian(X: torch.Tensor, s: torch.Tensor | None = None, stream=None,
                 tensor_cores: bool = True) -> torch.Tensor:
    """H = 2 X'^T X' (float32 [K, K]) of the input divided by s: awq_gptq_hessian_tc
    (tcgen05), or awq_gptq_hessian (CUDA cores) with tensor_cores=False."""
    _rowmajor(X, "X")
    T, K = X.shape
    s = torch.ones(K, dtype=torch.float32, device=X.device) if s is None else s
    H = torch.empty((K, K), dtype=torch.float32, device=X.device)
    args = (_dev(X, torch.float16, "X", row_strided=True), T, K, X.stride(0), _dev(s, torch.float32, "s"), _dev(H, torch.float32, "H"))
    if tensor_cores:
        need = int(lib().awq_gptq_hessian_workspace_bytes(T, K))
        ws = torch.empty(max(need, 256), dtype=torch.uint8, device=X.device)
        _check(lib().awq_gptq_hessian_tc(*args, ctypes.c_void_p(ws.data_ptr()), ws.numel(), _stream(stream)),
               "awq_gptq_hessian_tc")
    else:
        _check(lib().awq_gptq_hessian(*args, _stream(stream)), "awq_gptq_hessian")
    return H


def gptq_factor(H: torch.Tensor, damp: float = 0.01, stream=None) -> torch.Tensor:
    """U, upper, with (H + damp mean(diag H) I)^-1 = U^T U (float32 [K, K])."""
    K = H.shape[0]
    H = H.contiguous()
    U = torch.empty_like(H)
    ws = torch.empty(int(lib().awq_gptq_factor_workspace_bytes(K)), dtype=torch.uint8, device=H.device)
    _check(lib().awq_gptq_factor(_dev(H, torch.float32, "H"), K, float(damp), _dev(U, torch.float32, "U"),
                                 ctypes.c_void_p(ws.data_ptr()), ws.numel(), _stream(stream)), "awq_gptq_factor")
    return U


def gptq_quantize(W: torch.Tensor, s: torch.Tensor, U: torch.Tensor, bits: int = 4, group: int = 128,
                  zero_point: bool = True, stream=None) -> dict:
    """The GPTQ column sweep over RN32(W s) with factor U: packed codes, fp16
    scales and zeros (awq_pack's layout) and the fp16 W_hat."""
    W = W.contiguous()
    N, K = W.shape
    dev = W.device
    per = 16 if bits == 2 else 8
    o = dict(codes=torch.empty((N, K // per), dtype=torch.int32, device=dev),
             scales=torch.empty((N, K // group), dtype=torch.float16, device=dev),
             zeros=torch.empty((N, K // group), dtype=torch.float16, device=dev),
             W_hat=torch.empty_like(W), s_best=s)
    _check(lib().awq_gptq_quantize(_dev(W, torch.float16, "W"), N, K, _dev(s, torch.float32, "s"),
                                   _dev(U.contiguous(), torch.float32, "U"), _qcfg(bits, group, zero_point),
                                   _dev(o["codes"], torch.int32, "codes"), _dev(o["scales"], torch.float16, "scales"),
                                   _dev(o["zeros"], torch.float16, "zeros"), _dev(o["W_hat"], torch.float16, "W_hat"),
                                   _stream(stream)), "awq_gptq_quantize")
    return o


def gptq_layer(W: torch.Tensor, X: torch.Tensor, s: torch.Tensor | None = None, bits: int = 4, group: int = 128,
               zero_point: bool = True, damp: float = 0.01, stream=None) -> dict:
    """GPTQ on the layer scaled by s (s = 1: GPTQ alone): Hessian, factor, sweep,
    and the output error of the result."""
    K = W.shape[1]
    s = torch.ones(K, dtype=torch.float32, device=W.device) if s is None else s
    U = gptq_factor(gptq_hessian(X, s, stream), damp, stream)
    o = gptq_quantize(W, s, U, bits, group, zero_point, stream)
    o["loss"] = output_error(W, o["W_hat"], X, stream=stream)
    return o


def awq_gptq(W: torch.Tensor, X: torch.Tensor, bits: int = 4, group: int = 128, alphas: torch.Tensor | None = None,
             zero_point: bool = True, damp: float = 0.01, stream=None) -> dict:
    """AWQ's scale search, then GPTQ on the layer scaled by the chosen s.
    Returns the GPTQ result (codes, scales, zeros, W_hat, loss, s_best) plus the
    AWQ grid's losses and best index."""
    res = quantize_layer(W, X, alphas, bits, group, stream=stream, zero_point=zero_point)
    o = gptq_layer(W, X, res["s_best"], bits, group, zero_point, damp, stream)
    o["awq_losses"] = res["losses"]
    o["best_idx"] = res["best_idx"]
    return o


def get_status(stream=None) -> None:
    """Synchronise and raise if a kernel reported an error on the device."""
    _check(lib().awq_get_status(_stream(stream)), "awq_get_status")


def selftest_bounded_wait(stream=None) -> None:
    """Launch the bounded-wait self-test (see include/awq.h); the next get_status raises AWQError(TIMEOUT)."""
    _check(lib().awq_selftest_bounded_wait(_stream(stream)), "awq_selftest_bounded_wait")


def set_wait_timeout_ms(ms: int) -> None:
    lib().awq_set_wait_timeout_ms(int(ms))


def profile_next_search(begin: torch.cuda.Event, end: torch.cuda.Event) -> None:
    """Bracket the tensor-core kernel of the next search_layer call (this thread) with two events."""
    lib().awq_profile_next_search(ctypes.c_void_p(begin.cuda_event), ctypes.c_void_p(end.cuda_event))
