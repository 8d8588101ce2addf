"""Saving and reloading the packed output of the AWQ path.

The pages save the quantized model and load it back for inference ([QAS-QA]
"Как работает quantization-aware scaling в AWQ для защиты важных весов?" §9:
``save_quantized`` after ``quantize``), and what is kept is the low-bit weights
and their metadata ([AWQ-note] "AWQ: Activation-Aware Weight Quantization For
On-Device LLM Compression AND Acceleration", "Measures").  For this library
that is one layer's (or one group of layers sharing an input) result of
``pack`` / ``quantize_layer``:

  codes     int32 [N, K / per]   per = 16 codes a word at 2 bits, else 8
  scales    fp16  [N, K / group]
  zeros     fp16  [N, K / group]
  s_best    fp32  [K]            the chosen per-input-channel scale
  best_idx  int32 [1]            its index in the alpha grid
  losses    fp32  [n_alpha]      optional: the output error of every alpha
  alphas    fp32  [n_alpha]      optional: the grid
  a         fp32  [K]            optional: the activation statistic

with the quantizer configuration (bits, group size, zero point).  Every tensor
is copied to the host before writing (``torch.save``); ``load_quantized``
checks the format tag, the configuration and every shape and dtype before it
returns the tensors on the requested device, ready for ``qlinear``.  Host-side
plumbing only: nothing here computes.
"""
from __future__ import annotations

import torch

FORMAT = "awq-b200-packed-layer"
VERSION = 1

_REQUIRED = ("codes", "scales", "zeros", "s_best", "best_idx")
_OPTIONAL = ("losses", "alphas", "a")
_DTYPES = {"codes": torch.int32, "scales": torch.float16, "zeros": torch.float16, "s_best": torch.float32,
           "best_idx": torch.int32, "losses": torch.float32, "alphas": torch.float32, "a": torch.float32}


def _check_config(bits, group, zero_point):
    if bits not in (2, 3, 4):
        raise ValueError(f"bits must be 2, 3 or 4, got {bits!r}")
    if group not in (64, 128):
        raise ValueError(f"group size must be 64 or 128, got {group!r}")
    if not isinstance(zero_point, bool):
        raise ValueError(f"zero_point must be a bool, got {zero_point!r}")


def _check_tensors(t: dict, bits: int, group: int):
    for k in _REQUIRED:
        if k not in t:
            raise ValueError(f"missing tensor {k!r}")
    for k, v in t.items():
        if not isinstance(v, torch.Tensor):
            raise ValueError(f"{k!r} is not a tensor")
        if v.dtype != _DTYPES[k]:
            raise ValueError(f"{k!r} has dtype {v.dtype}, expected {_DTYPES[k]}")
    per = 16 if bits == 2 else 8
    if t["s_best"].dim() != 1:
        raise ValueError("s_best must be one-dimensional [K]")
    K = t["s_best"].shape[0]
    if t["codes"].dim() != 2:
        raise ValueError("codes must be [N, K / per]")
    N = t["codes"].shape[0]
    if K % group or K % per:
        raise ValueError(f"K = {K} is not a multiple of the group size {group} and of {per} codes a word")
    want = {"codes": (N, K // per), "scales": (N, K // group), "zeros": (N, K // group), "best_idx": (1,)}
    for k, shape in want.items():
        if tuple(t[k].shape) != shape:
            raise ValueError(f"{k!r} has shape {tuple(t[k].shape)}, expected {shape}")
    if "a" in t and tuple(t["a"].shape) != (K,):
        raise ValueError(f"'a' has shape {tuple(t['a'].shape)}, expected ({K},)")
    n = [t[k].numel() for k in ("losses", "alphas") if k in t]
    if len(n) == 2 and n[0] != n[1]:
        raise ValueError("losses and alphas have different lengths")
    if n and not 0 <= int(t["best_idx"].reshape(-1)[0]) < n[0]:
        raise ValueError(f"best_idx {int(t['best_idx'].reshape(-1)[0])} is outside the grid of {n[0]}")


def save_quantized(path, result: dict, bits: int, group: int, zero_point: bool = True,
                   alphas: torch.Tensor | None = None) -> None:
    """Write one packed result (the dict ``pack`` or ``quantize_layer`` returns;
    other keys are ignored) and its quantizer configuration to ``path``."""
    _check_config(bits, group, zero_point)
    t = {k: result[k] for k in _REQUIRED + _OPTIONAL if k in result}
    if alphas is not None:
        t["alphas"] = alphas
    _check_tensors(t, bits, group)
    blob = {"format": FORMAT, "version": VERSION, "bits": int(bits), "group_size": int(group),
            "zero_point": bool(zero_point),
            "tensors": {k: v.detach().to("cpu").contiguous() for k, v in t.items()}}
    torch.save(blob, path)


def load_quantized(path, device="cpu") -> dict:
    """Read a file written by ``save_quantized``.  Returns the tensors on
    ``device`` and the configuration under ``bits``, ``group_size`` and
    ``zero_point``; raises ValueError if the file is not of this format or its
    shapes do not match its configuration."""
    blob = torch.load(path, map_location="cpu", weights_only=True)
    if not isinstance(blob, dict) or blob.get("format") != FORMAT:
        raise ValueError(f"{path}: not a packed AWQ layer")
    if blob.get("version") != VERSION:
        raise ValueError(f"{path}: format version {blob.get('version')!r}, this library reads {VERSION}")
    bits, group, zp = blob.get("bits"), blob.get("group_size"), blob.get("zero_point")
    _check_config(bits, group, zp)
    t = blob.get("tensors")
    if not isinstance(t, dict) or set(t) - set(_REQUIRED + _OPTIONAL):
        raise ValueError(f"{path}: unexpected tensor set")
    _check_tensors(t, bits, group)
    out = {k: v.to(device) for k, v in t.items()}
    out.update(bits=bits, group_size=group, zero_point=zp)
    return out
