"""One layer's rows split across processes (one per GPU).

The output error of a layer is a sum over its output rows, and each row's
codes depend only on that row and the shared scale vector s ([AWQ-note] "AWQ:
Activation-Aware Weight Quantization For On-Device LLM Compression AND
Acceleration", "Measures": search the scales per layer against the error of
the layer's output).  So a layer shards by rows with one exchange:

1. every rank computes the statistics a from the (replicated) calibration input X;
2. every rank searches the alpha grid on its own rows with losses normalised by
   the layer's row count (awq_search_layer_part);
3. one all-reduce (sum) of the n_alpha losses gives every rank the layer's MSE;
4. every rank takes the same argmin and packs its own rows (awq_pack).

Steps 1, 2 and 4 run in the library's kernels; step 3 is torch.distributed
(NCCL between GPUs).  This module holds only that plumbing.
"""
from __future__ import annotations

import torch

from . import act_stats, default_alphas, pack, search_layer

ROW_UNIT = 256          # the search kernel's work unit is 256 rows: parts are whole units


def shard_rows(N: int, world: int, rank: int, unit: int = ROW_UNIT) -> tuple[int, int]:
    """Rows [r0, r1) of `rank`: contiguous blocks of whole `unit`s, as even as
    the units allow; trailing ranks may get no rows when N is small."""
    if world < 1 or not 0 <= rank < world or N < 0:
        raise ValueError("need world >= 1, 0 <= rank < world, N >= 0")
    units = -(-N // unit)
    per = -(-units // world)
    r0 = min(rank * per * unit, N)
    r1 = min(r0 + per * unit, N)
    return r0, r1


def quantize_layer_rows(W_part: torch.Tensor, X: torch.Tensor, rows_total: int, alphas: torch.Tensor | None = None,
                        bits: int = 4, group: int = 128, process_group=None, workspace: torch.Tensor | None = None,
                        zero_point: bool = True) -> dict:
    """The whole path for this rank's rows of a layer (see the module notes).

    W_part: this rank's rows of W (fp16 [n, K] on this rank's GPU, n may be 0);
    X: the full calibration input (fp16 [T, K], the same on every rank).
    Every rank of `process_group` must call this with the same rows_total,
    alphas and quantizer.  Returns the layer's losses (identical on every
    rank) and a; a rank with rows also gets best_idx, s_best and its part's
    codes, scales and zeros (a rank without rows has nothing to pack)."""
    import torch.distributed as dist

    dev = X.device
    al = default_alphas(device=dev) if alphas is None else alphas.to(dev)
    a = act_stats(X)
    n = W_part.shape[0]
    if n > 0:
        losses = search_layer(W_part, X, a, al, bits, group, workspace=workspace, zero_point=zero_point,
                              rows_total=rows_total)
    else:
        losses = torch.zeros(al.numel(), dtype=torch.float32, device=dev)
    if dist.is_available() and dist.is_initialized():
        dist.all_reduce(losses, op=dist.ReduceOp.SUM, group=process_group)
    if n > 0:
        res = pack(W_part, a, al, losses, bits, group, zero_point=zero_point)
    else:
        res = {}
    res["losses"] = losses
    res["a"] = a
    return res
