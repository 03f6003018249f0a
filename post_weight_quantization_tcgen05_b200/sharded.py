"""The path split over several GPUs, one process per GPU, torch.distributed for the exchange.

Hessian: H = sum over calibration tokens of x^T x is a sum over token chunks ("hipfire-calib-data"
dataset card: the statistics are sums over chunks), so each rank accumulates a disjoint token
range (`token_range`) into its own fp32 H with hq_hessian_accumulate, as many calls as it likes,
and one all-reduce (sum) of the K x K buffers (`allreduce_hessian`) leaves the layer's H on every
rank, exact up to the order of the fp32 sums.

GPTQ: given U, the rows of W are quantised independently (the sweep's feedback stays inside a
row), so each rank quantises a disjoint row range (`row_range`) with hq_gptq_quantize, factorising
the same H itself; the layer's qerr ("Exp 2026-08-18 GPTQ Int4", qerr definition) is
sqrt(sum num / sum den) over the ranks' numerator and denominator sums, which hq_qerr_terms
exposes and one all-reduce of two doubles adds up (`gptq_row_shard`).

Every arithmetic step runs in the library's kernels; this module only slices, calls and reduces.
"""

from __future__ import annotations

import math

import torch
import torch.distributed as dist


def split_range(n: int, rank: int, world: int) -> tuple[int, int]:
    """[start, stop) of part `rank` of n items in `world` contiguous parts whose sizes differ by
    at most one (the first n % world parts are one longer)."""
    if world < 1 or not 0 <= rank < world or n < 0:
        raise ValueError("bad split")
    base, extra = divmod(n, world)
    start = rank * base + min(rank, extra)
    return start, start + base + (1 if rank < extra else 0)


def token_range(T: int, rank: int, world: int) -> tuple[int, int]:
    """This rank's calibration tokens."""
    return split_range(T, rank, world)


def row_range(N: int, rank: int, world: int) -> tuple[int, int]:
    """This rank's rows of W."""
    return split_range(N, rank, world)


def allreduce_hessian(H: torch.Tensor, group=None) -> None:
    """H (each rank's partial sum over its tokens) <- the sum over all ranks, in place."""
    dist.all_reduce(H, op=dist.ReduceOp.SUM, group=group)


def combine_qerr_terms(terms: torch.Tensor, group=None) -> float:
    """terms = [numerator, denominator] of this rank's rows (fp64, any device the process group
    serves) -> the layer's qerr; 0 when every weight is zero."""
    dist.all_reduce(terms, op=dist.ReduceOp.SUM, group=group)
    num, den = (float(v) for v in terms.tolist())
    return 0.0 if den == 0.0 else math.sqrt(num / den)


def gptq_row_shard(hq, W_rows, H, group_size: int, damp: float, codes, scales, workspace, imp=None,
                   group=None) -> float:
    """Quantise this rank's rows W_rows [n, K] (codes [n, K/2], scales [n, K/group_size] out)
    against the layer's H, and return the qerr of the whole layer (every rank gets the same)."""
    hq.hq_gptq_quantize(W_rows, H, group_size, damp, codes, scales, workspace, imp=imp, want_qerr=False)
    terms = torch.empty(2, dtype=torch.float64, device=W_rows.device)
    hq.hq_qerr_terms(workspace, terms)
    return combine_qerr_terms(terms, group)
