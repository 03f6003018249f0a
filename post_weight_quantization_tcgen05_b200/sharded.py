"""The path split over several GPUs, one process per GPU, torch.distributed for the exchange.

Hessian: H = sum over calibration tokens of x^T x is a sum over token chunks ("hipfire-calib-data"
dataset card: the statistics are sums over chunks), so each rank accumulates a disjoint token
range (`token_range`) into its own fp32 H with hq_hessian_accumulate, as many calls as it likes.
`allreduce_hessian` then packs each rank's lower triangle (hq_hessian_pack_lower: K (K + 1) / 2
values, the half of H the path reads), sums the packed buffers with one all-reduce and unpacks
the sum into every rank's lower triangle: exact up to the order of the fp32 sums.

GPTQ: given U, the rows of W are quantised independently (the sweep's feedback stays inside a
row).  `gptq_row_shard` therefore factorises once: the root rank runs hq_gptq_factorize into a
factor buffer (plain bytes: the packed diagonal blocks of U' and the split U'^T), one broadcast
gives every rank that buffer, and each rank sweeps its own row range (`row_range`) with
hq_gptq_sweep.  The layer's qerr ("Exp 2026-08-18 GPTQ Int4", qerr definition) is
sqrt(sum num / sum den) over the ranks' numerator and denominator sums: hq_qerr_terms exposes
them, one all-reduce of two doubles adds them up and hq_qerr_from_terms takes the root.  A failed
factorisation is broadcast too (its header carries the status), so every rank raises the same
error after the same collective steps.

Every arithmetic step runs in the library's kernels; this module only slices, calls and
exchanges.
"""

from __future__ import annotations

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


def allreduce_hessian(hq, H: torch.Tensor, group=None) -> None:
    """H's lower triangle (each rank's partial sum over its tokens) <- the sum over all ranks, in
    place, exchanging the packed lower triangle only; H's strict upper triangle is untouched."""
    K = H.shape[0]
    packed = torch.empty(hq.hq_tril32_count(K), dtype=H.dtype, device=H.device)
    hq.hq_hessian_pack_lower(H, packed)
    dist.all_reduce(packed, op=dist.ReduceOp.SUM, group=group)
    hq.hq_hessian_unpack_lower(packed, K, H)


def combine_qerr_terms(hq, terms: torch.Tensor, group=None) -> float:
    """terms = [numerator, denominator] of this rank's rows (fp64, on this rank's device) -> the
    layer's qerr (hq_qerr_from_terms of the summed terms); every rank gets the same."""
    dist.all_reduce(terms, op=dist.ReduceOp.SUM, group=group)
    q = torch.empty(1, dtype=torch.float64, device=terms.device)
    hq.hq_qerr_from_terms(terms, q)
    return float(q.item())


def gptq_row_shard(hq, W_rows, H, group_size: int, damp: float, codes, scales, workspace=None, imp=None,
                   group=None, root: int = 0, factor_workspace=None) -> float:
    """Quantise this rank's rows W_rows [n, K] (codes [n, K/2], scales [n, K/group_size] out)
    against the layer's H, factorised once on `root` and broadcast; return the qerr of the whole
    layer (every rank gets the same).  H is read on the root only.  `workspace` (sweep scratch,
    hq_gptq_sweep_workspace_bytes) and `factor_workspace` (root only,
    hq_gptq_factor_workspace_bytes) are allocated when not given."""
    n, K = W_rows.shape
    dev = W_rows.device
    rank = dist.get_rank(group) if group is not None else dist.get_rank()
    factor = torch.empty(hq.hq_gptq_factor_bytes(K), dtype=torch.uint8, device=dev)
    failure = None
    if rank == root:
        if factor_workspace is None:
            factor_workspace = hq.alloc_workspace(hq.hq_gptq_factor_workspace_bytes(K), dev)
        try:
            hq.hq_gptq_factorize(H, damp, factor, factor_workspace)
        except hq.HQError as e:  # the factor's header records it: every rank's sweep reports it
            failure = e
    src = root if group is None else dist.get_global_rank(group, root)
    dist.broadcast(factor, src=src, group=group)
    if workspace is None:
        workspace = hq.alloc_workspace(hq.hq_gptq_sweep_workspace_bytes(n, K, group_size), dev)
    sweep_error = None
    try:
        hq.hq_gptq_sweep(W_rows, factor, group_size, codes, scales, workspace, imp=imp, want_qerr=False)
    except hq.HQError as e:
        sweep_error = e
    terms = torch.zeros(2, dtype=torch.float64, device=dev)
    if sweep_error is None:
        hq.hq_qerr_terms(workspace, terms)
    q = combine_qerr_terms(hq, terms, group)  # every rank takes this step, also after an error
    if sweep_error is not None:
        raise sweep_error
    if failure is not None:
        raise failure
    return q
