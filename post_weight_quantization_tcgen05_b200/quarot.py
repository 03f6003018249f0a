"""Rotate-then-GPTQ ("Exp 2026-08-18 GPTQ Int4", experiment summary: GPTQ composes with a
Hadamard rotation): W' = W R and H' = R^T H R with R = diag(signs) blockdiag(Hadamard_B / sqrt B)
(hq_hadamard_rotate_weights / hq_hadamard_rotate_hessian), then GPTQ on (W', H').  The codes
and scales describe W'; the layer is then fed R^T x (the activations rotated by the same signs
and blocks).  R is orthogonal, so the plain qerr of W' equals the un-rotated layer's
||W - Q' R^T|| / ||W||.  The random signs are drawn by the caller and passed in.

Every arithmetic step runs in the library's kernels; this module only allocates and calls.
"""

from __future__ import annotations

import torch


def random_signs(K: int, generator: torch.Generator, device="cuda") -> torch.Tensor:
    """fp32 [K] of +1 / -1 from `generator` (the method's random signs)."""
    bits = torch.randint(0, 2, (K,), generator=generator, device=generator.device, dtype=torch.int32)
    return (bits * 2 - 1).to(torch.float32).to(device)


def rotate_then_gptq(hq, W, H, signs, block: int, group: int, damp: float, codes, scales, workspace, imp=None):
    """GPTQ of W' = W R against H' = R^T H R (H read from its lower triangle).  Returns
    (qerr, W', H').  `imp`, when given, weights the columns of W', i.e. the ROTATED channels
    (the imatrix of the rotated layer is diag(H') / T, not diag(H) / T)."""
    N, K = W.shape
    Wr = torch.empty((N, K), dtype=torch.float32, device=W.device)
    Hr = torch.empty((K, K), dtype=torch.float32, device=W.device)
    hq.hq_hadamard_rotate_weights(W, signs, block, Wr)
    hq.hq_hadamard_rotate_hessian(H, signs, block, Hr)
    q = hq.hq_gptq_quantize(Wr, Hr, group, damp, codes, scales, workspace, imp=imp)
    return q, Wr, Hr
