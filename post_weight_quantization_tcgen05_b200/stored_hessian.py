"""Quantising against a Hessian read back from storage ("hipfire-calib-data" dataset card,
"REQUIRED: project to PSD before Cholesky"): the bf16 off-diagonals of the Bf16TrilDiagF32
format perturb the Gram matrix out of the positive semidefinite cone by about mean(diag H), so
a stored Hessian is decoded (hq_hessian_unpack_bf16tril), projected onto the PSD cone
(hq_hessian_project_psd) and only then factorised.  Raising the damping instead is the fallback
the pages measure and advise against (a damping near mean(diag H) turns GPTQ into
round-to-nearest); `quantize_with_damping_escalation` implements it for callers that skip the
projection: the damping is multiplied by `factor` after every failed factorisation, up to `cap`.

Every arithmetic step runs in the library's kernels; this module only sequences calls.
"""

from __future__ import annotations

import torch


def load_stored_hessian(hq, payload, K: int, project: bool = True, steps: int = 40, workspace=None):
    """Bf16TrilDiagF32 bytes (device uint8) -> fp32 [K, K] symmetric H on the same device,
    projected onto the PSD cone unless `project` is False."""
    H = torch.empty((K, K), dtype=torch.float32, device=payload.device)
    hq.hq_hessian_unpack_bf16tril(payload, K, H)
    if project:
        hq.hq_hessian_project_psd(H, workspace=workspace, steps=steps)
    return H


def quantize_with_damping_escalation(hq, W, H, group: int, damp: float, codes, scales, workspace, imp=None,
                                     factor: float = 10.0, cap: float = 1.0):
    """hq_gptq_quantize with damp, damp * factor, ... (at most `cap`) until the factorisation
    succeeds; returns (qerr, damp used).  Raises the last HQ_ERR_NOT_PD when even `cap` fails."""
    if not (damp > 0 and factor > 1 and cap >= damp):
        raise ValueError("need 0 < damp <= cap and factor > 1")
    d = float(damp)
    while True:
        try:
            return hq.hq_gptq_quantize(W, H, group, d, codes, scales, workspace, imp=imp), d
        except hq.HQError as e:
            if e.status != hq.HQ_ERR_NOT_PD or d >= cap:
                raise
            d = min(d * factor, cap)
