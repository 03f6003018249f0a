"""Shared helpers of the GPU parity tests: tolerance checks against the oracle."""

import numpy as np
import torch

# Tolerances stated for the path (codes, scales, loss, qerr, H); the codec is bit-exact.
H_REL_FRO = 1e-5
CODE_MATCH_MIN = 0.99
SCALE_REL = 1e-4
LOSS_REL = 0.01
QERR_REL = 0.01
# Teacher forcing (the oracle replays the GPU's own codes): the GPU's scales must match the
# oracle's on that trajectory to SCALE_REL, and every GPU code that differs from the code the
# oracle would pick there must be a near-tie: the oracle's w/s within TIE_TOL of the rounding
# boundary between the two codes.
TIE_TOL = 0.05


def to_np64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu", torch.float64).numpy()


def rel_fro(a, b) -> float:
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


def unpack_codes(codes_u8: torch.Tensor) -> np.ndarray:
    import oracle
    return oracle.unpack_int4(codes_u8.cpu().numpy())


def check_quant_parity(codes_gpu, scales_gpu, codes_ref, scales_ref, what=""):
    """Codes: >= 99 % identical and never off by more than 1; scales: relative 1e-4."""
    cg = np.asarray(codes_gpu, np.int16)
    cr = np.asarray(codes_ref, np.int16)
    assert cg.shape == cr.shape, what
    match = float(np.mean(cg == cr))
    maxdiff = int(np.max(np.abs(cg - cr))) if cg.size else 0
    sg = np.asarray(scales_gpu, np.float64)
    sr = np.asarray(scales_ref, np.float64)
    denom = np.maximum(np.abs(sr), 1e-30)
    srel = float(np.max(np.abs(sg - sr) / denom)) if sg.size else 0.0
    assert match >= CODE_MATCH_MIN, f"{what}: code match {match:.5f}"
    assert maxdiff <= 1, f"{what}: max code difference {maxdiff}"
    assert srel <= SCALE_REL, f"{what}: scale rel err {srel:.3e}"
    return match, maxdiff, srel


def scale_rel_err(sg, sr) -> np.ndarray:
    """|s_gpu - s_ref| / |s_ref| element-wise; two zero scales (an all-zero group) agree exactly."""
    sg = np.asarray(sg, np.float64)
    sr = np.asarray(sr, np.float64)
    return np.where(sr == 0.0, np.where(sg == 0.0, 0.0, np.inf), np.abs(sg - sr) / np.maximum(np.abs(sr), 1e-300))


def groups_before_divergence(codes_gpu, codes_ref, group):
    """Mask [N, K/group] of the groups whose first column lies at or before the row's first
    differing code (every group of a row without one).  A group's scale is taken from the
    current weights at its first column, which depend only on the codes of earlier columns, so
    up to that column both sweeps follow the same trajectory and their scales must agree."""
    cg = np.asarray(codes_gpu, np.int16)
    cr = np.asarray(codes_ref, np.int16)
    N, K = cg.shape
    diff = cg != cr
    first = np.where(diff.any(axis=1), diff.argmax(axis=1), K)
    starts = np.arange(K // group) * group
    return starts[None, :] <= first[:, None]


def check_gptq_parity(W64, U64, group, codes_gpu, scales_gpu, what=""):
    """Codes against the plain oracle (>= 99 % identical, never off by more than 1).  Scales
    against the plain oracle for every group that starts at or before the row's first
    differing code (relative 1e-4), and for the groups after it against the oracle forced onto
    the GPU's own code trajectory (relative 1e-4), where every differing code must also be a
    near-tie of the rounding rule."""
    import oracle
    ref_codes, ref_scales, _ = oracle.gptq_sweep(W64, U64, group)
    cg = np.asarray(codes_gpu, np.int16)
    cr = np.asarray(ref_codes, np.int16)
    match = float(np.mean(cg == cr))
    maxdiff = int(np.max(np.abs(cg - cr))) if cg.size else 0
    s_f, _, free_f, ratio_f = oracle.gptq_sweep_forced(W64, U64, group, codes_gpu)
    sg = np.asarray(scales_gpu, np.float64)
    sf = np.asarray(s_f, np.float64)
    srel = float(np.max(scale_rel_err(sg, sf))) if sg.size else 0.0
    before = groups_before_divergence(cg, cr, group)
    plain_err = scale_rel_err(sg, ref_scales)
    splain = float(np.max(plain_err[before])) if np.any(before) else 0.0
    splain_all = float(np.max(plain_err)) if sg.size else 0.0
    fr = np.asarray(free_f, np.int16)
    mism = cg != fr
    tie = 0.0
    if np.any(mism):
        boundary = (cg[mism] + fr[mism]) / 2.0
        r = np.asarray(ratio_f, np.float64)[mism]
        # a clamped free code (-8 / 7) with the GPU one step inside is a tie at the clamp edge too
        tie = float(np.max(np.where(np.abs(cg[mism] - fr[mism]) == 1, np.abs(r - boundary), np.inf)))
    print(f"[parity {what}] code match {match:.5f} maxdiff {maxdiff} | scale rel plain before divergence "
          f"{splain:.2e} ({int(before.sum())} of {before.size} groups; {splain_all:.2e} over all) forced {srel:.2e} "
          f"| forced mismatches {int(mism.sum())} worst tie distance {tie:.3e}")
    assert match >= CODE_MATCH_MIN, f"{what}: code match {match:.5f}"
    assert maxdiff <= 1, f"{what}: max code difference {maxdiff}"
    assert splain <= SCALE_REL, f"{what}: scale rel err against the plain oracle before divergence {splain:.3e}"
    assert srel <= SCALE_REL, f"{what}: teacher-forced scale rel err {srel:.3e}"
    assert tie <= TIE_TOL, f"{what}: a differing code is {tie:.3e} steps from its rounding boundary"
    return ref_codes, ref_scales


def split_tf32(x: torch.Tensor):
    """(hi, lo): hi = x with the low 13 mantissa bits cleared (a tf32 value), lo = x - hi
    (exact in fp32): the operand split the lazy-update kernel consumes."""
    hi = (x.view(torch.int32) & -8192).view(torch.float32)
    return hi, x - hi
