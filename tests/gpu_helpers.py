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


def check_gptq_parity(W64, U64, group, codes_gpu, scales_gpu, what=""):
    """Codes against the plain oracle (>= 99 % identical, never off by more than 1); scales and
    code validity against the oracle forced onto the GPU's code trajectory."""
    import oracle
    ref_codes, ref_scales, _ = oracle.gptq_sweep(W64, U64, group)
    cg = np.asarray(codes_gpu, np.int16)
    cr = np.asarray(ref_codes, np.int16)
    match = float(np.mean(cg == cr))
    maxdiff = int(np.max(np.abs(cg - cr))) if cg.size else 0
    s_f, _, free_f, ratio_f = oracle.gptq_sweep_forced(W64, U64, group, codes_gpu)
    sg = np.asarray(scales_gpu, np.float64)
    sf = np.asarray(s_f, np.float64)
    srel = float(np.max(np.abs(sg - sf) / np.maximum(np.abs(sf), 1e-30))) if sg.size else 0.0
    splain = float(np.max(np.abs(sg - np.asarray(ref_scales, np.float64)) /
                          np.maximum(np.abs(np.asarray(ref_scales, np.float64)), 1e-30))) if sg.size else 0.0
    fr = np.asarray(free_f, np.int16)
    mism = cg != fr
    tie = 0.0
    if np.any(mism):
        boundary = (cg[mism] + fr[mism]) / 2.0
        r = np.asarray(ratio_f, np.float64)[mism]
        # a clamped free code (-8 / 7) with the GPU one step inside is a tie at the clamp edge too
        tie = float(np.max(np.where(np.abs(cg[mism] - fr[mism]) == 1, np.abs(r - boundary), np.inf)))
    print(f"[parity {what}] code match {match:.5f} maxdiff {maxdiff} | scale rel forced {srel:.2e} "
          f"plain {splain:.2e} | forced mismatches {int(mism.sum())} worst tie distance {tie:.3e}")
    assert match >= CODE_MATCH_MIN, f"{what}: code match {match:.5f}"
    assert maxdiff <= 1, f"{what}: max code difference {maxdiff}"
    assert srel <= SCALE_REL, f"{what}: teacher-forced scale rel err {srel:.3e}"
    assert tie <= TIE_TOL, f"{what}: a differing code is {tie:.3e} steps from its rounding boundary"
    return ref_codes, ref_scales


def split_tf32(x: torch.Tensor):
    """(hi, lo): hi = x with the low 13 mantissa bits cleared (a tf32 value), lo = x - hi
    (exact in fp32): the operand split the lazy-update kernel consumes."""
    hi = (x.view(torch.int32) & -8192).view(torch.float32)
    return hi, x - hi
