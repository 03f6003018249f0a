"""fp64 CPU oracle: Hessian, damping, Cholesky chain, GPTQ sweep, RTN, qerr, layer loss,
Bf16TrilDiagF32 codec.

TEST INFRASTRUCTURE ONLY -- see ``oracle/__init__.py``.  numpy/scipy on the CPU; library
primitives (a matrix product, LAPACK's Cholesky and triangular solve) serve as single steps,
everything else is written out in the order the pages give it.  No blocking, no fusion.

Pages cited (by title and section):

* [calib]  "hipfire-calib-data" dataset card:
    - "Hessian storage: Bf16TrilDiagF32 (quant_type 130)": byte count K*4 + K*(K-1)/2*2,
      exact f32 diagonal, strict lower triangle as bf16 at index i*(i-1)/2 + j (i > j),
      mirrored on read, bf16 conversion by truncation (f32_bits >> 16).  Full Hessians XX^T.
    - "REQUIRED: project to PSD before Cholesky" / "The fix": damping is expressed as a
      multiple of mean(diag(H)); damping that dominates the diagonal turns GPTQ into
      round-to-nearest.  A stored (bf16) Hessian is made positive semidefinite by an
      eigendecomposition whose negative eigenvalues are clipped to zero, the matrix rebuilt
      from the clipped spectrum and then symmetrised.
* [gptq]   ork-driver wiki, "Exp 2026-08-18 GPTQ Int4":
    - experiment summary: error-compensated column-sequential int4 rounding (GPTQ), a
      Cholesky-based Hessian inverse plus an error-feedback sweep, uniform symmetric int4
      codes in [-8, 7] with a per-(row, group) scale, dequantisation w = code * scale; the
      plain baseline is symmetric absmax/7 rounding.
    - qerr definition: sqrt(sum_n sum_k imp[k](w - q)^2 / sum_n sum_k imp[k] w^2), imp = 1
      when no importance vector is given.
    - analytic check table (uniform weights: step absmax/7, RMS error step/sqrt(12)).
* [imat]   AtomicChat Qwen3.8-27B GGUF card, "The importance matrix": the calibration
  statistic is a sum over chunks, so partial results merge by addition; the importance
  matrix is the mean squared activation per channel.

Readings taken where the pages are silent (each also listed in the design notes):

* the group scale is taken from the *current* (error-compensated) weights of the group at
  its first column, s = fp32(absmax / 7); it is stored as fp32 and the same fp32 value is
  used for rounding and for dequantisation;
* the rounding decision is taken in the GPU kernel's precision: c = clamp(rint(fp32(w) / s),
  -8, 7) with an IEEE fp32 division and round-half-to-even; a group whose absmax is 0 has
  s = 0 and codes 0;
* damping lambda = damp * mean(diag H) added to the diagonal of the undamped H; a
  non-positive mean diagonal is an invalid input;
* U is the upper Cholesky factor of (H + lambda I)^-1, reached by the literal route
  (Cholesky, triangular inverse, H^-1 = L^-T L^-1, Cholesky of H^-1);
* columns are processed in natural order 0..K-1 (no activation ordering);
* qerr and the layer loss use the original weights W and q = code * scale; the loss uses
  the undamped H.
"""

from __future__ import annotations

import numpy as np
import scipy.linalg

__all__ = [
    "NotPositiveDefinite",
    "hessian",
    "hessian_accumulate",
    "imatrix",
    "damp_hessian",
    "project_psd",
    "hadamard_matrix",
    "hadamard_rotation",
    "rotate_weights",
    "rotate_hessian",
    "cholesky_lower",
    "upper_factor_of_inverse",
    "upper_factor_by_reversal",
    "gptq_sweep",
    "gptq_quantize",
    "gptq_sweep_forced",
    "rtn_quantize",
    "dequantize",
    "qerr",
    "layer_loss",
    "bf16tril_bytes",
    "bf16tril_encode",
    "bf16tril_decode",
    "truncate_f32_to_bf16_bits",
    "pack_int4",
    "unpack_int4",
]


class NotPositiveDefinite(ValueError):
    """Cholesky met a non-positive pivot: the damped Hessian is not positive definite."""


# ---------------------------------------------------------------------------------------
# Calibration Hessian  ([calib] "Hessian storage": full Hessians XX^T; [imat] sums over chunks)
# ---------------------------------------------------------------------------------------

def hessian(X) -> np.ndarray:
    """H = X^T X in fp64 for X laid out [tokens, channels] (the pages write XX^T with X laid
    out [channels, tokens]: the same K x K matrix).  Full symmetric result."""
    X64 = np.asarray(X, dtype=np.float64)
    if X64.ndim != 2:
        raise ValueError("X must be 2-D [T, K]")
    return X64.T @ X64


def hessian_accumulate(H, X) -> np.ndarray:
    """H + X^T X: the statistic is a sum over chunks, so chunked accumulation is addition
    ([imat] "The importance matrix")."""
    return np.asarray(H, dtype=np.float64) + hessian(X)


def imatrix(H, tokens: int) -> np.ndarray:
    """Importance = mean squared activation per channel = diag(H) / tokens
    ([gptq] qerr definition: diag(H)[k] = sum a_k^2 and the imatrix stores its mean)."""
    if tokens <= 0:
        raise ValueError("tokens must be positive")
    return np.diag(np.asarray(H, dtype=np.float64)).copy() / float(tokens)


# ---------------------------------------------------------------------------------------
# Damping and the Cholesky chain  ([calib] damping relative to mean(diag); [gptq] summary)
# ---------------------------------------------------------------------------------------

def damp_hessian(H, damp: float):
    """Return (H + lambda I, lambda) with lambda = damp * mean(diag H)."""
    H64 = np.asarray(H, dtype=np.float64)
    K = H64.shape[0]
    mean_diag = float(np.trace(H64)) / K
    if not mean_diag > 0.0:
        raise ValueError("mean(diag H) must be positive")
    lam = float(damp) * mean_diag
    return H64 + lam * np.eye(K), lam


def project_psd(H) -> np.ndarray:
    """[calib] "The fix": with H = V diag(l) V^T (symmetric eigendecomposition, LAPACK as one
    step), rebuild V diag(max(l, 0)) V^T, then return its symmetric part (P + P^T) / 2."""
    H64 = np.asarray(H, dtype=np.float64)
    l, V = np.linalg.eigh(H64)
    P = (V * np.maximum(l, 0.0)) @ V.T
    return (P + P.T) / 2.0


def hadamard_matrix(B: int) -> np.ndarray:
    """The orthonormal Walsh-Hadamard matrix of order B (a power of two), Sylvester ordering:
    M[i][j] = (-1)^popcount(i & j) / sqrt(B)."""
    if B < 1 or B & (B - 1):
        raise ValueError("B must be a power of two")
    i = np.arange(B)
    bits = np.bitwise_and.outer(i, i)
    parity = np.zeros((B, B), dtype=np.int64)
    while bits.any():
        parity ^= bits & 1
        bits >>= 1
    return (1.0 - 2.0 * parity) / np.sqrt(B)


def hadamard_rotation(signs, B: int) -> np.ndarray:
    """[gptq] experiment summary ("rotate then GPTQ"): R = diag(signs) blockdiag(M_B, ..., M_B),
    K = len(signs) a multiple of B."""
    s = np.asarray(signs, dtype=np.float64)
    K = s.size
    if K % B:
        raise ValueError("B must divide K")
    return s[:, None] * np.kron(np.eye(K // B), hadamard_matrix(B))


def rotate_weights(W, signs, B: int) -> np.ndarray:
    """W' = W R."""
    return np.asarray(W, dtype=np.float64) @ hadamard_rotation(signs, B)


def rotate_hessian(H, signs, B: int) -> np.ndarray:
    """H' = R^T H R, H taken as the symmetric matrix of its lower triangle."""
    L = np.tril(np.asarray(H, dtype=np.float64))
    Hs = L + np.tril(L, -1).T
    R = hadamard_rotation(signs, B)
    return R.T @ Hs @ R


def cholesky_lower(A) -> np.ndarray:
    """L with A = L L^T, L lower triangular with positive diagonal (LAPACK potrf as one step)."""
    try:
        return np.linalg.cholesky(np.asarray(A, dtype=np.float64))
    except np.linalg.LinAlgError as exc:
        raise NotPositiveDefinite(str(exc)) from None


def upper_factor_of_inverse(Hd) -> np.ndarray:
    """U upper triangular with U^T U = Hd^-1, by the literal "Cholesky-based Hessian inverse"
    route of [gptq]: L = chol(Hd); Hd^-1 = L^-T L^-1; U^T = chol(Hd^-1)."""
    L = cholesky_lower(Hd)
    K = L.shape[0]
    Linv = scipy.linalg.solve_triangular(L, np.eye(K), lower=True)
    Hinv = Linv.T @ Linv
    Lh = cholesky_lower(Hinv)
    return np.triu(Lh.T)


def upper_factor_by_reversal(Hd) -> np.ndarray:
    """The same U by a second route, used only to cross-check the first: with J the
    index reversal, J Hd J = M M^T (M lower) gives Hd = R R^T with R = J M J upper, so
    Hd^-1 = R^-T R^-1 and U = R^-1 = J M^-1 J (uniqueness of the Cholesky factor)."""
    Hd = np.asarray(Hd, dtype=np.float64)
    K = Hd.shape[0]
    M = cholesky_lower(Hd[::-1, ::-1])
    Minv = scipy.linalg.solve_triangular(M, np.eye(K), lower=True)
    return np.triu(Minv[::-1, ::-1])


# ---------------------------------------------------------------------------------------
# Quantiser and GPTQ sweep  ([gptq] experiment summary and analytic check)
# ---------------------------------------------------------------------------------------

_F32_SEVEN = np.float32(7.0)


def _group_scale(absmax) -> np.ndarray:
    """Per-(row, group) scale s = absmax / 7, as fp32 (fp32 absmax, IEEE fp32 division)."""
    return (np.asarray(absmax, dtype=np.float64).astype(np.float32) / _F32_SEVEN).astype(np.float32)


def _round_code(w, s) -> np.ndarray:
    """Code c = clamp(rint(fp32(w) / s), -8, 7), decided in fp32; s == 0 gives c = 0."""
    w32 = np.asarray(w, dtype=np.float64).astype(np.float32)
    s32 = np.asarray(s, dtype=np.float32)
    safe = np.where(s32 > 0, s32, np.float32(1.0))
    ratio = (w32 / safe).astype(np.float32)
    c = np.clip(np.rint(ratio), -8.0, 7.0)
    c = np.where(s32 > 0, c, 0.0)
    return c.astype(np.int8)


def gptq_sweep(W, U, group: int):
    """Error-compensated column-sequential sweep, unblocked (one column at a time).

    For j = 0..K-1 over every row at once:
      * at a group start (j % group == 0) the scale of the group is taken from the current
        weights of its columns, s = fp32(max |Wc[n, j:j+group]| / 7);
      * c = clamp(rint(Wc[n, j] / s), -8, 7), q = c * s;
      * e = (Wc[n, j] - q) / U[j, j];
      * Wc[n, k] -= e * U[j, k] for every k > j.
    Returns (codes int8 [N, K], scales fp32 [N, K/group], errors e fp64 [N, K]).
    """
    Wc = np.array(W, dtype=np.float64, copy=True)
    U = np.asarray(U, dtype=np.float64)
    N, K = Wc.shape
    if K % group:
        raise ValueError("group must divide K")
    codes = np.zeros((N, K), dtype=np.int8)
    scales = np.zeros((N, K // group), dtype=np.float32)
    E = np.zeros((N, K), dtype=np.float64)
    for j in range(K):
        g = j // group
        if j % group == 0:
            scales[:, g] = _group_scale(np.max(np.abs(Wc[:, j:j + group]), axis=1))
        s = scales[:, g]
        c = _round_code(Wc[:, j], s)
        q = c.astype(np.float64) * s.astype(np.float64)
        e = (Wc[:, j] - q) / U[j, j]
        if j + 1 < K:
            Wc[:, j + 1:] -= np.outer(e, U[j, j + 1:])
        codes[:, j] = c
        E[:, j] = e
    return codes, scales, E


def gptq_sweep_forced(W, U, group: int, forced_codes):
    """The same sweep with every code decision replaced by `forced_codes` (teacher forcing).

    Used to compare another implementation's scales and errors on ITS OWN code trajectory:
    once two implementations round one near-tie differently, the error feedback moves every
    later weight of that row, so plain element-wise comparison of later scales is meaningless.
    Besides (scales, errors) it returns, for every column, the code the unforced rule would
    pick from the same current weight, and the ratio w / s that rule rounds.
    Returns (scales fp32 [N, K/group], errors fp64 [N, K], free_codes int8 [N, K],
    ratios fp32 [N, K]).
    """
    Wc = np.array(W, dtype=np.float64, copy=True)
    U = np.asarray(U, dtype=np.float64)
    C = np.asarray(forced_codes).astype(np.float64)
    N, K = Wc.shape
    if K % group:
        raise ValueError("group must divide K")
    scales = np.zeros((N, K // group), dtype=np.float32)
    E = np.zeros((N, K), dtype=np.float64)
    free = np.zeros((N, K), dtype=np.int8)
    ratios = np.zeros((N, K), dtype=np.float32)
    for j in range(K):
        g = j // group
        if j % group == 0:
            scales[:, g] = _group_scale(np.max(np.abs(Wc[:, j:j + group]), axis=1))
        s = scales[:, g]
        free[:, j] = _round_code(Wc[:, j], s)
        safe = np.where(s > 0, s, np.float32(1.0))
        ratios[:, j] = np.where(s > 0, (Wc[:, j].astype(np.float32) / safe).astype(np.float32), 0.0)
        q = C[:, j] * s.astype(np.float64)
        e = (Wc[:, j] - q) / U[j, j]
        if j + 1 < K:
            Wc[:, j + 1:] -= np.outer(e, U[j, j + 1:])
        E[:, j] = e
    return scales, E, free, ratios


def gptq_quantize(W, H, group: int, damp: float):
    """Whole GPTQ path on an undamped Hessian: damp, U = upper Cholesky factor of the inverse,
    sweep.  Returns dict(codes, scales, errors, U, lam)."""
    Hd, lam = damp_hessian(H, damp)
    U = upper_factor_of_inverse(Hd)
    codes, scales, E = gptq_sweep(W, U, group)
    return {"codes": codes, "scales": scales, "errors": E, "U": U, "lam": lam}


def rtn_quantize(W, group: int):
    """Round-to-nearest with the same quantiser and no compensation (ork's absmax/7)."""
    W64 = np.asarray(W, dtype=np.float64)
    N, K = W64.shape
    if K % group:
        raise ValueError("group must divide K")
    Wg = W64.reshape(N, K // group, group)
    scales = _group_scale(np.max(np.abs(Wg), axis=2))
    codes = _round_code(Wg, scales[:, :, None]).reshape(N, K)
    return codes, scales


def dequantize(codes, scales, group: int) -> np.ndarray:
    """q = code * scale in fp64."""
    c = np.asarray(codes, dtype=np.float64)
    s = np.repeat(np.asarray(scales, dtype=np.float64), group, axis=1)
    return c * s


def qerr(W, codes, scales, group: int, imp=None) -> float:
    """sqrt(sum_n sum_k imp[k](w - q)^2 / sum_n sum_k imp[k] w^2), imp = 1 when None,
    with the original weights w.  An all-zero W gives 0."""
    W64 = np.asarray(W, dtype=np.float64)
    D = W64 - dequantize(codes, scales, group)
    if imp is None:
        imp64 = np.ones(W64.shape[1])
    else:
        imp64 = np.asarray(imp, dtype=np.float64)
    num = float(np.sum((D * D) @ imp64))
    den = float(np.sum((W64 * W64) @ imp64))
    return 0.0 if den == 0.0 else float(np.sqrt(num / den))


def layer_loss(W, codes, scales, group: int, H) -> float:
    """tr((W - Q) H (W - Q)^T) with the undamped H."""
    D = np.asarray(W, dtype=np.float64) - dequantize(codes, scales, group)
    return float(np.sum((D @ np.asarray(H, dtype=np.float64)) * D))


def pack_int4(codes) -> np.ndarray:
    """Two codes per byte, even column in the low nibble, 4-bit two's complement."""
    c = np.asarray(codes, dtype=np.int16)
    if c.shape[-1] % 2:
        raise ValueError("K must be even")
    lo = c[..., 0::2] & 0xF
    hi = c[..., 1::2] & 0xF
    return (lo | (hi << 4)).astype(np.uint8)


def unpack_int4(packed) -> np.ndarray:
    p = np.asarray(packed, dtype=np.int16)
    lo = p & 0xF
    hi = (p >> 4) & 0xF
    lo = np.where(lo >= 8, lo - 16, lo)
    hi = np.where(hi >= 8, hi - 16, hi)
    out = np.empty(p.shape[:-1] + (2 * p.shape[-1],), dtype=np.int8)
    out[..., 0::2] = lo
    out[..., 1::2] = hi
    return out


# ---------------------------------------------------------------------------------------
# Bf16TrilDiagF32 codec  ([calib] "Hessian storage: Bf16TrilDiagF32 (quant_type 130)")
# ---------------------------------------------------------------------------------------

def bf16tril_bytes(K: int) -> int:
    """K*4 + K*(K-1)/2 * 2 bytes."""
    return K * 4 + (K * (K - 1) // 2) * 2


def truncate_f32_to_bf16_bits(x) -> np.ndarray:
    """bf16 by truncation: the top 16 bits of the fp32 bit pattern (f32_bits >> 16)."""
    bits = np.ascontiguousarray(np.asarray(x, dtype=np.float32)).view(np.uint32)
    return (bits >> np.uint32(16)).astype(np.uint16)


def bf16tril_encode(H) -> bytes:
    """Diagonal as exact little-endian f32 (K*4 bytes), then the strict lower triangle as
    little-endian bf16 at index i*(i-1)/2 + j for i > j, written row by row."""
    H32 = np.ascontiguousarray(np.asarray(H, dtype=np.float32))
    K = H32.shape[0]
    if H32.shape != (K, K):
        raise ValueError("H must be square")
    diag = np.array([H32[i, i] for i in range(K)], dtype="<f4")
    tri = np.zeros(K * (K - 1) // 2, dtype="<u2")
    for i in range(1, K):
        base = i * (i - 1) // 2
        tri[base:base + i] = truncate_f32_to_bf16_bits(H32[i, :i])
    out = diag.tobytes() + tri.tobytes()
    assert len(out) == bf16tril_bytes(K)
    return out


def bf16tril_decode(buf, K: int) -> np.ndarray:
    """Full symmetric fp32 H: diagonal from the f32 block, H[i,j] = H[j,i] = bf16 bits << 16."""
    raw = bytes(buf) if not isinstance(buf, (bytes, bytearray)) else buf
    if len(raw) != bf16tril_bytes(K):
        raise ValueError("buffer size does not match K")
    diag = np.frombuffer(raw[:4 * K], dtype="<f4")
    tri = np.frombuffer(raw[4 * K:], dtype="<u2")
    H = np.zeros((K, K), dtype=np.float32)
    for i in range(1, K):
        base = i * (i - 1) // 2
        row = (tri[base:base + i].astype(np.uint32) << np.uint32(16)).view(np.float32)
        H[i, :i] = row
        H[:i, i] = row
    for i in range(K):
        H[i, i] = diag[i]
    return H
