"""Pins for the fp64 oracle: each checks it against something other than itself -- values
the pages print, closed forms, brute force on tiny inputs, invariants that a plausible
mistake (a dropped term, a wrong sign or index, a transposed operand) breaks.

CPU only.  The mutation tests at the end plant mistakes in copies of oracle routines (on the
CPU) and check that the pins catch them.
"""

import itertools
import math
import os

import numpy as np
import pytest

import oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _read_golden(name):
    rows = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            rows.append(line.split())
    return rows


def _spd(K, rng, cond_spread=3.0, corr=0.5):
    """A random symmetric positive definite matrix with varied diagonal scale."""
    A = rng.standard_normal((K, 2 * K))
    H = A @ A.T / (2 * K)
    H = (1 - corr) * np.diag(np.diag(H)) + corr * H
    d = np.exp(cond_spread * rng.standard_normal(K) / 2)
    return H * np.outer(d, d)


# ----------------------------------------------------------------------------- codec

def test_codec_size_formula_matches_page():
    for K, nbytes in _read_golden("bf16tril_sizes.txt"):
        K, nbytes = int(K), int(nbytes)
        assert O.bf16tril_bytes(K) == nbytes
        if K <= 128:
            H = np.zeros((K, K), np.float32)
            assert len(O.bf16tril_encode(H)) == nbytes


def test_codec_sizes_consistent_with_package_size():
    # The card: ~31.5 GB for 496 tensors, ~63 MB per Hessian on average; the K values it
    # names are 5120, 6144 and 17408.  The mean must lie inside the span of the formula.
    sizes = [O.bf16tril_bytes(K) for K in (5120, 6144, 17408)]
    assert min(sizes) < 63e6 < max(sizes)
    assert abs(31.5e9 / 496 - 63e6) / 63e6 < 0.01


def test_truncation_examples():
    for f32_bits, bf16_bits, *_ in _read_golden("bf16_truncation.txt"):
        x = np.array([int(f32_bits, 16)], dtype=np.uint32).view(np.float32)
        assert int(O.truncate_f32_to_bf16_bits(x)[0]) == int(bf16_bits, 16)


def test_codec_index_layout_and_mirror():
    # K = 4 with every entry distinct and exactly representable in bf16.
    K = 4
    H = np.zeros((K, K), np.float32)
    for i in range(K):
        for j in range(K):
            H[i, j] = 10 * i + j + 1 if i >= j else -1.0  # upper triangle never read
    buf = O.bf16tril_encode(H)
    diag = np.frombuffer(buf[:16], "<f4")
    tri = np.frombuffer(buf[16:], "<u2")
    assert list(diag) == [1.0, 12.0, 23.0, 34.0]
    as_f32 = (tri.astype(np.uint32) << 16).view(np.float32)
    # index i(i-1)/2 + j: (1,0)->0, (2,0)->1, (2,1)->2, (3,0)->3, (3,1)->4, (3,2)->5
    assert list(as_f32) == [11.0, 21.0, 22.0, 31.0, 32.0, 33.0]
    D = O.bf16tril_decode(buf, K)
    for i in range(K):
        for j in range(K):
            lo, hi = max(i, j), min(i, j)
            assert D[i, j] == 10 * lo + hi + 1


def test_codec_k1_and_k2():
    H1 = np.array([[3.5]], np.float32)
    b = O.bf16tril_encode(H1)
    assert len(b) == 4 and np.frombuffer(b, "<f4")[0] == 3.5
    assert O.bf16tril_decode(b, 1)[0, 0] == 3.5
    H2 = np.array([[1.0, 9.0], [np.float32(1.0000153), 2.0]], np.float32)
    b = O.bf16tril_encode(H2)
    assert len(b) == 10
    assert np.frombuffer(b[8:], "<u2")[0] == 0x3F80


def test_codec_truncation_invariants():
    rng = np.random.default_rng(1)
    K = 300
    H = (rng.standard_normal((K, K)) * np.exp(rng.standard_normal((K, K)) * 3)).astype(np.float32)
    H = np.tril(H) + np.tril(H, -1).T
    buf = O.bf16tril_encode(H)
    D = O.bf16tril_decode(buf, K)
    assert np.array_equal(np.diag(D), np.diag(H))            # diagonal exact
    off = ~np.eye(K, dtype=bool)
    h, d = H[off].astype(np.float64), D[off].astype(np.float64)
    nz = h != 0
    assert np.all(np.abs(d) <= np.abs(h))                     # truncation toward zero
    assert np.all(np.sign(d[nz]) == np.sign(h[nz]))
    rel = (np.abs(h[nz]) - np.abs(d[nz])) / np.abs(h[nz])
    assert rel.min() >= 0 and rel.max() < 2.0 ** -7
    # The card's "~0.391 %" bf16 step is the unit 2^-8 = 0.390625 %; truncation drops a
    # fraction u ~ U(0,1) of one bf16 ulp (2^-7 relative at mantissa m), so the relative
    # error is u 2^-7 / m: below 2 x 0.391 % always, and 2^-9 / ln 2 on average for the
    # log-uniform mantissas of these lognormal entries.
    assert abs(0.00391 - 2.0 ** -8) < 5e-6
    assert abs(rel.mean() - 2.0 ** -9 / math.log(2)) / (2.0 ** -9 / math.log(2)) < 0.03
    assert O.bf16tril_encode(D) == buf                         # encode∘decode∘encode = encode
    assert np.array_equal(D, D.T)


# ----------------------------------------------------------------------------- Hessian

def test_hessian_bruteforce_and_properties():
    rng = np.random.default_rng(2)
    T, K = 7, 5
    X = rng.standard_normal((T, K))
    H = O.hessian(X)
    for i in range(K):
        for j in range(K):
            s = 0.0
            for t in range(T):
                s += X[t, i] * X[t, j]
            assert abs(H[i, j] - s) < 1e-12
    assert np.array_equal(H, H.T)
    assert np.linalg.eigvalsh(H).min() > -1e-12
    # chunked accumulation is addition
    Hc = O.hessian_accumulate(O.hessian(X[:3]), X[3:])
    assert np.allclose(Hc, H, rtol=0, atol=1e-12)
    imp = O.imatrix(H, T)
    assert np.allclose(imp, (X ** 2).mean(axis=0), rtol=1e-14)


def test_damping_relative_to_mean_diag():
    H = np.diag([1.0, 2.0, 3.0, 6.0])
    Hd, lam = O.damp_hessian(H, 0.01)
    assert lam == pytest.approx(0.03)
    assert np.allclose(np.diag(Hd), [1.03, 2.03, 3.03, 6.03])
    with pytest.raises(ValueError):
        O.damp_hessian(np.zeros((3, 3)), 0.01)


def test_upper_factor_2x2_closed_form():
    a, b, c = 4.0, 1.5, 2.0
    det = a * c - b * b
    U = O.upper_factor_of_inverse(np.array([[a, b], [b, c]]))
    u11 = math.sqrt(c / det)
    u12 = -b / math.sqrt(c * det)
    u22 = 1.0 / math.sqrt(c)
    assert np.allclose(U, [[u11, u12], [0.0, u22]], rtol=1e-14, atol=1e-15)


def test_cholesky_chain_invariants():
    rng = np.random.default_rng(3)
    K = 96
    H = _spd(K, rng)
    Hd, lam = O.damp_hessian(H, 0.01)
    L = O.cholesky_lower(Hd)
    assert np.allclose(L @ L.T, Hd, rtol=0, atol=1e-12 * np.abs(Hd).max())
    U = O.upper_factor_of_inverse(Hd)
    assert np.array_equal(U, np.triu(U)) and np.all(np.diag(U) > 0)
    I = U @ Hd @ U.T
    assert np.abs(I - np.eye(K)).max() < 1e-9
    Ur = O.upper_factor_by_reversal(Hd)
    assert np.linalg.norm(U - Ur) / np.linalg.norm(U) < 1e-10


def test_not_positive_definite_raises():
    H = np.diag([5.0, 5.0, 5.0, -1.0])
    Hd, _ = O.damp_hessian(H, 0.01)
    with pytest.raises(O.NotPositiveDefinite):
        O.upper_factor_of_inverse(Hd)


# ----------------------------------------------------------------------------- quantiser

def _rtn_uniform_expected(G):
    # Given the group absmax M the other G-1 entries are U(-M, M); rounding on the step
    # M/7 leaves an error of variance (M/7)^2/12, the maximal entry none.  E[M^2] = G/(G+2),
    # E[w^2] = 1/3  ->  qerr^2 = (G-1) / (196 (G+2)), which tends to (1/14)^2.
    return math.sqrt((G - 1) / (196.0 * (G + 2)))


def test_page_analytic_table_arithmetic():
    g = {r[0]: (float(r[1]), float(r[2])) for r in _read_golden("rtn_uniform_analytic.txt")}
    step = 1.0 / 7.0
    assert abs(step - g["step"][0]) <= g["step"][1]
    assert abs(step / math.sqrt(12) - g["rms_quant_error"][0]) <= g["rms_quant_error"][1]
    assert abs(1 / math.sqrt(3) - g["rms_w"][0]) <= g["rms_w"][1]
    pred = (step / math.sqrt(12)) / (1 / math.sqrt(3))
    assert abs(pred - g["predicted_qerr"][0]) <= g["predicted_qerr"][1]
    assert abs(_rtn_uniform_expected(10 ** 9) - pred) < 1e-8
    # the measured 0.07117 is within 0.4 % of the prediction, as the page says
    assert abs(g["measured_qerr"][0] - pred) / pred < 0.004


@pytest.mark.parametrize("N,K,G", [(1024, 4096, 4096), (512, 4096, 128), (256, 4096, 32)])
def test_rtn_qerr_uniform_closed_form(N, K, G):
    rng = np.random.default_rng(4)
    W = rng.uniform(-1, 1, (N, K)).astype(np.float32)
    codes, scales = O.rtn_quantize(W, G)
    q = O.qerr(W, codes, scales, G)
    assert abs(q - _rtn_uniform_expected(G)) / _rtn_uniform_expected(G) < 0.003
    assert codes.min() >= -7 and codes.max() <= 7          # |w/s| <= 7 without compensation


def test_rtn_exact_grid_and_zero_group():
    rng = np.random.default_rng(5)
    N, K, G = 8, 64, 16
    s = np.float32(2.0 ** -5)
    codes = rng.integers(-7, 8, (N, K))
    codes[:, ::G] = 7  # every group reaches absmax 7 s exactly
    W = (codes * s).astype(np.float32)
    W[0, :G] = 0.0
    c, sc = O.rtn_quantize(W, G)
    expect = codes.copy()
    expect[0, :G] = 0
    assert np.array_equal(c, expect)
    assert sc[0, 0] == 0.0 and np.all(sc[:, 1:] == s)
    assert O.qerr(W, c, sc, G) == 0.0


def test_pack_int4_layout():
    codes = np.array([[-8, 7, -1, 0, 3, -3]], np.int8)
    p = O.pack_int4(codes)
    assert list(p[0]) == [0x78, 0x0F, 0xD3]
    assert np.array_equal(O.unpack_int4(p), codes)


# ----------------------------------------------------------------------------- GPTQ

def test_gptq_diagonal_hessian_is_rtn():
    rng = np.random.default_rng(6)
    N, K, G = 32, 256, 32
    W = rng.standard_normal((N, K)).astype(np.float32)
    H = np.diag(np.exp(rng.standard_normal(K)))
    r = O.gptq_quantize(W, H, G, 0.01)
    c, s = O.rtn_quantize(W, G)
    assert np.array_equal(r["codes"], c)
    assert np.array_equal(r["scales"], s)
    assert O.qerr(W, r["codes"], r["scales"], G) == O.qerr(W, c, s, G)


def test_gptq_large_damping_limit_is_rtn():
    # "once damp ~ mean(diag(H)) ... GPTQ degenerates to round-to-nearest"
    rng = np.random.default_rng(7)
    N, K, G = 32, 128, 32
    W = rng.uniform(-1, 1, (N, K)).astype(np.float32)
    H = _spd(K, rng, corr=0.9)
    r = O.gptq_quantize(W, H, G, 1e9)
    c, s = O.rtn_quantize(W, G)
    assert np.array_equal(r["codes"], c) and np.array_equal(r["scales"], s)
    r_small = O.gptq_quantize(W, H, G, 0.01)
    assert not np.array_equal(r_small["codes"], c)


def test_gptq_loss_identity():
    # D = W - Q = E U row by row and U H' U^T = I, so tr(D H' D^T) = sum e^2 exactly, and
    # the undamped loss is sum e^2 - lambda ||D||_F^2.
    rng = np.random.default_rng(8)
    N, K, G = 24, 192, 64
    W = rng.standard_normal((N, K)).astype(np.float32)
    H = _spd(K, rng, corr=0.8)
    r = O.gptq_quantize(W, H, G, 0.01)
    Hd, lam = O.damp_hessian(H, 0.01)
    D = W.astype(np.float64) - O.dequantize(r["codes"], r["scales"], G)
    lhs = float(np.sum((D @ Hd) * D))
    se2 = float(np.sum(r["errors"] ** 2))
    assert abs(lhs - se2) / se2 < 1e-9
    loss = O.layer_loss(W, r["codes"], r["scales"], G, H)
    assert abs(loss - (se2 - lam * float(np.sum(D * D)))) / loss < 1e-9
    assert np.allclose(D, r["errors"] @ r["U"], rtol=0, atol=1e-12)


def test_gptq_exact_grid_is_recovered():
    rng = np.random.default_rng(9)
    N, K, G = 16, 128, 32
    s = np.float32(2.0 ** -3)
    codes = rng.integers(-7, 8, (N, K))
    codes[:, ::G] = -7
    W = (codes * s).astype(np.float32)
    H = _spd(K, rng, corr=0.9)
    r = O.gptq_quantize(W, H, G, 0.01)
    assert np.array_equal(r["codes"], codes)
    assert np.all(r["errors"] == 0.0)
    assert O.qerr(W, r["codes"], r["scales"], G) == 0.0


def test_gptq_last_column_is_conditionally_optimal():
    # With all earlier codes fixed, the damped loss is a convex quadratic in the last
    # column's error; the sweep moves that column to its continuous conditional optimum
    # and rounds it, so no other code of the last column does better (the K = 2 argument,
    # applied to the final column of every row).
    rng = np.random.default_rng(10)
    N, K, G = 500, 8, 4
    W = rng.uniform(-1, 1, (N, K)).astype(np.float32)
    A = rng.standard_normal((K, K))
    H = A @ A.T + 0.5 * np.ones((K, K)) * K
    Hd, _ = O.damp_hessian(H, 0.01)
    r = O.gptq_quantize(W, H, G, 0.01)
    s_last = r["scales"][:, -1].astype(np.float64)
    D = W - O.dequantize(r["codes"], r["scales"], G)
    base = np.einsum("nk,kl,nl->n", D, Hd, D)
    moved = 0
    for alt in range(-8, 8):
        D2 = D.copy()
        D2[:, -1] = W[:, -1] - alt * s_last
        l2 = np.einsum("nk,kl,nl->n", D2, Hd, D2)
        assert np.all(base <= l2 * (1 + 1e-12) + 1e-300)
    # and the compensation really moved some last-column codes away from plain rounding
    c, _ = O.rtn_quantize(W, G)
    moved = int(np.sum(r["codes"][:, -1] != c[:, -1]))
    assert moved > 10


def test_gptq_k4_bruteforce():
    rng = np.random.default_rng(11)
    K, G = 4, 4
    H = np.array([[1.0, 0.7, 0.4, 0.2], [0.7, 1.0, 0.7, 0.4], [0.4, 0.7, 1.0, 0.7], [0.2, 0.4, 0.7, 1.0]])
    Hd, _ = O.damp_hessian(H, 0.01)
    grid = np.array(list(itertools.product(range(-8, 8), repeat=K)), dtype=np.float64)  # 65536 x 4
    N = 1000
    W = rng.uniform(-1, 1, (N, K)).astype(np.float32)
    r = O.gptq_quantize(W, H, G, 0.01)
    c, s = O.rtn_quantize(W, G)
    assert np.array_equal(r["scales"], s)
    Dg = W - O.dequantize(r["codes"], r["scales"], G)
    Dr = W - O.dequantize(c, s, G)
    lg = np.einsum("nk,kl,nl->n", Dg, Hd, Dg)
    lr = np.einsum("nk,kl,nl->n", Dr, Hd, Dr)
    for n in range(0, N, 5):  # brute force on every 5th row
        D = W[n].astype(np.float64)[None, :] - grid * float(s[n, 0])
        best = np.min(np.einsum("gk,kl,gl->g", D, Hd, D))
        assert best <= lg[n] * (1 + 1e-12) and best <= lr[n] * (1 + 1e-12)
    assert lg.sum() <= lr.sum()


def test_forced_sweep_reproduces_free_sweep_and_keeps_loss_identity():
    rng = np.random.default_rng(17)
    N, K, G = 16, 128, 32
    W = rng.standard_normal((N, K)).astype(np.float32)
    Hd, _ = O.damp_hessian(_spd(K, rng, corr=0.9), 0.01)
    U = O.upper_factor_of_inverse(Hd)
    codes, scales, E = O.gptq_sweep(W, U, G)
    s2, E2, free, ratios = O.gptq_sweep_forced(W, U, G, codes)
    assert np.array_equal(s2, scales) and np.array_equal(E2, E) and np.array_equal(free, codes)
    # forcing other codes: D = E U still holds, so tr(D H' D^T) = sum e^2 for ANY codes
    other = np.clip(codes + rng.integers(-1, 2, codes.shape), -8, 7)
    s3, E3, free3, _ = O.gptq_sweep_forced(W, U, G, other)
    D = W - O.dequantize(other, s3, G)
    assert abs(float(np.sum((D @ Hd) * D)) - float(np.sum(E3 ** 2))) / float(np.sum(E3 ** 2)) < 1e-9
    assert not np.array_equal(free3, other)


def test_gptq_scale_invariance_of_hessian():
    rng = np.random.default_rng(12)
    N, K, G = 16, 128, 32
    W = rng.standard_normal((N, K)).astype(np.float32)
    H = _spd(K, rng, corr=0.8)
    a = O.gptq_quantize(W, H, G, 0.01)
    b = O.gptq_quantize(W, 4.0 * H, G, 0.01)
    assert np.array_equal(a["codes"], b["codes"]) and np.array_equal(a["scales"], b["scales"])


def test_gptq_row_permutation():
    rng = np.random.default_rng(13)
    N, K, G = 20, 128, 64
    W = rng.standard_normal((N, K)).astype(np.float32)
    H = _spd(K, rng, corr=0.8)
    perm = rng.permutation(N)
    a = O.gptq_quantize(W, H, G, 0.01)
    b = O.gptq_quantize(W[perm], H, G, 0.01)
    assert np.array_equal(a["codes"][perm], b["codes"]) and np.array_equal(a["scales"][perm], b["scales"])


def test_group_scale_uses_compensated_weights():
    # 1 row, K = 4, group 2, worked by hand with exactly representable values.
    # Column 0: s = 0.875/7 = 0.125, 0.8125/0.125 = 6.5 rounds half-to-even to 6, q = 0.75,
    # e = 0.0625, and U[0, 2] = 1 moves W[0, 2] from 0.5 to 0.4375.  The scale of group 1
    # must then come from the moved weights: absmax(0.4375, 0.45) = 0.45, not 0.5.
    W = np.array([[0.8125, 0.875, 0.5, 0.45]], np.float32)
    U = np.eye(4)
    U[0, 2] = 1.0
    codes, scales, E = O.gptq_sweep(W, U, 2)
    assert scales[0, 0] == np.float32(0.125)
    assert codes[0, 0] == 6 and E[0, 0] == 0.0625
    assert codes[0, 1] == 7 and E[0, 1] == 0.0
    assert scales[0, 1] == np.float32(np.float32(0.45) / np.float32(7))
    assert scales[0, 1] != np.float32(np.float32(0.5) / np.float32(7))


def test_qerr_importance_properties():
    rng = np.random.default_rng(14)
    N, K, G = 32, 256, 32
    W = rng.uniform(-1, 1, (N, K)).astype(np.float32)
    c, s = O.rtn_quantize(W, G)
    imp = np.exp(rng.standard_normal(K))
    a = O.qerr(W, c, s, G, imp)
    assert a != O.qerr(W, c, s, G)                       # an importance vector moves the value
    assert a == pytest.approx(O.qerr(W, c, s, G, imp * 1024.0), rel=1e-13)  # scale cancels
    assert O.qerr(W, c, s, G, np.ones(K)) == pytest.approx(O.qerr(W, c, s, G), rel=1e-15)
    assert 0.0 <= a < 1.0


# ----------------------------------------------------------------------------- mutations

def _sweep_mutant(W, U, group, mutation):
    Wc = np.array(W, dtype=np.float64)
    N, K = Wc.shape
    codes = np.zeros((N, K), np.int8)
    scales = np.zeros((N, K // group), np.float32)
    E = np.zeros((N, K))
    for j in range(K):
        g = j // group
        if j % group == 0:
            scales[:, g] = O.hq_oracle._group_scale(np.max(np.abs(Wc[:, j:j + group]), axis=1))
        s = scales[:, g]
        c = O.hq_oracle._round_code(Wc[:, j], s)
        q = c * s.astype(np.float64)
        e = (Wc[:, j] - q) / U[j, j]
        row = U[j, j + 1:] if mutation != "transposed" else U[j + 1:, j]
        if mutation == "sign":
            Wc[:, j + 1:] += np.outer(e, row)
        elif mutation == "dropped_term":
            if j + 2 < K:
                Wc[:, j + 2:] -= np.outer(e, U[j, j + 2:])
        else:
            Wc[:, j + 1:] -= np.outer(e, row)
        codes[:, j] = c
        E[:, j] = e
    return codes, scales, E


@pytest.mark.parametrize("mutation", ["sign", "dropped_term", "transposed"])
def test_loss_identity_catches_planted_sweep_mistakes(mutation):
    rng = np.random.default_rng(15)
    N, K, G = 8, 64, 32
    W = rng.standard_normal((N, K)).astype(np.float32)
    H = _spd(K, rng, corr=0.8)
    Hd, _ = O.damp_hessian(H, 0.01)
    U = O.upper_factor_of_inverse(Hd)
    codes, scales, E = _sweep_mutant(W, U, G, mutation)
    D = W - O.dequantize(codes, scales, G)
    lhs = float(np.sum((D @ Hd) * D))
    assert abs(lhs - float(np.sum(E ** 2))) / float(np.sum(E ** 2)) > 1e-6


def test_truncation_pin_catches_round_to_nearest():
    x = np.array([0x3F808001], np.uint32).view(np.float32)
    bits = x.view(np.uint32).astype(np.uint64)
    rne = ((bits + 0x7FFF + ((bits >> 16) & 1)) >> 16).astype(np.uint16)  # a plausible mistake
    golden = {int(a, 16): int(b, 16) for a, b, *_ in _read_golden("bf16_truncation.txt")}
    assert int(rne[0]) != golden[0x3F808001]
    assert int(O.truncate_f32_to_bf16_bits(x)[0]) == golden[0x3F808001]


def test_factor_pins_catch_transposed_factor():
    rng = np.random.default_rng(16)
    K = 32
    Hd, _ = O.damp_hessian(_spd(K, rng, corr=0.8), 0.01)
    U = O.upper_factor_of_inverse(Hd)
    wrong = np.linalg.cholesky(np.linalg.inv(Hd))  # lower factor instead of upper
    assert np.abs(U @ Hd @ U.T - np.eye(K)).max() < 1e-9
    assert np.abs(np.triu(wrong) @ Hd @ np.triu(wrong).T - np.eye(K)).max() > 1e-3


# ----------------------------------------------------------------------------- PSD projection

def test_psd_projection_2x2_closed_form():
    """[calib] "The fix" on a 2 x 2 symmetric matrix with one negative eigenvalue: the result
    is l+ v v^T with l+ = (a + c)/2 + sqrt(((a - c)/2)^2 + b^2) and v the unit vector along
    (b, l+ - a), written out by hand."""
    for a, b, c in ((1.0, 2.0, 0.5), (-1.0, 0.3, 2.0), (0.2, -1.5, 0.1)):
        lp = (a + c) / 2 + math.sqrt(((a - c) / 2) ** 2 + b * b)
        lm = (a + c) / 2 - math.sqrt(((a - c) / 2) ** 2 + b * b)
        assert lm < 0 < lp
        v = np.array([b, lp - a])
        v /= np.linalg.norm(v)
        want = lp * np.outer(v, v)
        got = O.project_psd(np.array([[a, b], [b, c]]))
        assert np.allclose(got, want, rtol=0, atol=1e-14)


def test_psd_projection_diagonal_clips_and_psd_input_unchanged():
    d = np.array([3.0, -1.0, 0.0, 2.5, -4.0])
    assert np.array_equal(O.project_psd(np.diag(d)), np.diag(np.maximum(d, 0.0)))
    rng = np.random.default_rng(2)
    A = rng.standard_normal((40, 60))
    H = A @ A.T
    assert np.abs(O.project_psd(H) - H).max() <= 1e-12 * np.abs(H).max()


def test_psd_projection_nearest_psd_properties():
    """The projection onto the PSD cone (nearest in Frobenius norm): P is PSD, idempotent,
    orthogonal to H - P (<P, H - P> = 0), and ||H - P||^2 is the sum of the squared negative
    eigenvalues of H."""
    rng = np.random.default_rng(9)
    B = rng.standard_normal((50, 50))
    H = (B + B.T) / 2
    P = O.project_psd(H)
    l = np.linalg.eigvalsh(H)
    assert np.linalg.eigvalsh(P).min() >= -1e-12 * np.abs(l).max()
    assert np.abs(O.project_psd(P) - P).max() <= 1e-12 * np.abs(P).max()
    assert abs(np.sum(P * (H - P))) <= 1e-12 * np.sum(H * H)
    assert np.sum((H - P) ** 2) == pytest.approx(np.sum(l[l < 0] ** 2), rel=1e-10)


def test_psd_projection_of_a_bf16_stored_hessian_is_small():
    """[calib] "The fix": on a Hessian stored with bf16 off-diagonals, the projection removes
    less than bf16's own quantisation step (2^-8 relative); the stored matrix is indefinite."""
    import workloads as wl
    cfg = wl.correlated_config(16, 512, T=2048, group=128, seed=3)
    X = wl.make_activations(cfg, "cpu").double().numpy()
    H = (X.T @ X).astype(np.float32)
    Hs = O.bf16tril_decode(O.bf16tril_encode(H), 512)
    assert np.linalg.eigvalsh(Hs).min() < 0
    P = O.project_psd(Hs)
    rel = np.linalg.norm(P - Hs) / np.linalg.norm(Hs)
    assert 0 < rel < 2.0 ** -8


def test_psd_pins_catch_clipping_the_wrong_side():
    def wrong(H):
        l, V = np.linalg.eigh(np.asarray(H, dtype=np.float64))
        P = (V * np.minimum(l, 0.0)) @ V.T
        return (P + P.T) / 2
    d = np.array([3.0, -1.0])
    assert not np.array_equal(wrong(np.diag(d)), np.diag(np.maximum(d, 0.0)))


# ----------------------------------------------------------------------------- Hadamard rotation

def test_hadamard_matrix_sylvester_recursion_and_order_2():
    """The popcount definition against the Sylvester doubling M_2n = [[M, M], [M, -M]] / sqrt 2
    and the hand-written order 2."""
    assert np.allclose(O.hadamard_matrix(2), np.array([[1.0, 1.0], [1.0, -1.0]]) / math.sqrt(2), atol=1e-15)
    M = np.array([[1.0]])
    for n in (2, 4, 8, 16, 32, 64):
        M = np.block([[M, M], [M, -M]]) / math.sqrt(2)
        assert np.allclose(O.hadamard_matrix(n), M, atol=1e-14)
        assert np.allclose(O.hadamard_matrix(n) @ O.hadamard_matrix(n).T, np.eye(n), atol=1e-13)


def test_rotation_is_orthogonal_and_preserves_the_quadratic_form():
    """R orthogonal; W' R^T = W; H' = R^T H R has H's spectrum; the layer's output pairing
    W H W^T is unchanged (trace identity of the loss)."""
    rng = np.random.default_rng(6)
    K, B = 64, 16
    s = rng.choice([-1.0, 1.0], K)
    R = O.hadamard_rotation(s, B)
    assert np.allclose(R.T @ R, np.eye(K), atol=1e-13)
    W = rng.standard_normal((5, K))
    Wr = O.rotate_weights(W, s, B)
    assert np.allclose(Wr @ R.T, W, atol=1e-12)
    A = rng.standard_normal((K, 2 * K))
    H = A @ A.T
    Hr = O.rotate_hessian(np.tril(H), s, B)
    assert np.allclose(np.linalg.eigvalsh(Hr), np.linalg.eigvalsh(H), rtol=1e-10, atol=1e-9)
    assert np.trace(Wr @ Hr @ Wr.T) == pytest.approx(np.trace(W @ H @ W.T), rel=1e-12)


def test_rotation_pins_catch_a_missing_sign_vector():
    rng = np.random.default_rng(7)
    s = rng.choice([-1.0, 1.0], 32)
    W = rng.standard_normal((3, 32))
    wrong = W @ np.kron(np.eye(2), O.hadamard_matrix(16))  # signs dropped
    assert not np.allclose(wrong, O.rotate_weights(W, s, 16))
