"""GPU parity of each stage against the oracle on small and ragged shapes (all through the
C ABI).  Inputs are seeded; the oracle always sees the same bytes the GPU sees, and never
anything the CUDA path produced."""

import numpy as np
import pytest
import torch

import oracle
import workloads as wl
from gpu_helpers import (H_REL_FRO, LOSS_REL, QERR_REL, check_gptq_parity, rel_fro, to_np64, unpack_codes)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def hq():
    import post_weight_quantization_tcgen05_b200 as m
    return m


def _gen(seed, device="cuda"):
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


# ----------------------------------------------------------------------------- codec

def _random_h(K, seed):
    g = _gen(seed)
    H = torch.randn((K, K), generator=g, device="cuda") * torch.exp(3 * torch.randn((K, K), generator=g, device="cuda"))
    if K >= 4:
        bits = H.view(torch.int32)
        bits[1, 0] = 0x7F800000       # +inf
        bits[2, 0] = 0x7FC00001       # NaN
        bits[2, 1] = 0x7F800001       # NaN whose payload sits in the low half
        bits[3, 0] = 0x00000001       # smallest denormal
        bits[3, 1] = -0x80000000      # -0
        bits[3, 2] = 0x3F808001       # 1.0000153: truncation, not rounding
    return H


@pytest.mark.parametrize("K", [1, 2, 3, 4, 5, 12, 64, 127, 128, 129, 516, 1000, 2049, 2052])
def test_codec_encode_bit_exact(hq, cuda_device, K):
    H = _random_h(K, 100 + K)
    out = torch.full((hq.hq_bf16tril_bytes(K),), 0xAB, dtype=torch.uint8, device="cuda")
    hq.hq_hessian_pack_bf16tril(H, out)
    torch.cuda.synchronize()
    ref = oracle.bf16tril_encode(H.cpu().numpy())
    assert out.cpu().numpy().tobytes() == ref


@pytest.mark.parametrize("K", [1, 2, 3, 4, 12, 64, 68, 129, 516, 1000, 2049, 2052])
def test_codec_decode_bit_exact(hq, cuda_device, K):
    nb = hq.hq_bf16tril_bytes(K)
    g = _gen(200 + K)
    buf = torch.randint(0, 256, (nb,), generator=g, device="cuda", dtype=torch.int32).to(torch.uint8)
    Hf = torch.full((K, K), 7.0, device="cuda")
    hq.hq_hessian_unpack_bf16tril(buf, K, Hf)
    torch.cuda.synchronize()
    ref = oracle.bf16tril_decode(buf.cpu().numpy().tobytes(), K)
    assert np.array_equal(Hf.cpu().numpy().view(np.uint32), ref.view(np.uint32))


# ----------------------------------------------------------------------------- SYRK

def _syrk_check(hq, X, impl, chunks=1):
    T, K = X.shape
    H = torch.triu(torch.full((K, K), -123.0, device="cuda"), 1)  # sentinel above the diagonal
    bounds = np.linspace(0, T, chunks + 1).astype(int)
    for a, b in zip(bounds[:-1], bounds[1:]):
        hq.hq_debug_hessian_accumulate_impl(H, X[a:b].contiguous(), impl)
    torch.cuda.synchronize()
    ref = oracle.hessian(to_np64(X))
    Hn = to_np64(H)
    lo = np.tril(np.ones((K, K), bool))
    assert np.all(Hn[~lo] == -123.0), "strict upper triangle must not be touched"
    err = rel_fro(Hn[lo], ref[lo])
    assert err <= H_REL_FRO, err
    return err


@pytest.mark.parametrize("T,K", [(512, 128), (1, 64), (33, 7), (300, 200)])
def test_syrk_fp32_simt(hq, cuda_device, T, K):
    cfg = wl.small_config(wl.CONFIGS[0], N=1, K=K, T=T)
    X = wl.make_activations(cfg, "cuda")
    _syrk_check(hq, X, impl=0)


@pytest.mark.parametrize("T,K", [(64, 128), (1, 128), (100, 256), (4096, 384), (777, 1000), (129, 1032), (2048, 640)])
def test_syrk_bf16_tensor_core(hq, cuda_device, T, K):
    cfg = wl.small_config(wl.CONFIGS[1], N=1, K=K, T=T)
    X = wl.make_activations(cfg, "cuda")
    _syrk_check(hq, X, impl=0)


def test_syrk_bf16_chunked_and_simt_agree(hq, cuda_device):
    cfg = wl.small_config(wl.CONFIGS[1], N=1, K=512, T=3000)
    X = wl.make_activations(cfg, "cuda")
    _syrk_check(hq, X, impl=0, chunks=5)
    _syrk_check(hq, X, impl=1, chunks=2)


def test_syrk_wait_timeout_is_reported_and_the_stream_stays_usable(hq, cuda_device):
    """The bounded-wait failure path, made to run: the MMA issuer never releases the first
    operand stage, so the producer's wait to refill it runs out (limit 1e6 cycles, about half
    a millisecond) before it issues another load.  The call reports HQ_ERR_TIMEOUT through its
    status word, leaves H untouched (no tile finished) and returns; the next ordinary call on
    the same stream then computes the right H."""
    cfg = wl.small_config(wl.CONFIGS[1], N=1, K=128, T=512)
    X = wl.make_activations(cfg, "cuda")
    H = torch.zeros((128, 128), device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    hq.hq_debug_hessian_accumulate_timeout(H, X, status, wait_limit_cycles=1_000_000, withhold_stage=0)
    torch.cuda.synchronize()
    assert status.item() == hq.HQ_ERR_TIMEOUT
    assert torch.count_nonzero(H).item() == 0
    # the same kernel with the short limit and nothing withheld finishes normally
    status.zero_()
    hq.hq_debug_hessian_accumulate_timeout(H, X, status, wait_limit_cycles=1_000_000, withhold_stage=-1)
    torch.cuda.synchronize()
    assert status.item() == 0
    ref = oracle.hessian(to_np64(X))
    lo = np.tril(np.ones((128, 128), bool))
    assert rel_fro(to_np64(H)[lo], ref[lo]) <= H_REL_FRO
    # an ordinary call after the failed one
    H.zero_()
    hq.hq_hessian_accumulate(H, X, dev_status=status)
    torch.cuda.synchronize()
    assert status.item() == 0
    assert rel_fro(to_np64(H)[lo], ref[lo]) <= H_REL_FRO


# ----------------------------------------------------------------------------- factorisation

def _spd(K, seed, corr=0.7):
    rng = np.random.default_rng(seed)
    A = rng.standard_normal((K, 2 * K))
    H = A @ A.T / (2 * K)
    H = (1 - corr) * np.diag(np.diag(H)) + corr * H
    d = np.exp(rng.standard_normal(K))
    return (H * np.outer(d, d)).astype(np.float32)


@pytest.mark.parametrize("K", [128, 256, 640, 1152])
def test_factor_upper_cholesky_of_inverse(hq, cuda_device, K):
    H = _spd(K, K)
    Hd = torch.from_numpy(H).cuda()
    ws = hq.alloc_workspace(hq.hq_gptq_workspace_bytes(1, K, 128))
    Ut = torch.empty((K, K), device="cuda")
    hq.hq_debug_factor(Hd, 0.01, Ut, ws)
    Hdamp, _ = oracle.damp_hessian(H.astype(np.float64), 0.01)
    U = oracle.upper_factor_of_inverse(Hdamp)
    Ug = to_np64(Ut).T
    assert np.array_equal(Ug, np.triu(Ug))
    # fp64 factorisation, rounded once to fp32: the rounding alone gives about 2.5e-8 relative
    # Frobenius on U and 1.2e-7 on U H' U^T - I on these Hessians (kappa 1e3-1e4)
    assert rel_fro(Ug, U) < 1e-7
    I = Ug @ Hdamp @ Ug.T
    assert np.abs(I - np.eye(K)).max() < 1e-6
    # every entry within one fp32 ulp of the oracle's fp64 U (rounding is half an ulp), up to an
    # absolute 1e-10 max|U| for the small entries far from the diagonal, whose last bit an fp64
    # error of that size can flip
    assert np.all(np.abs(Ug - U) <= 2.0 ** -23 * np.abs(U) + 1e-10 * np.abs(U).max())


def test_factor_not_positive_definite(hq, cuda_device):
    K = 128
    H = np.eye(K, dtype=np.float32) * 5
    H[K // 2, K // 2] = -1.0
    ws = hq.alloc_workspace(hq.hq_gptq_workspace_bytes(1, K, 128))
    Ut = torch.empty((K, K), device="cuda")
    with pytest.raises(hq.HQError) as e:
        hq.hq_debug_factor(torch.from_numpy(H).cuda(), 0.01, Ut, ws)
    assert e.value.status == hq.HQ_ERR_NOT_PD
    with pytest.raises(hq.HQError) as e:
        hq.hq_debug_factor(torch.from_numpy(-np.eye(K, dtype=np.float32)).cuda(), 0.01, Ut, ws)
    assert e.value.status == hq.HQ_ERR_INVALID


# ----------------------------------------------------------------------------- GPTQ

def _run_gptq(hq, W, H, group, damp=0.01, imp=None, impl=0):
    N, K = W.shape
    codes, scales = hq.gptq_outputs(N, K, group)
    ws = hq.alloc_workspace(hq.hq_gptq_workspace_bytes(N, K, group))
    q = hq.hq_debug_gptq_quantize_impl(W, H, group, damp, codes, scales, ws, impl, imp=imp)
    torch.cuda.synchronize()
    return unpack_codes(codes), scales.cpu().numpy(), q


def _compare_gptq(W, H64, group, codes_g, scales_g, qerr_g, imp=None, damp=0.01, what=""):
    Wn = to_np64(W)
    Hd, _ = oracle.damp_hessian(H64, damp)
    U = oracle.upper_factor_of_inverse(Hd)
    rc, rs = check_gptq_parity(Wn, U, group, codes_g, scales_g, what)
    r = {"codes": rc, "scales": rs}
    q_ref = oracle.qerr(Wn, r["codes"], r["scales"], group, imp)
    assert abs(qerr_g - q_ref) <= QERR_REL * q_ref + 1e-12, (qerr_g, q_ref)
    l_ref = oracle.layer_loss(Wn, r["codes"], r["scales"], group, H64)
    l_gpu = oracle.layer_loss(Wn, codes_g, scales_g, group, H64)
    assert abs(l_gpu - l_ref) <= LOSS_REL * l_ref + 1e-12, (l_gpu, l_ref)
    # the GPU's own qerr equals the oracle's qerr of the GPU's codes (checks the reduction)
    q_of_gpu = oracle.qerr(Wn, codes_g, scales_g, group, imp)
    assert abs(qerr_g - q_of_gpu) <= 1e-6 * max(q_of_gpu, 1e-12)
    return r


def test_gptq_tiny_layer_pipeline(hq, cuda_device):
    """The tiny configuration end to end: SYRK on the GPU, then GPTQ; the oracle runs its own
    fp64 path from the same X and W."""
    cfg = wl.CONFIGS[0]
    X = wl.make_activations(cfg, "cuda")
    W = wl.make_weights(cfg, "cuda")
    H = torch.zeros((cfg.K, cfg.K), device="cuda")
    hq.hq_hessian_accumulate(H, X)
    codes, scales, q = _run_gptq(hq, W, H, cfg.group, cfg.damp)
    H64 = oracle.hessian(to_np64(X))
    _compare_gptq(W, H64, cfg.group, codes, scales, q, what="tiny")


@pytest.mark.parametrize("impl", [0, 1])
@pytest.mark.parametrize("N,K,group,wdt", [(64, 128, 32, "f32"), (33, 256, 64, "f32"), (1, 384, 128, "bf16"),
                                            (200, 512, 256, "bf16"), (130, 640, 128, "f32")])
def test_gptq_stage_correlated(hq, cuda_device, N, K, group, wdt, impl):
    """Strong compensation (low-rank correlated activations), ragged N, all group kinds,
    both trailing-update kernels; H given as the oracle's own fp32 Hessian."""
    cfg = wl.correlated_config(N, K, T=2 * K, group=group, seed=N + K)
    X = wl.make_activations(cfg, "cpu")
    H64 = oracle.hessian(X.double().numpy())
    H32 = H64.astype(np.float32)
    W = wl.make_weights(cfg, "cpu", N=N, K=K).to(wl.torch_dtype(wdt)).cuda()
    codes, scales, q = _run_gptq(hq, W, torch.from_numpy(H32).cuda(), group, impl=impl)
    _compare_gptq(W, H32.astype(np.float64), group, codes, scales, q, what=f"corr N={N} K={K} g={group}")


def test_gptq_diagonal_hessian_equals_rtn(hq, cuda_device):
    N, K, G = 96, 256, 32
    rng = np.random.default_rng(5)
    W = torch.from_numpy(rng.uniform(-1, 1, (N, K)).astype(np.float32)).cuda()
    H = torch.from_numpy(np.diag(np.exp(rng.standard_normal(K))).astype(np.float32)).cuda()
    c1, s1, q1 = _run_gptq(hq, W, H, G)
    codes, scales = hq.gptq_outputs(N, K, G)
    ws = hq.alloc_workspace(hq.hq_rtn_workspace_bytes(N, K, G))
    q2 = hq.hq_rtn_quantize(W, G, codes, scales, ws)
    c2, s2 = unpack_codes(codes), scales.cpu().numpy()
    assert np.array_equal(c1, c2) and np.array_equal(s1, s2) and abs(q1 - q2) <= 1e-12 * q2
    cr, sr = oracle.rtn_quantize(W.cpu().numpy(), G)
    assert np.array_equal(c2, cr) and np.array_equal(s2, sr)
    assert abs(q2 - oracle.qerr(W.cpu().numpy(), cr, sr, G)) < 1e-12


def test_gptq_outputs_independent_of_qerr_request_and_deterministic(hq, cuda_device):
    cfg = wl.correlated_config(160, 384, T=768, group=128, seed=3)
    X = wl.make_activations(cfg, "cpu")
    H = torch.from_numpy(oracle.hessian(X.double().numpy()).astype(np.float32)).cuda()
    W = wl.make_weights(cfg, "cuda", N=160, K=384)
    N, K, G = 160, 384, 128
    ws = hq.alloc_workspace(hq.hq_gptq_workspace_bytes(N, K, G))
    outs = []
    for want in (True, False, True):
        codes, scales = hq.gptq_outputs(N, K, G)
        qd = torch.zeros(1, dtype=torch.float64, device="cuda")
        q = hq.hq_gptq_quantize(W, H, G, 0.01, codes, scales, ws, want_qerr=want, qerr_dev=qd)
        torch.cuda.synchronize()
        outs.append((codes.cpu().numpy().tobytes(), scales.cpu().numpy().tobytes(), q, qd.item()))
    assert outs[0][0] == outs[1][0] == outs[2][0]
    assert outs[0][1] == outs[1][1] == outs[2][1]
    assert outs[1][2] is None and outs[0][2] == outs[2][2] == outs[0][3] == outs[1][3]


def test_gptq_importance_moves_qerr_and_scale_cancels(hq, cuda_device):
    cfg = wl.correlated_config(64, 256, T=512, group=64, seed=9)
    X = wl.make_activations(cfg, "cpu")
    H64 = oracle.hessian(X.double().numpy())
    H = torch.from_numpy(H64.astype(np.float32)).cuda()
    W = wl.make_weights(cfg, "cuda", N=64, K=256)
    imp = torch.empty(256, device="cuda")
    hq.hq_imatrix(H, 512, imp)
    torch.cuda.synchronize()
    assert np.allclose(imp.cpu().numpy(), oracle.imatrix(H.cpu().numpy().astype(np.float64), 512), rtol=1e-6)
    c0, s0, q0 = _run_gptq(hq, W, H, 64)
    c1, s1, q1 = _run_gptq(hq, W, H, 64, imp=imp)
    c2, s2, q2 = _run_gptq(hq, W, H, 64, imp=imp * 1024)
    assert np.array_equal(c0, c1) and np.array_equal(c1, c2)
    assert q0 != q1
    assert abs(q1 - q2) <= 1e-12 * q1
    assert abs(q1 - oracle.qerr(to_np64(W), c1, s1, 64, imp.cpu().numpy())) <= 1e-6 * q1


def test_gptq_hessian_power_of_two_scaling_is_bit_exact(hq, cuda_device):
    cfg = wl.correlated_config(96, 384, T=768, group=128, seed=4)
    X = wl.make_activations(cfg, "cpu")
    H = torch.from_numpy(oracle.hessian(X.double().numpy()).astype(np.float32)).cuda()
    W = wl.make_weights(cfg, "cuda", N=96, K=384)
    a = _run_gptq(hq, W, H, 128)
    b = _run_gptq(hq, W, H * 4.0, 128)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])


def test_gptq_row_permutation(hq, cuda_device):
    cfg = wl.correlated_config(100, 256, T=512, group=128, seed=6)
    X = wl.make_activations(cfg, "cpu")
    H = torch.from_numpy(oracle.hessian(X.double().numpy()).astype(np.float32)).cuda()
    W = wl.make_weights(cfg, "cuda", N=100, K=256)
    perm = torch.randperm(100, generator=_gen(1, "cpu")).cuda()
    a = _run_gptq(hq, W, H, 128)
    b = _run_gptq(hq, W[perm].contiguous(), H, 128)
    p = perm.cpu().numpy()
    assert np.array_equal(a[0][p], b[0]) and np.array_equal(a[1][p], b[1])


def test_gptq_exact_grid_recovered(hq, cuda_device):
    N, K, G = 64, 256, 32
    rng = np.random.default_rng(11)
    codes = rng.integers(-7, 8, (N, K))
    codes[:, ::G] = 7
    W = torch.from_numpy((codes * 2.0 ** -4).astype(np.float32)).cuda()
    cfg = wl.correlated_config(N, K, T=512, group=G, seed=12)
    X = wl.make_activations(cfg, "cpu")
    H = torch.from_numpy(oracle.hessian(X.double().numpy()).astype(np.float32)).cuda()
    c, s, q = _run_gptq(hq, W, H, G)
    assert np.array_equal(c, codes) and q == 0.0


def test_gptq_not_pd_reported(hq, cuda_device):
    K, N = 128, 8
    H = np.eye(K, dtype=np.float32) * 5
    H[3, 3] = -1.0
    W = torch.ones((N, K), device="cuda")
    with pytest.raises(hq.HQError) as e:
        _run_gptq(hq, W, torch.from_numpy(H).cuda(), 32)
    assert e.value.status == hq.HQ_ERR_NOT_PD


# ----------------------------------------------------------------------------- GPTQ edge cases

def _corr_layer(N, K, G, seed, wdt=torch.float32):
    cfg = wl.correlated_config(N, K, T=2 * K, group=G, seed=seed)
    X = wl.make_activations(cfg, "cpu")
    H32 = oracle.hessian(X.double().numpy()).astype(np.float32)
    W = wl.make_weights(cfg, "cpu", N=N, K=K).to(wdt)
    return W, H32


def test_gptq_zero_rows_and_zero_groups(hq, cuda_device):
    """An all-zero row gives codes 0 and scales 0 (absmax 0: s = 0, c = 0); a row whose first
    groups are zero keeps them zero (no error to feed back), so their scales are 0 too; a zero
    group after non-zero columns receives feedback and gets the oracle's non-zero scale."""
    N, K, G = 48, 512, 64
    W, H32 = _corr_layer(N, K, G, seed=21)
    W[0] = 0.0
    W[1, :2 * G] = 0.0
    W[2, 3 * G:4 * G] = 0.0
    W[3, K - G:] = 0.0
    Wd = W.cuda()
    codes, scales, q = _run_gptq(hq, Wd, torch.from_numpy(H32).cuda(), G)
    r = _compare_gptq(Wd, H32.astype(np.float64), G, codes, scales, q, what="zero rows/groups")
    assert np.all(codes[0] == 0) and np.all(scales[0] == 0.0)
    assert np.all(codes[1, :2 * G] == 0) and np.all(scales[1, :2] == 0.0) and np.all(scales[1, 2:] > 0.0)
    assert np.all(r["scales"][2, 3] > 0.0) and scales[2, 3] > 0.0
    assert np.all(r["codes"][0] == 0) and np.all(r["scales"][0] == 0.0) and np.all(r["scales"][1, :2] == 0.0)


def test_gptq_code_minus_eight_after_compensation(hq, cuda_device):
    """The clamp after compensation: H block-diagonal in 2 x 2 blocks [[4, 1.5], [1.5, 1]], so
    the first column of each pair feeds its error into the second with U'[0, 1] = -b/c (about
    -1.46 after damping).  Each pair is (6.6 s, -7 s) with s = absmax / 7: the first rounds up
    to 7 (residual -0.4 s) and pushes the second to about -7.59 s, which rounds to -8.  Negated
    rows push it to +7.59 s, which is clamped to +7."""
    N, K, G = 64, 256, 32
    H = np.zeros((K, K), np.float32)
    for p in range(0, K, 2):
        H[p:p + 2, p:p + 2] = [[4.0, 1.5], [1.5, 1.0]]
    rng = np.random.default_rng(8)
    amp = np.exp(rng.standard_normal((N, 1))) * 0.02
    pair = np.tile(np.array([6.6 / 7.0, -1.0]), K // 2)
    sign = np.where(np.arange(N) % 2 == 0, 1.0, -1.0)[:, None]
    W = torch.from_numpy((amp * sign * pair).astype(np.float32)).cuda()
    codes, scales, q = _run_gptq(hq, W, torch.from_numpy(H).cuda(), G)
    r = _compare_gptq(W, H.astype(np.float64), G, codes, scales, q, what="clamp")
    assert np.array_equal(codes, r["codes"]) and np.array_equal(scales, r["scales"])
    assert np.all(codes[0::2, 1::2] == -8) and np.all(codes[0::2, 0::2] == 7)
    assert np.all(codes[1::2, 1::2] == 7) and np.all(codes[1::2, 0::2] == -7)


@pytest.mark.parametrize("N,K,G,wdt", [(40, 128, 128, torch.float32), (24, 1024, 1024, torch.bfloat16),
                                      (1, 128, 32, torch.float32), (1, 128, 128, torch.bfloat16)])
def test_gptq_group_equals_k_and_single_row(hq, cuda_device, N, K, G, wdt):
    """One group spanning the whole row (a single scale per row, including a panel as wide as
    the group), and the smallest layer: one row of 128 columns."""
    W, H32 = _corr_layer(N, K, G, seed=N + K + G, wdt=wdt)
    Wd = W.cuda()
    codes, scales, q = _run_gptq(hq, Wd, torch.from_numpy(H32).cuda(), G)
    assert scales.shape == (N, K // G)
    _compare_gptq(Wd, H32.astype(np.float64), G, codes, scales, q, what=f"N={N} K={K} G={G}")


def test_gptq_non_finite_inputs(hq, cuda_device):
    """Non-finite inputs: a NaN weight leaves every other row's codes and scales exactly as
    without it (rows are independent); a Hessian with an infinite diagonal entry is refused as
    HQ_ERR_INVALID (mean(diag H) not finite); a NaN below the diagonal is reported as
    HQ_ERR_NOT_PD (the Cholesky pivot it reaches is not a positive number)."""
    N, K, G = 32, 256, 64
    W, H32 = _corr_layer(N, K, G, seed=31)
    Hd = torch.from_numpy(H32).cuda()
    Wd = W.cuda()
    c0, s0, _ = _run_gptq(hq, Wd, Hd, G)
    Wn = Wd.clone()
    Wn[5, 70] = float("nan")
    c1, s1, q1 = _run_gptq(hq, Wn, Hd, G)
    keep = np.arange(N) != 5
    assert np.array_equal(c0[keep], c1[keep]) and np.array_equal(s0[keep], s1[keep])
    assert np.isnan(q1)
    Hinf = Hd.clone()
    Hinf[7, 7] = float("inf")
    with pytest.raises(hq.HQError) as e:
        _run_gptq(hq, Wd, Hinf, G)
    assert e.value.status == hq.HQ_ERR_INVALID
    Hnan = Hd.clone()
    Hnan[100, 3] = float("nan")
    with pytest.raises(hq.HQError) as e:
        _run_gptq(hq, Wd, Hnan, G)
    assert e.value.status == hq.HQ_ERR_NOT_PD


# ----------------------------------------------------------------------------- RTN

@pytest.mark.parametrize("N,K,G", [(1, 2, 2), (37, 96, 32), (256, 4096, 128), (64, 4096, 4096)])
def test_rtn_bit_exact(hq, cuda_device, N, K, G):
    rng = np.random.default_rng(N * K)
    Wn = rng.uniform(-1, 1, (N, K)).astype(np.float32)
    W = torch.from_numpy(Wn).cuda()
    codes, scales = hq.gptq_outputs(N, K, G)
    ws = hq.alloc_workspace(hq.hq_rtn_workspace_bytes(N, K, G))
    q = hq.hq_rtn_quantize(W, G, codes, scales, ws)
    cr, sr = oracle.rtn_quantize(Wn, G)
    assert np.array_equal(unpack_codes(codes), cr)
    assert np.array_equal(scales.cpu().numpy(), sr)
    qr = oracle.qerr(Wn, cr, sr, G)
    assert abs(q - qr) <= 1e-12 * max(qr, 1e-300) + 1e-15


# ----------------------------------------------------------------------------- tf32 GEMM

def test_leaf_pivot_reciprocal_within_two_ulp(hq, cuda_device):
    """The leaf's Newton-Raphson reciprocal against the correctly rounded fp64 quotient, over
    pivots spanning the normal range (log-uniform magnitudes)."""
    g = _gen(77)
    e = torch.rand(1 << 20, generator=g, device="cuda", dtype=torch.float64) * 1200.0 - 600.0
    m = 1.0 + torch.rand(1 << 20, generator=g, device="cuda", dtype=torch.float64)
    d = m * torch.exp2(e.round())
    out = torch.empty_like(d)
    hq.hq_debug_rcp_f64(d, out)
    ref = 1.0 / d
    torch.cuda.synchronize()
    ulp = (ref.abs() * 2.0 ** -52)
    err = ((out - ref).abs() / ulp).max().item()
    assert err <= 2.0, err


@pytest.mark.parametrize("M,N,Kred,lower,tri,split", [
    (64, 64, 64, False, 0, False), (200, 136, 48, False, 0, True), (320, 192, 128, False, 3, True),
    (1280, 1280, 1280, False, 1, True), (1280, 1280, 1280, False, 2, True), (1280, 1280, 1280, True, 0, True),
    (2560, 2560, 2560, True, 0, False), (2560, 1280, 2560, False, 3, False)])
def test_f64_gemm_against_fp64(hq, cuda_device, M, N, Kred, lower, tri, split):
    """The factorisation's fp64 GEMM against torch's fp64 matmul, with its triangular-operand
    skipping (on operands that are zero there), the lower mask and the split-K path (which
    must also be bit-identical run to run)."""
    g = _gen(M * 5 + N + tri)
    A = torch.randn((M, Kred), generator=g, device="cuda", dtype=torch.float64)
    B = torch.randn((N, Kred), generator=g, device="cuda", dtype=torch.float64)
    if tri == 1:
        A = A.triu()
    elif tri == 2:
        A = A.tril()
    elif tri == 3:
        B = B.tril()
    C0 = torch.randn((M, N), generator=g, device="cuda", dtype=torch.float64)
    scratch = torch.empty(16 * M * N, device="cuda", dtype=torch.float64) if split else None
    C = C0.clone()
    hq.hq_debug_f64_gemm(C, A, B, alpha=-1.0, beta=1.0, lower=lower, tri=tri, scratch=scratch)
    C2 = C0.clone()
    hq.hq_debug_f64_gemm(C2, A, B, alpha=-1.0, beta=1.0, lower=lower, tri=tri, scratch=scratch)
    torch.cuda.synchronize()
    assert torch.equal(C, C2)
    ref = C0 - A @ B.T
    got = C
    if lower:
        mask = torch.ones((M, N), dtype=torch.bool, device="cuda").tril()
        assert torch.equal(got[~mask], C0[~mask])
        got, ref = got[mask], ref[mask]
    err = ((got - ref).norm() / ref.norm()).item()
    assert err < 1e-13, err


def _tri_operands(g, M, N, Kred, tri, garbage=False):
    """Random fp64 operands with the declared triangular one zero on its zero side inside the
    128-aligned band that the int8-sliced kernel reads; with `garbage`, NaN beyond that band
    (entries the kernel must never read)."""
    A = torch.randn((M, Kred), generator=g, device="cuda", dtype=torch.float64)
    B = torch.randn((N, Kred), generator=g, device="cuda", dtype=torch.float64)
    r = torch.arange(max(M, N), device="cuda")[:, None]
    k = torch.arange(Kred, device="cuda")[None, :]
    blk = (r // 128) * 128
    if tri == 1:
        A = A.triu()
        if garbage:
            A[(k < blk)[:M]] = float("nan")
    elif tri == 2:
        A = A.tril()
        if garbage:
            A[(k >= blk + 128)[:M]] = float("nan")
    elif tri == 3:
        B = B.tril()
        if garbage:
            B[(k >= blk + 128)[:N]] = float("nan")
    return A, B


@pytest.mark.parametrize("M,N,Kred,lower,tri,garbage", [
    (64, 64, 32, False, 0, False), (200, 136, 48, False, 0, False), (1000, 600, 300, False, 0, False),
    (1280, 1280, 1280, False, 1, True), (1280, 1280, 1280, False, 2, True), (1280, 1280, 1280, True, 0, False),
    (2560, 2560, 2560, True, 0, False), (2560, 1280, 2560, False, 3, True), (2560, 2560, 2560, False, 2, False),
    (384, 2560, 2560, False, 1, False)])
def test_i8x_gemm_against_fp64(hq, cuda_device, M, N, Kred, lower, tri, garbage):
    """The int8-sliced fp64 GEMM (7 slices, 28 tcgen05 kind::i8 products) against torch's fp64
    matmul: relative Frobenius error <= 1e-12 (per term the slicing keeps about 1.6e-14 of the
    product of the row maxima; Gaussian operands), bit-identical run to run, triangular
    operands read only inside their band, the lower mask, beta = 0 without reading C."""
    g = _gen(M * 3 + N + 17 * tri + Kred)
    A, B = _tri_operands(g, M, N, Kred, tri, garbage)
    Ar = torch.nan_to_num(A, nan=0.0)
    Br = torch.nan_to_num(B, nan=0.0)
    C0 = torch.randn((M, N), generator=g, device="cuda", dtype=torch.float64)
    C = C0.clone()
    hq.hq_debug_i8x_gemm(C, A, B, alpha=-1.0, beta=1.0, lower=lower, tri=tri)
    C2 = C0.clone()
    hq.hq_debug_i8x_gemm(C2, A, B, alpha=-1.0, beta=1.0, lower=lower, tri=tri)
    torch.cuda.synchronize()
    assert torch.equal(C, C2)
    prod = Ar @ Br.T
    ref = C0 - prod
    got = C
    if lower:
        mask = torch.ones((M, N), dtype=torch.bool, device="cuda").tril()
        assert torch.equal(got[~mask], C0[~mask])
        got, ref, prod = got[mask], ref[mask], prod[mask]
    err = ((got - ref).norm() / prod.norm()).item()
    assert err < 1e-12, err
    # beta = 0: C's previous contents (NaN here) are not read
    Cn = torch.full((M, N), float("nan"), device="cuda", dtype=torch.float64)
    hq.hq_debug_i8x_gemm(Cn, A, B, alpha=2.0, beta=0.0, lower=False, tri=tri)
    torch.cuda.synchronize()
    err0 = ((Cn - 2.0 * (Ar @ Br.T)).norm() / (2.0 * (Ar @ Br.T)).norm()).item()
    assert err0 < 1e-12, err0


@pytest.mark.parametrize("n,Kred,lower", [(1000, 700, True), (1000, 700, False), (136, 2048, True)])
def test_i8x_gemm_same_operand(hq, cuda_device, n, Kred, lower):
    """C -= T T^T with one tensor as both operands (the factorisation's A22 update): T is read and
    sliced once into both slice layouts; the result is bit-identical to the product with a copy
    of T as the second operand (sliced on its own) and within 1e-12 of torch's fp64 product.
    Sizes ragged against the 128-row and 64-row tile blocks."""
    g = _gen(n + Kred)
    T = torch.randn((n, Kred), generator=g, device="cuda", dtype=torch.float64)
    C0 = torch.randn((n, n), generator=g, device="cuda", dtype=torch.float64)
    C1, C2 = C0.clone(), C0.clone()
    hq.hq_debug_i8x_gemm(C1, T, T, alpha=-1.0, beta=1.0, lower=lower)
    hq.hq_debug_i8x_gemm(C2, T, T.clone(), alpha=-1.0, beta=1.0, lower=lower)
    torch.cuda.synchronize()
    assert torch.equal(C1, C2)
    prod = T @ T.T
    ref = C0 - prod
    if lower:
        mask = torch.ones((n, n), dtype=torch.bool, device="cuda").tril()
        assert torch.equal(C1[~mask], C0[~mask])
        C1, ref, prod = C1[mask], ref[mask], prod[mask]
    assert ((C1 - ref).norm() / prod.norm()).item() < 1e-12


def test_i8x_gemm_non_finite_rows_give_nan(hq, cuda_device):
    """A row with a NaN or an infinity gives a NaN row (A) or column (B) of the product, so that
    non-finite values still reach the factorisation's pivot check; every other entry is
    unaffected."""
    g = _gen(99)
    A = torch.randn((256, 512), generator=g, device="cuda", dtype=torch.float64)
    B = torch.randn((192, 512), generator=g, device="cuda", dtype=torch.float64)
    A[7, 100] = float("nan")
    B[33, 5] = float("inf")
    C = torch.zeros((256, 192), device="cuda", dtype=torch.float64)
    hq.hq_debug_i8x_gemm(C, A, B, alpha=1.0, beta=0.0)
    torch.cuda.synchronize()
    bad = torch.zeros_like(C, dtype=torch.bool)
    bad[7, :] = True
    bad[:, 33] = True
    assert torch.isnan(C[bad]).all()
    A[7, 100] = 0.0
    B[33, 5] = 0.0
    ref = A @ B.T
    assert ((C[~bad] - ref[~bad]).norm() / ref[~bad].norm()).item() < 1e-12


@pytest.mark.parametrize("M,N,Kred", [(5120, 384, 128), (5120, 4608, 512), (512, 512, 512), (512, 512, 1024),
                                       (1000, 600, 300), (132, 72, 36)])
def test_upd_gemm_against_fp64(hq, cuda_device, M, N, Kred):
    """The persistent 3xTF32 lazy-update kernel (every tile width it picks) against fp64:
    C -= A B^T with A, B given as tf32 part + remainder.  The tensor core's fp32 accumulation
    drifts with the number of chained MMAs (about 4e-6 relative at a contraction of 512), so
    the bound scales with the contraction."""
    from gpu_helpers import split_tf32
    g = _gen(M + 7 * N + Kred)
    A = torch.randn((M, Kred), generator=g, device="cuda")
    B = torch.randn((N, Kred), generator=g, device="cuda")
    C0 = torch.randn((M, N), generator=g, device="cuda")
    Ah, Al = split_tf32(A)
    Bh, Bl = split_tf32(B)
    C = C0.clone()
    hq.hq_debug_upd_gemm(C, Ah, Al, Bh, Bl)
    torch.cuda.synchronize()
    ref = C0.double() - A.double() @ B.double().T
    err = ((C.double() - ref).norm() / (A.double() @ B.double().T).norm()).item()
    assert err < 1e-6 + 1e-8 * Kred, err


def test_kernel_timing_records_every_launch(hq, cuda_device):
    """The event timing of kernel classes sees each factorisation leaf once per 128 columns
    and the algorithmic work it reports is the stated formula."""
    K = 512
    g = _gen(5)
    X = torch.randn((1024, K), generator=g, device="cuda")
    H = torch.zeros((K, K), device="cuda")
    hq.hq_hessian_accumulate(H, X)
    ws = hq.alloc_workspace(hq.hq_gptq_workspace_bytes(1, K, 128))
    Ut = torch.empty((K, K), device="cuda")
    hq.hq_debug_timing_start(["leaf", "f64_gemm_128", "f64_gemm_64"])
    hq.hq_debug_factor(H, 0.01, Ut, ws)
    hq.hq_debug_timing_stop()
    ms, work, n = hq.hq_debug_timing_read("leaf")
    assert n == K // 128 and ms > 0.0
    assert work == pytest.approx(n * 2.0 * 128 ** 3 / 3.0)
    ms64, work64, n64 = hq.hq_debug_timing_read("f64_gemm_64")
    assert n64 > 0 and ms64 > 0.0 and work64 > 0.0
    # nothing is recorded once timing is stopped
    hq.hq_debug_factor(H, 0.01, Ut, ws)
    assert hq.hq_debug_timing_read("leaf")[2] == n


def test_serialized_timing_gives_the_same_bits(hq, cuda_device):
    """hq_debug_timing_serialize only moves the factorisation's second-stream products onto the
    caller's stream: codes, scales and qerr are bit-identical (K = 4096 reaches the int8-sliced
    products on both streams)."""
    N, K, G = 256, 4096, 128
    cfg = wl.correlated_config(N, K, T=K, group=G, seed=11)
    X = wl.make_activations(cfg, "cuda")
    H = torch.zeros((K, K), device="cuda")
    hq.hq_hessian_accumulate(H, X)
    W = wl.make_weights(cfg, "cuda", N=N, K=K)
    base = _run_gptq(hq, W, H, G)
    hq.hq_debug_timing_serialize(True)
    try:
        ser = _run_gptq(hq, W, H, G)
    finally:
        hq.hq_debug_timing_serialize(False)
    assert np.array_equal(base[0], ser[0]) and np.array_equal(base[1], ser[1]) and base[2] == ser[2]
