"""GPU parity at the full sizes of the layer configurations, in the launch configuration the
benchmark times (one hq_hessian_accumulate over the layer's tokens, then hq_gptq_quantize).

GPTQ rows are independent given U, so the oracle sweeps a seeded sample of rows exactly; the
oracle's H and U are its own fp64 computations from the same X.  For the Hessian at scale
(4.19 M tokens) the oracle computes sampled entries of H as exact dot products.  Codes, and the
scales of every group up to a row's first differing code, are compared with the plain oracle,
which never takes the CUDA path's output as an input; only the scales after that point are
compared on the GPU's own code trajectory (the oracle replaying the GPU's codes)."""

import numpy as np
import pytest
import torch

import oracle
import workloads as wl
from gpu_helpers import H_REL_FRO, LOSS_REL, QERR_REL, check_gptq_parity, rel_fro, unpack_codes

pytestmark = [pytest.mark.gpu, pytest.mark.slow]


@pytest.fixture(scope="module")
def hq():
    import post_weight_quantization_tcgen05_b200 as m
    return m


def _oracle_hessian(X: torch.Tensor, rows_per_chunk: int = 8192) -> np.ndarray:
    """fp64 X^T X of a device tensor, chunk by chunk on the host (sum over chunks)."""
    K = X.shape[1]
    H = np.zeros((K, K))
    for a in range(0, X.shape[0], rows_per_chunk):
        H = oracle.hessian_accumulate(H, X[a:a + rows_per_chunk].double().cpu().numpy())
    return H


def _gpu_gptq(hq, W, H, cfg, imp=None):
    N, K = W.shape
    codes, scales = hq.gptq_outputs(N, K, cfg.group)
    ws = hq.alloc_workspace(hq.hq_gptq_workspace_bytes(N, K, cfg.group))
    q = hq.hq_gptq_quantize(W, H, cfg.group, cfg.damp, codes, scales, ws, imp=imp)
    torch.cuda.synchronize()
    return codes, scales, q


def _check_layer(hq, cfg, X, W, H_gpu, H64, n_sample=48, imp_gpu=None, imp64=None):
    """SYRK parity on the lower triangle, then GPTQ parity on sampled rows."""
    K = cfg.K
    lo = np.tril_indices(K)
    Hg = H_gpu.double().cpu().numpy()
    err = rel_fro(Hg[lo], H64[lo])
    assert err <= H_REL_FRO, f"H rel Frobenius {err:.3e}"
    codes, scales, q = _gpu_gptq(hq, W, H_gpu, cfg, imp_gpu)
    Wn = W.double().cpu().numpy()
    cg = unpack_codes(codes)
    sg = scales.cpu().numpy()
    # the GPU's layer qerr is the oracle's qerr of the GPU's codes (checks the reduction)
    q_of_gpu = oracle.qerr(Wn, cg, sg, cfg.group, imp64)
    assert abs(q - q_of_gpu) <= 1e-6 * q_of_gpu
    rng = np.random.default_rng(cfg.seed + 100)
    rows = np.sort(rng.choice(cfg.N, size=n_sample, replace=False))
    Hd, _ = oracle.damp_hessian(H64, cfg.damp)
    # the literal route at K <= 8192; the reversal route (pinned equal to it) above, for time
    U = oracle.upper_factor_of_inverse(Hd) if K <= 8192 else oracle.upper_factor_by_reversal(Hd)
    rc, rs = check_gptq_parity(Wn[rows], U, cfg.group, cg[rows], sg[rows], what=cfg.name)
    q_ref = oracle.qerr(Wn[rows], rc, rs, cfg.group, imp64)
    q_gpu_rows = oracle.qerr(Wn[rows], cg[rows], sg[rows], cfg.group, imp64)
    assert abs(q_gpu_rows - q_ref) <= QERR_REL * q_ref, (q_gpu_rows, q_ref)
    l_ref = oracle.layer_loss(Wn[rows], rc, rs, cfg.group, H64)
    l_gpu = oracle.layer_loss(Wn[rows], cg[rows], sg[rows], cfg.group, H64)
    assert abs(l_gpu - l_ref) <= LOSS_REL * l_ref, (l_gpu, l_ref)


def test_q_proj_layer_full_size(hq, cuda_device):
    cfg = wl.CONFIGS[1]
    X = wl.make_activations(cfg, "cuda")
    W = wl.make_weights(cfg, "cuda")
    H = torch.zeros((cfg.K, cfg.K), device="cuda")
    hq.hq_hessian_accumulate(H, X)
    H64 = _oracle_hessian(X)
    _check_layer(hq, cfg, X, W, H, H64)


def test_q_proj_layer_chunked_accumulation(hq, cuda_device):
    # the layer's 16 chunks of 512 tokens fed one by one give the same H within tolerance
    cfg = wl.CONFIGS[1]
    X = wl.make_activations(cfg, "cuda")
    H1 = torch.zeros((cfg.K, cfg.K), device="cuda")
    hq.hq_hessian_accumulate(H1, X)
    H2 = torch.zeros((cfg.K, cfg.K), device="cuda")
    for c in range(cfg.n_chunks):
        hq.hq_hessian_accumulate(H2, X[c * cfg.chunk:(c + 1) * cfg.chunk])
    torch.cuda.synchronize()
    lo = torch.ones((cfg.K, cfg.K), dtype=torch.bool, device="cuda").tril()
    d = ((H1 - H2)[lo].double().norm() / H1[lo].double().norm()).item()
    assert d <= H_REL_FRO


def test_gate_up_layer_full_size_with_imatrix(hq, cuda_device):
    cfg = wl.CONFIGS[2]
    X = wl.make_activations(cfg, "cuda")
    W = wl.make_weights(cfg, "cuda")
    H = torch.zeros((cfg.K, cfg.K), device="cuda")
    hq.hq_hessian_accumulate(H, X)
    imp = torch.empty(cfg.K, device="cuda")
    hq.hq_imatrix(H, cfg.T, imp)
    H64 = _oracle_hessian(X)
    imp64 = oracle.imatrix(H64, cfg.T)
    assert np.allclose(imp.cpu().numpy(), imp64, rtol=1e-5)
    _check_layer(hq, cfg, X, W, H, H64, n_sample=32, imp_gpu=imp, imp64=imp64)


def test_down_proj_layer_full_size(hq, cuda_device):
    """W [5120, 17408], X [65536, 17408] post-SiLU-like (positive, so H is dominated by a common
    component and the damped H is ill-conditioned, kappa ~ 1e5-1e6), group 128."""
    cfg = wl.CONFIGS[3]
    X = wl.make_activations(cfg, "cuda")
    W = wl.make_weights(cfg, "cuda")
    H = torch.zeros((cfg.K, cfg.K), device="cuda")
    hq.hq_hessian_accumulate(H, X)
    H64 = _oracle_hessian(X, rows_per_chunk=4096)
    _check_layer(hq, cfg, X, W, H, H64, n_sample=16)


def test_hessian_at_scale_sampled_and_codec(hq, cuda_device):
    """512 chunks of X bf16 [8192, 6144] streamed through the SYRK into one fp32 H; sampled
    entries against exact fp64 dot products; then the Bf16TrilDiagF32 codec on that H
    (checked by the definition's properties) and bit-exact against the oracle on a seeded H of
    the same size."""
    cfg = wl.CONFIGS[4]
    K = cfg.K
    scales = wl.channel_scales(cfg)
    rng = np.random.default_rng(44)
    ii = rng.integers(0, K, 48)
    jj = (rng.random(48) * (ii + 1)).astype(np.int64)
    ii = np.concatenate([ii, ii[:8]])
    jj = np.concatenate([jj, ii[:8]])
    # and entries of the last 8 tiles in the SYRK's order (each 8192-token call has 600 tiles on
    # 148 SMs: 4 whole rounds, then these 8 are cut by token segments over the idle SMs); they
    # lie in rows 5888 .. 6143, columns 5376 .. the diagonal
    ci = rng.integers(5888, K, 16)
    cj = 5376 + (rng.random(16) * (ci - 5376 + 1)).astype(np.int64)
    ii = np.concatenate([ii, ci])
    jj = np.concatenate([jj, cj])
    cols = np.unique(np.concatenate([ii, jj]))
    cols_t = torch.from_numpy(cols).cuda()
    pos = {c: n for n, c in enumerate(cols)}
    H = torch.zeros((K, K), device="cuda")
    acc = np.zeros(len(ii))
    for c in range(cfg.n_chunks):
        Xc = wl.make_activation_chunk(cfg, c, "cuda", scales)
        hq.hq_hessian_accumulate(H, Xc)
        sub = Xc[:, cols_t].double().cpu().numpy()
        acc += np.array([sub[:, pos[i]] @ sub[:, pos[j]] for i, j in zip(ii, jj)])
    torch.cuda.synchronize()
    got = H[torch.from_numpy(ii).cuda(), torch.from_numpy(jj).cuda()].double().cpu().numpy()
    assert rel_fro(got, acc) <= H_REL_FRO

    # codec on the accumulated H: every stored value is defined by H's own bits
    nb = hq.hq_bf16tril_bytes(K)
    out = torch.empty(nb, dtype=torch.uint8, device="cuda")
    hq.hq_hessian_pack_bf16tril(H, out)
    Hf = torch.empty((K, K), device="cuda")
    hq.hq_hessian_unpack_bf16tril(out, K, Hf)
    torch.cuda.synchronize()
    buf = out.cpu().numpy()
    Hb = H.cpu().numpy()
    assert np.array_equal(buf[:4 * K].view("<f4"), np.diag(Hb))
    tri = buf[4 * K:].view("<u2")
    for i in rng.integers(1, K, 32):
        base = i * (i - 1) // 2
        assert np.array_equal(tri[base:base + i], (Hb[i, :i].view(np.uint32) >> 16).astype(np.uint16))
    Hfn = Hf.cpu().numpy()
    assert np.array_equal(np.diag(Hfn), np.diag(Hb))
    assert np.array_equal(Hfn, Hfn.T)
    low = np.tril(np.ones((K, K), bool), -1)
    assert np.array_equal(Hfn[low].view(np.uint32), Hb[low].view(np.uint32) & 0xFFFF0000)

    # bit-exact against the oracle on a seeded H of the same size
    g = torch.Generator(device="cuda")
    g.manual_seed(4)
    Hg = torch.randn((K, K), generator=g, device="cuda") * 1000.0
    hq.hq_hessian_pack_bf16tril(Hg, out)
    torch.cuda.synchronize()
    ref = oracle.bf16tril_encode(Hg.cpu().numpy())
    assert out.cpu().numpy().tobytes() == ref
    hq.hq_hessian_unpack_bf16tril(out, K, Hf)
    torch.cuda.synchronize()
    assert np.array_equal(Hf.cpu().numpy().view(np.uint32), oracle.bf16tril_decode(ref, K).view(np.uint32))
