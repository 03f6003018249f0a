"""Rotate-then-GPTQ on the GPU: the Hadamard rotation of weights and Hessian against the oracle's
dense rotation, and GPTQ on the rotated layer against the oracle on the same rotated inputs."""

import numpy as np
import pytest
import torch

import oracle
import workloads as wl
from gpu_helpers import to_np64, unpack_codes

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def hq():
    import post_weight_quantization_tcgen05_b200 as m
    return m


@pytest.mark.parametrize("K,B,wdt", [(512, 256, "bf16"), (512, 128, "f32"), (384, 128, "bf16"), (256, 2, "f32"),
                                     (1024, 1024, "f32"), (96, 32, "bf16"), (64, 64, "f32"), (96, 16, "bf16"),
                                     (2048, 512, "bf16"), (1280, 256, "f32")])
def test_rotation_matches_oracle(hq, cuda_device, K, B, wdt):
    from post_weight_quantization_tcgen05_b200 import quarot
    g = torch.Generator(device="cuda")
    g.manual_seed(K + B)
    s = quarot.random_signs(K, g)
    cfg = wl.small_config(wl.CONFIGS[1], N=48, K=K, T=2 * K, seed=2)
    W = wl.make_weights(cfg, "cuda", N=48, K=K).to(wl.torch_dtype(wdt))
    X = wl.make_activations(cfg, "cuda")
    H = torch.zeros((K, K), device="cuda")
    hq.hq_hessian_accumulate(H, X)
    Wr = torch.empty((48, K), device="cuda")
    Hr = torch.empty((K, K), device="cuda")
    hq.hq_hadamard_rotate_weights(W, s, B, Wr)
    hq.hq_hadamard_rotate_hessian(H, s, B, Hr)
    torch.cuda.synchronize()
    sn = s.cpu().numpy()
    rw = oracle.rotate_weights(to_np64(W), sn, B)
    rh = oracle.rotate_hessian(to_np64(H), sn, B)
    ew = np.linalg.norm(to_np64(Wr) - rw) / np.linalg.norm(rw)
    eh = np.linalg.norm(to_np64(Hr) - rh) / np.linalg.norm(rh)
    assert ew < 1e-6 and eh < 1e-6, (ew, eh)
    # H' is symmetric: with blocks of 32 and more the off-diagonal blocks are written as exact
    # transposes of each other
    nb = K // B if B >= 32 else 0
    for bi in range(nb):
        for bj in range(bi):
            assert torch.equal(Hr[bi * B:(bi + 1) * B, bj * B:(bj + 1) * B],
                               Hr[bj * B:(bj + 1) * B, bi * B:(bi + 1) * B].T)
    # in place on fp32 weights gives the same bytes
    if wdt == "f32":
        W2 = W.clone()
        hq.hq_hadamard_rotate_weights(W2, s, B, W2)
        torch.cuda.synchronize()
        assert torch.equal(W2, Wr)


def test_rotate_then_gptq(hq, cuda_device):
    from post_weight_quantization_tcgen05_b200 import quarot
    N, K, G, B = 64, 512, 128, 256
    cfg = wl.correlated_config(N, K, T=4 * K, group=G, seed=8)
    X = wl.make_activations(cfg, "cuda")
    W = wl.make_weights(cfg, "cuda", N=N, K=K)
    H = torch.zeros((K, K), device="cuda")
    hq.hq_hessian_accumulate(H, X)
    g = torch.Generator(device="cuda")
    g.manual_seed(1042)
    s = quarot.random_signs(K, g)
    codes, scales = hq.gptq_outputs(N, K, G)
    ws = hq.alloc_workspace(hq.hq_gptq_workspace_bytes(N, K, G))
    q, Wr, Hr = quarot.rotate_then_gptq(hq, W, H, s, B, G, 0.01, codes, scales, ws)
    torch.cuda.synchronize()
    # the oracle's GPTQ on the same rotated inputs
    ref = oracle.gptq_quantize(to_np64(Wr), to_np64(Hr), G, 0.01)
    c = unpack_codes(codes)
    match = float(np.mean(c == ref["codes"]))
    assert match >= 0.99 and np.abs(c.astype(int) - ref["codes"].astype(int)).max() <= 1
    # the rotation is orthogonal: the error of W' is the un-rotated layer's error
    R = oracle.hadamard_rotation(s.cpu().numpy(), B)
    Qr = oracle.dequantize(c, scales.cpu().numpy(), G)
    Wn = to_np64(W)
    assert q == pytest.approx(np.linalg.norm(Wn - Qr @ R.T) / np.linalg.norm(Wn), rel=1e-4)


@pytest.mark.parametrize("B", [32, 256])
def test_rotation_unaligned_buffers(hq, cuda_device, B):
    """Buffers that are not 16-byte aligned take the shared-memory kernels: same values."""
    from post_weight_quantization_tcgen05_b200 import quarot
    N, K = 40, 512
    g = torch.Generator(device="cuda")
    g.manual_seed(B)
    s = quarot.random_signs(K, g)
    W = torch.randn((N, K), device="cuda", generator=g)
    Wr = torch.empty((N, K), device="cuda")
    hq.hq_hadamard_rotate_weights(W, s, B, Wr)
    buf = torch.empty(N * K + 1, device="cuda")
    Wu = buf[1:].view(N, K)
    hq.hq_hadamard_rotate_weights(W, s, B, Wu)
    hbuf = torch.empty(K * K + 1, device="cuda")
    Hu = hbuf[1:].view(K, K)
    A = torch.randn((K, K), device="cuda", generator=g, dtype=torch.float64)
    H = (A @ A.T).float()
    Hr = torch.empty((K, K), device="cuda")
    hq.hq_hadamard_rotate_hessian(H, s, B, Hr)
    hq.hq_hadamard_rotate_hessian(H, s, B, Hu)
    torch.cuda.synchronize()
    assert torch.allclose(Wu, Wr, rtol=1e-5, atol=1e-5 * float(Wr.abs().max()))
    assert torch.allclose(Hu, Hr, rtol=1e-5, atol=1e-5 * float(Hr.abs().max()))


@pytest.mark.parametrize("N,K,B", [(1500, 1024, 32), (9600, 1024, 256)])
def test_weight_rotation_beyond_one_wave(hq, cuda_device, N, K, B):
    """More blocks than one wave of warps holds (148 x 8 CTAs of 8 warps, 4 blocks each): the
    grid-stride loop of the weight rotation, against the oracle."""
    from post_weight_quantization_tcgen05_b200 import quarot
    assert N * (K // B) > 148 * 8 * 8 * 4
    g = torch.Generator(device="cuda")
    g.manual_seed(N + B)
    s = quarot.random_signs(K, g)
    W = (torch.randn((N, K), device="cuda", generator=g) * 0.02).to(torch.bfloat16)
    Wr = torch.empty((N, K), device="cuda")
    hq.hq_hadamard_rotate_weights(W, s, B, Wr)
    torch.cuda.synchronize()
    rw = oracle.rotate_weights(to_np64(W), s.cpu().numpy(), B)
    assert np.linalg.norm(to_np64(Wr) - rw) / np.linalg.norm(rw) < 1e-6
