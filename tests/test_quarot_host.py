"""Host logic of rotate-then-GPTQ ("Exp 2026-08-18 GPTQ Int4", experiment summary), on the CPU
with a stand-in for the library: the random signs, and the order and shapes of the calls."""

import types

import torch

from post_weight_quantization_tcgen05_b200 import quarot


def test_random_signs_are_plus_minus_one_and_seeded():
    g1 = torch.Generator(device="cpu")
    g1.manual_seed(7)
    g2 = torch.Generator(device="cpu")
    g2.manual_seed(7)
    a = quarot.random_signs(4096, g1, device="cpu")
    b = quarot.random_signs(4096, g2, device="cpu")
    assert a.dtype == torch.float32 and tuple(a.shape) == (4096,)
    assert torch.equal(a, b)
    assert set(a.unique().tolist()) == {-1.0, 1.0}
    assert 0.45 < float((a > 0).float().mean()) < 0.55


def test_rotate_then_gptq_calls_in_order_on_rotated_buffers():
    calls = []

    def rot_w(W, s, block, out):
        calls.append(("W", tuple(W.shape), block, tuple(out.shape), out.dtype))

    def rot_h(H, s, block, out):
        calls.append(("H", tuple(H.shape), block, tuple(out.shape), out.dtype))

    def quantize(W, H, group, damp, codes, scales, ws, imp=None):
        calls.append(("Q", tuple(W.shape), tuple(H.shape), group, damp, imp))
        return 0.25

    hq = types.SimpleNamespace(hq_hadamard_rotate_weights=rot_w, hq_hadamard_rotate_hessian=rot_h,
                               hq_gptq_quantize=quantize)
    W = torch.zeros((6, 8), dtype=torch.bfloat16)
    H = torch.zeros((8, 8))
    s = torch.ones(8)
    q, Wr, Hr = quarot.rotate_then_gptq(hq, W, H, s, 4, 4, 0.01, None, None, None)
    assert q == 0.25 and tuple(Wr.shape) == (6, 8) and Wr.dtype == torch.float32 and tuple(Hr.shape) == (8, 8)
    assert calls == [("W", (6, 8), 4, (6, 8), torch.float32), ("H", (8, 8), 4, (8, 8), torch.float32),
                     ("Q", (6, 8), (8, 8), 4, 0.01, None)]
