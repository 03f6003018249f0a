"""A representative run of the library's kernels on small seeded inputs, for the bounds-checking
build: every call is followed by a read of the bounds word.  Imported by tests/test_gpu_bounds.py
(with libhq.so) and run as a script in a child process with HQ_LIBRARY=libhq_bounds.so:

    HQ_LIBRARY=libhq_bounds.so python tests/bounds_workload.py OUT.pt

Shapes are ragged against the kernels' tiles and reach the int8-sliced products (K = 2048), the
fused panel sweep (a few rows per CTA) and the block-by-block sweep (more than 64 rows per CTA).
"""

from __future__ import annotations

import os
import sys

import torch


def _gen(seed: int) -> torch.Generator:
    g = torch.Generator(device="cuda")
    g.manual_seed(seed)
    return g


def _hessian(hq, T: int, K: int, seed: int, dtype=torch.bfloat16) -> torch.Tensor:
    X = torch.randn((T, K), device="cuda", generator=_gen(seed)).to(dtype)
    H = torch.zeros((K, K), device="cuda")
    hq.hq_hessian_accumulate(H, X)
    return H


def run_all(hq) -> tuple[dict, dict]:
    """(outputs, bounds words after each call)."""
    from post_weight_quantization_tcgen05_b200 import quarot
    out, words = {}, {}

    def mark(name):
        torch.cuda.synchronize()
        words[name] = hq.hq_debug_bounds_status()[1]

    hq.hq_debug_bounds_status()  # clear
    out["H_bf16"] = _hessian(hq, 1000, 384, 1)
    mark("syrk_bf16")
    out["H_f32"] = _hessian(hq, 300, 136, 2, dtype=torch.float32)
    mark("syrk_f32")

    # int8-sliced products (K = 2048) and the fused panel sweep (200 rows: 4 per CTA); at most
    # 1024 tokens per SYRK call here, so that no call cuts tiles into pieces (whose partial sums
    # arrive in a run-dependent order) and both builds see the same bits
    H = _hessian(hq, 1024, 2048, 3)
    W = (torch.randn((200, 2048), device="cuda", generator=_gen(4)) * 0.02).to(torch.bfloat16)
    codes, scales = hq.gptq_outputs(200, 2048, 128)
    ws = hq.alloc_workspace(hq.hq_gptq_workspace_bytes(200, 2048, 128))
    out["q_fused"] = torch.tensor(hq.hq_gptq_quantize(W, H, 128, 0.01, codes, scales, ws), dtype=torch.float64)
    out["codes_fused"], out["scales_fused"] = codes, scales
    mark("gptq_fused")

    # more than 64 rows per CTA: one block per sweep launch, tensor-core inner updates
    H2 = _hessian(hq, 512, 256, 5)
    W2 = (torch.randn((9600, 256), device="cuda", generator=_gen(6)) * 0.02).to(torch.bfloat16)
    codes2, scales2 = hq.gptq_outputs(9600, 256, 64)
    ws2 = hq.alloc_workspace(hq.hq_gptq_workspace_bytes(9600, 256, 64))
    out["q_blocks"] = torch.tensor(hq.hq_gptq_quantize(W2, H2, 64, 0.01, codes2, scales2, ws2), dtype=torch.float64)
    out["codes_blocks"], out["scales_blocks"] = codes2, scales2
    mark("gptq_blocks")

    for K in (1000, 1001):  # vectorised and scalar codec paths
        Hc = _hessian(hq, 64, K, 7, dtype=torch.float32)
        packed = torch.empty(hq.hq_bf16tril_bytes(K), dtype=torch.uint8, device="cuda")
        hq.hq_hessian_pack_bf16tril(Hc, packed)
        Hd = torch.empty((K, K), device="cuda")
        hq.hq_hessian_unpack_bf16tril(packed, K, Hd)
        out[f"packed_{K}"], out[f"decoded_{K}"] = packed, Hd
    mark("codec")

    Ht = out["H_f32"]
    p32 = torch.empty(hq.hq_tril32_count(136), dtype=torch.float32, device="cuda")
    hq.hq_hessian_pack_lower(Ht, p32)
    Hu = torch.zeros_like(Ht)
    hq.hq_hessian_unpack_lower(p32, 136, Hu)
    out["tril32"], out["tril32_back"] = p32, Hu
    mark("tril32")

    s = quarot.random_signs(512, _gen(8), device=torch.device("cuda"))
    Wr = torch.empty((40, 512), device="cuda")
    hq.hq_hadamard_rotate_weights((torch.randn((40, 512), device="cuda", generator=_gen(9))), s, 256, Wr)
    Hr = torch.empty((512, 512), device="cuda")
    hq.hq_hadamard_rotate_hessian(_hessian(hq, 600, 512, 10, dtype=torch.float32), s, 256, Hr)
    out["W_rot"], out["H_rot"] = Wr, Hr
    mark("hadamard")

    Wq = torch.randn((33, 256), device="cuda", generator=_gen(11))
    codes3, scales3 = hq.gptq_outputs(33, 256, 32)
    ws3 = hq.alloc_workspace(hq.hq_rtn_workspace_bytes(33, 256, 32))
    out["q_rtn"] = torch.tensor(hq.hq_rtn_quantize(Wq, 32, codes3, scales3, ws3), dtype=torch.float64)
    out["codes_rtn"], out["scales_rtn"] = codes3, scales3
    mark("rtn")
    return {k: v.cpu() for k, v in out.items()}, words


if __name__ == "__main__":
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import post_weight_quantization_tcgen05_b200 as hq_mod
    outputs, bound_words = run_all(hq_mod)
    enabled, _ = hq_mod.hq_debug_bounds_status()
    hq_mod.hq_debug_bounds_selftest()
    torch.cuda.synchronize()
    _, selftest_word = hq_mod.hq_debug_bounds_status()
    torch.save({"outputs": outputs, "words": bound_words, "enabled": enabled, "selftest": selftest_word,
                "library": os.path.basename(hq_mod._LIB_PATH)}, sys.argv[1])
