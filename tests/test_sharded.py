"""The multi-GPU split of the path (package module `sharded`): the host logic and the exchange
on CPU with two gloo ranks (partial Hessians over disjoint token ranges summed by one all-reduce;
qerr of a row-split layer from the ranks' numerator / denominator sums), and on one GPU the
pieces the split relies on: row shards quantise exactly like the whole layer, and hq_qerr_terms
gives sums whose ratio is the reported qerr."""

import math
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
from post_weight_quantization_tcgen05_b200 import sharded


@pytest.mark.parametrize("n", [0, 1, 5, 7, 128, 5120, 17408])
@pytest.mark.parametrize("world", [1, 2, 3, 8])
def test_split_range_covers_once_and_balances(n, world):
    parts = [sharded.split_range(n, r, world) for r in range(world)]
    assert parts[0][0] == 0 and parts[-1][1] == n
    for (a0, a1), (b0, b1) in zip(parts, parts[1:]):
        assert a1 == b0
    sizes = [b - a for a, b in parts]
    assert max(sizes) - min(sizes) <= 1 and min(sizes) >= 0
    assert sharded.token_range(n, world - 1, world) == parts[-1]
    assert sharded.row_range(n, 0, world) == parts[0]


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank: int, world: int, port: int, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        rng = np.random.default_rng(11)  # the same data on every rank
        T, K, N, G = 103, 64, 9, 32
        X = rng.standard_normal((T, K))
        # partial Hessian over this rank's tokens (a CPU stand-in for hq_hessian_accumulate)
        t0, t1 = sharded.token_range(T, rank, world)
        H = torch.from_numpy(X[t0:t1].T @ X[t0:t1])
        sharded.allreduce_hessian(H)
        h_err = float(np.abs(H.numpy() - X.T @ X).max() / np.abs(X.T @ X).max())
        # qerr of a row-split layer from the ranks' sums
        W = rng.uniform(-1, 1, (N, K))
        imp = rng.uniform(0.5, 2.0, K)
        codes, scales = oracle.rtn_quantize(W, G)
        r0, r1 = sharded.row_range(N, rank, world)
        D = W[r0:r1] - oracle.dequantize(codes[r0:r1], scales[r0:r1], G)
        terms = torch.tensor([float(np.sum((D * D) @ imp)), float(np.sum((W[r0:r1] ** 2) @ imp))],
                             dtype=torch.float64)
        q = sharded.combine_qerr_terms(terms)
        out.put((rank, h_err, q, oracle.qerr(W, codes, scales, G, imp)))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_hessian_allreduce_and_qerr_terms():
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(out.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for _, h_err, q, q_ref in res:
        assert h_err < 1e-13
        assert q == pytest.approx(q_ref, rel=1e-12)


@pytest.mark.gpu
def test_row_shards_quantise_like_the_layer_and_qerr_terms(cuda_device):
    import post_weight_quantization_tcgen05_b200 as hq
    import workloads as wl
    cfg = wl.correlated_config(96, 256, T=512, group=64, seed=5)
    X = wl.make_activations(cfg, "cuda")
    W = wl.make_weights(cfg, "cuda", N=96, K=256)
    K, G = 256, 64
    H = torch.zeros((K, K), device="cuda")
    # two partial Hessians over the two token halves, summed: the same H as one call
    for t0, t1 in (sharded.token_range(512, 0, 2), sharded.token_range(512, 1, 2)):
        hq.hq_hessian_accumulate(H, X[t0:t1])
    Hf = torch.zeros((K, K), device="cuda")
    hq.hq_hessian_accumulate(Hf, X)
    torch.cuda.synchronize()
    assert torch.allclose(H, Hf, rtol=1e-5, atol=1e-3)
    imp = torch.rand(K, device="cuda") + 0.5
    codes, scales = hq.gptq_outputs(96, K, G)
    ws = hq.alloc_workspace(hq.hq_gptq_workspace_bytes(96, K, G))
    q_full = hq.hq_gptq_quantize(W, Hf, G, 0.01, codes, scales, ws, imp=imp)
    terms = torch.empty(2, dtype=torch.float64, device="cuda")
    hq.hq_qerr_terms(ws, terms)
    num, den = terms.tolist()
    assert math.sqrt(num / den) == pytest.approx(q_full, rel=1e-15)
    # the rows in two shards: identical codes and scales, sums adding up to the layer's
    tot = [0.0, 0.0]
    for r in range(2):
        r0, r1 = sharded.row_range(96, r, 2)
        c, s = hq.gptq_outputs(r1 - r0, K, G)
        w2 = hq.alloc_workspace(hq.hq_gptq_workspace_bytes(r1 - r0, K, G))
        hq.hq_gptq_quantize(W[r0:r1].contiguous(), Hf, G, 0.01, c, s, w2, imp=imp, want_qerr=False)
        t = torch.empty(2, dtype=torch.float64, device="cuda")
        hq.hq_qerr_terms(w2, t)
        torch.cuda.synchronize()
        assert torch.equal(c, codes[r0:r1]) and torch.equal(s, scales[r0:r1])
        tot = [tot[0] + t[0].item(), tot[1] + t[1].item()]
    assert math.sqrt(tot[0] / tot[1]) == pytest.approx(q_full, rel=1e-12)
    # the whole exchange through a one-rank NCCL group
    os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
    os.environ["MASTER_PORT"] = str(_free_port())
    dist.init_process_group("nccl", rank=0, world_size=1)
    try:
        Hs = Hf.clone()
        sharded.allreduce_hessian(Hs)  # one rank: the sum is its own partial
        c, s = hq.gptq_outputs(96, K, G)
        q = sharded.gptq_row_shard(hq, W, Hs, G, 0.01, c, s, ws, imp=imp)
        torch.cuda.synchronize()
        assert torch.equal(Hs, Hf)
        assert torch.equal(c, codes) and torch.equal(s, scales)
        assert q == pytest.approx(q_full, rel=1e-15)
    finally:
        dist.destroy_process_group()
