"""The multi-GPU split of the path (package module `sharded`): the host logic and the exchange
on CPU with two gloo ranks and a stand-in for the library calls (partial Hessians summed through
the packed lower triangle; one factorisation on the root, broadcast; each rank's sweep of its
rows; qerr from the summed terms; a failed factorisation reported on every rank), and on one GPU
the library calls the split relies on, against the oracle."""

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


class _HostLib:
    """A CPU stand-in for the library calls the split makes (test infrastructure: the oracle
    plays the kernels), so that the exchange itself runs on gloo ranks without a GPU.  The factor
    buffer carries a status word and U (fp64) as bytes, like the real one carries its header and
    U' split; the sweep workspace keeps the qerr sums."""

    class HQError(RuntimeError):
        def __init__(self, status, where):
            self.status = status
            super().__init__(f"{where}: {status}")

    HQ_ERR_INVALID = 1
    HQ_ERR_NOT_PD = 3

    @staticmethod
    def alloc_workspace(n, device="cpu"):
        return torch.zeros(max(int(n), 1), dtype=torch.uint8, device=device)

    @staticmethod
    def hq_tril32_count(K):
        return K * (K + 1) // 2

    @staticmethod
    def hq_hessian_pack_lower(H, packed):
        i, j = np.tril_indices(H.shape[0])
        packed.copy_(H[torch.from_numpy(i), torch.from_numpy(j)])

    @staticmethod
    def hq_hessian_unpack_lower(packed, K, H):
        i, j = np.tril_indices(K)
        H[torch.from_numpy(i), torch.from_numpy(j)] = packed

    @staticmethod
    def hq_qerr_from_terms(terms, q):
        num, den = terms.tolist()
        q[0] = 0.0 if den == 0.0 else math.sqrt(num / den)

    @staticmethod
    def hq_gptq_factor_bytes(K):
        return 8 + 8 * K * K

    @staticmethod
    def hq_gptq_factor_workspace_bytes(K):
        return 1

    @staticmethod
    def hq_gptq_sweep_workspace_bytes(n, K, group):
        return 16

    @classmethod
    def hq_gptq_factorize(cls, H, damp, factor, ws):
        K = H.shape[0]
        Hn = H.double().numpy()
        Hs = np.tril(Hn) + np.tril(Hn, -1).T
        try:
            Hd, _ = oracle.damp_hessian(Hs, damp)
            U = oracle.upper_factor_of_inverse(Hd)
            status = 0
        except oracle.NotPositiveDefinite:
            U, status = np.zeros((K, K)), cls.HQ_ERR_NOT_PD
        except ValueError:  # mean(diag H) not positive
            U, status = np.zeros((K, K)), cls.HQ_ERR_INVALID
        factor[:8] = torch.from_numpy(np.array([status], np.int64).view(np.uint8))
        factor[8:] = torch.from_numpy(np.ascontiguousarray(U).view(np.uint8).ravel())
        if status:
            raise cls.HQError(status, "hq_gptq_factorize")

    @classmethod
    def hq_gptq_sweep(cls, W, factor, group, codes, scales, ws, imp=None, want_qerr=True):
        K = W.shape[1]
        status = int(factor[:8].numpy().view(np.int64)[0])
        if status:
            raise cls.HQError(status, "hq_gptq_sweep")
        U = factor[8:].numpy().view(np.float64).reshape(K, K)
        Wn = W.double().numpy()
        c, sc, _ = oracle.gptq_sweep(Wn, U, group)
        codes.copy_(torch.from_numpy(oracle.pack_int4(c)))
        scales.copy_(torch.from_numpy(sc))
        D = Wn - oracle.dequantize(c, sc, group)
        w = np.ones(K) if imp is None else imp.double().numpy()
        ws[:16] = torch.from_numpy(np.array([np.sum((D * D) @ w), np.sum((Wn * Wn) @ w)]).view(np.uint8))

    @staticmethod
    def hq_qerr_terms(ws, terms):
        terms.copy_(torch.from_numpy(ws[:16].numpy().view(np.float64).copy()))


def _rank_main(rank: int, world: int, port: int, out, not_pd: bool = False):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        hq = _HostLib()
        rng = np.random.default_rng(11)  # the same data on every rank
        T, K, N, G = 103, 64, 9, 32
        X = rng.standard_normal((T, K))
        # partial Hessian over this rank's tokens (a CPU stand-in for hq_hessian_accumulate),
        # upper triangle filled with garbage that the packed exchange must leave alone
        t0, t1 = sharded.token_range(T, rank, world)
        Hp = X[t0:t1].T @ X[t0:t1]
        H = torch.from_numpy(np.tril(Hp) + np.triu(np.full((K, K), -7.0 - rank), 1))
        sharded.allreduce_hessian(hq, H)
        Hn = H.numpy()
        lo = np.tril(np.ones((K, K), bool))
        h_err = float(np.abs(Hn[lo] - (X.T @ X)[lo]).max() / np.abs(X.T @ X).max())
        upper_kept = bool(np.all(Hn[~lo] == -7.0 - rank))
        # GPTQ with one factorisation on rank 0, broadcast, each rank its own rows
        W = rng.uniform(-1, 1, (N, K))
        imp = torch.from_numpy(rng.uniform(0.5, 2.0, K))
        r0, r1 = sharded.row_range(N, rank, world)
        codes = torch.zeros((r1 - r0, K // 2), dtype=torch.uint8)
        scales = torch.zeros((r1 - r0, K // G), dtype=torch.float32)
        Hbad = 5.0 * np.eye(K)
        Hbad[3, 3] = -1.0  # indefinite, positive mean diagonal
        Hg = torch.from_numpy(Hbad) if not_pd else H
        try:
            q = sharded.gptq_row_shard(hq, torch.from_numpy(W[r0:r1]), Hg if rank == 0 else None, G, 0.01, codes,
                                       scales, imp=imp)
            err = None
        except _HostLib.HQError as e:
            q, err = None, e.status
        out.put((rank, h_err, upper_kept, q, err, codes.numpy().copy(), scales.numpy().copy()))
    finally:
        dist.destroy_process_group()


def _run_two_ranks(not_pd=False):
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, out, not_pd)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted((out.get(timeout=120) for _ in procs), key=lambda r: r[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    return res


def test_two_gloo_ranks_hessian_allreduce_and_row_split_gptq():
    """Two gloo ranks: the packed lower-triangle all-reduce gives X^T X (upper triangles untouched);
    one factorisation on rank 0, broadcast, and each rank's sweep of its rows give the oracle's
    whole-layer codes, scales and qerr."""
    res = _run_two_ranks()
    rng = np.random.default_rng(11)
    T, K, N, G = 103, 64, 9, 32
    X = rng.standard_normal((T, K))
    W = rng.uniform(-1, 1, (N, K))
    imp = rng.uniform(0.5, 2.0, K)
    ref = oracle.gptq_quantize(W, X.T @ X, G, 0.01)
    q_ref = oracle.qerr(W, ref["codes"], ref["scales"], G, imp)
    codes = np.concatenate([oracle.unpack_int4(r[5]) for r in res])
    scales = np.concatenate([r[6] for r in res])
    for _, h_err, upper_kept, q, err, _, _ in res:
        assert h_err < 1e-13 and upper_kept and err is None
        assert q == pytest.approx(q_ref, rel=1e-10)
    assert np.array_equal(codes, ref["codes"])
    assert np.allclose(scales, ref["scales"], rtol=1e-6)


def test_two_gloo_ranks_failed_factorisation_reaches_every_rank():
    """A Hessian that is not positive definite on the root: every rank raises HQ_ERR_NOT_PD after
    the same collective steps (no rank is left waiting)."""
    res = _run_two_ranks(not_pd=True)
    assert [r[4] for r in res] == [_HostLib.HQ_ERR_NOT_PD, _HostLib.HQ_ERR_NOT_PD]


@pytest.mark.gpu
def test_row_shards_against_one_factorisation_match_the_oracle(cuda_device):
    """On one GPU: the token-split Hessian summed through the packed lower triangle; one
    hq_gptq_factorize, two hq_gptq_sweep row shards on separate sweep workspaces; their codes and
    scales are hq_gptq_quantize's bit for bit and match the plain oracle (codes >= 99 %, scales
    before divergence 1e-4, qerr 1 %); the shards' qerr sums combine through hq_qerr_from_terms."""
    import post_weight_quantization_tcgen05_b200 as hq
    import workloads as wl
    from gpu_helpers import QERR_REL, check_gptq_parity
    N, K, G = 96, 384, 64
    cfg = wl.correlated_config(N, K, T=768, group=G, seed=5)
    X = wl.make_activations(cfg, "cuda")
    W = wl.make_weights(cfg, "cuda", N=N, K=K)
    parts = []
    for r in range(2):
        t0, t1 = sharded.token_range(768, r, 2)
        Hr = torch.zeros((K, K), device="cuda")
        hq.hq_hessian_accumulate(Hr, X[t0:t1])
        p = torch.empty(hq.hq_tril32_count(K), device="cuda")
        hq.hq_hessian_pack_lower(Hr, p)
        parts.append(p)
    H = torch.full((K, K), 5.0, device="cuda")
    hq.hq_hessian_unpack_lower(parts[0] + parts[1], K, H)
    Hf = torch.zeros((K, K), device="cuda")
    hq.hq_hessian_accumulate(Hf, X)
    torch.cuda.synchronize()
    lo = torch.ones((K, K), dtype=torch.bool, device="cuda").tril()
    assert torch.allclose(H[lo], Hf[lo], rtol=1e-5, atol=1e-3) and bool((H[~lo] == 5.0).all())
    imp = torch.rand(K, device="cuda") + 0.5
    codes, scales = hq.gptq_outputs(N, K, G)
    ws = hq.alloc_workspace(hq.hq_gptq_workspace_bytes(N, K, G))
    q_full = hq.hq_gptq_quantize(W, H, G, 0.01, codes, scales, ws, imp=imp)
    factor = torch.empty(hq.hq_gptq_factor_bytes(K), dtype=torch.uint8, device="cuda")
    hq.hq_gptq_factorize(H, 0.01, factor, hq.alloc_workspace(hq.hq_gptq_factor_workspace_bytes(K)))
    terms = torch.zeros(2, dtype=torch.float64, device="cuda")
    for r in range(2):
        r0, r1 = sharded.row_range(N, r, 2)
        c, s = hq.gptq_outputs(r1 - r0, K, G)
        w2 = hq.alloc_workspace(hq.hq_gptq_sweep_workspace_bytes(r1 - r0, K, G))
        hq.hq_gptq_sweep(W[r0:r1].contiguous(), factor, G, c, s, w2, imp=imp, want_qerr=False)
        t = torch.empty(2, dtype=torch.float64, device="cuda")
        hq.hq_qerr_terms(w2, t)
        torch.cuda.synchronize()
        assert torch.equal(c, codes[r0:r1]) and torch.equal(s, scales[r0:r1])
        terms += t
    q = torch.empty(1, dtype=torch.float64, device="cuda")
    hq.hq_qerr_from_terms(terms, q)
    assert q.item() == pytest.approx(q_full, rel=1e-12)
    # against the oracle: its own fp64 Hessian of the same X, its own U
    H64 = oracle.hessian(X.double().cpu().numpy())
    Hd, _ = oracle.damp_hessian(H64, 0.01)
    Wn = W.double().cpu().numpy()
    cg = oracle.unpack_int4(codes.cpu().numpy())
    rc, rs = check_gptq_parity(Wn, oracle.upper_factor_of_inverse(Hd), G, cg, scales.cpu().numpy(), "row shards")
    q_ref = oracle.qerr(Wn, rc, rs, G, imp.cpu().numpy())
    assert abs(q.item() - q_ref) <= QERR_REL * q_ref


@pytest.mark.gpu
def test_sharded_module_through_a_one_rank_nccl_group(cuda_device):
    """The module's exchange over a real NCCL group of one rank (the broadcast and all-reduces are
    then identities): the layer's codes against the oracle."""
    import post_weight_quantization_tcgen05_b200 as hq
    import workloads as wl
    from gpu_helpers import QERR_REL, check_gptq_parity
    N, K, G = 64, 256, 64
    cfg = wl.correlated_config(N, K, T=512, group=G, seed=8)
    X = wl.make_activations(cfg, "cuda")
    W = wl.make_weights(cfg, "cuda", N=N, K=K)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(_free_port())
    dist.init_process_group("nccl", rank=0, world_size=1)
    try:
        H = torch.zeros((K, K), device="cuda")
        hq.hq_hessian_accumulate(H, X)
        sharded.allreduce_hessian(hq, H)
        codes, scales = hq.gptq_outputs(N, K, G)
        q = sharded.gptq_row_shard(hq, W, H, G, 0.01, codes, scales)
        torch.cuda.synchronize()
    finally:
        dist.destroy_process_group()
    H64 = oracle.hessian(X.double().cpu().numpy())
    Hd, _ = oracle.damp_hessian(H64, 0.01)
    Wn = W.double().cpu().numpy()
    cg = oracle.unpack_int4(codes.cpu().numpy())
    rc, rs = check_gptq_parity(Wn, oracle.upper_factor_of_inverse(Hd), G, cg, scales.cpu().numpy(), "nccl one rank")
    q_ref = oracle.qerr(Wn, rc, rs, G)
    assert abs(q - q_ref) <= QERR_REL * q_ref
