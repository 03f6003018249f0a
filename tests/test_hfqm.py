"""HFQM calibration packages ("hipfire-calib-data" dataset card, ".calib.hfq — HFQM
calibration package"): the framing against a package written out by hand from the card's
layout (tests/golden/hfqm_small.txt), round trips of the reader and writer, refusals of
malformed packages, and on the GPU a package of real Hessians through the library's codec."""

import os

import numpy as np
import pytest
import torch

from post_weight_quantization_tcgen05_b200 import hfqm

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "hfqm_small.txt")


def _golden_bytes() -> bytes:
    out = b""
    for line in open(GOLDEN):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        out += bytes.fromhex("".join(line.split()[1:]))
    return out


def test_framing_matches_the_hand_built_package():
    g = _golden_bytes()
    assert len(g) == 80
    e = hfqm.Entry("t.imatrix", hfqm.QT_F32, (2,), 0, 8)
    got = hfqm.build_package(7, {"a": 1}, [e], [np.array([1.0, 2.0], dtype="<f4").tobytes()])
    assert got == g
    arch, meta, entries = hfqm.parse_package(g)
    assert arch == 7 and meta == {"a": 1}
    assert entries == [hfqm.Entry("t.imatrix", 0, (2,), 0, 8, 72)]


def test_round_trip_of_several_entries_and_unicode_metadata(tmp_path):
    rng = np.random.default_rng(4)
    meta = {"arch": "qwen3.8", "note": "calibration — 4.5M tokens", "n": [1, 2, 3]}
    entries, payloads = [], []
    for i, K in enumerate((4, 9)):
        p = rng.integers(0, 256, K * 4 + K * (K - 1), dtype=np.uint8).tobytes()
        entries.append(hfqm.Entry(f"layers.{i}.w.hessian", hfqm.QT_BF16_TRIL_DIAG_F32, (K, K), 0, len(p)))
        payloads.append(p)
        q = rng.random(K).astype("<f4").tobytes()
        entries.append(hfqm.Entry(f"layers.{i}.w.imatrix", hfqm.QT_F32, (K,), 0, len(q)))
        payloads.append(q)
    buf = hfqm.build_package(3, meta, entries, payloads)
    arch, m, got = hfqm.parse_package(buf)
    assert arch == 3 and m == meta and len(got) == 4
    for e, g, p in zip(entries, got, payloads):
        assert (g.name, g.quant_type, g.shape, g.group_size, g.data_size) == \
            (e.name, e.quant_type, e.shape, e.group_size, e.data_size)
        assert buf[g.offset:g.offset + g.data_size] == p


def test_malformed_packages_are_refused():
    g = _golden_bytes()
    with pytest.raises(ValueError):
        hfqm.parse_package(b"HFQX" + g[4:])
    with pytest.raises(ValueError):
        hfqm.parse_package(g[:20])
    bad = bytearray(g)
    bad[12] = 2  # n_entries in the header no longer matches the index
    with pytest.raises(ValueError):
        hfqm.parse_package(bytes(bad))
    with pytest.raises(ValueError):
        hfqm.parse_package(g[:-1])  # payload cut short


@pytest.mark.gpu
def test_package_of_hessians_through_the_codec(tmp_path, cuda_device):
    import post_weight_quantization_tcgen05_b200 as hq
    import workloads as wl
    tensors = []
    for i, K in enumerate((256, 384)):
        cfg = wl.small_config(wl.CONFIGS[1], N=8, K=K, T=1024, seed=i + 1)
        X = wl.make_activations(cfg, "cuda")
        H = torch.zeros((K, K), device="cuda")
        hq.hq_hessian_accumulate(H, X)
        imp = torch.empty(K, device="cuda")
        hq.hq_imatrix(H, cfg.T, imp)
        tensors.append((f"layers.{i}.mlp", H, imp))
    path = str(tmp_path / "m.calib.hfq")
    hfqm.write_package(hq, path, 42, {"tokens": 1024}, tensors)
    arch, meta, entries, buf = hfqm.read_package(path)
    assert arch == 42 and meta == {"tokens": 1024} and len(entries) == 4
    for (name, H, imp), eh, ei in zip(tensors, entries[0::2], entries[1::2]):
        K = H.shape[0]
        assert eh.name == name + ".hessian" and eh.shape == (K, K)
        ref = torch.empty((K, K), device="cuda")
        tril = torch.empty(hq.hq_bf16tril_bytes(K), dtype=torch.uint8, device="cuda")
        hq.hq_hessian_pack_bf16tril(H, tril)
        hq.hq_hessian_unpack_bf16tril(tril, K, ref)
        got = hfqm.load_hessian(hq, buf, eh)
        torch.cuda.synchronize()
        assert torch.equal(got, ref)
        assert torch.equal(hfqm.load_imatrix(buf, ei), imp)
        proj = hfqm.load_hessian(hq, buf, eh, project=True)
        assert float(torch.linalg.norm(proj - ref) / torch.linalg.norm(ref)) < 1e-3
