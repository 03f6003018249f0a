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
    """Hessians from the oracle (fp64 X^T X of seeded activations, rounded to fp32) are written
    into a package through the library's encoder and read back through its decoder: every
    .hessian payload is the oracle's Bf16TrilDiagF32 encoding of the same matrix byte for byte,
    load_hessian returns the oracle's decoding bit for bit, and the .imatrix payload is the
    importance vector written."""
    import oracle
    import post_weight_quantization_tcgen05_b200 as hq
    import workloads as wl
    tensors, ref_H = [], []
    for i, K in enumerate((256, 384)):
        cfg = wl.small_config(wl.CONFIGS[1], N=8, K=K, T=1024, seed=i + 1)
        X = wl.make_activations(cfg, "cpu")
        H32 = oracle.hessian(X.double().numpy()).astype(np.float32)
        imp32 = oracle.imatrix(H32.astype(np.float64), cfg.T).astype(np.float32)
        tensors.append((f"layers.{i}.mlp", torch.from_numpy(H32).cuda(), torch.from_numpy(imp32).cuda()))
        ref_H.append(H32)
    path = str(tmp_path / "m.calib.hfq")
    hfqm.write_package(hq, path, 42, {"tokens": 1024}, tensors)
    arch, meta, entries, buf = hfqm.read_package(path)
    assert arch == 42 and meta == {"tokens": 1024} and len(entries) == 4
    for (name, H, imp), H32, eh, ei in zip(tensors, ref_H, entries[0::2], entries[1::2]):
        K = H.shape[0]
        assert eh.name == name + ".hessian" and eh.shape == (K, K) and eh.quant_type == 130
        enc = oracle.bf16tril_encode(H32)
        assert bytes(buf[eh.offset:eh.offset + eh.data_size]) == enc
        got = hfqm.load_hessian(hq, buf, eh)
        torch.cuda.synchronize()
        assert np.array_equal(got.cpu().numpy().view(np.uint32), oracle.bf16tril_decode(enc, K).view(np.uint32))
        assert torch.equal(hfqm.load_imatrix(buf, ei), imp)
        proj = hfqm.load_hessian(hq, buf, eh, project=True)
        ref_proj = oracle.project_psd(oracle.bf16tril_decode(enc, K).astype(np.float64))
        err = np.linalg.norm(proj.double().cpu().numpy() - ref_proj) / np.linalg.norm(ref_proj)
        assert err < 1e-5, err
