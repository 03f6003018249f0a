"""The bounds-checking build (libhq_bounds.so, HQ_DEBUG_BOUNDS) on a representative run of the
kernels: no index check fails, the results are bit-identical to libhq.so's, and a check that
fails by construction is recorded with its file tag and line."""

import os
import subprocess
import sys

import pytest
import torch

import bounds_workload

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def hq():
    import post_weight_quantization_tcgen05_b200 as m
    return m


def test_bounds_build_finds_no_violation_and_changes_no_bit(hq, cuda_device, tmp_path):
    lib = os.path.join(ROOT, "post_weight_quantization_tcgen05_b200", "libhq_bounds.so")
    assert os.path.exists(lib), "libhq_bounds.so not built (build.py --all)"
    ref, ref_words = bounds_workload.run_all(hq)
    assert all(w == 0 for w in ref_words.values())  # the regular build never records
    out = tmp_path / "bounds.pt"
    env = dict(os.environ, HQ_LIBRARY="libhq_bounds.so")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "tests", "bounds_workload.py"), str(out)],
                       env=env, cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stdout + r.stderr
    res = torch.load(out)
    assert res["library"] == "libhq_bounds.so" and res["enabled"] is True
    bad = {k: (w >> 16, w & 0xFFFF) for k, w in res["words"].items() if w != 0}
    assert not bad, f"index checks failed (file tag, line): {bad}"
    for k, v in ref.items():
        assert torch.equal(v, res["outputs"][k]), k
    tag, line = res["selftest"] >> 16, res["selftest"] & 0xFFFF
    assert tag == hq.bounds_file_tag("api.cu") and line > 0, res["selftest"]
