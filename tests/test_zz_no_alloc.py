"""hq_rtn_quantize_noalloc against hq_rtn_quantize.

The allocation-free entry point serves callers that cannot give the library scratch memory
(an application whose device memory is all reserved by its own pool, a service that forbids
allocation after start-up, a plugin under another framework's allocator).  It must produce
exactly what the workspace entry point produces, call after call, although every call reuses
the same library-owned scratch array.  This file is collected last on purpose.
"""

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def hq():
    import post_weight_quantization_tcgen05_b200 as m
    return m


def _reference(hq, W, G, imp):
    N, K = W.shape
    codes, scales = hq.gptq_outputs(N, K, G)
    ws = hq.alloc_workspace(hq.hq_rtn_workspace_bytes(N, K, G))
    q = hq.hq_rtn_quantize(W, G, codes, scales, ws, imp=imp)
    return codes.cpu().numpy(), scales.cpu().numpy(), q


def test_noalloc_matches_workspace_entry_point_twice(hq, cuda_device):
    g = torch.Generator(device="cuda")
    g.manual_seed(123)
    cases = [(96, 256, 32, torch.float32, False), (700, 512, 128, torch.bfloat16, True)]
    for N, K, G, dt, use_imp in cases:  # two calls in a row on the shared scratch
        W = (torch.randn((N, K), generator=g, device="cuda") * 0.05).to(dt)
        imp = torch.rand(K, generator=g, device="cuda") + 0.5 if use_imp else None
        codes, scales = hq.gptq_outputs(N, K, G)
        qd = torch.zeros(1, dtype=torch.float64, device="cuda")
        q = hq.hq_rtn_quantize_noalloc(W, G, codes, scales, imp=imp, qerr_dev=qd)
        torch.cuda.synchronize()
        rc, rs, rq = _reference(hq, W, G, imp)
        assert np.array_equal(codes.cpu().numpy(), rc)
        assert np.array_equal(scales.cpu().numpy(), rs)
        assert abs(q - rq) <= 1e-12 * rq and qd.item() == q


def test_noalloc_commits_no_memory_after_its_first_call(hq, cuda_device):
    """The property the entry point exists for: once a first call on the device has loaded the
    library's scratch array, later calls leave the device's free memory unchanged."""
    N, K, G = 256, 1024, 64
    g = torch.Generator(device="cuda")
    g.manual_seed(5)
    W = torch.randn((N, K), generator=g, device="cuda")
    codes, scales = hq.gptq_outputs(N, K, G)
    qd = torch.zeros(1, dtype=torch.float64, device="cuda")
    hq.hq_rtn_quantize_noalloc(W, G, codes, scales, qerr_dev=qd, want_qerr=False)  # warm-up
    torch.cuda.synchronize()
    free0 = torch.cuda.mem_get_info()[0]
    for _ in range(2):
        hq.hq_rtn_quantize_noalloc(W, G, codes, scales, qerr_dev=qd, want_qerr=False)
    torch.cuda.synchronize()
    assert torch.cuda.mem_get_info()[0] == free0


def test_noalloc_at_exactly_the_scratch_limit(hq, cuda_device):
    """N * (K / group) equal to the scratch's capacity is accepted and matches the workspace
    entry point."""
    N, K, G = 8192, 2048, 16
    assert N * (K // G) == hq.HQ_RTN_NOALLOC_MAX_GROUPS
    g = torch.Generator(device="cuda")
    g.manual_seed(9)
    W = torch.rand((N, K), generator=g, device="cuda") * 2.0 - 1.0
    codes, scales = hq.gptq_outputs(N, K, G)
    q = hq.hq_rtn_quantize_noalloc(W, G, codes, scales)
    torch.cuda.synchronize()
    rc, rs, rq = _reference(hq, W, G, None)
    assert np.array_equal(codes.cpu().numpy(), rc)
    assert np.array_equal(scales.cpu().numpy(), rs)
    assert abs(q - rq) <= 1e-12 * rq


def test_noalloc_refuses_more_groups_than_its_scratch(hq, cuda_device):
    W = torch.zeros((8, 64), device="cuda")
    codes, scales = hq.gptq_outputs(8, 64, 32)
    raw = hq.lib.hq_rtn_quantize_noalloc  # N * (K / group) beyond the scratch: refused, nothing launched
    limit = hq.HQ_RTN_NOALLOC_MAX_GROUPS
    st = raw(W.data_ptr(), hq.HQ_F32, limit // 2 + 1, 64, 32, None, codes.data_ptr(), scales.data_ptr(),
                    None, None, None)
    assert st == hq.HQ_ERR_UNSUPPORTED
