"""Host logic of the stored-Hessian helpers ("hipfire-calib-data" card, "REQUIRED: project to PSD
before Cholesky"), on the CPU with a stand-in for the library: the damping escalation's
sequence and refusals, and the decode-then-project order of load_stored_hessian."""

import types

import pytest
import torch

from post_weight_quantization_tcgen05_b200 import stored_hessian


class _Err(Exception):
    def __init__(self, status):
        super().__init__(f"status {status}")
        self.status = status


def _fake_library(works_from: float, other_error_at=None):
    """hq_gptq_quantize fails with NOT_PD below `works_from` (and with another status at
    `other_error_at`); records every damping it is called with."""
    calls = []

    def quantize(W, H, group, damp, codes, scales, ws, imp=None):
        calls.append(damp)
        if other_error_at is not None and damp >= other_error_at:
            raise _Err(5)
        if damp < works_from:
            raise _Err(3)
        return 0.125

    return types.SimpleNamespace(HQError=_Err, HQ_ERR_NOT_PD=3, hq_gptq_quantize=quantize), calls


def test_escalation_multiplies_until_the_factorisation_succeeds():
    hq, calls = _fake_library(works_from=0.5)
    q, d = stored_hessian.quantize_with_damping_escalation(hq, None, None, 128, 0.01, None, None, None)
    assert q == 0.125 and d == pytest.approx(1.0)
    assert calls == pytest.approx([0.01, 0.1, 1.0])


def test_escalation_stops_at_the_cap_and_raises():
    hq, calls = _fake_library(works_from=2.0)
    with pytest.raises(_Err) as e:
        stored_hessian.quantize_with_damping_escalation(hq, None, None, 128, 0.01, None, None, None, cap=0.5)
    assert e.value.status == 3
    assert calls == pytest.approx([0.01, 0.1, 0.5])


def test_first_success_needs_no_escalation():
    hq, calls = _fake_library(works_from=0.0)
    _, d = stored_hessian.quantize_with_damping_escalation(hq, None, None, 128, 0.01, None, None, None)
    assert d == 0.01 and calls == [0.01]


def test_other_errors_are_not_escalated():
    hq, calls = _fake_library(works_from=1.0, other_error_at=0.05)
    with pytest.raises(_Err) as e:
        stored_hessian.quantize_with_damping_escalation(hq, None, None, 128, 0.01, None, None, None)
    assert e.value.status == 5
    assert calls == pytest.approx([0.01, 0.1])


@pytest.mark.parametrize("damp,factor,cap", [(0.0, 10.0, 1.0), (0.01, 1.0, 1.0), (0.5, 10.0, 0.1)])
def test_escalation_refuses_bad_arguments(damp, factor, cap):
    hq, calls = _fake_library(works_from=0.0)
    with pytest.raises(ValueError):
        stored_hessian.quantize_with_damping_escalation(hq, None, None, 128, damp, None, None, None,
                                                        factor=factor, cap=cap)
    assert calls == []


def test_load_decodes_then_projects():
    order = []

    def unpack(payload, K, H):
        order.append(("unpack", K, tuple(H.shape)))

    def project(H, workspace=None, steps=40):
        order.append(("project", steps))

    hq = types.SimpleNamespace(hq_hessian_unpack_bf16tril=unpack, hq_hessian_project_psd=project)
    payload = torch.zeros(16, dtype=torch.uint8)
    H = stored_hessian.load_stored_hessian(hq, payload, 3, steps=12)
    assert H.dtype == torch.float32 and tuple(H.shape) == (3, 3)
    assert order == [("unpack", 3, (3, 3)), ("project", 12)]
    order.clear()
    stored_hessian.load_stored_hessian(hq, payload, 3, project=False)
    assert order == [("unpack", 3, (3, 3))]
