"""The device status word: a condition raised on a plan is reported once by
gtq_status and then cleared, and decoding goes on giving correct results.

The condition is set from the host with gtq_raise_status, the same bit a
kernel sets when a bounded wait expires or a norm is clamped, so no GPU is
made to fault or hang."""

import numpy as np
import pytest

torch = pytest.importorskip("torch")

import decode_attention_13_b200 as gtq  # noqa: E402
from tests.test_gpu_parity import Case, check_case  # noqa: E402

pytestmark = pytest.mark.gpu


def test_raised_timeout_is_reported_once_then_cleared():
    c = Case(1, 2, 4, 300, 3, 3, seed=41)
    c.quantize()
    c.decode()
    assert gtq.gtq_status(c.plan) == gtq.GTQ_OK
    gtq.gtq_raise_status(c.plan, gtq.GTQ_ERR_TIMEOUT)
    assert gtq.gtq_status(c.plan) == gtq.GTQ_ERR_TIMEOUT
    assert gtq.gtq_status(c.plan) == gtq.GTQ_OK


def test_timeout_takes_precedence_over_overflow():
    c = Case(1, 1, 2, 100, 2, 2, seed=42)
    gtq.gtq_raise_status(c.plan, gtq.GTQ_ERR_OVERFLOW)
    assert gtq.gtq_status(c.plan) == gtq.GTQ_ERR_OVERFLOW
    gtq.gtq_raise_status(c.plan, gtq.GTQ_ERR_OVERFLOW)
    gtq.gtq_raise_status(c.plan, gtq.GTQ_ERR_TIMEOUT)
    assert gtq.gtq_status(c.plan) == gtq.GTQ_ERR_TIMEOUT
    assert gtq.gtq_status(c.plan) == gtq.GTQ_OK


def test_only_device_conditions_can_be_raised():
    c = Case(1, 1, 2, 64, 2, 2, seed=43)
    with pytest.raises(gtq.GtqError):
        gtq.gtq_raise_status(c.plan, gtq.GTQ_ERR_INVALID)
    assert gtq.gtq_status(c.plan) == gtq.GTQ_OK


def test_decoding_after_a_reported_condition():
    # the caller's recovery: read the status, build a fresh plan; both the fresh
    # plan and the old one (whose merge state was not disturbed) decode correctly
    c = Case(1, 2, 4, 700, 3, 3, seed=44)
    c.quantize()
    gtq.gtq_raise_status(c.plan, gtq.GTQ_ERR_TIMEOUT)
    assert gtq.gtq_status(c.plan) == gtq.GTQ_ERR_TIMEOUT
    check_case(c, quantized=True)
    fresh = Case(1, 2, 4, 700, 3, 3, seed=44)
    ref = check_case(fresh)
    assert np.all(np.isfinite(ref))
