"""Bounded waits: a wait that nothing completes ends with a status, not a hang.

The probe kernel waits on a shared-memory barrier that no thread ever arrives
on, with a 2 ms limit; the device records SQA_ERR_TIMEOUT, the host reads it,
and the context stays usable for the next launch.
"""
import pytest

from helpers import attn_inputs, run_attn

pytestmark = pytest.mark.gpu


def test_stuck_wait_times_out_and_context_survives():
    import reduced_query_head_b200 as sqa
    assert sqa.sqa_device_status() == sqa.SQA_OK
    assert sqa.sqa_check_wait_timeout(2_000_000) == sqa.SQA_ERR_TIMEOUT
    assert sqa.sqa_device_status() == sqa.SQA_OK           # read-and-clear
    qb, kb, vb = attn_inputs(1, 256, 4, 2, 64, 1)
    out = run_attn(qb, kb, vb, False, 0.125)              # still launches and completes
    assert out.isfinite().all()


def test_short_wait_limit_does_not_disturb_normal_runs():
    import reduced_query_head_b200 as sqa
    prev = sqa.sqa_set_wait_limit_ns(200_000_000)
    try:
        qb, kb, vb = attn_inputs(1, 4096, 8, 2, 64, 2)
        run_attn(qb, kb, vb, True, 0.125)
        assert sqa.sqa_device_status() == sqa.SQA_OK
    finally:
        sqa.sqa_set_wait_limit_ns(prev)
