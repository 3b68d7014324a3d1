"""Failure detection without a GPU fault.

Every wait inside the library's kernels is bounded. When one runs out, the
kernel records MFA_ERR_TIMEOUT in the device status word, skips the work that
depended on it and returns, so the context stays usable. The self-test entry
point makes one such wait run out on purpose: the decode call's combine kernel
waits for two partial outputs whose flags nothing ever sets. The test checks
the reported status, the elapsed time against the limit, and that the next
ordinary call is correct.
"""
import numpy as np
import pytest
import torch

from decode_attention_08_b200 import inputs as gen
from decode_attention_08_b200 import mfa

from helpers import assert_close, decode_atol, oracle_decode, run_decode

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("limit_ms", [1, 20])
def test_bounded_wait_runs_out_and_reports_timeout(limit_ms):
    assert mfa.read_status() == 0
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    start.record()
    mfa.selftest_wait_timeout(limit_ms * 1_000_000)
    end.record()
    assert mfa.read_status() == mfa.STATUS_CODES["MFA_ERR_TIMEOUT"]
    elapsed = start.elapsed_time(end)
    assert limit_ms <= elapsed < limit_ms + 50, elapsed
    assert mfa.read_status() == 0  # cleared by the previous read


def test_context_stays_usable_after_a_timeout():
    mfa.selftest_wait_timeout(2_000_000)
    assert mfa.read_status() == mfa.STATUS_CODES["MFA_ERR_TIMEOUT"]
    lens = [3000, 1, 129, 700]
    dec = gen.make_decode_inputs(701, len(lens), lens)
    got = run_decode(dec)  # asserts a clean status
    ref, _ = oracle_decode(dec)
    assert_close(got, ref, decode_atol(dec, ref, torch.float32), "after timeout")


def test_selftest_rejects_bad_limits():
    with pytest.raises(mfa.MfaError):
        mfa.selftest_wait_timeout(0)
    with pytest.raises(mfa.MfaError):
        mfa.selftest_wait_timeout(10**11)
