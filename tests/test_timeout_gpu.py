"""Failure detection without a GPU fault: a bounded device wait runs out.

The self-test kernel waits on a barrier that nothing completes; the wait
gives up after the limit, the device error word reports
FA_ERR_DEVICE_TIMEOUT, the host reads and clears it, and the same context
then runs attention correctly.  Nothing traps, faults or hangs.
"""
import time

import pytest
import torch

import exact_attention_143_b200 as fa
import oracle
from seeded_inputs import make_qkv
from tests.parity import check_o, to64

pytestmark = pytest.mark.gpu


def test_wait_timeout_is_reported_and_context_survives():
    assert fa.get_device_error() == fa.FA_OK
    t0 = time.perf_counter()
    status = fa.selftest_wait_timeout(50_000_000)  # 50 ms
    elapsed = time.perf_counter() - t0
    assert status == fa.FA_ERR_DEVICE_TIMEOUT
    assert elapsed < 5.0
    assert fa.get_device_error() == fa.FA_OK  # the word was cleared by the read
    q, k, v = make_qkv(1, 200, 200, 2, 2, 64, torch.float16, 30)
    o, lse = fa.fa_fwd(q.cuda(), k.cuda(), v.cuda(), causal=True)
    torch.cuda.synchronize()
    assert fa.get_device_error() == fa.FA_OK
    o_ref, _ = oracle.attention_fwd(to64(q), to64(k), to64(v), 0.125, True)
    check_o(o, o_ref, torch.float16)


def test_selftest_rejects_bad_limit():
    with pytest.raises(fa.FAError):
        fa.selftest_wait_timeout(0)
