"""Fault path of the bounded waits, exercised without faulting the GPU.

A self-test kernel waits on a barrier that nothing will complete, with a short
bound.  The wait must run out, record FA_ERR_DEVICE_TIMEOUT in the device status
word and return; the context must stay usable for normal work afterwards.
"""
import pytest
import torch

import oracle
import parity
import workloads

pytestmark = pytest.mark.gpu


def test_wait_timeout_is_reported_and_context_survives():
    import exact_attention_132_b200 as fa
    assert fa.fa_get_device_status() == 0
    fa.fa_debug_wait_timeout_selftest(2000)        # 2 ms bound
    code = fa.fa_get_device_status()
    assert code >> 24 == fa.FA_ERR_DEVICE_TIMEOUT
    assert code & 0xFFFFFF == 99                   # the self-test's wait site
    assert fa.fa_get_device_status() == 0          # reading clears the word
    # the context still runs real work correctly
    w = workloads.make_small(1, 2, 256, 64, True, seed=1, backward=False)
    q, k, v = workloads.make_bf16_inputs(w)
    o, lse = fa.attention_forward(q.cuda(), k.cuda(), v.cuda(), causal=True)
    o_ref, lse_ref = oracle.attention_fwd(q, k, v, w.sm_scale, True)
    parity.assert_fwd_ok(o, lse, o_ref, lse_ref)
    assert fa.fa_get_device_status() == 0


def test_selftest_rejects_bad_bound():
    import exact_attention_132_b200 as fa
    with pytest.raises(fa.FAError):
        fa.fa_debug_wait_timeout_selftest(0)
