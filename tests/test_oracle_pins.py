"""Pins of the fp64 oracle against facts other than itself (CPU only)."""
import numpy as np
import pytest

import oracle
import oracle_checks as oc
import workloads


@pytest.mark.parametrize("check", oc.FWD_CHECKS, ids=lambda f: f.__name__)
def test_oracle_forward_pins(check):
    assert check(oracle.attention_fwd)


@pytest.mark.parametrize("check", oc.BWD_CHECKS, ids=lambda f: f.__name__)
def test_oracle_backward_pins(check):
    assert check(oracle.attention_bwd)


def test_oracle_finite_differences():
    assert oc.check_finite_differences(oracle.attention_bwd, oracle.attention_fwd)


def test_oracle_matches_pages_fp32_magnitude():
    assert oc.check_fp32_sdpa_magnitude(oracle.attention_fwd)


@pytest.mark.parametrize("check", oc.PROBS_CHECKS, ids=lambda f: f.__name__)
def test_softmax_probs_pins(check):
    """P from the two-pass definition: rows sum to one, and P is the brute force's weights."""
    assert check(oracle.softmax_probs)


@pytest.mark.parametrize("causal", [False, True])
def test_online_equals_two_pass(causal):
    """Tiling independence: the blocked online softmax with random block sizes equals
    the two-pass definition, including K outlier rows that force max changes."""
    w = workloads.make_small(1, 2, 300, 32, causal, seed=9, backward=False)
    w = w.with_shape(outlier_frac=0.05)
    q, k, v = workloads.make_bf16_inputs(w)
    rng = np.random.default_rng(0)
    blocks = rng.integers(1, 97, size=17)
    o1, l1 = oracle.attention_fwd(q, k, v, w.sm_scale, causal)
    o2, l2 = oracle.attention_fwd_online(q, k, v, w.sm_scale, causal, blocks)
    assert np.abs(o1 - o2).max() <= 1e-12 * max(1.0, np.abs(o1).max())
    assert np.abs(l1 - l2).max() <= 1e-12 * np.abs(l1).max()


def test_row_subset_matches_full():
    w = workloads.make_small(2, 2, 200, 16, True, seed=4, backward=True)
    q, k, v, do = workloads.make_bf16_inputs(w)
    o, lse = oracle.attention_fwd(q, k, v, w.sm_scale, True)
    picks = np.array([[0, 0, 0], [1, 1, 199], [0, 1, 57], [1, 0, 128]])
    o2, l2 = oracle.attention_fwd_rows(q, k, v, w.sm_scale, True, picks)
    for n, (b, h, i) in enumerate(picks):
        assert np.abs(o2[n] - o[b, h, i]).max() < 1e-13
        assert abs(l2[n] - lse[b, h, i]) < 1e-13
    dq, _, _ = oracle.attention_bwd(q, k, v, do, w.sm_scale, True)
    dq2 = oracle.attention_bwd_rows_dq(q, k, v, do, w.sm_scale, True, picks)
    for n, (b, h, i) in enumerate(picks):
        assert np.abs(dq2[n] - dq[b, h, i]).max() < 1e-12
    dqh, dkh, dvh = oracle.attention_bwd(q, k, v, do, w.sm_scale, True, heads=[(1, 0)])
    _, dk, dv = oracle.attention_bwd(q, k, v, do, w.sm_scale, True)
    assert np.abs(dkh[0] - dk[1, 0]).max() < 1e-13 and np.abs(dvh[0] - dv[1, 0]).max() < 1e-13


def test_row_blocking_is_exact(monkeypatch):
    """Rows processed in blocks (for long heads) give the same numbers as one block."""
    from oracle import attention_ref as ar
    w = workloads.make_small(1, 1, 130, 8, True, seed=5)
    q, k, v, do = workloads.make_bf16_inputs(w)
    o1, l1 = ar.attention_fwd(q, k, v, 0.3, True)
    g1 = ar.attention_bwd(q, k, v, do, 0.3, True)
    monkeypatch.setattr(ar, "ROW_BLOCK", 17)
    o2, l2 = ar.attention_fwd(q, k, v, 0.3, True)
    g2 = ar.attention_bwd(q, k, v, do, 0.3, True)
    assert np.abs(o1 - o2).max() < 1e-14 and np.abs(l1 - l2).max() < 1e-14
    for a, b in zip(g1, g2):
        assert np.abs(a - b).max() < 1e-13


@pytest.mark.parametrize("check", oc.DEC_CHECKS, ids=lambda f: f.__name__)
def test_oracle_decode_pins(check):
    assert check(oracle.attention_decode)


@pytest.mark.parametrize("check", oc.GQA_BWD_CHECKS, ids=lambda f: f.__name__)
def test_oracle_gqa_backward_pins(check):
    assert check(oracle.attention_bwd_gqa)
