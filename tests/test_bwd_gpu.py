"""bf16 backward: CUDA path (through the C ABI) vs the fp64 oracle's chain rule."""
import numpy as np
import pytest
import torch

import oracle
import parity
import workloads

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def fa():
    import exact_attention_132_b200 as m
    return m


def run_fwd_bwd(fa, q, k, v, do, causal, scale):
    qc, kc, vc, dc = (t.cuda() for t in (q, k, v, do))
    o, lse = fa.attention_forward(qc, kc, vc, causal=causal, scale=scale)
    dq, dk, dv = fa.attention_backward(qc, kc, vc, o, dc, lse, causal=causal, scale=scale)
    torch.cuda.synchronize()
    return o, lse, (dq, dk, dv)


SMALL = [
    (1, 2, 128, 64, False), (1, 2, 256, 64, True), (2, 2, 500, 64, True), (1, 2, 640, 64, False),
    (2, 3, 1000, 64, True),
    (1, 2, 384, 128, True), (2, 1, 700, 128, False),
    (1, 2, 256, 256, True), (1, 1, 330, 256, False),
    (1, 1, 1, 64, True), (1, 1, 50, 128, True),
    (1, 2, 300, 96, True), (1, 1, 257, 96, False), (1, 1, 200, 192, True), (1, 1, 130, 192, False),
]


@pytest.mark.parametrize("B,H,N,d,causal", SMALL)
def test_bwd_small_matches_oracle(fa, B, H, N, d, causal):
    w = workloads.make_small(B, H, N, d, causal, seed=N * 3 + d + 1, backward=True)
    q, k, v, do = workloads.make_bf16_inputs(w)
    _, _, got = run_fwd_bwd(fa, q, k, v, do, causal, w.sm_scale)
    ref = oracle.attention_bwd(q, k, v, do, w.sm_scale, causal)
    errs = parity.assert_grads_ok(got, ref, tag=w.name)
    print(w.name, errs)
    assert fa.fa_get_device_status() == 0


def test_bwd_d64_workload_full():
    """B=1 H=8 N=8192 d=64 causal: every gradient element vs the oracle."""
    import exact_attention_132_b200 as fa
    w = workloads.WORKLOADS["fwdbwd_d64"]
    q, k, v, do = workloads.make_bf16_inputs(w)
    o, lse, got = run_fwd_bwd(fa, q, k, v, do, True, w.sm_scale)
    ref = oracle.attention_bwd(q, k, v, do, w.sm_scale, True)
    errs = parity.assert_grads_ok(got, ref, tag=w.name)
    print("fwdbwd_d64", errs)
    o_ref, lse_ref = oracle.attention_fwd(q, k, v, w.sm_scale, True)
    parity.assert_fwd_ok(o, lse, o_ref, lse_ref, tag=w.name)


def test_bwd_d256_workload_full_size_heads():
    """B=2 H=8 N=16384 d=256 non-causal, N(0, 0.5^2): run at full size; two whole heads
    (every row, every gradient element) are checked against the oracle."""
    import exact_attention_132_b200 as fa
    w = workloads.WORKLOADS["fwdbwd_d256"]
    q, k, v, do = workloads.make_bf16_inputs(w)
    o, lse, got = run_fwd_bwd(fa, q, k, v, do, False, w.sm_scale)
    heads = [(0, 0), (1, 5)]
    ref = oracle.attention_bwd(q, k, v, do, w.sm_scale, False, heads=heads)
    sel = [torch.stack([g[b, h].cpu() for b, h in heads]) for g in got]
    errs = parity.assert_grads_ok(sel, ref, tag=w.name)
    print("fwdbwd_d256 heads", heads, errs)
    o_ref, lse_ref = oracle.attention_fwd_heads(q, k, v, w.sm_scale, False, heads)
    og = torch.stack([o[b, h].cpu() for b, h in heads])
    lg = torch.stack([lse[b, h].cpu() for b, h in heads])
    parity.assert_fwd_ok(og, lg, o_ref, lse_ref, tag=w.name)
    for g in got:
        assert torch.isfinite(g.float()).all()


def test_bwd_invariants_at_full_size():
    """Properties that hold at any size: sum_j dK_j = 0 and sum_j dV_j = sum_i dO_i per head."""
    import exact_attention_132_b200 as fa
    w = workloads.WORKLOADS["fwdbwd_d64"]
    q, k, v, do = workloads.make_bf16_inputs(w)
    _, _, (dq, dk, dv) = run_fwd_bwd(fa, q, k, v, do, True, w.sm_scale)
    sdk = dk.double().sum(2)
    sdv = dv.double().sum(2)
    sdo = do.double().sum(2).cuda()
    scale_k = dk.double().abs().sum(2).max()
    assert (sdk.abs().max() / scale_k) < 2e-2
    assert ((sdv - sdo).abs().max() / sdo.abs().max()) < 2e-2


def test_bwd_is_deterministic(fa):
    w = workloads.make_small(1, 2, 512, 128, True, seed=11, backward=True)
    q, k, v, do = (t.cuda() for t in workloads.make_bf16_inputs(w))
    o, lse = fa.attention_forward(q, k, v, causal=True)
    g1 = fa.attention_backward(q, k, v, o, do, lse, causal=True)
    g2 = fa.attention_backward(q, k, v, o, do, lse, causal=True)
    assert all(torch.equal(a, b) for a, b in zip(g1, g2))


def test_bwd_d64_repeatability(fa):
    """At d = 64 dQ is summed over key tiles by fp32 reduce-adds in whatever order the
    CTAs reach them, so only its last bits may differ between runs; dK and dV, which
    each CTA owns, repeat exactly."""
    w = workloads.make_small(2, 3, 1000, 64, True, seed=12, backward=True)
    q, k, v, do = (t.cuda() for t in workloads.make_bf16_inputs(w))
    o, lse = fa.attention_forward(q, k, v, causal=True)
    dq1, dk1, dv1 = fa.attention_backward(q, k, v, o, do, lse, causal=True)
    dq2, dk2, dv2 = fa.attention_backward(q, k, v, o, do, lse, causal=True)
    assert torch.equal(dk1, dk2) and torch.equal(dv1, dv2)
    diff = (dq1.float() - dq2.float()).abs()
    # at most one bf16 rounding step of the value
    assert bool((diff <= dq1.float().abs() * 2.0 ** -7 + 1e-30).all())


def test_bwd_workspace_too_small_raises(fa):
    q = torch.zeros(1, 1, 128, 64, dtype=torch.bfloat16, device="cuda")
    lse = torch.zeros(1, 1, 128, dtype=torch.float32, device="cuda")
    ws = torch.empty(16, dtype=torch.uint8, device="cuda")
    with pytest.raises(fa.FAError) as ei:
        fa.attention_backward(q, q, q, q, q, lse, workspace=ws)
    assert ei.value.status == fa.FA_ERR_INVALID_ARG
