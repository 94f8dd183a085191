"""Large shapes: a long sequence (forward and backward), many heads, and a large FP8
problem, checked on sampled rows / heads against the oracle (each row still sees its full
key set) — the sizes where the work-item counts, tile counts and 64-bit offsets are
largest."""
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


def _sampled(o, lse, q, k, v, w, picks):
    o_ref, lse_ref = oracle.attention_fwd_rows(q, k, v, w.sm_scale, w.causal, picks)
    og, lg = o.cpu(), lse.cpu()
    got_o = np.stack([parity.to64(og[b, h, i]) for b, h, i in picks])
    got_l = np.array([float(lg[b, h, i]) for b, h, i in picks])
    return got_o, got_l, o_ref, lse_ref


@pytest.mark.parametrize("d", [64, 128])
def test_long_sequence_forward(fa, d):
    """N = 131072, causal: 1024 query tiles and 1024 key tiles per head."""
    w = workloads.make_small(1, 2, 131072, d, True, seed=11 + d, backward=False)
    q, k, v = workloads.make_bf16_inputs(w, with_grad_out=False)
    o, lse = fa.attention_forward(q.cuda(), k.cuda(), v.cuda(), causal=True, scale=w.sm_scale)
    torch.cuda.synchronize()
    picks = parity.sample_rows(1, 2, w.N, n_heads=2, n_rows=12, seed=d,
                               extra_rows=(65535, 65536, 131071 - 64))
    parity.assert_fwd_ok(*_sampled(o, lse, q, k, v, w, picks), tag=w.name)
    assert fa.fa_get_device_status() == 0


def test_long_sequence_backward_dq_rows(fa):
    """N = 65536, d = 64, causal backward: sampled dQ rows (row i of dQ needs only row i
    of P and dP), and dK, dV finite."""
    w = workloads.make_small(1, 1, 65536, 64, True, seed=5, backward=True)
    q, k, v, do = workloads.make_bf16_inputs(w)
    qc, kc, vc, dc = q.cuda(), k.cuda(), v.cuda(), do.cuda()
    o, lse = fa.attention_forward(qc, kc, vc, causal=True, scale=w.sm_scale)
    dq, dk, dv = fa.attention_backward(qc, kc, vc, o, dc, lse, causal=True, scale=w.sm_scale)
    torch.cuda.synchronize()
    picks = parity.sample_rows(1, 1, w.N, n_heads=1, n_rows=10, seed=3)
    ref = oracle.attention_bwd_rows_dq(q, k, v, do, w.sm_scale, True, picks)
    dqc = dq.cpu()
    got = np.stack([parity.to64(dqc[b, h, i]) for b, h, i in picks])
    err = np.linalg.norm(got - ref) / np.linalg.norm(ref)
    assert err <= parity.GRAD_REL_FRO, err
    assert torch.isfinite(dk.float()).all() and torch.isfinite(dv.float()).all()
    assert fa.fa_get_device_status() == 0


def test_many_heads(fa):
    """B = 32, H = 64 (2048 heads, 2048 work items of two query tiles): every head goes
    through the scheduler; a spread of heads is checked in full."""
    w = workloads.make_small(32, 64, 200, 64, True, seed=21, backward=False)
    q, k, v = workloads.make_bf16_inputs(w, with_grad_out=False)
    o, lse = fa.attention_forward(q.cuda(), k.cuda(), v.cuda(), causal=True, scale=w.sm_scale)
    torch.cuda.synchronize()
    heads = [(0, 0), (5, 17), (16, 32), (31, 63), (20, 1)]
    o_ref, lse_ref = oracle.attention_fwd_heads(q, k, v, w.sm_scale, True, heads)
    og, lg = o.cpu(), lse.cpu()
    got_o = np.stack([parity.to64(og[b, h]) for b, h in heads])
    got_l = np.stack([parity.to64(lg[b, h]) for b, h in heads])
    parity.assert_fwd_ok(got_o, got_l, o_ref, lse_ref, tag="many heads")


def test_fp8_long_sequence(fa):
    """FP8 forward at N = 131072, d = 128, causal, on sampled rows."""
    w = workloads.make_small(1, 1, 131072, 128, True, seed=8, backward=False)
    inp = workloads.make_fp8_inputs(w)
    args = [inp[n].cuda() for n in ("q8", "k8", "v8", "qs", "ks", "vs")]
    o, lse = fa.attention_forward_fp8(*args, causal=True, scale=w.sm_scale)
    torch.cuda.synchronize()
    qd, kd, vd = (workloads.dequantize_e4m3_per_tile(inp[n + "8"], inp[n + "s"]) for n in "qkv")
    picks = parity.sample_rows(1, 1, w.N, n_heads=1, n_rows=12, seed=4)
    err = parity.fwd_errors(*_sampled(o, lse, qd, kd, vd, w, picks))
    assert parity.o_ok(err, parity.FP8_O_MAX_ABS), err
    assert fa.fa_get_device_status() == 0
