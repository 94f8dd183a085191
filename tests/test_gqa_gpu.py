"""Grouped query heads (GQA / MQA) at full sequence length: forward and backward through
the C ABI vs the fp64 oracle (query head h reads key/value head h // g)."""
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


def _inputs(B, Hq, Hkv, N, d, seed, with_do):
    q, k, v = workloads.make_decode_inputs(B, Hq, Hkv, N, N, d, seed=seed)
    if not with_do:
        return q, k, v
    do = workloads.make_decode_inputs(B, Hq, Hkv, N, N, d, seed=seed + 1)[0]
    return q, k, v, do


FWD = [
    # (B, Hq, Hkv, N, d, causal)
    (1, 8, 2, 777, 128, True), (2, 4, 1, 513, 64, False), (1, 6, 3, 300, 256, True),
    (1, 4, 2, 1000, 64, True), (2, 8, 4, 256, 128, False),
]


@pytest.mark.parametrize("B,Hq,Hkv,N,d,causal", FWD)
def test_gqa_forward_matches_oracle(fa, B, Hq, Hkv, N, d, causal):
    q, k, v = _inputs(B, Hq, Hkv, N, d, seed=N + Hq * 10 + d, with_do=False)
    scale = 1.0 / np.sqrt(d)
    o, lse = fa.attention_forward_gqa(q.cuda(), k.cuda(), v.cuda(), causal=causal, scale=scale)
    torch.cuda.synchronize()
    # Nq == Nk: the decoding oracle's end-aligned mask is the lower triangle
    o_ref, lse_ref = oracle.attention_decode(q, k, v, scale, causal)
    parity.assert_fwd_ok(o, lse, o_ref, lse_ref, tag=f"gqa fwd {B},{Hq},{Hkv},{N},{d},{causal}")
    assert fa.fa_get_device_status() == 0


BWD = [
    (1, 4, 2, 300, 64, True), (1, 8, 1, 257, 128, False), (1, 4, 2, 200, 256, True),
    (2, 6, 3, 400, 128, True), (2, 4, 1, 513, 64, False),
]


@pytest.mark.parametrize("B,Hq,Hkv,N,d,causal", BWD)
def test_gqa_backward_matches_oracle(fa, B, Hq, Hkv, N, d, causal):
    q, k, v, do = _inputs(B, Hq, Hkv, N, d, seed=N + Hq + d, with_do=True)
    scale = 1.0 / np.sqrt(d)
    qc, kc, vc, doc = q.cuda(), k.cuda(), v.cuda(), do.cuda()
    o, lse = fa.attention_forward_gqa(qc, kc, vc, causal=causal, scale=scale)
    dq, dk, dv = fa.attention_backward_gqa(qc, kc, vc, o, doc, lse, causal=causal, scale=scale)
    torch.cuda.synchronize()
    rq, rk, rv = oracle.attention_bwd_gqa(q, k, v, do, scale, causal)
    for name, got, ref in (("dq", dq, rq), ("dk", dk, rk), ("dv", dv, rv)):
        err = parity.rel_fro(got, ref)
        assert err <= parity.GRAD_REL_FRO, (name, err)
    assert fa.fa_get_device_status() == 0


def test_gqa_one_group_equals_plain_entry_points(fa):
    """Hkv == Hq through the grouped entry points is the ordinary forward and backward."""
    q, k, v, do = (t.cuda() for t in _inputs(1, 2, 2, 333, 128, seed=3, with_do=True))
    o1, l1 = fa.attention_forward_gqa(q, k, v, causal=True)
    o2, l2 = fa.attention_forward(q, k, v, causal=True)
    g1 = fa.attention_backward_gqa(q, k, v, o1, do, l1, causal=True)
    g2 = fa.attention_backward(q, k, v, o2, do, l2, causal=True)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
    for a, b in zip(g1, g2):
        assert torch.equal(a, b)
