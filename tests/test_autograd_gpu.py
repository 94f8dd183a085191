"""Autograd wrapper: gradients through torch.autograd against the fp64 oracle."""
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


@pytest.mark.parametrize("B,Hq,Hkv,N,d,causal", [(1, 4, 4, 300, 64, True), (2, 4, 2, 257, 128, False),
                                                 (1, 2, 1, 200, 256, True)])
def test_autograd_matches_oracle(fa, B, Hq, Hkv, N, d, causal):
    q, k, v = workloads.make_decode_inputs(B, Hq, Hkv, N, N, d, seed=N + d)
    do = workloads.make_decode_inputs(B, Hq, Hkv, N, N, d, seed=N + d + 1)[0]
    scale = 1.0 / np.sqrt(d)
    qc, kc, vc = (t.cuda().requires_grad_(True) for t in (q, k, v))
    o = fa.attention(qc, kc, vc, causal=causal, scale=scale)
    (o.float() * do.cuda().float()).sum().backward()
    torch.cuda.synchronize()
    o_ref, _ = oracle.attention_decode(q, k, v, scale, causal)
    assert parity.o_ok(parity.fwd_errors(o.detach(), np.zeros(1), o_ref, np.zeros(1)), parity.O_MAX_ABS)
    rq, rk, rv = oracle.attention_bwd_gqa(q, k, v, do, scale, causal)
    for name, got, ref in (("dq", qc.grad, rq), ("dk", kc.grad, rk), ("dv", vc.grad, rv)):
        assert parity.rel_fro(got, ref) <= parity.GRAD_REL_FRO, name
