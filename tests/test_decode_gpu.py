"""Decoding (few queries, long K/V, grouped heads): CUDA path through the C ABI vs the
fp64 oracle on the same seeded inputs, with the bf16 forward tolerances."""
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


CASES = [
    # (B, Hq, Hkv, Nq, Nk, d, causal)
    (2, 4, 4, 1, 1000, 128, True),        # plain decoding, one key/value head per query head
    (1, 8, 2, 1, 4097, 128, True),        # GQA g=4, ragged key tail, several splits
    (2, 8, 1, 2, 777, 64, True),          # MQA, two queries
    (1, 16, 2, 16, 2000, 128, True),      # 128 query rows per key/value head
    (1, 4, 2, 3, 130, 256, False),        # d=256, two key tiles, non-causal
    (1, 2, 2, 5, 5, 64, True),            # Nq == Nk: the ordinary causal forward
    (1, 6, 3, 1, 1, 128, False),          # one key
    (3, 4, 2, 7, 300, 64, False),
    (1, 8, 2, 2, 1500, 96, True),         # stored head dims on the 128 / 256 kernels
    (1, 4, 4, 1, 700, 192, True),
]


@pytest.mark.parametrize("B,Hq,Hkv,Nq,Nk,d,causal", CASES)
def test_decode_matches_oracle(fa, B, Hq, Hkv, Nq, Nk, d, causal):
    q, k, v = workloads.make_decode_inputs(B, Hq, Hkv, Nq, Nk, d, seed=Nk * 3 + Nq + d)
    scale = 1.0 / np.sqrt(d)
    o, lse = fa.attention_decode(q.cuda(), k.cuda(), v.cuda(), causal=causal, scale=scale)
    torch.cuda.synchronize()
    o_ref, lse_ref = oracle.attention_decode(q, k, v, scale, causal)
    parity.assert_fwd_ok(o, lse, o_ref, lse_ref, tag=f"dec {B},{Hq},{Hkv},{Nq},{Nk},{d},{causal}")
    assert fa.fa_get_device_status() == 0


def test_decode_square_equals_forward(fa):
    """Nq == Nk with Hq == Hkv is the forward: both paths agree within rounding."""
    q, k, v = workloads.make_decode_inputs(1, 2, 2, 100, 100, 128, seed=5)
    qc, kc, vc = q.cuda(), k.cuda(), v.cuda()
    o1, l1 = fa.attention_decode(qc, kc, vc, causal=True)
    o2, l2 = fa.attention_forward(qc, kc, vc, causal=True)
    torch.cuda.synchronize()
    assert (o1.float() - o2.float()).abs().max().item() <= 1e-2
    assert (l1 - l2).abs().max().item() <= 1e-3


def test_decode_bench_workload_full(fa):
    """The benchmark's decoding workload (B=8, Hq=32, Hkv=8, Nq=1, Nk=32768, d=128)
    against the oracle on every row."""
    w = workloads.DECODE_WORKLOADS["decode_d128"]
    q, k, v = workloads.make_decode_inputs(w.B, w.Hq, w.Hkv, w.Nq, w.Nk, w.d, seed=w.seed)
    o, lse = fa.attention_decode(q.cuda(), k.cuda(), v.cuda(), causal=w.causal, scale=w.sm_scale)
    torch.cuda.synchronize()
    o_ref, lse_ref = oracle.attention_decode(q, k, v, w.sm_scale, w.causal)
    parity.assert_fwd_ok(o, lse, o_ref, lse_ref, tag=w.name)


def test_decode_workspace_too_small_is_rejected(fa):
    q, k, v = (t.cuda() for t in workloads.make_decode_inputs(1, 4, 2, 1, 512, 64, seed=9))
    o = torch.empty_like(q)
    need = fa.fa_decode_workspace_size(1, 4, 2, 1, 512, 64)
    ws = torch.empty(max(need - 256, 16), dtype=torch.uint8, device="cuda")
    with pytest.raises(fa.FAError):
        fa.fa_decode(q, k, v, o, None, ws)
