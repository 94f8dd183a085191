"""FP8 backward: gradients for the dequantised inputs of the FP8 forward (CUDA path through
the C ABI) vs the fp64 oracle's chain rule on the same dequantised values.

The CUDA path starts from the FP8 forward's O and LSE, so its D_i = dO . O carries the
forward's e4m3 rounding of P, while the oracle uses the exact O; the inputs it
recomputes from are the dequantised values rounded to bf16.  No tolerance is given for
an FP8 backward: the bf16 gradient bound applies (measured 0.3-1.0 %)."""
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
    # (B, H, N, d, causal)
    (1, 2, 256, 64, True), (1, 2, 300, 128, False), (1, 1, 515, 128, True),
    (2, 1, 200, 96, True), (1, 1, 257, 256, True), (1, 1, 130, 192, False),
]


@pytest.mark.parametrize("B,H,N,d,causal", CASES)
def test_fp8_bwd_matches_oracle(fa, B, H, N, d, causal):
    w = workloads.make_small(B, H, N, d, causal, seed=N + 5 * d + 3, backward=True)
    inp = workloads.make_fp8_inputs(w)
    do = workloads.make_bf16_inputs(w)[3]
    dev = {n: inp[n].cuda() for n in ("q8", "k8", "v8", "qs", "ks", "vs")}
    args = [dev[n] for n in ("q8", "k8", "v8", "qs", "ks", "vs")]
    o, lse = fa.attention_forward_fp8(*args, causal=causal, scale=w.sm_scale)
    dq, dk, dv = fa.attention_backward_fp8(*args, o, do.cuda(), lse, causal=causal, scale=w.sm_scale)
    torch.cuda.synchronize()
    qd, kd, vd = (workloads.dequantize_e4m3_per_tile(inp[n + "8"], inp[n + "s"]) for n in "qkv")
    rq, rk, rv = oracle.attention_bwd(qd, kd, vd, do, w.sm_scale, causal)
    errs = {n: parity.rel_fro(g, r) for n, g, r in (("dq", dq, rq), ("dk", dk, rk), ("dv", dv, rv))}
    print(w.name, errs)
    for n, e in errs.items():
        assert e <= parity.GRAD_REL_FRO, (n, errs)
    assert fa.fa_get_device_status() == 0


def test_fp8_bwd_workspace_too_small_is_rejected(fa):
    w = workloads.make_small(1, 1, 128, 64, True, seed=2, backward=True)
    inp = workloads.make_fp8_inputs(w)
    args = [inp[n].cuda() for n in ("q8", "k8", "v8", "qs", "ks", "vs")]
    o = torch.zeros((1, 1, 128, 64), dtype=torch.bfloat16, device="cuda")
    lse = torch.zeros((1, 1, 128), dtype=torch.float32, device="cuda")
    grads = [torch.empty_like(o) for _ in range(3)]
    need = fa.fa_bwd_fp8_workspace_size(1, 1, 128, 64)
    ws = torch.empty(need - 256, dtype=torch.uint8, device="cuda")
    with pytest.raises(fa.FAError):
        fa.fa_bwd_fp8(*args, o, o, lse, *grads, ws, causal=True)
