"""FP8 e4m3 forward: CUDA path vs the fp64 oracle on the dequantised inputs."""
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


def run_fp8(fa, inp, causal, scale):
    dev = {n: inp[n].cuda() for n in ("q8", "k8", "v8", "qs", "ks", "vs")}
    o, lse = fa.attention_forward_fp8(dev["q8"], dev["k8"], dev["v8"], dev["qs"], dev["ks"],
                                      dev["vs"], causal=causal, scale=scale)
    torch.cuda.synchronize()
    return o, lse


def dequant(inp):
    return [workloads.dequantize_e4m3_per_tile(inp[n + "8"], inp[n + "s"]) for n in "qkv"]


@pytest.mark.parametrize("B,H,N,d,causal", [
    (1, 2, 256, 128, True), (2, 2, 640, 128, False), (1, 3, 1000, 128, True),
    (1, 1, 130, 128, False),
    # narrower and wider heads: 64 and 96 on the 128 kernel, 192 and 256 on the 256 kernel
    (1, 2, 515, 64, True), (1, 1, 300, 96, False), (1, 2, 700, 256, True),
    (2, 1, 257, 192, False),
])
def test_fp8_small_matches_oracle(fa, B, H, N, d, causal):
    w = workloads.make_small(B, H, N, d, causal, seed=N + 17 + d, backward=False)
    inp = workloads.make_fp8_inputs(w)
    o, lse = run_fp8(fa, inp, causal, w.sm_scale)
    qd, kd, vd = dequant(inp)
    o_ref, lse_ref = oracle.attention_fwd(qd, kd, vd, w.sm_scale, causal)
    err = parity.fwd_errors(o, lse, o_ref, lse_ref)
    print(w.name, err)
    assert parity.o_ok(err, parity.FP8_O_MAX_ABS), err
    assert np.isfinite(parity.to64(lse)).all()


def test_fp8_workload_full_size_eight_whole_heads(fa):
    """B=1 H=32 N=32768 d=128 causal, per-128-row-tile scales, run at full size: eight whole
    heads (every row, so every query tile and every work item of those heads) checked
    against the oracle on the dequantised inputs, plus finiteness of the whole output."""
    w = workloads.WORKLOADS["fp8_d128"]
    inp = workloads.make_fp8_inputs(w)
    o, lse = run_fp8(fa, inp, True, w.sm_scale)
    og, lg = o.cpu(), lse.cpu()
    assert torch.isfinite(og.float()).all() and torch.isfinite(lg).all()
    # first, last and six seeded heads in between
    rng = np.random.default_rng(8)
    heads = sorted({0, w.H - 1} | set(rng.choice(np.arange(1, w.H - 1), size=6, replace=False).tolist()))
    assert len(heads) == 8
    worst = 0.0
    for h in heads:
        qd, kd, vd = (workloads.dequantize_e4m3_per_tile(inp[n + "8"][:, h:h + 1], inp[n + "s"][:, h:h + 1])
                      for n in "qkv")
        o_ref, lse_ref = oracle.attention_fwd(qd, kd, vd, w.sm_scale, True)
        err = parity.fwd_errors(og[:, h:h + 1], lg[:, h:h + 1], o_ref, lse_ref)
        print("fp8_d128 head", h, err)
        assert parity.o_ok(err, parity.FP8_O_MAX_ABS), (h, err)
        worst = max(worst, err["o_max_abs"])
    print("fp8_d128 eight whole heads, O max abs", worst)
