"""Host-side checks of the seeded input recipes (no attention arithmetic here)."""
import math

import torch

import workloads


def test_seeded_inputs_are_reproducible():
    w = workloads.make_small(1, 2, 130, 16, True, seed=3)
    a = workloads.make_bf16_inputs(w)
    b = workloads.make_bf16_inputs(w)
    assert all(torch.equal(x, y) for x, y in zip(a, b))
    assert a[0].dtype == torch.bfloat16 and a[0].shape == (1, 2, 130, 16)


def test_outlier_rows_are_exact_multiples():
    w = workloads.WORKLOADS["fwd_d128"].with_shape(B=1, H=2, N=512)
    q, k, v = workloads.make_bf16_inputs(w)
    w0 = w.with_shape(outlier_frac=0.0)
    _, k0, _ = workloads.make_bf16_inputs(w0)
    ratio = (k.float() / k0.float().where(k0.float() != 0, torch.ones(()))).abs()
    changed = (k != k0).any(-1)
    assert int(changed[0, 0].sum()) <= 5 and int(changed.sum()) >= 2
    assert torch.allclose(ratio[changed], torch.full_like(ratio[changed], 8.0))


def test_fp8_quantisation_recipe():
    x = torch.randn(1, 2, 300, 16, generator=torch.Generator().manual_seed(1))
    xq, s = workloads.quantize_e4m3_per_tile(x)
    assert xq.dtype == torch.float8_e4m3fn and s.shape == (1, 2, 3)
    deq = workloads.dequantize_e4m3_per_tile(xq, s)
    for t in range(3):
        tile = x[:, :, t * 128:(t + 1) * 128]
        assert torch.allclose(s[:, :, t], tile.abs().amax(dim=(2, 3)) / 448.0)
        # the tile's largest magnitude maps to +-448 exactly
        assert float(xq[:, :, t * 128:(t + 1) * 128].float().abs().amax()) == 448.0
    rel = ((deq - x.double()).abs() / x.double().abs().clamp_min(1e-3)).max()
    assert rel < 2 ** -3   # e4m3 keeps 3 mantissa bits; subnormals only near zero
    z = torch.zeros(1, 1, 128, 8)
    zq, zs = workloads.quantize_e4m3_per_tile(z)
    assert float(zs) == 1.0 and float(zq.float().abs().sum()) == 0.0


def test_flop_counts():
    w = workloads.WORKLOADS["fwd_d128"]
    assert w.fwd_flops() == 4 * 4 * 16 * 4096 ** 2 * 128 / 2
    assert workloads.WORKLOADS["fwdbwd_d256"].bwd_flops() == 2.5 * 4 * 2 * 8 * 16384 ** 2 * 256
    assert math.isclose(workloads.WORKLOADS["fwd_d128"].sm_scale, 1 / math.sqrt(128))
