"""Accuracy of the software exp2 the kernels run on the FMA pipe for part of the
exponentials (FA4's partial software exponential, "FlashAttentionとは？…"
(issoh.co.jp), section FA4のB200で1613TFLOPs…).

The library evaluates it, the special-function-unit ex2 and CUDA's exp2f on the same
fp32 inputs (fa_debug_exp2); the values are compared here with float64 2^x.  Bounds:
relative error <= 7.5e-5 (the degree-3 minimax fit's) on (-125.99, 127]; <= 1.5e-4 on
[-126, -125.99], where 2^n = 2^-126 meets a polynomial value just below one and the
exponent-field add yields a subnormal encoding that loses the implicit leading bit
(measured 9.1e-5 at x = -125.99992 before the bound was stated this way); at and below
the clamp at -126 the result stands in for anything smaller and lies in [0, 2^-126].
"""
import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

POLY_REL = 7.5e-5
EDGE_REL = 1.5e-4


@pytest.fixture(scope="module")
def fa():
    import exact_attention_132_b200 as m
    return m


def _inputs():
    rng = np.random.default_rng(11)
    dense = np.linspace(-126.0, 127.0, 2_000_001)
    near_int = (np.arange(-126, 128)[:, None] + np.array([-0.5, -0.49999, -1e-6, 0.0, 1e-6,
                                                          0.49999, 0.5])[None, :]).ravel()
    rand = rng.uniform(-126.0, 127.0, size=1_000_000)
    small = rng.uniform(-1.0, 1.0, size=100_000)     # the softmax's common range
    x = np.concatenate([dense, near_int, rand, small]).astype(np.float32)
    return x[(x > -126.0) & (x <= 127.0)]


def test_software_exp2_relative_error_bound(fa):
    x = _inputs()
    y_poly, y_sfu, y_lib = (t.cpu().numpy().astype(np.float64)
                            for t in fa.fa_debug_exp2(torch.from_numpy(x).cuda()))
    exact = np.exp2(x.astype(np.float64))
    rel = np.abs(y_poly / exact - 1.0)
    edge = x <= -125.99
    print("software exp2: max rel err", rel[~edge].max(), "at x =", x[~edge][rel[~edge].argmax()],
          "; bottom edge", rel[edge].max())
    assert rel[~edge].max() <= POLY_REL
    assert rel[edge].max() <= EDGE_REL
    # the same bounds against CUDA's exp2f (itself within 2 ulp of the exact value)
    rel_lib = np.abs(y_poly / y_lib - 1.0)
    assert rel_lib[~edge].max() <= POLY_REL + 3e-7
    assert rel_lib[edge].max() <= EDGE_REL + 3e-7
    # the special-function unit is the form the software one replaces; sanity only
    assert np.abs(y_sfu / exact - 1.0).max() <= 1e-5


def test_software_exp2_at_and_below_the_clamp(fa):
    x = np.concatenate([[-126.0, -126.25, -126.5, -127.0, -130.0, -149.0, -200.0, -1e4,
                         -3.0e38], np.linspace(-300.0, -126.0, 10001)]).astype(np.float32)
    y_poly, _, _ = (t.cpu().numpy().astype(np.float64)
                    for t in fa.fa_debug_exp2(torch.from_numpy(x).cuda()))
    assert np.all(np.isfinite(y_poly))
    assert np.all(y_poly >= 0.0)
    assert np.all(y_poly <= 2.0 ** -126)
    # just above the clamp the bound holds again
    x2 = np.float32([-125.99, -125.75, -125.5, -125.25])
    y2, _, _ = (t.cpu().numpy().astype(np.float64) for t in fa.fa_debug_exp2(torch.from_numpy(x2).cuda()))
    assert np.abs(y2 / np.exp2(x2.astype(np.float64)) - 1.0).max() <= POLY_REL
    x3 = np.float32([-125.99992, -125.9999, -125.995])
    y3, _, _ = (t.cpu().numpy().astype(np.float64) for t in fa.fa_debug_exp2(torch.from_numpy(x3).cuda()))
    assert np.abs(y3 / np.exp2(x3.astype(np.float64)) - 1.0).max() <= EDGE_REL


def test_software_exp2_odd_count_and_empty(fa):
    x = torch.tensor([0.0, 1.0, -1.0, 3.5, -7.25], device="cuda")
    y_poly, _, _ = fa.fa_debug_exp2(x)
    want = np.exp2(np.float64([0.0, 1.0, -1.0, 3.5, -7.25]))
    assert np.abs(y_poly.cpu().numpy() / want - 1.0).max() <= POLY_REL
    e = fa.fa_debug_exp2(torch.empty(0, device="cuda"))
    assert all(t.numel() == 0 for t in e)
