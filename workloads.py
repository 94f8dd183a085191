"""Seeded synthetic inputs for the attention workloads.

This module holds only input recipes: shapes, seeds, value distributions and
the FP8 input quantisation that the FP8 workload starts from.  It contains none
of the attention arithmetic.  Both the fp64 oracle (via tests and bench) and the
CUDA path receive their inputs from here, so the two sides see bit-identical
values.

Workloads (all tensors [B, H, N, d], d contiguous):

* ``fwd_small``   forward, B=1 H=8  N=1024  d=64,  causal, scale 1/8
* ``fwd_d128``    forward, B=4 H=16 N=4096  d=128, causal, scale 1/sqrt(128);
                  1% of K rows per head multiplied by 8 (forces running-max
                  changes in the online softmax)
* ``fwdbwd_d64``  forward+backward, B=1 H=8 N=8192 d=64, causal, scale 1/8
* ``fwdbwd_d256`` forward+backward, B=2 H=8 N=16384 d=256, non-causal,
                  values N(0, 0.5^2), scale 1/16
* ``fp8_d128``    FP8 e4m3 forward, B=1 H=32 N=32768 d=128, causal,
                  scale 1/sqrt(128); per-128-row-tile fp32 scales

Generation: ``torch.Generator('cpu').manual_seed(seed)``, ``randn`` in fp32,
then round-to-nearest-even to bf16 (or quantise to e4m3 for the FP8 case).
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import torch

FP8_TILE_ROWS = 128          # rows that share one FP8 scale
E4M3_MAX = 448.0             # largest finite float8_e4m3fn value


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    N: int
    d: int
    causal: bool
    backward: bool = False
    fp8: bool = False
    std: float = 1.0
    outlier_frac: float = 0.0   # fraction of K rows per head scaled by outlier_mul
    outlier_mul: float = 8.0
    seed: int = 1000
    scale: float = field(default=0.0)

    @property
    def sm_scale(self) -> float:
        return self.scale if self.scale > 0 else 1.0 / math.sqrt(self.d)

    def fwd_flops(self) -> float:
        """Algorithmic forward FLOPs: 4*B*H*N^2*d, halved when causal."""
        f = 4.0 * self.B * self.H * self.N * self.N * self.d
        return f / 2 if self.causal else f

    def bwd_flops(self) -> float:
        """Algorithmic backward FLOPs: 2.5x the forward count."""
        return 2.5 * self.fwd_flops()

    def with_shape(self, **kw) -> "Workload":
        d = dict(self.__dict__)
        d.update(kw)
        return Workload(**d)


WORKLOADS = {
    "fwd_small": Workload("fwd_small", 1, 8, 1024, 64, True, seed=1001, scale=1.0 / 8),
    "fwd_d128": Workload("fwd_d128", 4, 16, 4096, 128, True, seed=1002,
                         outlier_frac=0.01, outlier_mul=8.0),
    "fwdbwd_d64": Workload("fwdbwd_d64", 1, 8, 8192, 64, True, backward=True, seed=1003,
                           scale=1.0 / 8),
    "fwdbwd_d256": Workload("fwdbwd_d256", 2, 8, 16384, 256, False, backward=True, std=0.5,
                            seed=1004, scale=1.0 / 16),
    "fp8_d128": Workload("fp8_d128", 1, 32, 32768, 128, True, fp8=True, seed=1005),
}


def _randn(gen: torch.Generator, shape, std: float) -> torch.Tensor:
    x = torch.randn(shape, generator=gen, dtype=torch.float32)
    if std != 1.0:
        x = x * std
    return x


def make_bf16_inputs(w: Workload, with_grad_out: bool | None = None):
    """Return CPU bf16 tensors q, k, v (and dO when the workload has a backward).

    K outlier rows: for every (b, h), floor(outlier_frac * N) distinct row
    indices are drawn from the same generator and those rows of K are
    multiplied by ``outlier_mul`` after the bf16 rounding (x8 is exact in bf16).
    """
    gen = torch.Generator("cpu").manual_seed(w.seed)
    shape = (w.B, w.H, w.N, w.d)
    q = _randn(gen, shape, w.std).to(torch.bfloat16)
    k = _randn(gen, shape, w.std).to(torch.bfloat16)
    v = _randn(gen, shape, w.std).to(torch.bfloat16)
    n_out = int(math.floor(w.outlier_frac * w.N))
    if n_out > 0:
        for b in range(w.B):
            for h in range(w.H):
                rows = torch.randperm(w.N, generator=gen)[:n_out]
                k[b, h, rows] = (k[b, h, rows].float() * w.outlier_mul).to(torch.bfloat16)
    want_do = w.backward if with_grad_out is None else with_grad_out
    if want_do:
        do = _randn(gen, shape, w.std).to(torch.bfloat16)
        return q, k, v, do
    return q, k, v


def quantize_e4m3_per_tile(x: torch.Tensor, tile_rows: int = FP8_TILE_ROWS):
    """Per-(b, h, 128-row tile) e4m3 quantisation of an fp32 [B,H,N,d] tensor.

    scale_t = amax(|x_tile|) / 448 (1 when the tile is all zero);
    x_q = float8_e4m3fn(RNE(x / scale_t)), saturating at +-448.
    Returns (x_q as torch.float8_e4m3fn, scales fp32 [B, H, ceil(N/128)]).
    A ragged last tile uses its own rows only.
    """
    B, H, N, d = x.shape
    nt = (N + tile_rows - 1) // tile_rows
    pad = nt * tile_rows - N
    xp = torch.nn.functional.pad(x, (0, 0, 0, pad)) if pad else x
    xt = xp.reshape(B, H, nt, tile_rows, d)
    amax = xt.abs().amax(dim=(3, 4))
    scales = torch.where(amax > 0, amax / E4M3_MAX, torch.ones_like(amax)).to(torch.float32)
    y = xt / scales[..., None, None]
    y = y.clamp(-E4M3_MAX, E4M3_MAX)
    xq = y.to(torch.float8_e4m3fn).reshape(B, H, nt * tile_rows, d)[:, :, :N].contiguous()
    return xq, scales.contiguous()


def dequantize_e4m3_per_tile(xq: torch.Tensor, scales: torch.Tensor,
                             tile_rows: int = FP8_TILE_ROWS) -> torch.Tensor:
    """Exact dequantised values x_q * scale_t as float64 (what the oracle consumes)."""
    B, H, N, d = xq.shape
    idx = torch.arange(N) // tile_rows
    s = scales.to(torch.float64)[:, :, idx]            # [B,H,N]
    return xq.to(torch.float64) * s[..., None]


def make_fp8_inputs(w: Workload):
    """FP8 workload: fp32 N(0, std^2) q, k, v quantised per 128-row tile to e4m3.

    Returns dict with q8, k8, v8 (float8_e4m3fn), qs, ks, vs (fp32 scales) and
    the fp32 originals (for reporting the quantisation error only).
    """
    gen = torch.Generator("cpu").manual_seed(w.seed)
    shape = (w.B, w.H, w.N, w.d)
    out = {}
    for name in ("q", "k", "v"):
        x = _randn(gen, shape, w.std)
        xq, s = quantize_e4m3_per_tile(x)
        out[name + "8"] = xq
        out[name + "s"] = s
        out[name + "32"] = x
    return out


def make_small(B: int, H: int, N: int, d: int, causal: bool, seed: int = 7, std: float = 1.0,
               backward: bool = True, scale: float = 0.0) -> Workload:
    """An ad-hoc small workload for parity tests (several tiles plus a ragged tail)."""
    return Workload(f"small_b{B}h{H}n{N}d{d}{'c' if causal else ''}", B, H, N, d, causal,
                    backward=backward, std=std, seed=seed, scale=scale)


# ----------------------------------------------------------------------------- decoding
@dataclass(frozen=True)
class DecodeWorkload:
    """Few queries against a long key/value sequence with grouped heads."""
    name: str
    B: int
    Hq: int
    Hkv: int
    Nq: int
    Nk: int
    d: int
    causal: bool
    seed: int
    std: float = 1.0

    @property
    def sm_scale(self) -> float:
        return 1.0 / math.sqrt(self.d)

    def flops(self) -> float:
        """4 * B * Hq * Nq * Nk * d (every query sees almost every key; the end-aligned
        causal mask hides at most Nq - 1 keys)."""
        return 4.0 * self.B * self.Hq * self.Nq * self.Nk * self.d

    def bytes(self) -> int:
        """Algorithmic HBM bytes: Q, K, V read and O written in bf16, LSE in fp32."""
        return 2 * (self.B * self.Hq * self.Nq * self.d * 2 + self.B * self.Hkv * self.Nk * self.d * 2) \
            + 4 * self.B * self.Hq * self.Nq


DECODE_WORKLOADS = {
    # one new token per sequence, 32 query heads sharing 8 key/value heads, 32k cache
    "decode_d128": DecodeWorkload("decode_d128", 8, 32, 8, 1, 32768, 128, True, seed=1006),
}


def make_decode_inputs(B: int, Hq: int, Hkv: int, Nq: int, Nk: int, d: int, seed: int,
                       std: float = 1.0):
    """CPU bf16 q [B, Hq, Nq, d], k, v [B, Hkv, Nk, d], N(0, std^2), one seeded generator."""
    gen = torch.Generator("cpu").manual_seed(seed)
    q = _randn(gen, (B, Hq, Nq, d), std).to(torch.bfloat16)
    k = _randn(gen, (B, Hkv, Nk, d), std).to(torch.bfloat16)
    v = _randn(gen, (B, Hkv, Nk, d), std).to(torch.bfloat16)
    return q, k, v
