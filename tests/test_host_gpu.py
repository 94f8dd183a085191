"""Host-buffer forward (fa_fwd_host): chunked copies overlapping the kernels must give
exactly fa_fwd's results, and match the fp64 oracle."""
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
    # (B, H, N, d, causal): one chunk, several chunks with a short last one, more heads
    # than chunks
    (1, 1, 300, 64, True), (2, 5, 257, 128, False), (1, 16, 640, 128, True),
    (3, 3, 130, 256, True), (1, 9, 200, 96, False),
]


@pytest.mark.parametrize("B,H,N,d,causal", CASES)
def test_host_forward_equals_device_forward(fa, B, H, N, d, causal):
    w = workloads.make_small(B, H, N, d, causal, seed=N + H + d, backward=False)
    q, k, v = workloads.make_bf16_inputs(w, with_grad_out=False)
    o_h, lse_h = fa.attention_forward_host(q.pin_memory(), k.pin_memory(), v.pin_memory(),
                                           causal=causal, scale=w.sm_scale)
    o_d, lse_d = fa.attention_forward(q.cuda(), k.cuda(), v.cuda(), causal=causal, scale=w.sm_scale)
    torch.cuda.synchronize()
    assert torch.equal(o_h, o_d.cpu()) and torch.equal(lse_h, lse_d.cpu())
    if B * H * N <= 4000:
        o_ref, lse_ref = oracle.attention_fwd(q, k, v, w.sm_scale, causal)
        parity.assert_fwd_ok(o_h, lse_h, o_ref, lse_ref, tag=w.name)
    assert fa.fa_get_device_status() == 0


def test_host_forward_pageable_inputs_and_no_lse(fa):
    w = workloads.make_small(1, 4, 200, 64, True, seed=4, backward=False)
    q, k, v = workloads.make_bf16_inputs(w, with_grad_out=False)
    o = torch.empty_like(q)   # pageable host memory
    ws = torch.empty(fa.fa_fwd_host_workspace_size(1, 4, 200, 64), dtype=torch.uint8, device="cuda")
    stream = torch.cuda.current_stream()
    fa.fa_fwd_host(q, k, v, o, None, ws, scale=w.sm_scale, causal=True, stream=stream)
    stream.synchronize()
    o_d, _ = fa.attention_forward(q.cuda(), k.cuda(), v.cuda(), causal=True, scale=w.sm_scale)
    assert torch.equal(o, o_d.cpu())
