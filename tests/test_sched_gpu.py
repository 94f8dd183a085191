"""Dynamic work distribution of the forward kernels: per-stream item counters that every
launch leaves at zero.  Back-to-back launches on one stream and overlapping launches on
several streams must each compute every item exactly once (results equal a lone launch)."""
import pytest
import torch

import workloads

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def fa():
    import exact_attention_132_b200 as m
    return m


def _inputs(B, H, N, d, causal, seed):
    w = workloads.make_small(B, H, N, d, causal, seed=seed, backward=False)
    return w, [t.cuda() for t in workloads.make_bf16_inputs(w, with_grad_out=False)]


@pytest.mark.parametrize("d", [64, 128, 256])
def test_back_to_back_launches_on_one_stream(fa, d):
    w, (q, k, v) = _inputs(2, 4, 1000, d, True, seed=d)
    ref_o, ref_l = fa.attention_forward(q, k, v, causal=True, scale=w.sm_scale)
    o, lse = torch.empty_like(ref_o), torch.empty_like(ref_l)
    for _ in range(20):
        o.zero_()
        fa.fa_fwd(q, k, v, o, lse, scale=w.sm_scale, causal=True)
    torch.cuda.synchronize()
    assert torch.equal(o, ref_o) and torch.equal(lse, ref_l)
    assert fa.fa_get_device_status() == 0


def test_overlapping_launches_on_several_streams(fa):
    # causal d=128 (two-tile kernel) and d=256 (one-tile kernel) problems, each on its
    # own stream, launched repeatedly so that their kernels overlap on the GPU
    probs = [_inputs(4, 8, 2048, 128, True, seed=1), _inputs(1, 8, 2048, 256, True, seed=2),
             _inputs(2, 8, 1536, 64, False, seed=3)]
    refs = [fa.attention_forward(q, k, v, causal=w.causal, scale=w.sm_scale)
            for w, (q, k, v) in probs]
    torch.cuda.synchronize()
    streams = [torch.cuda.Stream() for _ in probs]
    outs = [(torch.empty_like(r[0]), torch.empty_like(r[1])) for r in refs]
    for _ in range(10):
        for (w, (q, k, v)), (o, lse), s in zip(probs, outs, streams):
            with torch.cuda.stream(s):
                o.zero_()
                fa.fa_fwd(q, k, v, o, lse, scale=w.sm_scale, causal=w.causal, stream=s)
    torch.cuda.synchronize()
    for (o, lse), (ro, rl) in zip(outs, refs):
        assert torch.equal(o, ro) and torch.equal(lse, rl)
    assert fa.fa_get_device_status() == 0


def test_forward_and_decode_replay_from_a_cuda_graph(fa):
    """Captured once and replayed: each replay must draw its work items afresh (the
    counter is back at zero after every launch) and the decode merge must still wait for
    its split kernel."""
    w, (q, k, v) = _inputs(2, 8, 1500, 128, True, seed=31)
    o_ref, l_ref = fa.attention_forward(q, k, v, causal=True, scale=w.sm_scale)
    kd, vd = k[:, :2].contiguous(), v[:, :2].contiguous()
    qd = q[:, :, -2:].contiguous()
    od_ref, ld_ref = fa.attention_decode(qd, kd, vd, causal=True, scale=w.sm_scale)
    torch.cuda.synchronize()
    o, lse = torch.empty_like(o_ref), torch.empty_like(l_ref)
    od, ld = torch.empty_like(od_ref), torch.empty_like(ld_ref)
    ws = torch.empty(fa.fa_decode_workspace_size(2, 8, 2, 2, 1500, 128), dtype=torch.uint8,
                     device="cuda")
    s = torch.cuda.Stream()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        # warm-up outside the capture (first-use setup such as kernel attributes)
        fa.fa_fwd(q, k, v, o, lse, scale=w.sm_scale, causal=True, stream=s)
        fa.fa_decode(qd, kd, vd, od, ld, ws, scale=w.sm_scale, causal=True, stream=s)
    s.synchronize()
    with torch.cuda.graph(g, stream=s):
        fa.fa_fwd(q, k, v, o, lse, scale=w.sm_scale, causal=True, stream=s)
        fa.fa_decode(qd, kd, vd, od, ld, ws, scale=w.sm_scale, causal=True, stream=s)
    for _ in range(5):
        o.zero_()
        od.zero_()
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(o, o_ref) and torch.equal(lse, l_ref)
        assert torch.equal(od, od_ref) and torch.equal(ld, ld_ref)
    assert fa.fa_get_device_status() == 0


@pytest.mark.parametrize("d", [64, 128])
def test_backward_replays_from_a_cuda_graph(fa, d):
    """The backward's chained launches (programmatic dependents; at d = 64 the zeroing
    row-dot pass, the dK/dV pass with its dQ reduce-adds and the convert pass) captured
    once and replayed: every replay starts from zeroed dQ sums and matches eager runs."""
    w, (q, k, v) = _inputs(1, 4, 700, d, True, seed=40 + d)
    do = torch.randn_like(q.float()).to(torch.bfloat16)
    o, lse = fa.attention_forward(q, k, v, causal=True, scale=w.sm_scale)
    ref = fa.attention_backward(q, k, v, o, do, lse, causal=True, scale=w.sm_scale)
    torch.cuda.synchronize()
    dq, dk, dv = (torch.empty_like(q) for _ in range(3))
    ws = torch.empty(fa.fa_bwd_workspace_size(1, 4, 700, d), dtype=torch.uint8, device="cuda")
    s = torch.cuda.Stream()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        fa.fa_bwd(q, k, v, o, do, lse, dq, dk, dv, ws, scale=w.sm_scale, causal=True, stream=s)
    s.synchronize()
    with torch.cuda.graph(g, stream=s):
        fa.fa_bwd(q, k, v, o, do, lse, dq, dk, dv, ws, scale=w.sm_scale, causal=True, stream=s)
    for _ in range(4):
        dq.zero_()
        dk.zero_()
        dv.zero_()
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(dk, ref[1]) and torch.equal(dv, ref[2])
        if d == 64:   # dQ sums in varying order: equal to within its last bits
            diff = (dq.float() - ref[0].float()).abs()
            assert bool((diff <= ref[0].float().abs() * 2.0 ** -7 + 1e-30).all())
        else:
            assert torch.equal(dq, ref[0])
    assert fa.fa_get_device_status() == 0
