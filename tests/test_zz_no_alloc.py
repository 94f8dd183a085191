"""fa_bwd_noalloc: the backward entry point for callers that cannot allocate.

Some callers cannot give the library a workspace: a plugin whose host program
owns all device memory through its own pool, or a latency-critical path that
cannot afford cudaMalloc's implicit device-wide synchronisation.  For them the
library keeps the backward's per-row scratch in a fixed array of its own.  This
test calls that entry point through the C ABI and checks that it gives the same
gradients as fa_bwd with a caller workspace, and as the fp64 oracle, on two
calls in a row per shape and across shapes (so a stale scratch from an earlier
call would show).  It lives in its own file, collected last, and depends on no state
left by other tests.
"""
import pytest
import torch

import oracle
import parity
import workloads

pytestmark = pytest.mark.gpu

# Every kernel pair the entry point can launch: d = 64 (its own two-pass dK/dV + dQ
# kernels, causal and not), the d = 128 and d = 256 kernels, and a ragged tail.  The
# first shape also runs in the workspace backward's oracle-checked suite.
SHAPES = [(1, 2, 384, 128, True), (2, 2, 500, 64, False), (1, 2, 640, 64, True),
          (1, 2, 320, 256, False), (1, 1, 200, 256, True)]


def test_noalloc_backward_matches_workspace_backward_and_oracle_two_calls():
    import exact_attention_132_b200 as fa
    for B, H, N, d, causal in SHAPES:
        w = workloads.make_small(B, H, N, d, causal, seed=31 + N, backward=True)
        q_c, k_c, v_c, do_c = workloads.make_bf16_inputs(w)
        q, k, v, do = (t.cuda() for t in (q_c, k_c, v_c, do_c))
        o, lse = fa.attention_forward(q, k, v, causal=causal, scale=w.sm_scale)
        ref = fa.attention_backward(q, k, v, o, do, lse, causal=causal, scale=w.sm_scale)
        exact = oracle.attention_bwd(q_c, k_c, v_c, do_c, w.sm_scale, causal)
        for call in range(2):      # the second call finds the first one's scratch contents
            got = tuple(torch.full_like(q, float("nan")) for _ in range(3))
            fa.fa_bwd_noalloc(q, k, v, o, do, lse, *got, scale=w.sm_scale, causal=causal)
            torch.cuda.synchronize()
            errs = {n: parity.rel_fro(g, r.float().cpu().double().numpy())
                    for n, g, r in zip(("dq", "dk", "dv"), got, ref)}
            assert all(e <= parity.GRAD_REL_FRO for e in errs.values()), (w.name, call, errs)
            parity.assert_grads_ok(got, exact, tag=(w.name, call, "oracle"))
        assert fa.fa_get_device_status() == 0


def test_noalloc_rejects_problems_beyond_its_scratch():
    import exact_attention_132_b200 as fa
    too_many = fa.FA_BWD_NOALLOC_MAX_ROWS // 64 + 1     # B*H*N just past the limit with H=64
    st = fa.lib.fa_bwd_noalloc(16, 16, 16, 16, 16, 16, 16, 16, 16, 1, 64, too_many, 64,
                               0.125, 0, None)
    assert st == fa.FA_ERR_INVALID_ARG
    assert "exceeds the fixed scratch" in fa.fa_last_error_string()
