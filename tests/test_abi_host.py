"""Host-side checks of the C ABI that need no GPU: the library loads, exports every
symbol include/fa.h declares, and rejects bad arguments before any CUDA call."""
import ctypes
import os
import re
import subprocess

import pytest

import exact_attention_132_b200 as fa

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    text = open(os.path.join(ROOT, "include", "fa.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(fa_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for required in ("fa_fwd", "fa_fwd_fp8", "fa_bwd", "fa_bwd_workspace_size",
                     "fa_last_error_string", "fa_get_device_status"):
        assert required in names


def test_library_exports_every_declared_symbol():
    out = subprocess.run(["nm", "-D", "--defined-only", fa.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\bT (fa_[a-z0-9_]+)$", out, flags=re.M))
    missing = [n for n in declared_functions() if n not in exported]
    assert not missing, missing
    for n in declared_functions():
        assert hasattr(fa.lib, n)


def test_version():
    assert fa.fa_version() >= 100


def test_forward_kernel_names():
    # every supported head dim names a kernel whose tile matches it; others name none
    for d, fp8 in ((64, False), (128, False), (256, False), (128, True)):
        name = fa.fa_fwd_kernel_name(d, fp8)
        assert name and name.startswith("fa_fwd_") and f"<{d}," in name
        assert ("e4m3" in name) == fp8
    assert fa.fa_fwd_kernel_name(80) is None
    # stored head dims 96 and 192 run on the 128 and 256 kernels
    assert fa.fa_fwd_kernel_name(96) == fa.fa_fwd_kernel_name(128)
    assert fa.fa_fwd_kernel_name(192) == fa.fa_fwd_kernel_name(256)
    assert fa.fa_fwd_kernel_name(80, True) is None
    assert fa.fa_fwd_kernel_name(64, True) == fa.fa_fwd_kernel_name(128, True)
    assert "<256," in fa.fa_fwd_kernel_name(192, True)


def _fwd(q=1, k=1, v=1, o=1, lse=None, B=1, H=1, N=128, d=128, scale=0.1, causal=0):
    P = lambda x: None if x is None else ctypes.c_void_p(16 * x)
    return fa.lib.fa_fwd(P(q), P(k), P(v), P(o), P(lse), B, H, N, d, scale, causal, None)


def test_argument_errors_return_before_any_cuda_call():
    assert _fwd(q=None) == fa.FA_ERR_INVALID_ARG
    assert "q is NULL" in fa.fa_last_error_string()
    assert _fwd(B=-1) == fa.FA_ERR_INVALID_ARG
    assert _fwd(scale=0.0) == fa.FA_ERR_INVALID_ARG
    assert _fwd(scale=float("nan")) == fa.FA_ERR_INVALID_ARG
    assert _fwd(scale=-1.0) == fa.FA_ERR_INVALID_ARG
    assert _fwd(d=80) == fa.FA_ERR_UNSUPPORTED
    assert _fwd(d=32) == fa.FA_ERR_UNSUPPORTED
    # misaligned pointer
    assert fa.lib.fa_fwd(ctypes.c_void_p(18), ctypes.c_void_p(16), ctypes.c_void_p(16),
                         ctypes.c_void_p(16), None, 1, 1, 128, 64, 0.1, 0, None) == fa.FA_ERR_INVALID_ARG
    assert "aligned" in fa.fa_last_error_string()


def test_empty_problems_are_a_no_op():
    assert _fwd(q=None, k=None, v=None, o=None, N=0) == fa.FA_OK
    assert _fwd(q=None, k=None, v=None, o=None, B=0) == fa.FA_OK
    assert fa.lib.fa_bwd(None, None, None, None, None, None, None, None, None, None, 0,
                         1, 4, 0, 64, 0.125, 1, None) == fa.FA_OK
    assert fa.fa_bwd_workspace_size(0, 4, 128, 64) == 0


def test_fp8_and_bwd_argument_errors():
    P = lambda x: ctypes.c_void_p(16 * x)
    st = fa.lib.fa_fwd_fp8(P(1), P(1), P(1), None, P(1), P(1), P(1), None, 1, 1, 256, 128, 0.1, 1, None)
    assert st == fa.FA_ERR_INVALID_ARG
    st = fa.lib.fa_fwd_fp8(P(1), P(1), P(1), P(1), P(1), P(1), P(1), None, 1, 1, 256, 80, 0.1, 1, None)
    assert st == fa.FA_ERR_UNSUPPORTED
    need = fa.fa_bwd_workspace_size(2, 3, 1000, 64)
    assert need >= 2 * 3 * 1000 * 4 and need % 256 == 0
    st = fa.lib.fa_bwd(P(1), P(1), P(1), P(1), P(1), P(1), P(1), P(1), P(1), P(1), need - 256,
                       2, 3, 1000, 64, 0.125, 0, None)
    assert st == fa.FA_ERR_INVALID_ARG and "workspace" in fa.fa_last_error_string()


def test_fp8_bwd_argument_errors():
    P = lambda x: ctypes.c_void_p(16 * x)
    need = fa.fa_bwd_fp8_workspace_size(1, 2, 300, 128)
    # three bf16 copies of the inputs plus the D_i rows, each 256-byte aligned
    assert need >= 3 * 2 * 300 * 128 * 2 + 2 * 300 * 4 and need % 256 == 0
    assert fa.fa_bwd_fp8_workspace_size(0, 2, 300, 128) == 0
    args = [P(1)] * 13
    st = fa.lib.fa_bwd_fp8(*args, need, 1, 2, 300, 80, 0.1, 1, None)
    assert st == fa.FA_ERR_UNSUPPORTED
    st = fa.lib.fa_bwd_fp8(*args, need - 256, 1, 2, 300, 128, 0.1, 1, None)
    assert st == fa.FA_ERR_INVALID_ARG and "workspace" in fa.fa_last_error_string()
    no_scale = args[:3] + [None] + args[4:]
    st = fa.lib.fa_bwd_fp8(*no_scale, need, 1, 2, 300, 128, 0.1, 1, None)
    assert st == fa.FA_ERR_INVALID_ARG and "scale" in fa.fa_last_error_string()
    assert fa.lib.fa_bwd_fp8(*([None] * 13), 0, 1, 2, 0, 128, 0.1, 1, None) == fa.FA_OK


def test_host_forward_argument_errors():
    P = lambda x: ctypes.c_void_p(16 * x)
    need = fa.fa_fwd_host_workspace_size(2, 8, 1000, 128)
    assert need > 0 and need % 256 == 0
    assert fa.fa_fwd_host_workspace_size(0, 8, 1000, 128) == 0
    st = fa.lib.fa_fwd_host(None, P(1), P(1), P(1), None, P(1), need, 2, 8, 1000, 128, 0.1, 1, None)
    assert st == fa.FA_ERR_INVALID_ARG and "host" in fa.fa_last_error_string()
    st = fa.lib.fa_fwd_host(P(1), P(1), P(1), P(1), None, P(1), need - 256, 2, 8, 1000, 128, 0.1, 1,
                            None)
    assert st == fa.FA_ERR_INVALID_ARG and "workspace" in fa.fa_last_error_string()
    st = fa.lib.fa_fwd_host(P(1), P(1), P(1), P(1), None, P(1), need, 2, 8, 1000, 80, 0.1, 1, None)
    assert st == fa.FA_ERR_UNSUPPORTED
    assert fa.lib.fa_fwd_host(None, None, None, None, None, None, 0, 2, 8, 0, 128, 0.1, 1,
                              None) == fa.FA_OK


def test_python_wrappers_validate_shapes():
    import torch
    q = torch.zeros(1, 2, 8, 64, dtype=torch.bfloat16)
    with pytest.raises(TypeError):
        fa.fa_fwd(q.float(), q, q, q)
    with pytest.raises(ValueError):
        fa.fa_fwd(q, q[:, :1], q, q)
    with pytest.raises(ValueError):
        fa.fa_fwd(q, q, q, q)   # CPU tensors are rejected: no CPU path exists


def _dec(q=1, k=1, v=1, o=1, lse=None, B=1, Hq=8, Hkv=2, Nq=1, Nk=300, d=128, scale=0.1,
         causal=0, ws=1, ws_bytes=1 << 30):
    P = lambda x: None if x is None else ctypes.c_void_p(16 * x)
    return fa.lib.fa_decode(P(q), P(k), P(v), P(o), P(lse), B, Hq, Hkv, Nq, Nk, d, scale, causal,
                            P(ws), ws_bytes, None)


def test_decode_argument_errors_return_before_any_cuda_call():
    assert _dec(d=80) == 2                              # unsupported head dim
    assert _dec(Hq=6, Hkv=4) == 1                       # Hq not a multiple of Hkv
    assert _dec(Hq=64, Hkv=1, Nq=4) == 1                # 256 rows per key/value head
    assert _dec(Nk=0) == 1
    assert _dec(causal=1, Nq=4, Nk=3) == 1              # causal needs Nq <= Nk
    assert _dec(scale=float("nan")) == 1
    assert _dec(B=-1) == 1
    assert _dec(Nq=0) == 0 and _dec(B=0) == 0           # empty problems are no-ops
    assert fa.fa_decode_workspace_size(1, 6, 4, 1, 100, 128) == 0


def test_noalloc_backward_argument_errors_return_before_any_cuda_call():
    # the Python constant is the header's limit
    hdr = open(os.path.join(ROOT, "include", "fa.h")).read()
    m = re.search(r"#define\s+FA_BWD_NOALLOC_MAX_ROWS\s+\(1 << (\d+)\)", hdr)
    assert m and fa.FA_BWD_NOALLOC_MAX_ROWS == 1 << int(m.group(1))
    P = lambda x: ctypes.c_void_p(16 * x)
    ptrs = [P(1)] * 9

    def call(B=1, H=2, N=256, d=128, scale=0.125, ps=ptrs):
        return fa.lib.fa_bwd_noalloc(*ps, B, H, N, d, scale, 1, None)

    assert call(d=80) == fa.FA_ERR_UNSUPPORTED
    assert call(N=-1) == fa.FA_ERR_INVALID_ARG
    assert call(scale=float("nan")) == fa.FA_ERR_INVALID_ARG
    # one row past the fixed scratch, and exactly at it with a null pointer (so that the
    # size check passes and the pointer check answers, still before any CUDA call)
    H, N = 32, fa.FA_BWD_NOALLOC_MAX_ROWS // 32
    assert call(B=1, H=H, N=N + 1) == fa.FA_ERR_INVALID_ARG
    assert "exceeds the fixed scratch" in fa.fa_last_error_string()
    nulls = ptrs[:6] + [None] + ptrs[7:]
    assert call(B=1, H=H, N=N, ps=nulls) == fa.FA_ERR_INVALID_ARG
    assert "dq" in fa.fa_last_error_string()
    # empty problems launch nothing and touch no pointer
    assert call(B=0, ps=[None] * 9) == fa.FA_OK


def test_exp2_probe_argument_errors_return_before_any_cuda_call():
    P = ctypes.c_void_p(256)
    assert fa.lib.fa_debug_exp2(P, P, P, P, -1, None) == fa.FA_ERR_INVALID_ARG
    assert fa.lib.fa_debug_exp2(None, P, P, P, 8, None) == fa.FA_ERR_INVALID_ARG
    assert fa.lib.fa_debug_exp2(P, P, None, P, 8, None) == fa.FA_ERR_INVALID_ARG
    assert fa.lib.fa_debug_exp2(None, None, None, None, 0, None) == fa.FA_OK
