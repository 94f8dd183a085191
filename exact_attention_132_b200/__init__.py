"""Python binding of libfa.so: exact fused attention for B200 (sm_100a).

Argument marshalling only: every function here checks shapes/dtypes, takes the
device pointers and the current CUDA stream from torch, and calls the C entry
point of the same name (declared in include/fa.h).  All arithmetic runs in the
library's CUDA kernels; there is no Python or CPU fallback, and importing this
package fails if the library has not been built
(``python exact_attention_132_b200/build.py``).
"""
from __future__ import annotations

import ctypes
import math
import os

import torch

__all__ = [
    "FAError", "fa_fwd", "fa_fwd_fp8", "fa_bwd", "fa_bwd_workspace_size", "fa_last_error_string",
    "fa_get_device_status", "fa_debug_wait_timeout_selftest", "fa_debug_exp2", "fa_version",
    "fa_fwd_kernel_name",
    "fa_decode", "fa_decode_workspace_size", "fa_fwd_gqa", "fa_bwd_gqa", "attention_forward",
    "attention_decode", "attention_forward_gqa", "attention_backward_gqa",
    "attention_forward_fp8", "attention_backward", "LIB_PATH", "lib",
]

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libfa.so")

FA_OK, FA_ERR_INVALID_ARG, FA_ERR_UNSUPPORTED, FA_ERR_CUDA, FA_ERR_DEVICE_TIMEOUT = range(5)
STATUS_NAMES = {0: "FA_OK", 1: "FA_ERR_INVALID_ARG", 2: "FA_ERR_UNSUPPORTED", 3: "FA_ERR_CUDA",
                4: "FA_ERR_DEVICE_TIMEOUT"}


class FAError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"{STATUS_NAMES.get(status, status)}: {msg}")
        self.status = status


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with "
                          "`python exact_attention_132_b200/build.py`")
    L = ctypes.CDLL(LIB_PATH)
    vp, i, f, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
    L.fa_fwd.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, f, i, vp]
    L.fa_fwd_fp8.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, f, i, vp]
    L.fa_bwd_workspace_size.argtypes = [i, i, i, i]
    L.fa_bwd_workspace_size.restype = sz
    L.fa_bwd.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, i, i, i, i, f, i, vp]
    L.fa_bwd_noalloc.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, f, i, vp]
    L.fa_bwd_noalloc.restype = ctypes.c_int
    L.fa_last_error_string.argtypes = []
    L.fa_last_error_string.restype = ctypes.c_char_p
    L.fa_get_device_status.argtypes = [vp, ctypes.POINTER(ctypes.c_int)]
    L.fa_debug_wait_timeout_selftest.argtypes = [i, vp]
    L.fa_debug_exp2.argtypes = [vp, vp, vp, vp, i, vp]
    L.fa_debug_exp2.restype = ctypes.c_int
    L.fa_version.argtypes = []
    L.fa_fwd_gqa.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, f, i, vp]
    L.fa_fwd_gqa.restype = ctypes.c_int
    L.fa_bwd_gqa.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, i, i, i, i, i, f, i, vp]
    L.fa_bwd_gqa.restype = ctypes.c_int
    L.fa_decode_workspace_size.argtypes = [i, i, i, i, i, i]
    L.fa_decode_workspace_size.restype = sz
    L.fa_decode.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, i, f, i, vp, sz, vp]
    L.fa_decode.restype = ctypes.c_int
    L.fa_fwd_kernel_name.argtypes = [i, i]
    L.fa_fwd_kernel_name.restype = ctypes.c_char_p
    L.fa_fwd_host_workspace_size.argtypes = [i, i, i, i]
    L.fa_fwd_host_workspace_size.restype = sz
    L.fa_fwd_host.argtypes = [vp, vp, vp, vp, vp, vp, sz, i, i, i, i, f, i, vp]
    L.fa_fwd_host.restype = ctypes.c_int
    L.fa_bwd_fp8_workspace_size.argtypes = [i, i, i, i]
    L.fa_bwd_fp8_workspace_size.restype = sz
    L.fa_bwd_fp8.argtypes = [vp] * 13 + [sz, i, i, i, i, f, i, vp]
    L.fa_bwd_fp8.restype = ctypes.c_int
    for name in ("fa_fwd", "fa_fwd_fp8", "fa_bwd", "fa_get_device_status",
                 "fa_debug_wait_timeout_selftest", "fa_version"):
        getattr(L, name).restype = ctypes.c_int
    return L


lib = _load()


def fa_last_error_string() -> str:
    return lib.fa_last_error_string().decode()


def _check(status: int) -> None:
    if status != FA_OK:
        raise FAError(status, fa_last_error_string())


def _ptr(t) -> int | None:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr() if t.numel() > 0 else None


def _stream(stream) -> int | None:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream if torch.cuda.is_available() else None
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _bhnd(t: torch.Tensor, name: str, dtype) -> tuple:
    if t.dim() != 4:
        raise ValueError(f"{name} must be [B, H, N, d], got shape {tuple(t.shape)}")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if t.numel() and not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    return tuple(t.shape)


def fa_fwd(q, k, v, o, lse=None, scale: float | None = None, causal: bool = False, stream=None):
    """O = softmax(scale Q K^T) V into ``o`` (bf16) and row logsumexp into ``lse`` (fp32)."""
    B, H, N, d = _bhnd(q, "q", torch.bfloat16)
    for t, n in ((k, "k"), (v, "v"), (o, "o")):
        if _bhnd(t, n, torch.bfloat16) != (B, H, N, d):
            raise ValueError(f"{n} shape differs from q")
    if lse is not None and (tuple(lse.shape) != (B, H, N) or lse.dtype != torch.float32):
        raise ValueError("lse must be fp32 [B, H, N]")
    sc = 1.0 / math.sqrt(d) if scale is None else float(scale)
    _check(lib.fa_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, H, N, d, sc,
                      1 if causal else 0, _stream(stream)))


def fa_fwd_fp8(q8, k8, v8, q_scale, k_scale, v_scale, o, lse=None, scale: float | None = None,
               causal: bool = False, stream=None):
    """FP8 e4m3 forward with per-128-row-tile fp32 scales; bf16 output."""
    B, H, N, d = _bhnd(q8, "q8", torch.float8_e4m3fn)
    for t, n in ((k8, "k8"), (v8, "v8")):
        if _bhnd(t, n, torch.float8_e4m3fn) != (B, H, N, d):
            raise ValueError(f"{n} shape differs from q8")
    if _bhnd(o, "o", torch.bfloat16) != (B, H, N, d):
        raise ValueError("o shape differs from q8")
    nt = (N + 127) // 128
    for t, n in ((q_scale, "q_scale"), (k_scale, "k_scale"), (v_scale, "v_scale")):
        if tuple(t.shape) != (B, H, nt) or t.dtype != torch.float32 or not t.is_contiguous():
            raise ValueError(f"{n} must be contiguous fp32 [B, H, ceil(N/128)]")
    if lse is not None and (tuple(lse.shape) != (B, H, N) or lse.dtype != torch.float32):
        raise ValueError("lse must be fp32 [B, H, N]")
    sc = 1.0 / math.sqrt(d) if scale is None else float(scale)
    _check(lib.fa_fwd_fp8(_ptr(q8), _ptr(k8), _ptr(v8), _ptr(q_scale), _ptr(k_scale),
                          _ptr(v_scale), _ptr(o), _ptr(lse), B, H, N, d, sc,
                          1 if causal else 0, _stream(stream)))


def fa_bwd_workspace_size(B: int, H: int, N: int, d: int) -> int:
    return int(lib.fa_bwd_workspace_size(B, H, N, d))


def fa_bwd(q, k, v, o, dO, lse, dq, dk, dv, workspace, scale: float | None = None,
           causal: bool = False, stream=None):
    """dQ, dK, dV (bf16) of L = sum(O * dO), recomputing P from the saved ``lse``."""
    B, H, N, d = _bhnd(q, "q", torch.bfloat16)
    for t, n in ((k, "k"), (v, "v"), (o, "o"), (dO, "dO"), (dq, "dq"), (dk, "dk"), (dv, "dv")):
        if _bhnd(t, n, torch.bfloat16) != (B, H, N, d):
            raise ValueError(f"{n} shape differs from q")
    if tuple(lse.shape) != (B, H, N) or lse.dtype != torch.float32:
        raise ValueError("lse must be fp32 [B, H, N]")
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    sc = 1.0 / math.sqrt(d) if scale is None else float(scale)
    _check(lib.fa_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(dO), _ptr(lse), _ptr(dq), _ptr(dk),
                      _ptr(dv), _ptr(workspace), ws_bytes, B, H, N, d, sc, 1 if causal else 0,
                      _stream(stream)))


FA_BWD_NOALLOC_MAX_ROWS = 1 << 21


def fa_bwd_noalloc(q, k, v, o, dO, lse, dq, dk, dv, scale: float | None = None,
                   causal: bool = False, stream=None):
    """fa_bwd without a workspace argument, for callers that cannot allocate device
    memory: the library uses its own fixed scratch (B*H*N <= FA_BWD_NOALLOC_MAX_ROWS).
    Calls that overlap on the GPU share that scratch and race; serialise them."""
    B, H, N, d = _bhnd(q, "q", torch.bfloat16)
    for t, n in ((k, "k"), (v, "v"), (o, "o"), (dO, "dO"), (dq, "dq"), (dk, "dk"), (dv, "dv")):
        if _bhnd(t, n, torch.bfloat16) != (B, H, N, d):
            raise ValueError(f"{n} shape differs from q")
    if tuple(lse.shape) != (B, H, N) or lse.dtype != torch.float32:
        raise ValueError("lse must be fp32 [B, H, N]")
    sc = 1.0 / math.sqrt(d) if scale is None else float(scale)
    _check(lib.fa_bwd_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(dO), _ptr(lse), _ptr(dq),
                              _ptr(dk), _ptr(dv), B, H, N, d, sc, 1 if causal else 0,
                              _stream(stream)))


def fa_get_device_status(stream=None) -> int:
    code = ctypes.c_int(0)
    _check(lib.fa_get_device_status(_stream(stream), ctypes.byref(code)))
    return code.value


def fa_debug_wait_timeout_selftest(timeout_us: int, stream=None) -> None:
    _check(lib.fa_debug_wait_timeout_selftest(int(timeout_us), _stream(stream)))


def fa_debug_exp2(x: torch.Tensor, stream=None):
    """(software 2^x, special-function-unit ex2, exp2f) of the fp32 CUDA tensor x."""
    if x.dtype != torch.float32 or not x.is_cuda or not x.is_contiguous():
        raise ValueError("x must be a contiguous fp32 CUDA tensor")
    outs = tuple(torch.empty_like(x) for _ in range(3))
    _check(lib.fa_debug_exp2(_ptr(x), *(_ptr(t) for t in outs), x.numel(), _stream(stream)))
    return outs


def fa_version() -> int:
    return int(lib.fa_version())


def fa_fwd_kernel_name(head_dim: int, fp8: bool = False) -> str | None:
    """Name and tile configuration of the forward kernel launched for this head dim."""
    r = lib.fa_fwd_kernel_name(int(head_dim), int(bool(fp8)))
    return None if r is None else r.decode()


# ------------------------------------------------------------------ allocating helpers
def attention_forward(q, k, v, causal: bool = False, scale: float | None = None):
    """Allocate O and LSE with torch and run fa_fwd; returns (o, lse)."""
    B, H, N, d = q.shape
    o = torch.empty_like(q)
    lse = torch.empty((B, H, N), dtype=torch.float32, device=q.device)
    fa_fwd(q, k, v, o, lse, scale=scale, causal=causal)
    return o, lse


def attention_forward_fp8(q8, k8, v8, q_scale, k_scale, v_scale, causal: bool = False,
                          scale: float | None = None):
    B, H, N, d = q8.shape
    o = torch.empty((B, H, N, d), dtype=torch.bfloat16, device=q8.device)
    lse = torch.empty((B, H, N), dtype=torch.float32, device=q8.device)
    fa_fwd_fp8(q8, k8, v8, q_scale, k_scale, v_scale, o, lse, scale=scale, causal=causal)
    return o, lse


def attention_backward(q, k, v, o, dO, lse, causal: bool = False, scale: float | None = None,
                       workspace=None):
    """Allocate dQ/dK/dV (and the workspace unless given) and run fa_bwd."""
    B, H, N, d = q.shape
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    if workspace is None:
        nbytes = fa_bwd_workspace_size(B, H, N, d)
        workspace = torch.empty(max(nbytes, 1), dtype=torch.uint8, device=q.device)
    fa_bwd(q, k, v, o, dO, lse, dq, dk, dv, workspace, scale=scale, causal=causal)
    return dq, dk, dv


def fa_fwd_host_workspace_size(B: int, H: int, N: int, d: int) -> int:
    return int(lib.fa_fwd_host_workspace_size(B, H, N, d))


def fa_fwd_host(q, k, v, o, lse, workspace, scale: float | None = None, causal: bool = False,
                stream=None):
    """Forward on host (CPU) bf16 tensors [B, H, N, d]: chunks of heads are copied in,
    computed and copied out with the copies overlapping the kernels.  o (and lse, fp32
    [B, H, N], or None) are host tensors written once ``stream`` completes; workspace is a
    device tensor of fa_fwd_host_workspace_size bytes."""
    shp = tuple(q.shape)
    if len(shp) != 4:
        raise ValueError("q must be [B, H, N, d]")
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (o, "o")):
        if t.dtype != torch.bfloat16 or tuple(t.shape) != shp or not t.is_contiguous():
            raise TypeError(f"{n} must be a contiguous bf16 tensor of q's shape")
        if t.is_cuda:
            raise ValueError(f"{n} must be in host memory")
    B, H, N, d = shp
    if lse is not None and (tuple(lse.shape) != (B, H, N) or lse.dtype != torch.float32
                            or lse.is_cuda or not lse.is_contiguous()):
        raise ValueError("lse must be a contiguous host fp32 [B, H, N] tensor")
    if workspace is None or not workspace.is_cuda:
        raise ValueError("workspace must be a device tensor")
    ws_bytes = workspace.numel() * workspace.element_size()
    sc = 1.0 / math.sqrt(d) if scale is None else float(scale)
    _check(lib.fa_fwd_host(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                           lse.data_ptr() if lse is not None else None, _ptr(workspace), ws_bytes,
                           B, H, N, d, sc, 1 if causal else 0, _stream(stream)))


def attention_forward_host(q, k, v, causal: bool = False, scale: float | None = None,
                           device=None):
    """Allocate page-locked o / lse and the device workspace, run fa_fwd_host on the
    current stream of ``device`` and wait for it."""
    B, H, N, d = q.shape
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    o = torch.empty((B, H, N, d), dtype=torch.bfloat16).pin_memory()
    lse = torch.empty((B, H, N), dtype=torch.float32).pin_memory()
    ws = torch.empty(max(1, fa_fwd_host_workspace_size(B, H, N, d)), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    fa_fwd_host(q, k, v, o, lse, ws, scale=scale, causal=causal, stream=stream)
    stream.synchronize()
    return o, lse


def fa_bwd_fp8_workspace_size(B: int, H: int, N: int, d: int) -> int:
    return int(lib.fa_bwd_fp8_workspace_size(B, H, N, d))


def fa_bwd_fp8(q8, k8, v8, q_scale, k_scale, v_scale, o, dO, lse, dq, dk, dv, workspace,
               scale: float | None = None, causal: bool = False, stream=None):
    """Gradients (bf16) for the dequantised inputs of the FP8 forward: o and lse are
    fa_fwd_fp8's outputs; the workspace holds bf16 copies of q8, k8, v8 times their tile
    scales and the row sums of the backward."""
    B, H, N, d = _bhnd(q8, "q8", torch.float8_e4m3fn)
    for t, n in ((k8, "k8"), (v8, "v8")):
        if _bhnd(t, n, torch.float8_e4m3fn) != (B, H, N, d):
            raise ValueError(f"{n} shape differs from q8")
    for t, n in ((o, "o"), (dO, "dO"), (dq, "dq"), (dk, "dk"), (dv, "dv")):
        if _bhnd(t, n, torch.bfloat16) != (B, H, N, d):
            raise ValueError(f"{n} shape differs from q8")
    nt = (N + 127) // 128
    for t, n in ((q_scale, "q_scale"), (k_scale, "k_scale"), (v_scale, "v_scale")):
        if tuple(t.shape) != (B, H, nt) or t.dtype != torch.float32 or not t.is_contiguous():
            raise ValueError(f"{n} must be contiguous fp32 [B, H, ceil(N/128)]")
    if tuple(lse.shape) != (B, H, N) or lse.dtype != torch.float32:
        raise ValueError("lse must be fp32 [B, H, N]")
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    sc = 1.0 / math.sqrt(d) if scale is None else float(scale)
    _check(lib.fa_bwd_fp8(_ptr(q8), _ptr(k8), _ptr(v8), _ptr(q_scale), _ptr(k_scale),
                          _ptr(v_scale), _ptr(o), _ptr(dO), _ptr(lse), _ptr(dq), _ptr(dk),
                          _ptr(dv), _ptr(workspace), ws_bytes, B, H, N, d, sc,
                          1 if causal else 0, _stream(stream)))


def attention_backward_fp8(q8, k8, v8, q_scale, k_scale, v_scale, o, dO, lse,
                           causal: bool = False, scale: float | None = None):
    """Allocate dQ/dK/dV and the workspace and run fa_bwd_fp8."""
    B, H, N, d = q8.shape
    dq, dk, dv = (torch.empty((B, H, N, d), dtype=torch.bfloat16, device=q8.device)
                  for _ in range(3))
    nbytes = fa_bwd_fp8_workspace_size(B, H, N, d)
    workspace = torch.empty(max(nbytes, 1), dtype=torch.uint8, device=q8.device)
    fa_bwd_fp8(q8, k8, v8, q_scale, k_scale, v_scale, o, dO, lse, dq, dk, dv, workspace,
               scale=scale, causal=causal)
    return dq, dk, dv


# ------------------------------------------------------------------ decoding (GQA / MQA)
def fa_decode_workspace_size(B: int, Hq: int, Hkv: int, Nq: int, Nk: int, d: int) -> int:
    return int(lib.fa_decode_workspace_size(B, Hq, Hkv, Nq, Nk, d))


def fa_decode(q, k, v, o, lse, workspace, scale: float | None = None, causal: bool = False,
              stream=None):
    """Few queries ([B, Hq, Nq, d]) against long K/V ([B, Hkv, Nk, d]); causal queries sit
    at the end of the sequence.  Writes o (bf16) and lse (fp32 [B, Hq, Nq], or None)."""
    B, Hq, Nq, d = _bhnd(q, "q", torch.bfloat16)
    Bk, Hkv, Nk, dk = _bhnd(k, "k", torch.bfloat16)
    if (Bk, dk) != (B, d) or tuple(v.shape) != tuple(k.shape) or v.dtype != torch.bfloat16:
        raise ValueError("k and v must be bf16 [B, Hkv, Nk, d] with q's B and d")
    if not v.is_contiguous():
        raise ValueError("v must be contiguous")
    if _bhnd(o, "o", torch.bfloat16) != (B, Hq, Nq, d):
        raise ValueError("o shape differs from q")
    if lse is not None and (tuple(lse.shape) != (B, Hq, Nq) or lse.dtype != torch.float32):
        raise ValueError("lse must be fp32 [B, Hq, Nq]")
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    sc = 1.0 / math.sqrt(d) if scale is None else float(scale)
    _check(lib.fa_decode(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, Hq, Hkv, Nq, Nk, d, sc,
                         1 if causal else 0, _ptr(workspace), ws_bytes, _stream(stream)))


def attention_decode(q, k, v, causal: bool = False, scale: float | None = None):
    """Allocate O, LSE and the workspace with torch and run fa_decode; returns (o, lse)."""
    B, Hq, Nq, d = q.shape
    Hkv, Nk = k.shape[1], k.shape[2]
    o = torch.empty_like(q)
    lse = torch.empty((B, Hq, Nq), dtype=torch.float32, device=q.device)
    nbytes = fa_decode_workspace_size(B, Hq, Hkv, Nq, Nk, d)
    ws = torch.empty(max(nbytes, 16), dtype=torch.uint8, device=q.device)
    fa_decode(q, k, v, o, lse, ws, scale=scale, causal=causal)
    return o, lse


# ------------------------------------------------------------------ grouped heads, full length
def _gqa_shapes(q, k):
    B, Hq, N, d = _bhnd(q, "q", torch.bfloat16)
    Bk, Hkv, Nk, dk = _bhnd(k, "k", torch.bfloat16)
    if (Bk, Nk, dk) != (B, N, d):
        raise ValueError("k must be [B, Hkv, N, d] with q's B, N and d")
    return B, Hq, Hkv, N, d


def fa_fwd_gqa(q, k, v, o, lse, scale: float | None = None, causal: bool = False, stream=None):
    """Forward with Hq query heads on Hkv key/value heads (query head h reads h // g)."""
    B, Hq, Hkv, N, d = _gqa_shapes(q, k)
    if _bhnd(v, "v", torch.bfloat16) != (B, Hkv, N, d):
        raise ValueError("v shape differs from k")
    if _bhnd(o, "o", torch.bfloat16) != (B, Hq, N, d):
        raise ValueError("o shape differs from q")
    if lse is not None and (tuple(lse.shape) != (B, Hq, N) or lse.dtype != torch.float32):
        raise ValueError("lse must be fp32 [B, Hq, N]")
    sc = 1.0 / math.sqrt(d) if scale is None else float(scale)
    _check(lib.fa_fwd_gqa(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, Hq, Hkv, N, d, sc,
                          1 if causal else 0, _stream(stream)))


def fa_bwd_gqa(q, k, v, o, dO, lse, dq, dk, dv, workspace, scale: float | None = None,
               causal: bool = False, stream=None):
    """Backward with grouped heads; dk, dv sum over the query heads of each group."""
    B, Hq, Hkv, N, d = _gqa_shapes(q, k)
    for t, n, h in ((v, "v", Hkv), (o, "o", Hq), (dO, "dO", Hq), (dq, "dq", Hq), (dk, "dk", Hkv),
                    (dv, "dv", Hkv)):
        if _bhnd(t, n, torch.bfloat16) != (B, h, N, d):
            raise ValueError(f"{n} has the wrong shape")
    if tuple(lse.shape) != (B, Hq, N) or lse.dtype != torch.float32:
        raise ValueError("lse must be fp32 [B, Hq, N]")
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    sc = 1.0 / math.sqrt(d) if scale is None else float(scale)
    _check(lib.fa_bwd_gqa(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(dO), _ptr(lse), _ptr(dq),
                          _ptr(dk), _ptr(dv), _ptr(workspace), ws_bytes, B, Hq, Hkv, N, d, sc,
                          1 if causal else 0, _stream(stream)))


def attention_forward_gqa(q, k, v, causal: bool = False, scale: float | None = None):
    """Allocate O and LSE with torch and run fa_fwd_gqa; returns (o, lse)."""
    B, Hq, N, d = q.shape
    o = torch.empty_like(q)
    lse = torch.empty((B, Hq, N), dtype=torch.float32, device=q.device)
    fa_fwd_gqa(q, k, v, o, lse, scale=scale, causal=causal)
    return o, lse


def attention_backward_gqa(q, k, v, o, dO, lse, causal: bool = False, scale: float | None = None):
    """Allocate dQ/dK/dV and the workspace and run fa_bwd_gqa; returns (dq, dk, dv)."""
    B, Hq, N, d = q.shape
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    ws = torch.empty(max(fa_bwd_workspace_size(B, Hq, N, d), 16), dtype=torch.uint8, device=q.device)
    fa_bwd_gqa(q, k, v, o, dO, lse, dq, dk, dv, ws, scale=scale, causal=causal)
    return dq, dk, dv


# ------------------------------------------------------------------ autograd
class _Attention(torch.autograd.Function):
    """O = softmax(scale Q K^T) V with the library's forward, and its backward by
    recomputation from the saved logsumexp.  Grouped heads when K and V have fewer
    heads than Q."""

    @staticmethod
    def forward(ctx, q, k, v, causal, scale):
        q, k, v = q.contiguous(), k.contiguous(), v.contiguous()
        o, lse = attention_forward_gqa(q, k, v, causal=causal, scale=scale)
        ctx.save_for_backward(q, k, v, o, lse)
        ctx.causal, ctx.scale = causal, scale
        return o

    @staticmethod
    def backward(ctx, do):
        q, k, v, o, lse = ctx.saved_tensors
        dq, dk, dv = attention_backward_gqa(q, k, v, o, do.contiguous(), lse, causal=ctx.causal,
                                            scale=ctx.scale)
        return dq, dk, dv, None, None


def attention(q, k, v, causal: bool = False, scale: float | None = None):
    """Differentiable exact attention on bf16 CUDA tensors q [B, Hq, N, d], k and v
    [B, Hkv, N, d] (Hq a multiple of Hkv); scale defaults to 1/sqrt(d)."""
    return _Attention.apply(q, k, v, causal, scale)
