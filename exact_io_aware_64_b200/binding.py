"""ctypes binding for libfa.so (include/fa.h).

Argument marshalling only: it checks that tensors are CUDA, contiguous and of the right
shape and dtype, allocates outputs with torch when the caller does not pass them, and
hands raw pointers and the current CUDA stream to the C ABI.  Every step of the
computation runs in the library's kernels; there is no fallback.
"""
from __future__ import annotations

import ctypes
import math
import os
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libfa.so")

FA_OK = 0
FA_ERR_INVALID_ARG = 1
FA_ERR_UNSUPPORTED = 2
FA_ERR_CUDA = 3
FA_ERR_TIMEOUT = 4

_lib = None

_vp = ctypes.c_void_p
_i = ctypes.c_int
_f = ctypes.c_float
_sz = ctypes.c_size_t

SIGNATURES = {
    "fa_abi_version": ([], _i),
    "fa_fwd": ([_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _f, _i, _vp], _i),
    "fa_fwd_qk": ([_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _f, _i, _vp], _i),
    "fa_fwd_varlen": ([_vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _f, _i, _vp],
                      _i),
    "fa_fwd_packed": ([_vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _i, _f, _i,
                       _vp], _i),
    "fa_fwd_f32": ([_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _f, _i, _vp], _i),
    "fa_fwd_f32_qk": ([_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _f, _i, _vp], _i),
    "fa_fwd_f32_varlen": ([_vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _f, _i,
                           _vp], _i),
    "fa_fwd_f32_packed": ([_vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _i, _f,
                           _i, _vp], _i),
    "fa_bwd_workspace_bytes": ([_i, _i, _i, _i], _sz),
    "fa_bwd": ([_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _f, _i, _vp, _sz,
                _vp], _i),
    "fa_bwd_qk": ([_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _f, _i, _vp,
                   _sz, _vp], _i),
    "fa_bwd_varlen": ([_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i,
                       _i, _f, _i, _vp, _sz, _vp], _i),
    "fa_bwd_packed": ([_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i,
                       _i, _i, _i, _f, _i, _vp, _sz, _vp], _i),
    "fa_bwd_f32": ([_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _f, _i, _vp,
                    _sz, _vp], _i),
    "fa_bwd_f32_qk": ([_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _f, _i,
                       _vp, _sz, _vp], _i),
    "fa_bwd_f32_varlen": ([_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i,
                           _i, _i, _f, _i, _vp, _sz, _vp], _i),
    "fa_bwd_f32_packed": ([_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i,
                           _i, _i, _i, _i, _f, _i, _vp, _sz, _vp], _i),
    "fa_merge": ([_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _vp], _i),
    "fa_accumulate": ([_vp, _vp, _vp, _sz, _vp], _i),
    "fa_selftest_timeout": ([ctypes.c_longlong, _vp], _i),
    "fa_bwd_noalloc": ([_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _f, _i,
                        _vp], _i),
    "fa_bwd_noalloc_max_scratch_bytes": ([], _sz),
    "fa_trace_events": ([ctypes.POINTER(_vp), _i], _i),
    "fa_status_string": ([_i], ctypes.c_char_p),
    "fa_last_error_message": ([], ctypes.c_char_p),
    "fa_check_device_error": ([_vp], _i),
}


class FAError(RuntimeError):
    def __init__(self, call: str, status: int, message: str):
        super().__init__(f"{call} failed: {status_name(status)}: {message}")
        self.status = status


def lib() -> ctypes.CDLL:
    """Load libfa.so (built in place by ``python -m exact_io_aware_64_b200.build``)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"{LIB_PATH} is missing: build it with python -m exact_io_aware_64_b200.build")
        L = ctypes.CDLL(LIB_PATH)
        for name, (args, res) in SIGNATURES.items():
            fn = getattr(L, name)
            fn.argtypes = args
            fn.restype = res
        _lib = L
    return _lib


def status_name(status: int) -> str:
    return lib().fa_status_string(status).decode()


def _check(call: str, status: int) -> None:
    if status != FA_OK:
        raise FAError(call, status, lib().fa_last_error_message().decode())


def _stream_handle(stream: Optional[torch.cuda.Stream]) -> int:
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _check_bhnd(name: str, t: torch.Tensor, shape, dtype) -> None:
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def fwd(Q: torch.Tensor, K: torch.Tensor, V: torch.Tensor, scale: Optional[float] = None,
        causal: bool = False, O: Optional[torch.Tensor] = None,
        LSE: Optional[torch.Tensor] = None, want_lse: bool = True,
        stream: Optional[torch.cuda.Stream] = None):
    """Exact attention forward through ``fa_fwd`` / ``fa_fwd_qk`` (bf16; the latter when
    Nq != Nk) or ``fa_fwd_f32`` / ``fa_fwd_f32_qk`` (float32).

    Q: [B, H, Nq, d]; K, V: [B, H, Nk, d]; CUDA tensors, contiguous, all bf16 or all
    float32.  With Nq != Nk the queries are the last Nq of the Nk tokens (causal masking
    aligned at the bottom right).
    Returns (O, LSE); LSE is None when ``want_lse`` is False and none is passed.
    """
    B, H, Nq, d = Q.shape
    Nk = K.shape[2]
    dtype = Q.dtype
    if dtype not in (torch.bfloat16, torch.float32):
        raise ValueError("Q, K, V must be bfloat16 or float32")
    _check_bhnd("Q", Q, (B, H, Nq, d), dtype)
    for name, t in (("K", K), ("V", V)):
        _check_bhnd(name, t, (B, H, Nk, d), dtype)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if O is None:
        O = torch.empty_like(Q)
    _check_bhnd("O", O, (B, H, Nq, d), dtype)
    if LSE is None and want_lse:
        LSE = torch.empty((B, H, Nq), device=Q.device, dtype=torch.float32)
    if LSE is not None:
        _check_bhnd("LSE", LSE, (B, H, Nq), torch.float32)
    with torch.cuda.device(Q.device):
        if dtype == torch.float32 and Nq == Nk:
            name = "fa_fwd_f32"
            st = lib().fa_fwd_f32(_ptr(Q), _ptr(K), _ptr(V), _ptr(O), _ptr(LSE), B, H, Nq, d,
                                  float(scale), int(bool(causal)), _stream_handle(stream))
        elif dtype == torch.float32:
            name = "fa_fwd_f32_qk"
            st = lib().fa_fwd_f32_qk(_ptr(Q), _ptr(K), _ptr(V), _ptr(O), _ptr(LSE), B, H, Nq,
                                     Nk, d, float(scale), int(bool(causal)),
                                     _stream_handle(stream))
        elif Nq == Nk:
            name = "fa_fwd"
            st = lib().fa_fwd(_ptr(Q), _ptr(K), _ptr(V), _ptr(O), _ptr(LSE), B, H, Nq, d,
                              float(scale), int(bool(causal)), _stream_handle(stream))
        else:
            name = "fa_fwd_qk"
            st = lib().fa_fwd_qk(_ptr(Q), _ptr(K), _ptr(V), _ptr(O), _ptr(LSE), B, H, Nq, Nk,
                                 d, float(scale), int(bool(causal)), _stream_handle(stream))
    _check(name, st)
    return O, LSE


def workspace_bytes(B: int, H: int, N: int, d: int) -> int:
    return int(lib().fa_bwd_workspace_bytes(B, H, N, d))


def bwd(Q: torch.Tensor, K: torch.Tensor, V: torch.Tensor, O: torch.Tensor,
        dO: torch.Tensor, LSE: torch.Tensor, scale: Optional[float] = None,
        causal: bool = False, dQ: Optional[torch.Tensor] = None,
        dK: Optional[torch.Tensor] = None, dV: Optional[torch.Tensor] = None,
        workspace: Optional[torch.Tensor] = None,
        stream: Optional[torch.cuda.Stream] = None):
    """Exact attention backward through ``fa_bwd`` / ``fa_bwd_qk`` (bf16; the latter when
    Nq != Nk) or ``fa_bwd_f32`` / ``fa_bwd_f32_qk`` (float32).

    Q, O, dO: [B, H, Nq, d]; K, V: [B, H, Nk, d]; CUDA tensors, contiguous, all bf16 or
    all float32; LSE: [B, H, Nq] float32.  Returns (dQ, dK, dV) in the inputs' dtype."""
    B, H, Nq, d = Q.shape
    Nk = K.shape[2]
    dtype = Q.dtype
    if dtype not in (torch.bfloat16, torch.float32):
        raise ValueError("Q, K, V, O, dO must be bfloat16 or float32")
    for name, t in (("Q", Q), ("O", O), ("dO", dO)):
        _check_bhnd(name, t, (B, H, Nq, d), dtype)
    for name, t in (("K", K), ("V", V)):
        _check_bhnd(name, t, (B, H, Nk, d), dtype)
    _check_bhnd("LSE", LSE, (B, H, Nq), torch.float32)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    dQ = torch.empty_like(Q) if dQ is None else dQ
    dK = torch.empty_like(K) if dK is None else dK
    dV = torch.empty_like(V) if dV is None else dV
    _check_bhnd("dQ", dQ, (B, H, Nq, d), dtype)
    for name, t in (("dK", dK), ("dV", dV)):
        _check_bhnd(name, t, (B, H, Nk, d), dtype)
    need = workspace_bytes(B, H, Nq, d)
    if workspace is None:
        workspace = torch.empty(max(need, 1), device=Q.device, dtype=torch.uint8)
    ws_bytes = workspace.numel() * workspace.element_size()
    ptrs = (_ptr(Q), _ptr(K), _ptr(V), _ptr(O), _ptr(dO), _ptr(LSE), _ptr(dQ), _ptr(dK),
            _ptr(dV))
    tail = (float(scale), int(bool(causal)), _ptr(workspace), ws_bytes, _stream_handle(stream))
    with torch.cuda.device(Q.device):
        if dtype == torch.float32 and Nq == Nk:
            name = "fa_bwd_f32"
            st = lib().fa_bwd_f32(*ptrs, B, H, Nq, d, *tail)
        elif dtype == torch.float32:
            name = "fa_bwd_f32_qk"
            st = lib().fa_bwd_f32_qk(*ptrs, B, H, Nq, Nk, d, *tail)
        elif Nq == Nk:
            name = "fa_bwd"
            st = lib().fa_bwd(*ptrs, B, H, Nq, d, *tail)
        else:
            name = "fa_bwd_qk"
            st = lib().fa_bwd_qk(*ptrs, B, H, Nq, Nk, d, *tail)
    _check(name, st)
    return dQ, dK, dV


def bwd_noalloc(Q: torch.Tensor, K: torch.Tensor, V: torch.Tensor, O: torch.Tensor,
                dO: torch.Tensor, LSE: torch.Tensor, scale: Optional[float] = None,
                causal: bool = False, dQ: Optional[torch.Tensor] = None,
                dK: Optional[torch.Tensor] = None, dV: Optional[torch.Tensor] = None,
                stream: Optional[torch.cuda.Stream] = None):
    """Backward through ``fa_bwd_noalloc``: the library's fixed scratch replaces the
    workspace, for callers that cannot allocate device memory.  Outputs may be passed in
    so that nothing is allocated here either.  Returns (dQ, dK, dV)."""
    B, H, N, d = Q.shape
    for name, t in (("Q", Q), ("K", K), ("V", V), ("O", O), ("dO", dO)):
        _check_bhnd(name, t, (B, H, N, d), torch.bfloat16)
    _check_bhnd("LSE", LSE, (B, H, N), torch.float32)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    dQ = torch.empty_like(Q) if dQ is None else dQ
    dK = torch.empty_like(K) if dK is None else dK
    dV = torch.empty_like(V) if dV is None else dV
    for name, t in (("dQ", dQ), ("dK", dK), ("dV", dV)):
        _check_bhnd(name, t, (B, H, N, d), torch.bfloat16)
    with torch.cuda.device(Q.device):
        st = lib().fa_bwd_noalloc(_ptr(Q), _ptr(K), _ptr(V), _ptr(O), _ptr(dO), _ptr(LSE),
                                  _ptr(dQ), _ptr(dK), _ptr(dV), B, H, N, d, float(scale),
                                  int(bool(causal)), _stream_handle(stream))
    _check("fa_bwd_noalloc", st)
    return dQ, dK, dV


def _layout_dtype(Q: torch.Tensor) -> torch.dtype:
    if Q.dtype not in (torch.bfloat16, torch.float32):
        raise ValueError("Q, K, V must be bfloat16 or float32")
    return Q.dtype


def _check_seqlens(seqlens_q: torch.Tensor, seqlens_k: torch.Tensor, B: int, device) -> None:
    for name, t in (("seqlens_q", seqlens_q), ("seqlens_k", seqlens_k)):
        if not t.is_cuda or t.device != device:
            raise ValueError(f"{name} must be on the inputs' CUDA device")
        if t.dtype != torch.int32 or tuple(t.shape) != (B,) or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous int32 tensor of shape ({B},)")


def fwd_varlen(Q: torch.Tensor, K: torch.Tensor, V: torch.Tensor, seqlens_q: torch.Tensor,
               seqlens_k: torch.Tensor, scale: Optional[float] = None, causal: bool = False,
               O: Optional[torch.Tensor] = None, LSE: Optional[torch.Tensor] = None,
               stream: Optional[torch.cuda.Stream] = None):
    """Forward over a padded batch through ``fa_fwd_varlen`` (bf16) or
    ``fa_fwd_f32_varlen`` (float32): sequence b uses its first seqlens_q[b] query rows of
    Q [B, H, Nq, d] and seqlens_k[b] key rows of K, V [B, H, Nk, d].  Rows of O and LSE
    past a sequence's length are not written (outputs allocated here start as zeros and
    -inf).  Returns (O, LSE)."""
    B, H, Nq, d = Q.shape
    Nk = K.shape[2]
    dtype = _layout_dtype(Q)
    _check_bhnd("Q", Q, (B, H, Nq, d), dtype)
    for name, t in (("K", K), ("V", V)):
        _check_bhnd(name, t, (B, H, Nk, d), dtype)
    _check_seqlens(seqlens_q, seqlens_k, B, Q.device)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if O is None:
        O = torch.zeros_like(Q)
    if LSE is None:
        LSE = torch.full((B, H, Nq), float("-inf"), device=Q.device, dtype=torch.float32)
    _check_bhnd("O", O, (B, H, Nq, d), dtype)
    _check_bhnd("LSE", LSE, (B, H, Nq), torch.float32)
    name = "fa_fwd_varlen" if dtype == torch.bfloat16 else "fa_fwd_f32_varlen"
    with torch.cuda.device(Q.device):
        st = getattr(lib(), name)(_ptr(Q), _ptr(K), _ptr(V), _ptr(O), _ptr(LSE),
                                  _ptr(seqlens_q), _ptr(seqlens_k), B, H, Nq, Nk, d,
                                  float(scale), int(bool(causal)), _stream_handle(stream))
    _check(name, st)
    return O, LSE


def bwd_varlen(Q: torch.Tensor, K: torch.Tensor, V: torch.Tensor, O: torch.Tensor,
               dO: torch.Tensor, LSE: torch.Tensor, seqlens_q: torch.Tensor,
               seqlens_k: torch.Tensor, scale: Optional[float] = None, causal: bool = False,
               dQ: Optional[torch.Tensor] = None, dK: Optional[torch.Tensor] = None,
               dV: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
               stream: Optional[torch.cuda.Stream] = None):
    """Backward over a padded batch through ``fa_bwd_varlen`` (bf16) or
    ``fa_bwd_f32_varlen`` (float32), the gradient of ``fwd_varlen`` with the same lengths.
    Rows past a sequence's lengths are not written (gradients allocated here start as
    zeros).  Returns (dQ, dK, dV)."""
    B, H, Nq, d = Q.shape
    Nk = K.shape[2]
    dtype = _layout_dtype(Q)
    for name, t in (("Q", Q), ("O", O), ("dO", dO)):
        _check_bhnd(name, t, (B, H, Nq, d), dtype)
    for name, t in (("K", K), ("V", V)):
        _check_bhnd(name, t, (B, H, Nk, d), dtype)
    _check_bhnd("LSE", LSE, (B, H, Nq), torch.float32)
    _check_seqlens(seqlens_q, seqlens_k, B, Q.device)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    dQ = torch.zeros_like(Q) if dQ is None else dQ
    dK = torch.zeros_like(K) if dK is None else dK
    dV = torch.zeros_like(V) if dV is None else dV
    _check_bhnd("dQ", dQ, (B, H, Nq, d), dtype)
    for name, t in (("dK", dK), ("dV", dV)):
        _check_bhnd(name, t, (B, H, Nk, d), dtype)
    need = workspace_bytes(B, H, Nq, d)
    if workspace is None:
        workspace = torch.empty(max(need, 1), device=Q.device, dtype=torch.uint8)
    ws_bytes = workspace.numel() * workspace.element_size()
    name = "fa_bwd_varlen" if dtype == torch.bfloat16 else "fa_bwd_f32_varlen"
    with torch.cuda.device(Q.device):
        st = getattr(lib(), name)(_ptr(Q), _ptr(K), _ptr(V), _ptr(O), _ptr(dO), _ptr(LSE),
                                  _ptr(dQ), _ptr(dK), _ptr(dV), _ptr(seqlens_q),
                                  _ptr(seqlens_k), B, H, Nq, Nk, d, float(scale),
                                  int(bool(causal)), _ptr(workspace), ws_bytes,
                                  _stream_handle(stream))
    _check(name, st)
    return dQ, dK, dV


def _check_packed(name: str, t: torch.Tensor, tokens: int, H: int, d: int,
                  dtype: torch.dtype = torch.bfloat16) -> None:
    _check_bhnd(name, t, (tokens, H, d), dtype)


def _check_cu(cu_q: torch.Tensor, cu_k: torch.Tensor, device) -> int:
    for name, t in (("cu_seqlens_q", cu_q), ("cu_seqlens_k", cu_k)):
        if not t.is_cuda or t.device != device or t.dtype != torch.int32 or t.dim() != 1 \
                or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous int32 CUDA vector on the inputs' device")
    if cu_q.numel() != cu_k.numel() or cu_q.numel() < 1:
        raise ValueError("cu_seqlens_q and cu_seqlens_k must both have B+1 entries")
    return cu_q.numel() - 1


def fwd_packed(Q: torch.Tensor, K: torch.Tensor, V: torch.Tensor, cu_seqlens_q: torch.Tensor,
               cu_seqlens_k: torch.Tensor, max_seqlen_q: int, max_seqlen_k: int,
               scale: Optional[float] = None, causal: bool = False,
               O: Optional[torch.Tensor] = None, LSE: Optional[torch.Tensor] = None,
               stream: Optional[torch.cuda.Stream] = None):
    """Forward over a packed batch through ``fa_fwd_packed`` (bf16) or
    ``fa_fwd_f32_packed`` (float32): Q [total_q, H, d], K and V [total_k, H, d], sequences
    delimited by the int32 start arrays (B+1 entries).
    Returns (O [total_q, H, d], LSE [H, total_q])."""
    total_q, H, d = Q.shape
    total_k = K.shape[0]
    dtype = _layout_dtype(Q)
    _check_packed("Q", Q, total_q, H, d, dtype)
    for name, t in (("K", K), ("V", V)):
        _check_packed(name, t, total_k, H, d, dtype)
    B = _check_cu(cu_seqlens_q, cu_seqlens_k, Q.device)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    O = torch.zeros_like(Q) if O is None else O
    LSE = torch.full((H, total_q), float("-inf"), device=Q.device) if LSE is None else LSE
    _check_packed("O", O, total_q, H, d, dtype)
    _check_bhnd("LSE", LSE, (H, total_q), torch.float32)
    name = "fa_fwd_packed" if dtype == torch.bfloat16 else "fa_fwd_f32_packed"
    with torch.cuda.device(Q.device):
        st = getattr(lib(), name)(_ptr(Q), _ptr(K), _ptr(V), _ptr(O), _ptr(LSE),
                                  _ptr(cu_seqlens_q), _ptr(cu_seqlens_k), B, H,
                                  int(max_seqlen_q), int(max_seqlen_k), total_q, total_k, d,
                                  float(scale), int(bool(causal)), _stream_handle(stream))
    _check(name, st)
    return O, LSE


def bwd_packed(Q: torch.Tensor, K: torch.Tensor, V: torch.Tensor, O: torch.Tensor,
               dO: torch.Tensor, LSE: torch.Tensor, cu_seqlens_q: torch.Tensor,
               cu_seqlens_k: torch.Tensor, max_seqlen_q: int, max_seqlen_k: int,
               scale: Optional[float] = None, causal: bool = False,
               dQ: Optional[torch.Tensor] = None, dK: Optional[torch.Tensor] = None,
               dV: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
               stream: Optional[torch.cuda.Stream] = None):
    """Backward over a packed batch through ``fa_bwd_packed`` (bf16) or
    ``fa_bwd_f32_packed`` (float32), the gradient of ``fwd_packed`` with the same start
    arrays.  Returns (dQ, dK, dV)."""
    total_q, H, d = Q.shape
    total_k = K.shape[0]
    dtype = _layout_dtype(Q)
    for name, t in (("Q", Q), ("O", O), ("dO", dO)):
        _check_packed(name, t, total_q, H, d, dtype)
    for name, t in (("K", K), ("V", V)):
        _check_packed(name, t, total_k, H, d, dtype)
    _check_bhnd("LSE", LSE, (H, total_q), torch.float32)
    B = _check_cu(cu_seqlens_q, cu_seqlens_k, Q.device)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    dQ = torch.zeros_like(Q) if dQ is None else dQ
    dK = torch.zeros_like(K) if dK is None else dK
    dV = torch.zeros_like(V) if dV is None else dV
    _check_packed("dQ", dQ, total_q, H, d, dtype)
    for name, t in (("dK", dK), ("dV", dV)):
        _check_packed(name, t, total_k, H, d, dtype)
    need = workspace_bytes(B, H, int(max_seqlen_q), d)
    if workspace is None:
        workspace = torch.empty(max(need, 1), device=Q.device, dtype=torch.uint8)
    ws_bytes = workspace.numel() * workspace.element_size()
    name = "fa_bwd_packed" if dtype == torch.bfloat16 else "fa_bwd_f32_packed"
    with torch.cuda.device(Q.device):
        st = getattr(lib(), name)(_ptr(Q), _ptr(K), _ptr(V), _ptr(O), _ptr(dO), _ptr(LSE),
                                  _ptr(dQ), _ptr(dK), _ptr(dV), _ptr(cu_seqlens_q),
                                  _ptr(cu_seqlens_k), B, H, int(max_seqlen_q),
                                  int(max_seqlen_k), total_q, total_k, d, float(scale),
                                  int(bool(causal)), _ptr(workspace), ws_bytes,
                                  _stream_handle(stream))
    _check(name, st)
    return dQ, dK, dV


def merge(O_acc: torch.Tensor, LSE_acc: torch.Tensor, O_part: torch.Tensor,
          LSE_part: torch.Tensor, O_out: Optional[torch.Tensor] = None,
          stream: Optional[torch.cuda.Stream] = None):
    """Merge a partial result over a block of keys into a float32 accumulator in place
    through ``fa_merge``.  O_acc [B, H, N, d] float32, LSE_acc [B, H, N] float32 (-inf:
    empty), O_part [B, H, N, d] bf16, LSE_part [B, H, N] float32; O_out, if given, gets
    the merged O as bf16.  Returns (O_acc, LSE_acc)."""
    B, H, N, d = O_acc.shape
    _check_bhnd("O_acc", O_acc, (B, H, N, d), torch.float32)
    _check_bhnd("LSE_acc", LSE_acc, (B, H, N), torch.float32)
    _check_bhnd("O_part", O_part, (B, H, N, d), torch.bfloat16)
    _check_bhnd("LSE_part", LSE_part, (B, H, N), torch.float32)
    if O_out is not None:
        _check_bhnd("O_out", O_out, (B, H, N, d), torch.bfloat16)
    with torch.cuda.device(O_acc.device):
        st = lib().fa_merge(_ptr(O_acc), _ptr(LSE_acc), _ptr(O_part), _ptr(LSE_part),
                            _ptr(O_out), B, H, N, d, _stream_handle(stream))
    _check("fa_merge", st)
    return O_acc, LSE_acc


def accumulate(acc: torch.Tensor, part: torch.Tensor, out: Optional[torch.Tensor] = None,
               stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
    """acc += part (float32 += bf16, same shape, contiguous) through ``fa_accumulate``;
    ``out``, if given, receives acc rounded to bf16.  Returns acc."""
    if acc.dtype != torch.float32 or part.dtype != torch.bfloat16:
        raise ValueError("acc must be float32 and part bfloat16")
    if acc.shape != part.shape or (out is not None and out.shape != acc.shape):
        raise ValueError("acc, part and out must have the same shape")
    for name, t in (("acc", acc), ("part", part), ("out", out)):
        if t is not None and (not t.is_cuda or not t.is_contiguous()):
            raise ValueError(f"{name} must be a contiguous CUDA tensor")
    if out is not None and out.dtype != torch.bfloat16:
        raise ValueError("out must be bfloat16")
    with torch.cuda.device(acc.device):
        st = lib().fa_accumulate(_ptr(acc), _ptr(part), _ptr(out), acc.numel(),
                                 _stream_handle(stream))
    _check("fa_accumulate", st)
    return acc


class trace_kernels:
    """Context manager: record the given torch.cuda.Events at kernel boundaries of the
    library calls made inside it (fa_trace_events).  events[0] before the first kernel
    of each call, events[k] after its k-th kernel."""

    def __init__(self, events):
        for e in events:
            e.record()  # make sure the underlying cudaEvent_t exists
        self._arr = (_vp * len(events))(*[e.cuda_event for e in events])
        self._n = len(events)

    def __enter__(self):
        _check("fa_trace_events", lib().fa_trace_events(self._arr, self._n))
        return self

    def __exit__(self, *exc):
        lib().fa_trace_events(None, 0)


def check_device_error(stream: Optional[torch.cuda.Stream] = None) -> None:
    """Synchronise the stream and raise FAError if a kernel reported a wait timeout."""
    _check("fa_check_device_error", lib().fa_check_device_error(_stream_handle(stream)))
