"""Thin Python binding of libkda (ctypes).  Argument marshalling only: every step of
the scan and of the convolution runs in the CUDA library; PyTorch supplies device
memory and the current stream.

There is no fallback.  If ``libkda.so`` has not been built, or a call is made with
tensors that are not on a CUDA device, these functions raise.
"""
from __future__ import annotations

import ctypes
import os
import threading
from typing import Optional, Sequence, Tuple

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libkda.so")

KDA_F32, KDA_BF16 = 0, 1
MSC_TEXT, MSC_IMAGE, MSC_VIDEO = 0, 1, 2
STATUS = {0: "KDA_OK", 1: "KDA_ERR_INVALID_ARG", 2: "KDA_ERR_UNSUPPORTED", 3: "KDA_ERR_CUDA",
          4: "KDA_ERR_TIMEOUT", 5: "KDA_ERR_WORKSPACE"}

# Every symbol include/kda.h declares.
EXPORTED = ("kda_status_string", "kda_last_device_error", "kda_forward_workspace_size",
            "kda_forward", "mshortconv_forward", "kda_mshortconv_workspace_size",
            "kda_mshortconv_forward", "kda_kernel_launches", "kda_profile_enable",
            "kda_profile_collect", "kda_forward_noalloc", "kda_debug_drop_handoff", "kda_fma_probe",
            "kda_forward_gated", "kda_forward_varlen", "kda_forward_varlen_workspace_size",
            "kda_sp_workspace_size", "kda_sp_transition", "kda_sp_prefix", "kda_sp_output",
            "kda_backward", "kda_backward_workspace_size", "mshortconv_backward",
            "kda_mshortconv_backward", "kda_mshortconv_backward_workspace_size", "kda_forward_plan")


class KdaError(RuntimeError):
    def __init__(self, fn: str, code: int):
        super().__init__(f"{fn} failed: {STATUS.get(code, code)}")
        self.code = code


class MscSegment(ctypes.Structure):
    _fields_ = [("modality", ctypes.c_int32), ("reserved", ctypes.c_int32),
                ("start", ctypes.c_int64), ("F", ctypes.c_int32), ("Hgt", ctypes.c_int32),
                ("Wid", ctypes.c_int32), ("weight_set", ctypes.c_int32)]


_lib = None
_lock = threading.Lock()


def load_library(path: str = LIB_PATH):
    """Loads libkda.so and declares its signatures (raises if it is missing)."""
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        if not os.path.exists(path):
            raise ImportError(f"{path} is missing: build it with "
                              "`python -m linear_attention_sequence_mshortconv_b200.build`")
        lib = ctypes.CDLL(path)
        P, I, Z = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
        lib.kda_status_string.restype = ctypes.c_char_p
        lib.kda_status_string.argtypes = [I]
        lib.kda_last_device_error.restype = I
        lib.kda_last_device_error.argtypes = []
        lib.kda_forward_workspace_size.restype = Z
        lib.kda_forward_workspace_size.argtypes = [I, I, I, I, I, I, I, I]
        lib.kda_forward.restype = I
        lib.kda_forward.argtypes = [P, P, P, P, P, P, P, P, I, I, I, I, I, I, I, I, P, Z, P]
        lib.mshortconv_forward.restype = I
        lib.mshortconv_forward.argtypes = [P, P, I, I, I, I, P, I, I, P, I, P, I, P, I, P]
        lib.kda_mshortconv_workspace_size.restype = Z
        lib.kda_mshortconv_workspace_size.argtypes = [I, I, I, I, I, I, I]
        lib.kda_mshortconv_forward.restype = I
        lib.kda_mshortconv_forward.argtypes = [P, P, P, P, I, I, P, P, P, P, P, P, P, P,
                                               I, I, I, I, I, I, I, P, Z, P]
        lib.kda_forward_noalloc.restype = I
        lib.kda_forward_noalloc.argtypes = [P, P, P, P, P, P, P, P, I, I, I, I, I, I, I, I, P]
        lib.kda_kernel_launches.restype = ctypes.c_uint64
        lib.kda_kernel_launches.argtypes = []
        lib.kda_profile_enable.restype = None
        lib.kda_profile_enable.argtypes = [I]
        lib.kda_debug_drop_handoff.restype = None
        lib.kda_debug_drop_handoff.argtypes = [I]
        lib.kda_forward_gated.restype = I
        lib.kda_forward_gated.argtypes = [P, P, P, P, P, P, P, P, ctypes.c_float, P, P, I, I, I, I, I, I, I,
                                          I, P, Z, P]
        lib.kda_forward_varlen.restype = I
        lib.kda_forward_varlen.argtypes = [P, P, P, P, P, P, P, P, P, I, I, I, I, I, I, I, P, Z, P]
        lib.kda_forward_varlen_workspace_size.restype = Z
        lib.kda_forward_varlen_workspace_size.argtypes = [P, I, I, I, I, I, I, I]
        lib.kda_sp_workspace_size.restype = Z
        lib.kda_sp_workspace_size.argtypes = [I, I, I, I, I, I]
        lib.kda_sp_transition.restype = I
        lib.kda_sp_transition.argtypes = [P, P, P, P, P, P, I, I, I, I, I, I, P, Z, P]
        lib.kda_sp_prefix.restype = I
        lib.kda_sp_prefix.argtypes = [P, I, I, P, P, I, I, I, P]
        lib.kda_sp_output.restype = I
        lib.kda_sp_output.argtypes = [P, P, P, P, P, P, P, P, I, I, I, I, I, I, I, P, Z, P]
        lib.kda_backward_workspace_size.restype = Z
        lib.kda_backward_workspace_size.argtypes = [I, I, I, I, I]
        lib.kda_backward.restype = I
        lib.kda_backward.argtypes = [P, P, P, P, P, P, P, P, P, P, P, P, P, P, I, I, I, I, I, I, I, P, Z, P]
        lib.mshortconv_backward.restype = I
        lib.mshortconv_backward.argtypes = [P, P, P, I, I, I, I, P, I, I, P, I, P, I, P, I, P, P, P, P]
        lib.kda_mshortconv_backward_workspace_size.restype = Z
        lib.kda_mshortconv_backward_workspace_size.argtypes = [I, I, I, I, I]
        lib.kda_mshortconv_backward.restype = I
        lib.kda_mshortconv_backward.argtypes = [P, P, P, P, I, I, P, P, P, P, P, P, P, I, P, P, P, P, P, P, P,
                                                P, P, P, I, I, I, I, I, P, Z, P]
        lib.kda_forward_plan.restype = I
        lib.kda_forward_plan.argtypes = [I, I, I, I, I, I, I, I, ctypes.POINTER(ctypes.c_int),
                                         ctypes.POINTER(ctypes.c_int)]
        lib.kda_fma_probe.restype = I
        lib.kda_fma_probe.argtypes = [ctypes.POINTER(ctypes.c_double)]
        lib.kda_profile_collect.restype = I
        lib.kda_profile_collect.argtypes = [ctypes.c_char_p, ctypes.POINTER(ctypes.c_double),
                                            ctypes.POINTER(ctypes.c_int)]
        _lib = lib
        return lib


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return KDA_F32
    if t.dtype == torch.bfloat16:
        return KDA_BF16
    raise TypeError(f"unsupported dtype {t.dtype} (bf16 or fp32)")


def _dev(t: Optional[torch.Tensor], name: str, dtype=None):
    if t is None:
        return None
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _check(fn: str, rc: int):
    if rc != 0:
        raise KdaError(fn, rc)


def _code(dtype) -> int:
    return KDA_F32 if dtype == torch.float32 else KDA_BF16


def workspace_size(B, T, H, Dk, Dv, dtype=torch.bfloat16, chunk=0, o_dtype=None) -> int:
    lib = load_library()
    return int(lib.kda_forward_workspace_size(B, T, H, Dk, Dv, _code(dtype),
                                              _code(o_dtype or dtype), chunk))


def forward(q, k, v, g, beta, S0=None, *, chunk: int = 0, o=None, S_T=None,
            want_state: bool = True, workspace=None, stream=None, o_dtype=None):
    """KDA forward scan (Eq. 14) with readout o_t = S_t^T q_t.

    q, k, g: [B,T,H,Dk]; v: [B,T,H,Dv]; beta: [B,T,H] -- all bf16 or all fp32 CUDA
    tensors; S0: [B,H,Dk,Dv] fp32 or None.  o_dtype: torch.float32 or torch.bfloat16
    (default: the input dtype).  chunk: 0 (the dtype's default), 16, 32, 64 or 128; only
    64 runs on the tensor cores.  Returns (o, S_T or None)."""
    lib = load_library()
    B, T, H, Dk = q.shape
    Dv = v.shape[-1]
    dt = _dtype_code(q)
    for name, t, shape in (("k", k, (B, T, H, Dk)), ("g", g, (B, T, H, Dk)),
                           ("v", v, (B, T, H, Dv)), ("beta", beta, (B, T, H))):
        if tuple(t.shape) != shape:
            raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {shape}")
        if t.dtype != q.dtype:
            raise TypeError(f"{name} dtype {t.dtype} differs from q's {q.dtype}")
    o_dtype = o_dtype or (o.dtype if o is not None else q.dtype)
    if o is None:
        o = torch.empty((B, T, H, Dv), dtype=o_dtype, device=q.device)
    if S_T is None and want_state:
        S_T = torch.empty((B, H, Dk, Dv), dtype=torch.float32, device=q.device)
    if S0 is not None and tuple(S0.shape) != (B, H, Dk, Dv):
        raise ValueError("S0 shape")
    ws_ptr, ws_bytes = None, 0
    if workspace is not None:
        ws_ptr, ws_bytes = _dev(workspace, "workspace"), workspace.numel() * workspace.element_size()
    rc = lib.kda_forward(_dev(q, "q"), _dev(k, "k"), _dev(v, "v"), _dev(g, "g"),
                         _dev(beta, "beta"), _dev(S0, "S0", torch.float32), _dev(o, "o", o_dtype),
                         _dev(S_T, "S_T", torch.float32), B, T, H, Dk, Dv, dt, _code(o_dtype),
                         chunk, ws_ptr, ws_bytes, _stream(stream))
    _check("kda_forward", rc)
    return o, S_T


def forward_gated(q, k, v, g, beta, gate, gamma=None, eps: float = 1e-6, S0=None, *, chunk: int = 0,
                  o=None, S_T=None, want_state: bool = True, workspace=None, stream=None, o_dtype=None):
    """kda_forward_gated: the scan of forward() with the output side of Eq. 15 applied,
    y = Sigmoid(gate) * gamma_h * RMSNorm(S_t^T q_t) per (token, head).  gate: [B,T,H,Dv]
    in q's dtype; gamma: [H,Dv] fp32 or None.  Returns (y, S_T or None)."""
    lib = load_library()
    B, T, H, Dk = q.shape
    Dv = v.shape[-1]
    dt = _dtype_code(q)
    for name, t, shape in (("k", k, (B, T, H, Dk)), ("g", g, (B, T, H, Dk)),
                           ("v", v, (B, T, H, Dv)), ("beta", beta, (B, T, H)), ("gate", gate, (B, T, H, Dv))):
        if tuple(t.shape) != shape:
            raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {shape}")
        if t.dtype != q.dtype:
            raise TypeError(f"{name} dtype {t.dtype} differs from q's {q.dtype}")
    if gamma is not None and tuple(gamma.shape) != (H, Dv):
        raise ValueError("gamma shape")
    o_dtype = o_dtype or (o.dtype if o is not None else q.dtype)
    if o is None:
        o = torch.empty((B, T, H, Dv), dtype=o_dtype, device=q.device)
    if S_T is None and want_state:
        S_T = torch.empty((B, H, Dk, Dv), dtype=torch.float32, device=q.device)
    if S0 is not None and tuple(S0.shape) != (B, H, Dk, Dv):
        raise ValueError("S0 shape")
    ws_ptr, ws_bytes = None, 0
    if workspace is not None:
        ws_ptr, ws_bytes = _dev(workspace, "workspace"), workspace.numel() * workspace.element_size()
    rc = lib.kda_forward_gated(_dev(q, "q"), _dev(k, "k"), _dev(v, "v"), _dev(g, "g"), _dev(beta, "beta"),
                               _dev(S0, "S0", torch.float32), _dev(gate, "gate"),
                               _dev(gamma, "gamma", torch.float32), float(eps), _dev(o, "o", o_dtype),
                               _dev(S_T, "S_T", torch.float32), B, T, H, Dk, Dv, dt, _code(o_dtype),
                               chunk, ws_ptr, ws_bytes, _stream(stream))
    _check("kda_forward_gated", rc)
    return o, S_T


def _cu_array(cu_seqlens):
    arr = (ctypes.c_int32 * len(cu_seqlens))(*[int(x) for x in cu_seqlens])
    return arr, len(cu_seqlens) - 1


def varlen_workspace_size(cu_seqlens, H, Dk, Dv, dtype=torch.bfloat16, chunk: int = 0, o_dtype=None) -> int:
    arr, n = _cu_array(cu_seqlens)
    return int(load_library().kda_forward_varlen_workspace_size(
        ctypes.cast(arr, ctypes.c_void_p), n, H, Dk, Dv, _code(dtype), _code(o_dtype or dtype), chunk))


def forward_varlen(q, k, v, g, beta, cu_seqlens, S0=None, *, chunk: int = 0, o=None, S_T=None,
                   want_state: bool = True, workspace=None, stream=None, o_dtype=None):
    """kda_forward_varlen: packed samples on one token axis, the state reset at every
    sample start.  q, k, g: [T_total,H,Dk]; v: [T_total,H,Dv]; beta: [T_total,H];
    cu_seqlens: host sequence of n+1 offsets (0, ..., T_total); S0: [n,H,Dk,Dv] fp32 or
    None.  Returns (o [T_total,H,Dv], S_T [n,H,Dk,Dv] or None)."""
    lib = load_library()
    T, H, Dk = q.shape
    Dv = v.shape[-1]
    arr, n = _cu_array(cu_seqlens)
    if n < 0 or int(arr[n]) != T:
        raise ValueError("cu_seqlens must end at the packed length")
    dt = _dtype_code(q)
    for name, t, shape in (("k", k, (T, H, Dk)), ("g", g, (T, H, Dk)), ("v", v, (T, H, Dv)), ("beta", beta, (T, H))):
        if tuple(t.shape) != shape:
            raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {shape}")
        if t.dtype != q.dtype:
            raise TypeError(f"{name} dtype {t.dtype} differs from q's {q.dtype}")
    o_dtype = o_dtype or (o.dtype if o is not None else q.dtype)
    if o is None:
        o = torch.empty((T, H, Dv), dtype=o_dtype, device=q.device)
    if S_T is None and want_state:
        S_T = torch.empty((n, H, Dk, Dv), dtype=torch.float32, device=q.device)
    if S0 is not None and tuple(S0.shape) != (n, H, Dk, Dv):
        raise ValueError("S0 shape")
    ws_ptr, ws_bytes = None, 0
    if workspace is not None:
        ws_ptr, ws_bytes = _dev(workspace, "workspace"), workspace.numel() * workspace.element_size()
    rc = lib.kda_forward_varlen(_dev(q, "q"), _dev(k, "k"), _dev(v, "v"), _dev(g, "g"), _dev(beta, "beta"),
                                _dev(S0, "S0", torch.float32), _dev(o, "o", o_dtype), _dev(S_T, "S_T", torch.float32),
                                ctypes.cast(arr, ctypes.c_void_p), n, H, Dk, Dv, dt, _code(o_dtype), chunk,
                                ws_ptr, ws_bytes, _stream(stream))
    _check("kda_forward_varlen", rc)
    return o, S_T


def _shard_inputs(q, k, v, g, beta):
    B, T, H, D = q.shape
    for name, t, shape in (("k", k, (B, T, H, D)), ("g", g, (B, T, H, D)), ("v", v, (B, T, H, D)),
                           ("beta", beta, (B, T, H))):
        if tuple(t.shape) != shape:
            raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {shape}")
        if t.dtype != q.dtype:
            raise TypeError(f"{name} dtype {t.dtype} differs from q's {q.dtype}")
    return B, T, H, D, _dtype_code(q)


def _ws(workspace):
    if workspace is None:
        return None, 0
    return _dev(workspace, "workspace"), workspace.numel() * workspace.element_size()


def sp_workspace_size(B, T, H, D, dtype=torch.bfloat16, chunk: int = 0) -> int:
    """Bytes of the workspace one shard's kda_sp_transition / kda_sp_output share."""
    return int(load_library().kda_sp_workspace_size(B, T, H, D, _code(dtype), chunk))


def sp_workspace(q, chunk: int = 0):
    """A workspace tensor for the shard q belongs to (None if the shard needs none)."""
    B, T, H, D = q.shape
    n = sp_workspace_size(B, T, H, D, q.dtype, chunk)
    return torch.empty(n, dtype=torch.uint8, device=q.device) if n else None


def sp_transition(q, k, v, g, beta, workspace, *, chunk: int = 0, MN=None, stream=None):
    """kda_sp_transition: the shard's affine map S_out = M S_in + N as MN [B,H,2,D,D]
    fp32 (block 0 = N, block 1 = M).  `workspace` (see sp_workspace) must be passed
    unchanged to sp_output for the same shard."""
    lib = load_library()
    B, T, H, D, dt = _shard_inputs(q, k, v, g, beta)
    if MN is None:
        MN = torch.empty((B, H, 2, D, D), dtype=torch.float32, device=q.device)
    ws_ptr, ws_bytes = _ws(workspace)
    rc = lib.kda_sp_transition(_dev(q, "q"), _dev(k, "k"), _dev(v, "v"), _dev(g, "g"), _dev(beta, "beta"),
                               _dev(MN, "MN", torch.float32), B, T, H, D, dt, chunk, ws_ptr, ws_bytes,
                               _stream(stream))
    _check("kda_sp_transition", rc)
    return MN


def sp_prefix(MN_all, r: int, S0=None, *, S_in=None, stream=None):
    """kda_sp_prefix: entry state [B,H,D,D] of shard r from the ranks' maps
    MN_all [R,B,H,2,D,D] (rank order) and the rows' S0 (None = zeros)."""
    lib = load_library()
    R, B, H, two, D, D2 = MN_all.shape
    if two != 2 or D2 != D:
        raise ValueError("MN_all must be [R,B,H,2,D,D]")
    if S0 is not None and tuple(S0.shape) != (B, H, D, D):
        raise ValueError("S0 shape")
    if S_in is None:
        S_in = torch.empty((B, H, D, D), dtype=torch.float32, device=MN_all.device)
    rc = lib.kda_sp_prefix(_dev(MN_all, "MN_all", torch.float32), R, int(r), _dev(S0, "S0", torch.float32),
                           _dev(S_in, "S_in", torch.float32), B, H, D, _stream(stream))
    _check("kda_sp_prefix", rc)
    return S_in


def sp_output(q, k, v, g, beta, S_in, workspace, *, chunk: int = 0, o=None, S_T=None,
              want_state: bool = True, o_dtype=None, stream=None):
    """kda_sp_output: the shard's scan from S_in, reusing what sp_transition left in
    `workspace`.  Returns (o [B,T,H,D], S_T or None)."""
    lib = load_library()
    B, T, H, D, dt = _shard_inputs(q, k, v, g, beta)
    o_dtype = o_dtype or (o.dtype if o is not None else q.dtype)
    if o is None:
        o = torch.empty((B, T, H, D), dtype=o_dtype, device=q.device)
    if S_T is None and want_state:
        S_T = torch.empty((B, H, D, D), dtype=torch.float32, device=q.device)
    if S_in is not None and tuple(S_in.shape) != (B, H, D, D):
        raise ValueError("S_in shape")
    ws_ptr, ws_bytes = _ws(workspace)
    rc = lib.kda_sp_output(_dev(q, "q"), _dev(k, "k"), _dev(v, "v"), _dev(g, "g"), _dev(beta, "beta"),
                           _dev(S_in, "S_in", torch.float32), _dev(o, "o", o_dtype), _dev(S_T, "S_T", torch.float32),
                           B, T, H, D, dt, _code(o_dtype), chunk, ws_ptr, ws_bytes, _stream(stream))
    _check("kda_sp_output", rc)
    return o, S_T


def backward_workspace_size(B, T, H, Dk, Dv) -> int:
    return int(load_library().kda_backward_workspace_size(B, T, H, Dk, Dv))


def backward(q, k, v, g, beta, do, S0=None, dS_T=None, *, want_dS0: bool = True, workspace=None,
             stream=None, out=None):
    """kda_backward: gradients (fp32) of L with dL/do = do and dL/dS_T = dS_T through the
    scan of forward().  q, k, v, g, beta, S0 as passed to forward(); do: [B,T,H,Dv] bf16
    or fp32.  Returns (dq, dk, dv, dg, dbeta, dS0 or None); `out` may hold preallocated
    fp32 tensors in that order."""
    lib = load_library()
    B, T, H, Dk = q.shape
    Dv = v.shape[-1]
    dt = _dtype_code(q)
    for name, t, shape in (("k", k, (B, T, H, Dk)), ("g", g, (B, T, H, Dk)),
                           ("v", v, (B, T, H, Dv)), ("beta", beta, (B, T, H))):
        if tuple(t.shape) != shape:
            raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {shape}")
        if t.dtype != q.dtype:
            raise TypeError(f"{name} dtype {t.dtype} differs from q's {q.dtype}")
    if tuple(do.shape) != (B, T, H, Dv):
        raise ValueError("do shape")
    for name, t in (("S0", S0), ("dS_T", dS_T)):
        if t is not None and tuple(t.shape) != (B, H, Dk, Dv):
            raise ValueError(f"{name} shape")
    f = dict(dtype=torch.float32, device=q.device)
    if out is None:
        out = (torch.empty((B, T, H, Dk), **f), torch.empty((B, T, H, Dk), **f),
               torch.empty((B, T, H, Dv), **f), torch.empty((B, T, H, Dk), **f),
               torch.empty((B, T, H), **f), torch.empty((B, H, Dk, Dv), **f) if want_dS0 else None)
    dq, dk, dv, dg, dbeta, dS0 = out
    ws_ptr, ws_bytes = _ws(workspace)
    rc = lib.kda_backward(_dev(q, "q"), _dev(k, "k"), _dev(v, "v"), _dev(g, "g"), _dev(beta, "beta"),
                          _dev(S0, "S0", torch.float32), _dev(do, "do"), _dev(dS_T, "dS_T", torch.float32),
                          _dev(dq, "dq", torch.float32), _dev(dk, "dk", torch.float32),
                          _dev(dv, "dv", torch.float32), _dev(dg, "dg", torch.float32),
                          _dev(dbeta, "dbeta", torch.float32), _dev(dS0, "dS0", torch.float32),
                          B, T, H, Dk, Dv, dt, _dtype_code(do), ws_ptr, ws_bytes, _stream(stream))
    _check("kda_backward", rc)
    return dq, dk, dv, dg, dbeta, dS0


NOALLOC_SCRATCH_BYTES = 32 << 20


def forward_noalloc(q, k, v, g, beta, S0=None, *, chunk: int = 0, o=None, S_T=None,
                    stream=None, o_dtype=None):
    """kda_forward_noalloc: the same scan as forward() with its scratch taken from the
    array compiled into the library (no device allocation inside the call).  The
    caller supplies every tensor, outputs included (created here only for convenience
    when not given)."""
    lib = load_library()
    B, T, H, Dk = q.shape
    Dv = v.shape[-1]
    o_dtype = o_dtype or (o.dtype if o is not None else q.dtype)
    if o is None:
        o = torch.empty((B, T, H, Dv), dtype=o_dtype, device=q.device)
    if S_T is None:
        S_T = torch.empty((B, H, Dk, Dv), dtype=torch.float32, device=q.device)
    rc = lib.kda_forward_noalloc(_dev(q, "q"), _dev(k, "k", q.dtype), _dev(v, "v", q.dtype),
                                 _dev(g, "g", q.dtype), _dev(beta, "beta", q.dtype),
                                 _dev(S0, "S0", torch.float32), _dev(o, "o", o_dtype),
                                 _dev(S_T, "S_T", torch.float32), B, T, H, Dk, Dv,
                                 _dtype_code(q), _code(o_dtype), chunk, _stream(stream))
    _check("kda_forward_noalloc", rc)
    return o, S_T


def make_segments(segments: Sequence[Sequence[int]]):
    """(modality, start, F, Hgt, Wid, weight_set) tuples -> ctypes array (host)."""
    rows = list(segments)
    arr = (MscSegment * max(1, len(rows)))()
    for i, (m, s, F, Hh, W, ws) in enumerate(rows):
        arr[i] = MscSegment(int(m), 0, int(s), int(F), int(Hh), int(W), int(ws))
    return arr, len(rows)


def mshortconv(x, segments, Kt, w_text=None, w_image=None, w_video=None, *, y=None,
               stream=None):
    """Depthwise modality-aware short convolution of x [B,T,C] (section 3.4)."""
    lib = load_library()
    B, T, C = x.shape
    dt = _dtype_code(x)
    if y is None:
        y = torch.empty_like(x)
    segs, n = make_segments(segments)

    def wsets(w):
        return (0 if w is None else int(w.shape[0]))

    rc = lib.mshortconv_forward(_dev(x, "x"), _dev(y, "y", x.dtype), B, T, C, dt,
                                ctypes.cast(segs, ctypes.c_void_p), n, int(Kt),
                                _dev(w_text, "w_text", torch.float32), wsets(w_text),
                                _dev(w_image, "w_image", torch.float32), wsets(w_image),
                                _dev(w_video, "w_video", torch.float32), wsets(w_video),
                                _stream(stream))
    _check("mshortconv_forward", rc)
    return y


def mshortconv_backward(x, dy, segments, Kt, w_text=None, w_image=None, w_video=None, *,
                        want_dw: bool = True, stream=None):
    """mshortconv_backward: (dx [B,T,C] fp32, dw_text, dw_image, dw_video) for dL/dy = dy
    through mshortconv(x, ...); each dw has its weight's shape (None where the weight is
    None or want_dw is False)."""
    lib = load_library()
    B, T, C = x.shape
    if tuple(dy.shape) != (B, T, C) or dy.dtype != x.dtype:
        raise ValueError("dy must match x in shape and dtype")
    dt = _dtype_code(x)
    dx = torch.empty((B, T, C), dtype=torch.float32, device=x.device)
    segs, n = make_segments(segments)
    dws = [None if (w is None or not want_dw) else torch.empty_like(w, dtype=torch.float32)
           for w in (w_text, w_image, w_video)]

    def wsets(w):
        return (0 if w is None else int(w.shape[0]))

    rc = lib.mshortconv_backward(_dev(x, "x"), _dev(dy, "dy"), _dev(dx, "dx", torch.float32), B, T, C, dt,
                                 ctypes.cast(segs, ctypes.c_void_p), n, int(Kt),
                                 _dev(w_text, "w_text", torch.float32), wsets(w_text),
                                 _dev(w_image, "w_image", torch.float32), wsets(w_image),
                                 _dev(w_video, "w_video", torch.float32), wsets(w_video),
                                 *[_dev(d, "dw", torch.float32) for d in dws], _stream(stream))
    _check("mshortconv_backward", rc)
    return (dx, *dws)


def mshortconv_workspace_size(B, T, H, D, dtype=torch.bfloat16, chunk=0, o_dtype=None) -> int:
    lib = load_library()
    return int(lib.kda_mshortconv_workspace_size(B, T, H, D, _code(dtype),
                                                 _code(o_dtype or dtype), chunk))


def mshortconv_kda_forward(xq, xk, xv, segments, Kt, wq, wk, wv, g, beta, S0=None, *,
                           chunk: int = 0, o=None, S_T=None, want_state: bool = True,
                           workspace=None, stream=None, o_dtype=None):
    """Fused Eq. 13 -> Eq. 14: conv of x_q, x_k, x_v, per-head L2 norm of q and k,
    KDA scan.  x*: [B,T,H*D]; w* = (w_text [1,C,Kt], w_image [1,C,3,3], w_video [1,C,3,3,3]);
    g: [B,T,H,D]; beta: [B,T,H]."""
    lib = load_library()
    B, T, H, D = g.shape
    dt = _dtype_code(xq)
    o_dtype = o_dtype or (o.dtype if o is not None else xq.dtype)
    if o is None:
        o = torch.empty((B, T, H, D), dtype=o_dtype, device=xq.device)
    if S_T is None and want_state:
        S_T = torch.empty((B, H, D, D), dtype=torch.float32, device=xq.device)
    segs, n = make_segments(segments)
    arrs = []
    for name, w in (("wq", wq), ("wk", wk), ("wv", wv)):
        a = (ctypes.c_void_p * 3)()
        for i in range(3):
            a[i] = _dev(w[i], f"{name}[{i}]", torch.float32) if w[i] is not None else None
        arrs.append(a)
    ws_ptr, ws_bytes = None, 0
    if workspace is not None:
        ws_ptr, ws_bytes = _dev(workspace, "workspace"), workspace.numel() * workspace.element_size()
    rc = lib.kda_mshortconv_forward(_dev(xq, "xq"), _dev(xk, "xk"), _dev(xv, "xv"),
                                    ctypes.cast(segs, ctypes.c_void_p), n, int(Kt),
                                    ctypes.cast(arrs[0], ctypes.c_void_p),
                                    ctypes.cast(arrs[1], ctypes.c_void_p),
                                    ctypes.cast(arrs[2], ctypes.c_void_p),
                                    _dev(g, "g", xq.dtype), _dev(beta, "beta", xq.dtype),
                                    _dev(S0, "S0", torch.float32), _dev(o, "o", o_dtype),
                                    _dev(S_T, "S_T", torch.float32), B, T, H, D, dt,
                                    _code(o_dtype), chunk,
                                    ws_ptr, ws_bytes, _stream(stream))
    _check("kda_mshortconv_forward", rc)
    return o, S_T


def mshortconv_kda_backward_workspace_size(B, T, H, D, dtype=torch.bfloat16) -> int:
    return int(load_library().kda_mshortconv_backward_workspace_size(B, T, H, D, _code(dtype)))


def mshortconv_kda_backward(xq, xk, xv, segments, Kt, wq, wk, wv, g, beta, do, S0=None, dS_T=None, *,
                            want_dS0: bool = True, workspace=None, stream=None):
    """kda_mshortconv_backward: gradients (fp32) through mshortconv_kda_forward for
    dL/do = do and dL/dS_T = dS_T.  Returns a dict with dxq, dxk, dxv ([B,T,H*D]),
    dwq, dwk, dwv (tuples shaped like wq, wk, wv; None where the weight is None), dg,
    dbeta, dS0."""
    lib = load_library()
    B, T, H, D = g.shape
    C = H * D
    dt = _dtype_code(xq)
    f = dict(dtype=torch.float32, device=xq.device)
    out = {"dxq": torch.empty((B, T, C), **f), "dxk": torch.empty((B, T, C), **f),
           "dxv": torch.empty((B, T, C), **f), "dg": torch.empty((B, T, H, D), **f),
           "dbeta": torch.empty((B, T, H), **f),
           "dS0": torch.empty((B, H, D, D), **f) if want_dS0 else None}
    segs, n = make_segments(segments)
    warrs, dwarrs = [], []
    for name, w in (("wq", wq), ("wk", wk), ("wv", wv)):
        a, da = (ctypes.c_void_p * 3)(), (ctypes.c_void_p * 3)()
        dws = []
        for i in range(3):
            a[i] = _dev(w[i], f"{name}[{i}]", torch.float32) if w[i] is not None else None
            dw = torch.empty_like(w[i], dtype=torch.float32) if w[i] is not None else None
            da[i] = _dev(dw, f"d{name}[{i}]", torch.float32) if dw is not None else None
            dws.append(dw)
        warrs.append(a)
        dwarrs.append(da)
        out["d" + name] = tuple(dws)
    ws_ptr, ws_bytes = _ws(workspace)
    cp = lambda a: ctypes.cast(a, ctypes.c_void_p)
    rc = lib.kda_mshortconv_backward(_dev(xq, "xq"), _dev(xk, "xk"), _dev(xv, "xv"), cp(segs), n, int(Kt),
                                     cp(warrs[0]), cp(warrs[1]), cp(warrs[2]), _dev(g, "g", xq.dtype),
                                     _dev(beta, "beta", xq.dtype), _dev(S0, "S0", torch.float32), _dev(do, "do"),
                                     _dtype_code(do), _dev(dS_T, "dS_T", torch.float32),
                                     _dev(out["dxq"], "dxq"), _dev(out["dxk"], "dxk"), _dev(out["dxv"], "dxv"),
                                     cp(dwarrs[0]), cp(dwarrs[1]), cp(dwarrs[2]), _dev(out["dg"], "dg"),
                                     _dev(out["dbeta"], "dbeta"), _dev(out["dS0"], "dS0"), B, T, H, D, dt,
                                     ws_ptr, ws_bytes, _stream(stream))
    _check("kda_mshortconv_backward", rc)
    return out


def forward_plan(B, T, H, Dk, Dv, dtype=torch.bfloat16, chunk: int = 0, o_dtype=None):
    """(segments, chunks per segment) of kda_forward's tensor-core split on this device
    ((0, 0) off that path)."""
    P, L = ctypes.c_int(0), ctypes.c_int(0)
    _check("kda_forward_plan", load_library().kda_forward_plan(B, T, H, Dk, Dv, _code(dtype),
                                                               _code(o_dtype or dtype), chunk,
                                                               ctypes.byref(P), ctypes.byref(L)))
    return P.value, L.value


def kernel_launches() -> int:
    """Kernels launched by libkda in this process so far."""
    return int(load_library().kda_kernel_launches())


def profile_enable(on: bool = True) -> None:
    load_library().kda_profile_enable(1 if on else 0)


def profile_collect(name: str):
    """(total device ms, launches) of kernel `name` since the last collection, or None."""
    ms, n = ctypes.c_double(0.0), ctypes.c_int(0)
    rc = load_library().kda_profile_collect(name.encode(), ctypes.byref(ms), ctypes.byref(n))
    return None if rc != 0 else (ms.value, n.value)


def debug_drop_handoff(on: bool) -> None:
    """Test hook: while on, the tensor-core scan withholds one hand-off between its warp
    roles per CTA, so a bounded wait runs out and the call reports a timeout."""
    load_library().kda_debug_drop_handoff(1 if on else 0)


def fma_probe() -> float:
    """Measured fp32 FMA rate of the current GPU (FMAs per second)."""
    r = ctypes.c_double(0.0)
    _check("kda_fma_probe", load_library().kda_fma_probe(ctypes.byref(r)))
    return r.value


def last_device_error() -> int:
    """Reads and clears the device status word (0 = no device-side failure)."""
    return int(load_library().kda_last_device_error())
