"""Python binding of libkda.so (argument marshalling only).

Every step of the operator runs in the CUDA library; this module only checks
that the tensors are CUDA tensors of the right dtype and shape, fills the C
argument structs declared in include/kda.h and calls them on the current
torch stream.  There is no CPU path: without the CUDA library, a GPU, or with
host tensors, every call raises.
"""
from __future__ import annotations

import ctypes
import os
import threading
from typing import Optional, Tuple

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_PKG, "libkda.so")
_lib = None
_lock = threading.Lock()

KDA_OK = 0
KDA_ERR_INVALID_ARG = 1
KDA_ERR_UNSUPPORTED = 2
KDA_ERR_CUDA = 3
KDA_ERR_DEVICE_TIMEOUT = 4
KDA_ERR_DEVICE_CHECK = 5
KDA_F32 = 0
KDA_BF16 = 1
KDA_GATE_CHANNEL = 0
KDA_GATE_HEAD = 1

EXPORTED = ("kda_prefill", "kda_prefill_workspace_size", "kda_decode", "kda_get_device_status",
            "kda_status_string", "kda_version", "kda_prefill_noalloc", "kda_short_conv",
            "kda_prefill_backward", "kda_prefill_backward_workspace_size", "kda_debug_set_fault",
            "kda_debug_timeout_site")
KDA_FAULT_STARVE_STATE_LOADS = 1


class KdaError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {status_string(status)}")


class PrefillArgs(ctypes.Structure):
    _fields_ = [("dtype", ctypes.c_int), ("num_seqs", ctypes.c_int),
                ("total_tokens", ctypes.c_int), ("H", ctypes.c_int), ("dk", ctypes.c_int),
                ("dv", ctypes.c_int), ("q", ctypes.c_void_p), ("k", ctypes.c_void_p),
                ("v", ctypes.c_void_p), ("log_alpha", ctypes.c_void_p),
                ("beta", ctypes.c_void_p), ("cu_seqlens", ctypes.c_void_p),
                ("pad_mask", ctypes.c_void_p), ("init_state", ctypes.c_void_p),
                ("o", ctypes.c_void_p), ("final_state", ctypes.c_void_p),
                ("chunk", ctypes.c_int), ("workspace", ctypes.c_void_p),
                ("workspace_bytes", ctypes.c_size_t), ("gate", ctypes.c_int)]


class DecodeArgs(ctypes.Structure):
    _fields_ = [("dtype", ctypes.c_int), ("B", ctypes.c_int), ("H", ctypes.c_int),
                ("dk", ctypes.c_int), ("dv", ctypes.c_int), ("q", ctypes.c_void_p),
                ("k", ctypes.c_void_p), ("v", ctypes.c_void_p),
                ("log_alpha", ctypes.c_void_p), ("beta", ctypes.c_void_p),
                ("mask", ctypes.c_void_p), ("state", ctypes.c_void_p), ("o", ctypes.c_void_p),
                ("gate", ctypes.c_int)]


class ConvArgs(ctypes.Structure):
    _fields_ = [("dtype", ctypes.c_int), ("num_seqs", ctypes.c_int),
                ("total_tokens", ctypes.c_int), ("D", ctypes.c_int), ("width", ctypes.c_int),
                ("x", ctypes.c_void_p), ("weight", ctypes.c_void_p), ("bias", ctypes.c_void_p),
                ("cu_seqlens", ctypes.c_void_p), ("pad_mask", ctypes.c_void_p),
                ("state_in", ctypes.c_void_p), ("state_out", ctypes.c_void_p),
                ("y", ctypes.c_void_p)]


class BackwardArgs(ctypes.Structure):
    _fields_ = [("dtype", ctypes.c_int), ("num_seqs", ctypes.c_int),
                ("total_tokens", ctypes.c_int), ("H", ctypes.c_int), ("dk", ctypes.c_int),
                ("dv", ctypes.c_int), ("q", ctypes.c_void_p), ("k", ctypes.c_void_p),
                ("v", ctypes.c_void_p), ("log_alpha", ctypes.c_void_p),
                ("beta", ctypes.c_void_p), ("cu_seqlens", ctypes.c_void_p),
                ("pad_mask", ctypes.c_void_p), ("init_state", ctypes.c_void_p),
                ("gate", ctypes.c_int), ("grad_o", ctypes.c_void_p),
                ("grad_final_state", ctypes.c_void_p), ("grad_q", ctypes.c_void_p),
                ("grad_k", ctypes.c_void_p), ("grad_v", ctypes.c_void_p),
                ("grad_log_alpha", ctypes.c_void_p), ("grad_beta", ctypes.c_void_p),
                ("grad_init_state", ctypes.c_void_p), ("workspace", ctypes.c_void_p),
                ("workspace_bytes", ctypes.c_size_t)]


def library_path() -> str:
    return _LIB_PATH


def load(build_if_stale: bool = True) -> ctypes.CDLL:
    """Load libkda.so (compiling it with nvcc first if it is missing or stale)."""
    global _lib
    with _lock:
        if _lib is None:
            if build_if_stale:
                from . import build as _build
                _build.build()
            if not os.path.exists(_LIB_PATH):
                raise RuntimeError(f"libkda.so not found at {_LIB_PATH}; build it first")
            lib = ctypes.CDLL(_LIB_PATH)
            lib.kda_prefill.argtypes = [ctypes.POINTER(PrefillArgs), ctypes.c_void_p]
            lib.kda_prefill.restype = ctypes.c_int
            lib.kda_prefill_workspace_size.argtypes = [ctypes.POINTER(PrefillArgs)]
            lib.kda_prefill_workspace_size.restype = ctypes.c_size_t
            lib.kda_decode.argtypes = [ctypes.POINTER(DecodeArgs), ctypes.c_void_p]
            lib.kda_decode.restype = ctypes.c_int
            lib.kda_short_conv.argtypes = [ctypes.POINTER(ConvArgs), ctypes.c_void_p]
            lib.kda_short_conv.restype = ctypes.c_int
            lib.kda_prefill_backward.argtypes = [ctypes.POINTER(BackwardArgs), ctypes.c_void_p]
            lib.kda_prefill_backward.restype = ctypes.c_int
            lib.kda_prefill_backward_workspace_size.argtypes = [ctypes.POINTER(BackwardArgs)]
            lib.kda_prefill_backward_workspace_size.restype = ctypes.c_size_t
            lib.kda_get_device_status.argtypes = [ctypes.c_void_p]
            lib.kda_get_device_status.restype = ctypes.c_int
            lib.kda_status_string.argtypes = [ctypes.c_int]
            lib.kda_status_string.restype = ctypes.c_char_p
            lib.kda_version.restype = ctypes.c_int
            lib.kda_prefill_noalloc.argtypes = [ctypes.POINTER(PrefillArgs), ctypes.c_void_p]
            lib.kda_prefill_noalloc.restype = ctypes.c_int
            lib.kda_debug_set_fault.argtypes = [ctypes.c_int, ctypes.c_longlong]
            lib.kda_debug_set_fault.restype = ctypes.c_int
            lib.kda_debug_timeout_site.argtypes = [ctypes.c_void_p]
            lib.kda_debug_timeout_site.restype = ctypes.c_int
            _lib = lib
    return _lib


def status_string(status: int) -> str:
    return load().kda_status_string(int(status)).decode()


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream_handle(stream) -> ctypes.c_void_p:
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _check_cuda(name: str, t: Optional[torch.Tensor], dtype=None, shape=None):
    if t is None:
        return
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor (the operator has no CPU path)")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return KDA_BF16
    if t.dtype == torch.float32:
        return KDA_F32
    raise TypeError(f"q/k/v must be bfloat16 or float32, got {t.dtype}")


def prefill_args(q, k, v, log_alpha, beta, cu_seqlens, pad_mask=None, init_state=None,
                 o=None, final_state=None, chunk: int = 0, workspace=None) -> PrefillArgs:
    """Fill a kda_prefill_args struct from tensors (no validation beyond shapes)."""
    N, H, dk = q.shape
    dv = v.shape[2]
    a = PrefillArgs()
    a.dtype = _dtype_code(q)
    a.num_seqs = cu_seqlens.numel() - 1
    a.total_tokens = N
    a.H, a.dk, a.dv = H, dk, dv
    a.q, a.k, a.v = _ptr(q), _ptr(k), _ptr(v)
    a.log_alpha, a.beta, a.cu_seqlens = _ptr(log_alpha), _ptr(beta), _ptr(cu_seqlens)
    a.pad_mask, a.init_state = _ptr(pad_mask), _ptr(init_state)
    a.o, a.final_state = _ptr(o), _ptr(final_state)
    a.chunk = int(chunk)
    a.workspace = _ptr(workspace)
    a.workspace_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    a.gate = gate_layout(log_alpha)
    return a


def gate_layout(log_alpha) -> int:
    """KDA_GATE_HEAD for a [rows, H] log_alpha (one gate per token and head), else
    KDA_GATE_CHANNEL ([rows, H, dk])."""
    return KDA_GATE_HEAD if log_alpha is not None and log_alpha.dim() == 2 else KDA_GATE_CHANNEL


def prefill_workspace_bytes(num_seqs: int) -> int:
    a = PrefillArgs()
    a.num_seqs = int(num_seqs)
    return int(load().kda_prefill_workspace_size(ctypes.byref(a)))


def prefill_workspace_size_for(q, k, v, log_alpha, beta, cu_seqlens, chunk: int = 0) -> int:
    """kda_prefill_workspace_size() for these tensors (at least 1 byte)."""
    a = prefill_args(q, k, v, log_alpha, beta, cu_seqlens, chunk=chunk)
    return max(int(load().kda_prefill_workspace_size(ctypes.byref(a))), 1)


def prefill_workspace(q, k, v, log_alpha, beta, cu_seqlens, chunk: int = 0) -> torch.Tensor:
    """A device workspace of the size kda_prefill_workspace_size() states for these
    arguments (for callers that allocate it once, e.g. before a CUDA graph capture)."""
    a = prefill_args(q, k, v, log_alpha, beta, cu_seqlens, chunk=chunk)
    nbytes = int(load().kda_prefill_workspace_size(ctypes.byref(a)))
    return torch.empty(max(nbytes, 1), dtype=torch.uint8, device=q.device)


def prefill(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, log_alpha: torch.Tensor,
            beta: torch.Tensor, cu_seqlens: torch.Tensor, pad_mask: Optional[torch.Tensor] = None,
            init_state: Optional[torch.Tensor] = None, o: Optional[torch.Tensor] = None,
            final_state: Optional[torch.Tensor] = None, chunk: int = 0,
            workspace: Optional[torch.Tensor] = None, want_final_state: bool = True,
            stream=None) -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
    """KDA chunkwise prefill (kda_prefill).  Returns (o, final_state).

    q, k [N,H,dk] and v [N,H,dv] bf16 or fp32; log_alpha [N,H,dk] fp32 (per-channel gate) or
    [N,H] fp32 (one gate per token and head); beta [N,H] fp32;
    cu_seqlens [B+1] int32; pad_mask [N] uint8 or None; init_state [B,H,dk,dv] fp32 or None.
    Outputs are allocated here when not given (torch allocates; the library does not).
    """
    lib = load()
    N, H, dk = q.shape
    dv = v.shape[2]
    B = cu_seqlens.numel() - 1
    _check_cuda("q", q, shape=(N, H, dk))
    _check_cuda("k", k, dtype=q.dtype, shape=(N, H, dk))
    _check_cuda("v", v, dtype=q.dtype, shape=(N, H, dv))
    _check_cuda("log_alpha", log_alpha, torch.float32,
                (N, H) if gate_layout(log_alpha) == KDA_GATE_HEAD else (N, H, dk))
    _check_cuda("beta", beta, torch.float32, (N, H))
    _check_cuda("cu_seqlens", cu_seqlens, torch.int32, (B + 1,))
    _check_cuda("pad_mask", pad_mask, torch.uint8, (N,))
    _check_cuda("init_state", init_state, torch.float32, (B, H, dk, dv))
    if o is None:
        o = torch.empty((N, H, dv), dtype=q.dtype, device=q.device)
    _check_cuda("o", o, q.dtype, (N, H, dv))
    if final_state is None and want_final_state:
        final_state = torch.empty((B, H, dk, dv), dtype=torch.float32, device=q.device)
    _check_cuda("final_state", final_state, torch.float32, (B, H, dk, dv))
    a = prefill_args(q, k, v, log_alpha, beta, cu_seqlens, pad_mask, init_state, o, final_state,
                     chunk, workspace)
    if workspace is None:
        # the library states its own need (span table; per-chunk items of the two-kernel path)
        nbytes = int(lib.kda_prefill_workspace_size(ctypes.byref(a)))
        if nbytes:
            workspace = torch.empty(nbytes, dtype=torch.uint8, device=q.device)
            a.workspace = _ptr(workspace)
            a.workspace_bytes = nbytes
    st = lib.kda_prefill(ctypes.byref(a), _stream_handle(stream))
    if st != KDA_OK:
        raise KdaError(st, "kda_prefill")
    return o, final_state


def decode(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, log_alpha: torch.Tensor,
           beta: torch.Tensor, state: torch.Tensor, mask: Optional[torch.Tensor] = None,
           o: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """One KDA decode step (kda_decode); ``state`` [B,H,dk,dv] fp32 is updated in place.
    log_alpha is [B,H,dk] (per-channel gate) or [B,H] (one gate per row and head)."""
    lib = load()
    B, H, dk = q.shape
    dv = v.shape[2]
    _check_cuda("q", q, shape=(B, H, dk))
    _check_cuda("k", k, q.dtype, (B, H, dk))
    _check_cuda("v", v, q.dtype, (B, H, dv))
    _check_cuda("log_alpha", log_alpha, torch.float32,
                (B, H) if gate_layout(log_alpha) == KDA_GATE_HEAD else (B, H, dk))
    _check_cuda("beta", beta, torch.float32, (B, H))
    _check_cuda("mask", mask, torch.uint8, (B,))
    _check_cuda("state", state, torch.float32, (B, H, dk, dv))
    if o is None:
        o = torch.empty((B, H, dv), dtype=q.dtype, device=q.device)
    _check_cuda("o", o, q.dtype, (B, H, dv))
    a = DecodeArgs()
    a.dtype = _dtype_code(q)
    a.B, a.H, a.dk, a.dv = B, H, dk, dv
    a.q, a.k, a.v = _ptr(q), _ptr(k), _ptr(v)
    a.log_alpha, a.beta, a.mask = _ptr(log_alpha), _ptr(beta), _ptr(mask)
    a.state, a.o = _ptr(state), _ptr(o)
    a.gate = gate_layout(log_alpha)
    st = lib.kda_decode(ctypes.byref(a), _stream_handle(stream))
    if st != KDA_OK:
        raise KdaError(st, "kda_decode")
    return o


def short_conv(x: torch.Tensor, weight: torch.Tensor, cu_seqlens: torch.Tensor,
               bias: Optional[torch.Tensor] = None, pad_mask: Optional[torch.Tensor] = None,
               state_in: Optional[torch.Tensor] = None, state_out: Optional[torch.Tensor] = None,
               y: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """Padding-correct short causal convolution (kda_short_conv).  x [N,D] bf16 or fp32,
    weight [D,W] fp32, bias [D] fp32, state_in/state_out [B,W-1,D] fp32 (may be the same
    tensor).  Returns y [N,D] (allocated here when not given)."""
    lib = load()
    N, D = x.shape
    W = weight.shape[1]
    B = cu_seqlens.numel() - 1
    _check_cuda("x", x, shape=(N, D))
    _check_cuda("weight", weight, torch.float32, (D, W))
    _check_cuda("bias", bias, torch.float32, (D,))
    _check_cuda("cu_seqlens", cu_seqlens, torch.int32, (B + 1,))
    _check_cuda("pad_mask", pad_mask, torch.uint8, (N,))
    _check_cuda("state_in", state_in, torch.float32, (B, W - 1, D))
    _check_cuda("state_out", state_out, torch.float32, (B, W - 1, D))
    if y is None:
        y = torch.empty((N, D), dtype=x.dtype, device=x.device)
    _check_cuda("y", y, x.dtype, (N, D))
    a = ConvArgs()
    a.dtype = _dtype_code(x)
    a.num_seqs, a.total_tokens, a.D, a.width = B, N, D, W
    a.x, a.weight, a.bias = _ptr(x), _ptr(weight), _ptr(bias)
    a.cu_seqlens, a.pad_mask = _ptr(cu_seqlens), _ptr(pad_mask)
    a.state_in, a.state_out, a.y = _ptr(state_in), _ptr(state_out), _ptr(y)
    st = lib.kda_short_conv(ctypes.byref(a), _stream_handle(stream))
    if st != KDA_OK:
        raise KdaError(st, "kda_short_conv")
    return y


def prefill_backward(q, k, v, log_alpha, beta, cu_seqlens, grad_o, grad_final_state=None,
                     pad_mask=None, init_state=None, want_grad_init_state: bool = True,
                     workspace=None, stream=None):
    """Backward of the prefill (kda_prefill_backward).  Returns a dict of fp32 CUDA
    tensors dq, dk, dv, dlog_alpha (log_alpha's layout), dbeta and dS0 (None unless
    wanted).  grad_o [N,H,dv] and grad_final_state [B,H,dk,dv] are fp32."""
    lib = load()
    N, H, dk = q.shape
    dv = v.shape[2]
    B = cu_seqlens.numel() - 1
    gate = gate_layout(log_alpha)
    _check_cuda("q", q, shape=(N, H, dk))
    _check_cuda("k", k, q.dtype, (N, H, dk))
    _check_cuda("v", v, q.dtype, (N, H, dv))
    _check_cuda("log_alpha", log_alpha, torch.float32, (N, H) if gate == KDA_GATE_HEAD else (N, H, dk))
    _check_cuda("beta", beta, torch.float32, (N, H))
    _check_cuda("cu_seqlens", cu_seqlens, torch.int32, (B + 1,))
    _check_cuda("pad_mask", pad_mask, torch.uint8, (N,))
    _check_cuda("init_state", init_state, torch.float32, (B, H, dk, dv))
    _check_cuda("grad_o", grad_o, torch.float32, (N, H, dv))
    _check_cuda("grad_final_state", grad_final_state, torch.float32, (B, H, dk, dv))
    f32 = dict(dtype=torch.float32, device=q.device)
    g = {"dq": torch.empty((N, H, dk), **f32), "dk": torch.empty((N, H, dk), **f32),
         "dv": torch.empty((N, H, dv), **f32), "dlog_alpha": torch.empty(tuple(log_alpha.shape), **f32),
         "dbeta": torch.empty((N, H), **f32),
         "dS0": torch.empty((B, H, dk, dv), **f32) if want_grad_init_state else None}
    a = BackwardArgs()
    a.dtype = _dtype_code(q)
    a.num_seqs, a.total_tokens, a.H, a.dk, a.dv = B, N, H, dk, dv
    a.q, a.k, a.v = _ptr(q), _ptr(k), _ptr(v)
    a.log_alpha, a.beta, a.cu_seqlens = _ptr(log_alpha), _ptr(beta), _ptr(cu_seqlens)
    a.pad_mask, a.init_state, a.gate = _ptr(pad_mask), _ptr(init_state), gate
    a.grad_o, a.grad_final_state = _ptr(grad_o), _ptr(grad_final_state)
    a.grad_q, a.grad_k, a.grad_v = _ptr(g["dq"]), _ptr(g["dk"]), _ptr(g["dv"])
    a.grad_log_alpha, a.grad_beta, a.grad_init_state = _ptr(g["dlog_alpha"]), _ptr(g["dbeta"]), _ptr(g["dS0"])
    if workspace is None:
        nbytes = int(lib.kda_prefill_backward_workspace_size(ctypes.byref(a)))
        workspace = torch.empty(max(nbytes, 1), dtype=torch.uint8, device=q.device)
    a.workspace = _ptr(workspace)
    a.workspace_bytes = workspace.numel() * workspace.element_size()
    st = lib.kda_prefill_backward(ctypes.byref(a), _stream_handle(stream))
    if st != KDA_OK:
        raise KdaError(st, "kda_prefill_backward")
    return g


def prefill_backward_workspace_bytes(N: int, B: int, H: int, dk: int, dv: int) -> int:
    """kda_prefill_backward_workspace_size() for these sizes (at least 1 byte)."""
    a = BackwardArgs()
    a.num_seqs, a.total_tokens, a.H, a.dk, a.dv = B, N, H, dk, dv
    return max(int(load().kda_prefill_backward_workspace_size(ctypes.byref(a))), 1)


def get_device_status(stream=None) -> int:
    """Synchronise the stream and return (and clear) the latched device status."""
    return int(load().kda_get_device_status(_stream_handle(stream)))


def debug_set_fault(fault: int, wait_cycles: int = 0) -> None:
    """kda_debug_set_fault: plant a test fault and set the bounded-wait limit (tests only;
    ``debug_set_fault(0)`` restores normal operation and the default limit)."""
    st = load().kda_debug_set_fault(int(fault), int(wait_cycles))
    if st != KDA_OK:
        raise KdaError(st, "kda_debug_set_fault")


def debug_timeout_site(stream=None) -> int:
    """kda_debug_timeout_site: code of the first bounded wait that ran out (0 = none)."""
    return int(load().kda_debug_timeout_site(_stream_handle(stream)))


def raw_prefill(args: PrefillArgs, stream=None) -> int:
    """Call kda_prefill with a prepared struct; returns the status code."""
    return int(load().kda_prefill(ctypes.byref(args), _stream_handle(stream)))


NOALLOC_MAX_SEQS = 4096


def prefill_noalloc(q, k, v, log_alpha, beta, cu_seqlens, o, final_state=None,
                    pad_mask=None, init_state=None, chunk: int = 0, stream=None):
    """kda_prefill_noalloc: the prefill with its scratch taken from a fixed array inside
    the library, for callers that cannot allocate device memory at call time.  The
    outputs ``o`` (and ``final_state``, if wanted) must be given; nothing is allocated."""
    lib = load()
    a = prefill_args(q, k, v, log_alpha, beta, cu_seqlens, pad_mask, init_state, o,
                     final_state, chunk, None)
    st = lib.kda_prefill_noalloc(ctypes.byref(a), _stream_handle(stream))
    if st != KDA_OK:
        raise KdaError(st, "kda_prefill_noalloc")
    return o, final_state
