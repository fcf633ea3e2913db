"""Thin ctypes binding of libgdn.so (the C ABI declared in include/gdn.h).

Argument marshalling only: every step of the forward and backward passes runs
in the CUDA kernels of libgdn.so.  PyTorch provides device memory and the current stream.
There is no fallback: if the library is missing or the device is not a CUDA
device, the call raises.
"""
from __future__ import annotations

import ctypes
import os
import threading
from typing import Optional, Tuple

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libgdn.so")

GDN_OK = 0
GDN_ERR_INVALID_ARG = 1
GDN_ERR_UNSUPPORTED = 2
GDN_ERR_ALIGNMENT = 3
GDN_ERR_CUDA = 4
GDN_ERR_DEVICE_CHECK = 5
GDN_ERR_FAULT_INJECTED = 6

GDN_F32, GDN_BF16 = 0, 1
GDN_INV_EXACT, GDN_INV_NEUMANN, GDN_INV_NEUMANN_RESIDUAL = 0, 1, 2
KERNELS = {"auto": 0, "simt": 1, "tc": 2, "recurrent": 3, "tc_split": 4}
KERNEL_NAMES = {v: k for k, v in KERNELS.items()}
MODES = {"exact": GDN_INV_EXACT, "neumann": GDN_INV_NEUMANN, "residual": GDN_INV_NEUMANN_RESIDUAL}

EXPORTS = ("gdn_chunk_fwd", "gdn_select_kernel", "gdn_workspace_bytes", "gdn_device_check",
           "gdn_status_string", "gdn_last_error", "gdn_abi_version", "gdn_chunk_fwd_static_scratch",
           "gdn_chunk_bwd", "gdn_bwd_workspace_bytes", "gdn_debug_chunk_T", "gdn_select_segments")
STATIC_SCRATCH_BYTES = 24 << 20   # GDN_STATIC_SCRATCH_BYTES


class GDNError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{status_string(status)}: {message}")
        self.status = status


class FwdArgs(ctypes.Structure):
    """Mirror of ``gdn_fwd_args``."""
    _fields_ = [
        ("B", ctypes.c_int32), ("T", ctypes.c_int32), ("H", ctypes.c_int32),
        ("dk", ctypes.c_int32), ("dv", ctypes.c_int32), ("chunk", ctypes.c_int32),
        ("io_dtype", ctypes.c_int32), ("o_dtype", ctypes.c_int32),
        ("q", ctypes.c_void_p), ("k", ctypes.c_void_p), ("v", ctypes.c_void_p),
        ("alpha", ctypes.c_void_p), ("alpha_per_channel", ctypes.c_int32),
        ("beta", ctypes.c_void_p), ("precond", ctypes.c_int32),
        ("rho_decay", ctypes.c_float), ("rho_eps", ctypes.c_float),
        ("erase", ctypes.c_void_p), ("write", ctypes.c_void_p),
        ("S0", ctypes.c_void_p), ("o", ctypes.c_void_p), ("S_T", ctypes.c_void_p),
        ("mode", ctypes.c_int32), ("neumann_N", ctypes.c_int32),
        ("kernel", ctypes.c_int32), ("dv_split", ctypes.c_int32),
        ("workspace", ctypes.c_void_p), ("workspace_bytes", ctypes.c_uint64),
        ("residual_S", ctypes.c_int32),
        ("precond_x", ctypes.c_float), ("precond_query", ctypes.c_int32),
        ("seq_segments", ctypes.c_int32),
    ]


class BwdArgs(ctypes.Structure):
    """Mirror of ``gdn_bwd_args``."""
    _fields_ = [
        ("B", ctypes.c_int32), ("T", ctypes.c_int32), ("H", ctypes.c_int32),
        ("dk", ctypes.c_int32), ("dv", ctypes.c_int32), ("chunk", ctypes.c_int32),
        ("io_dtype", ctypes.c_int32), ("do_dtype", ctypes.c_int32),
        ("q", ctypes.c_void_p), ("k", ctypes.c_void_p), ("v", ctypes.c_void_p),
        ("alpha", ctypes.c_void_p), ("beta", ctypes.c_void_p), ("S0", ctypes.c_void_p),
        ("grad_o", ctypes.c_void_p), ("grad_S_T", ctypes.c_void_p),
        ("grad_q", ctypes.c_void_p), ("grad_k", ctypes.c_void_p), ("grad_v", ctypes.c_void_p),
        ("grad_alpha", ctypes.c_void_p), ("grad_beta", ctypes.c_void_p),
        ("grad_S0", ctypes.c_void_p),
        ("workspace", ctypes.c_void_p), ("workspace_bytes", ctypes.c_uint64),
        ("mode", ctypes.c_int32), ("neumann_N", ctypes.c_int32), ("residual_S", ctypes.c_int32),
    ]


_lock = threading.Lock()
_lib = None


def lib() -> ctypes.CDLL:
    """Load libgdn.so (raises if it has not been built)."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                                   "`python -m chunked_gated_delta_14_b200.build`")
            L = ctypes.CDLL(LIB_PATH)
            L.gdn_chunk_fwd.argtypes = [ctypes.POINTER(FwdArgs), ctypes.c_void_p]
            L.gdn_chunk_fwd.restype = ctypes.c_int
            L.gdn_select_kernel.argtypes = [ctypes.POINTER(FwdArgs)]
            L.gdn_select_kernel.restype = ctypes.c_int32
            L.gdn_select_segments.argtypes = [ctypes.POINTER(FwdArgs)]
            L.gdn_select_segments.restype = ctypes.c_int32
            L.gdn_workspace_bytes.argtypes = [ctypes.POINTER(FwdArgs)]
            L.gdn_workspace_bytes.restype = ctypes.c_uint64
            L.gdn_device_check.argtypes = [ctypes.c_void_p]
            L.gdn_device_check.restype = ctypes.c_int
            L.gdn_status_string.argtypes = [ctypes.c_int]
            L.gdn_status_string.restype = ctypes.c_char_p
            L.gdn_last_error.argtypes = []
            L.gdn_last_error.restype = ctypes.c_char_p
            L.gdn_abi_version.argtypes = []
            L.gdn_abi_version.restype = ctypes.c_int32
            L.gdn_chunk_fwd_static_scratch.argtypes = [ctypes.POINTER(FwdArgs), ctypes.c_void_p]
            L.gdn_chunk_fwd_static_scratch.restype = ctypes.c_int
            L.gdn_chunk_bwd.argtypes = [ctypes.POINTER(BwdArgs), ctypes.c_void_p]
            L.gdn_chunk_bwd.restype = ctypes.c_int
            L.gdn_bwd_workspace_bytes.argtypes = [ctypes.POINTER(BwdArgs)]
            L.gdn_bwd_workspace_bytes.restype = ctypes.c_uint64
            L.gdn_debug_chunk_T.argtypes = [ctypes.POINTER(FwdArgs), ctypes.c_int32, ctypes.c_int32,
                                            ctypes.c_int32, ctypes.c_void_p, ctypes.c_void_p]
            L.gdn_debug_chunk_T.restype = ctypes.c_int
            _lib = L
    return _lib


def status_string(s: int) -> str:
    try:
        return lib().gdn_status_string(int(s)).decode()
    except Exception:  # pragma: no cover - message formatting only
        return f"status {s}"


def last_error() -> str:
    return lib().gdn_last_error().decode()


def abi_version() -> int:
    return int(lib().gdn_abi_version())


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _dtype_code(dt: torch.dtype) -> int:
    if dt == torch.bfloat16:
        return GDN_BF16
    if dt == torch.float32:
        return GDN_F32
    raise TypeError(f"unsupported dtype {dt}; use torch.bfloat16 or torch.float32")


def _check(t: Optional[torch.Tensor], name: str, shape, dtype=None):
    if t is None:
        return
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.device.type != "cuda":
        raise ValueError(f"{name} must be a CUDA tensor (got {t.device})")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} has dtype {t.dtype}, expected {dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def make_args(**kw) -> FwdArgs:
    a = FwdArgs()
    a.rho_decay = 0.99
    a.rho_eps = 1e-6
    for k, v in kw.items():
        setattr(a, k, v)
    return a


def select_kernel(args: FwdArgs) -> int:
    """Kernel gdn_chunk_fwd would launch (1 simt, 2 fused tc, 3 recurrent, 4 split tc)
    or -status. Host only."""
    return int(lib().gdn_select_kernel(ctypes.byref(args)))


def select_segments(args: FwdArgs) -> int:
    """Sequence segments gdn_chunk_fwd would use (1 or 3) or -status. Host only."""
    return int(lib().gdn_select_segments(ctypes.byref(args)))


def workspace_bytes(args: FwdArgs) -> int:
    """Device workspace gdn_chunk_fwd needs for ``args`` (host only)."""
    return int(lib().gdn_workspace_bytes(ctypes.byref(args)))


_ws_cache = {}


def clear_workspace_cache(device: Optional[torch.device] = None) -> None:
    """Drop the cached workspaces (all devices, or one), e.g. when a stream that
    was used for calls is retired.  Each cached buffer holds its bytes until it
    is dropped: about 96 MiB for a split-kernel forward of the 4 x 16 x 4096
    benchmark shape, 263 MB for the SIMT two-gate forward of 2 x 16 x 4096,
    1.4 GB for the scalar-rule backward of the benchmark shape; the fused and
    the recurrent forward need none."""
    for key in list(_ws_cache):
        if device is None or (key[0] == device.type and key[1] == device.index):
            del _ws_cache[key]


def workspace_for(args, device: torch.device,
                  stream: Optional[torch.cuda.Stream] = None) -> Optional[torch.Tensor]:
    """A cached device buffer of at least the workspace ``args`` needs, or None.

    One buffer per (device, stream, direction): calls ordered on one stream
    reuse it, calls on different streams never share one, and forward
    (FwdArgs) and backward (BwdArgs) calls keep separate buffers.  ``stream``
    is the stream the call will run on (default: the device's current one).
    Buffers stay cached until ``clear_workspace_cache``."""
    bwd = isinstance(args, BwdArgs)
    need = bwd_workspace_bytes(args) if bwd else workspace_bytes(args)
    if need == 0:
        return None
    current = torch.cuda.current_stream(device)
    if stream is None:
        stream = current
    key = (device.type, device.index, stream.cuda_stream, bwd)
    buf = _ws_cache.get(key)
    if buf is None or buf.numel() < need:
        buf = torch.empty(need, dtype=torch.uint8, device=device)
        if stream.cuda_stream != current.cuda_stream:
            buf.record_stream(stream)   # freed blocks wait for the stream that used them
        _ws_cache[key] = buf
    return buf


def call(args: FwdArgs, stream: Optional[int] = None) -> None:
    """Raw gdn_chunk_fwd call; raises GDNError on a non-OK status."""
    s = lib().gdn_chunk_fwd(ctypes.byref(args), ctypes.c_void_p(stream or 0))
    if s != GDN_OK:
        raise GDNError(s, last_error())


def call_static_scratch(args: FwdArgs, stream: Optional[int] = None) -> None:
    """Raw gdn_chunk_fwd_static_scratch call (tensor-core kernel, the library's
    fixed scratch; args.workspace must be 0); raises GDNError on a non-OK status."""
    s = lib().gdn_chunk_fwd_static_scratch(ctypes.byref(args), ctypes.c_void_p(stream or 0))
    if s != GDN_OK:
        raise GDNError(s, last_error())


def call_debug_chunk_T(args: FwdArgs, b: int, h: int, n: int, T_out: int,
                       stream: Optional[int] = None) -> None:
    """Raw gdn_debug_chunk_T call (T_out: device pointer of 4096 floats); raises
    GDNError on a non-OK status."""
    s = lib().gdn_debug_chunk_T(ctypes.byref(args), int(b), int(h), int(n), ctypes.c_void_p(T_out),
                                ctypes.c_void_p(stream or 0))
    if s != GDN_OK:
        raise GDNError(s, last_error())


def debug_chunk_T(q, k, v, alpha=None, beta=None, *, b: int = 0, h: int = 0, n: int = 0,
                  mode: str = "exact", N: int = 3, S0=None) -> torch.Tensor:
    """The 64 x 64 fp32 T the fused kernel forms for chunk n of sequence (b, h)
    (exact inverse or masked Neumann series), from one gdn_debug_chunk_T call."""
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    o = torch.empty((B, T, H, dv), device=q.device, dtype=torch.float32)
    S_T = torch.empty((B, H, dk, dv), device=q.device, dtype=torch.float32)
    T_out = torch.full((64, 64), float("nan"), device=q.device, dtype=torch.float32)
    args = make_args(B=B, T=T, H=H, dk=dk, dv=dv, chunk=64, io_dtype=_dtype_code(q.dtype), o_dtype=GDN_F32,
                     q=_ptr(q), k=_ptr(k), v=_ptr(v), alpha=_ptr(alpha), beta=_ptr(beta), S0=_ptr(S0),
                     o=_ptr(o), S_T=_ptr(S_T), mode=MODES[mode], neumann_N=int(N), kernel=KERNELS["tc"])
    stream = torch.cuda.current_stream(q.device)
    with torch.cuda.device(q.device):
        call_debug_chunk_T(args, b, h, n, T_out.data_ptr(), stream.cuda_stream)
    return T_out


def device_check(stream: Optional[int] = None) -> None:
    """Synchronise and raise GDNError if a kernel recorded a device-side failure."""
    s = lib().gdn_device_check(ctypes.c_void_p(stream or 0))
    if s != GDN_OK:
        raise GDNError(s, last_error())


def chunk_fwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
              alpha: Optional[torch.Tensor] = None, beta: Optional[torch.Tensor] = None, *,
              erase: Optional[torch.Tensor] = None, write: Optional[torch.Tensor] = None,
              precond: int = 0, rho_decay: float = 0.99, rho_eps: float = 1e-6,
              precond_x: float = 2.0, precond_query: bool = False,
              S0: Optional[torch.Tensor] = None, chunk: int = 64, mode: str = "exact",
              N: int = 3, S: int = 8, o_dtype: Optional[torch.dtype] = None, kernel: str = "auto",
              dv_split: int = 0, segments: int = 0, out: Optional[torch.Tensor] = None,
              final_state: bool = True, S_T: Optional[torch.Tensor] = None,
              stream: Optional[torch.cuda.Stream] = None
              ) -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
    """Chunkwise gated delta-rule forward; returns ``(o, S_T)``.

    q, k: [B, T, H, dk]; v: [B, T, H, dv] (bf16 or fp32, same dtype).
    alpha: [B, T, H] or [B, T, H, dk] fp32 decay (None = 1); beta: [B, T, H]
    fp32 (None = 1).  erase [B, T, H, dk], write [B, T, H, dv] gates and
    ``precond`` select the preconditioned two-gate rule: 1 (or True) the
    moving-average factor 1/sqrt(rho + eps), 2 Diag(A_t)^-1, 3 that squashed into
    [1/precond_x, precond_x]; ``precond_query`` moves the factor to the query.  S0 / S_T:
    [B, H, dk, dv] fp32 (h = S^T).  ``o_dtype`` defaults to q's dtype.
    ``mode``: "exact", "neumann" (masked series to order N) or "residual" (the
    masked series corrected with S residual terms).  ``segments``: 0 lets the
    library choose, 1 forces one pass over the chunks, 3 three sequence segments
    (split tensor-core kernels, scalar rule, chunk 64, B = 1).
    """
    if q.dim() != 4:
        raise ValueError("q must be [B, T, H, dk]")
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    io = q.dtype
    _check(q, "q", (B, T, H, dk), io)
    _check(k, "k", (B, T, H, dk), io)
    _check(v, "v", (B, T, H, dv), io)
    per_channel = alpha is not None and alpha.dim() == 4
    _check(alpha, "alpha", (B, T, H, dk) if per_channel else (B, T, H), torch.float32)
    _check(beta, "beta", (B, T, H), torch.float32)
    _check(erase, "erase", (B, T, H, dk), io)
    _check(write, "write", (B, T, H, dv), io)
    _check(S0, "S0", (B, H, dk, dv), torch.float32)
    od = o_dtype or io
    if out is None:
        out = torch.empty((B, T, H, dv), device=q.device, dtype=od)
    _check(out, "out", (B, T, H, dv), od)
    if final_state and S_T is None:
        S_T = torch.empty((B, H, dk, dv), device=q.device, dtype=torch.float32)
    if not final_state:
        S_T = None
    _check(S_T, "S_T", (B, H, dk, dv), torch.float32)
    args = make_args(
        B=B, T=T, H=H, dk=dk, dv=dv, chunk=int(chunk), io_dtype=_dtype_code(io),
        o_dtype=_dtype_code(od), q=_ptr(q), k=_ptr(k), v=_ptr(v), alpha=_ptr(alpha),
        alpha_per_channel=int(per_channel), beta=_ptr(beta), precond=int(precond),
        precond_x=float(precond_x), precond_query=int(bool(precond_query)),
        rho_decay=float(rho_decay), rho_eps=float(rho_eps), erase=_ptr(erase),
        write=_ptr(write), S0=_ptr(S0), o=_ptr(out), S_T=_ptr(S_T), mode=MODES[mode],
        neumann_N=int(N), residual_S=int(S), kernel=KERNELS[kernel], dv_split=int(dv_split),
        seq_segments=int(segments))
    if stream is None:
        stream = torch.cuda.current_stream(q.device)
    ws = workspace_for(args, q.device, stream)
    if ws is not None:
        args.workspace = ws.data_ptr()
        args.workspace_bytes = ws.numel()
    with torch.cuda.device(q.device):
        call(args, stream.cuda_stream)
    return out, S_T


# ------------------------------------------------------------------ backward

def make_bwd_args(**kw) -> BwdArgs:
    a = BwdArgs()
    for k, v in kw.items():
        setattr(a, k, v)
    return a


def bwd_workspace_bytes(args: BwdArgs) -> int:
    """Device workspace gdn_chunk_bwd needs for ``args`` (0 if invalid; host only)."""
    return int(lib().gdn_bwd_workspace_bytes(ctypes.byref(args)))


def call_bwd(args: BwdArgs, stream: Optional[int] = None) -> None:
    """Raw gdn_chunk_bwd call; raises GDNError on a non-OK status."""
    s = lib().gdn_chunk_bwd(ctypes.byref(args), ctypes.c_void_p(stream or 0))
    if s != GDN_OK:
        raise GDNError(s, last_error())


def chunk_bwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
              alpha: Optional[torch.Tensor], beta: Optional[torch.Tensor],
              grad_o: torch.Tensor, *, S0: Optional[torch.Tensor] = None,
              grad_S_T: Optional[torch.Tensor] = None, chunk: int = 64,
              want_S0: bool = True, mode: str = "exact", N: int = 3, S: int = 8,
              stream: Optional[torch.cuda.Stream] = None) -> dict:
    """Gradients of the gated delta rule (scalar alpha and beta, exact inverse).

    Inputs as ``chunk_fwd``; ``grad_o`` [B, T, H, dv] (bf16 or fp32) is dL/do
    and ``grad_S_T`` [B, H, dk, dv] fp32 (or None) dL/dS_T.  Returns a dict of
    fp32 tensors ``dq``, ``dk``, ``dv``, ``dalpha`` / ``dbeta`` (None when the
    gate is None) and ``dS0`` (None unless ``want_S0``).  ``mode`` is the chunk
    inverse of the forward being differentiated: "exact", "neumann" (the
    masked truncated series of order ``N``) or "residual" (that series with ``S``
    correction terms).
    """
    if q.dim() != 4:
        raise ValueError("q must be [B, T, H, dk]")
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    io = q.dtype
    _check(q, "q", (B, T, H, dk), io)
    _check(k, "k", (B, T, H, dk), io)
    _check(v, "v", (B, T, H, dv), io)
    _check(alpha, "alpha", (B, T, H), torch.float32)
    _check(beta, "beta", (B, T, H), torch.float32)
    _check(S0, "S0", (B, H, dk, dv), torch.float32)
    _check(grad_o, "grad_o", (B, T, H, dv))
    _check(grad_S_T, "grad_S_T", (B, H, dk, dv), torch.float32)
    f32 = dict(device=q.device, dtype=torch.float32)
    g = dict(dq=torch.empty((B, T, H, dk), **f32), dk=torch.empty((B, T, H, dk), **f32),
             dv=torch.empty((B, T, H, dv), **f32),
             dalpha=None if alpha is None else torch.empty((B, T, H), **f32),
             dbeta=None if beta is None else torch.empty((B, T, H), **f32),
             dS0=torch.empty((B, H, dk, dv), **f32) if want_S0 else None)
    args = make_bwd_args(
        B=B, T=T, H=H, dk=dk, dv=dv, chunk=int(chunk), io_dtype=_dtype_code(io),
        do_dtype=_dtype_code(grad_o.dtype), q=_ptr(q), k=_ptr(k), v=_ptr(v), alpha=_ptr(alpha),
        beta=_ptr(beta), S0=_ptr(S0), grad_o=_ptr(grad_o), grad_S_T=_ptr(grad_S_T),
        grad_q=_ptr(g["dq"]), grad_k=_ptr(g["dk"]), grad_v=_ptr(g["dv"]),
        grad_alpha=_ptr(g["dalpha"]), grad_beta=_ptr(g["dbeta"]), grad_S0=_ptr(g["dS0"]),
        mode=MODES[mode], neumann_N=int(N), residual_S=int(S))
    if stream is None:
        stream = torch.cuda.current_stream(q.device)
    ws = workspace_for(args, q.device, stream)
    if ws is not None:
        args.workspace = ws.data_ptr()
        args.workspace_bytes = ws.numel()
    with torch.cuda.device(q.device):
        call_bwd(args, stream.cuda_stream)
    return g


class GatedDeltaRule(torch.autograd.Function):
    """Differentiable gated delta rule: forward by ``chunk_fwd``, backward by
    ``chunk_bwd``, both with the same chunk inverse (``mode`` "exact", "neumann"
    of order ``N``, or "residual" with ``S`` correction terms); both run in
    libgdn.so."""

    @staticmethod
    def forward(ctx, q, k, v, alpha, beta, S0, chunk, mode="exact", N=3, S=8):
        o, S_T = chunk_fwd(q, k, v, alpha, beta, S0=S0, chunk=chunk, mode=mode, N=N, S=S)
        ctx.save_for_backward(q, k, v, alpha, beta, S0)
        ctx.chunk, ctx.mode, ctx.N, ctx.S = chunk, mode, N, S
        return o, S_T

    @staticmethod
    def backward(ctx, grad_o, grad_S_T):
        q, k, v, alpha, beta, S0 = ctx.saved_tensors
        if grad_o is None:
            grad_o = torch.zeros(v.shape, device=v.device, dtype=torch.float32)
        g = chunk_bwd(q, k, v, alpha, beta, grad_o.contiguous(), S0=S0,
                      grad_S_T=None if grad_S_T is None else grad_S_T.float().contiguous(),
                      chunk=ctx.chunk, want_S0=S0 is not None and ctx.needs_input_grad[5],
                      mode=ctx.mode, N=ctx.N, S=ctx.S)
        cast = lambda t, like: None if t is None else t.to(like.dtype)
        return (cast(g["dq"], q), cast(g["dk"], k), cast(g["dv"], v), g["dalpha"], g["dbeta"],
                g["dS0"], None, None, None, None)


def gated_delta_rule(q, k, v, alpha=None, beta=None, S0=None, chunk: int = 64, mode: str = "exact",
                     N: int = 3, S: int = 8):
    """``(o, S_T)`` of the gated delta rule with autograd support (see GatedDeltaRule);
    ``mode`` "neumann" uses the masked truncated series of order ``N`` as the chunk
    inverse in both passes, "residual" that series with ``S`` correction terms."""
    if mode not in ("exact", "neumann", "residual"):
        raise ValueError("gated_delta_rule: mode must be 'exact', 'neumann' or 'residual'")
    return GatedDeltaRule.apply(q, k, v, alpha, beta, S0, chunk, mode, N, S)
