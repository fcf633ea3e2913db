"""ctypes wrapper of the fp64 token-by-token oracle (``gdn_oracle.c``).

Test infrastructure only.  Inputs may be numpy arrays or CPU torch tensors of
any float dtype; they are widened to float64 exactly as the CUDA path receives
them (bf16 values widen losslessly).  The forward functions return
``(o, h_T)`` as float64 numpy arrays with ``o`` shaped [B, T, H, d_v] and
``h_T`` shaped [B, H, d_k, d_v] (the transposed state h = S^T);
``gated_delta_bwd`` returns the gradients of the gated delta rule.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gdn_oracle.c")
_LIB = os.path.join(_HERE, "libgdn_oracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile the C oracle in place with gcc (OpenMP)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-shared", "-fPIC", _SRC,
                               "-o", tmp, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            dp = ctypes.POINTER(ctypes.c_double)
            i = ctypes.c_int
            lib.oracle_gated_delta_fwd.argtypes = [i, i, i, i, i, dp, dp, dp, dp, dp, dp,
                                                   dp, dp, i]
            lib.oracle_gated_delta_fwd.restype = None
            lib.oracle_precond_two_gate_fwd.argtypes = [i, i, i, i, i, dp, dp, dp, dp, dp,
                                                        dp, i, ctypes.c_double,
                                                        ctypes.c_double, ctypes.c_double, i,
                                                        dp, dp, dp, i]
            lib.oracle_precond_two_gate_fwd.restype = None
            lib.oracle_gated_delta_bwd.argtypes = [i, i, i, i, i, dp, dp, dp, dp, dp, dp, dp,
                                                   dp, dp, dp, dp, dp, dp, dp, i]
            lib.oracle_gated_delta_bwd.restype = None
            _lib = lib
    return _lib


def _f64(x):
    if x is None:
        return None
    if hasattr(x, "detach"):  # torch tensor
        x = x.detach().to("cpu").double().numpy()
    return np.ascontiguousarray(x, dtype=np.float64)


def _ptr(a):
    if a is None:
        return None
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def _threads(nthreads):
    if nthreads is not None:
        return int(nthreads)
    return len(os.sched_getaffinity(0))


def gated_delta_fwd(q, k, v, alpha=None, beta=None, h0=None, nthreads=None):
    """S_t = S_{t-1} alpha_t (I - beta_t k_t k_t^T) + beta_t v_t k_t^T, o_t = S_t q_t.

    alpha, beta: [B, T, H] or None (meaning 1).  h0: [B, H, d_k, d_v] or None.
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    alpha, beta, h0 = _f64(alpha), _f64(beta), _f64(h0)
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    assert k.shape == q.shape and v.shape[:3] == q.shape[:3]
    for a in (alpha, beta):
        assert a is None or a.shape == (B, T, H)
    assert h0 is None or h0.shape == (B, H, dk, dv)
    o = np.zeros((B, T, H, dv))
    hT = np.zeros((B, H, dk, dv))
    _load().oracle_gated_delta_fwd(B, T, H, dk, dv, _ptr(q), _ptr(k), _ptr(v), _ptr(alpha),
                                   _ptr(beta), _ptr(h0), _ptr(o), _ptr(hT),
                                   _threads(nthreads))
    return o, hT


def precond_two_gate_fwd(q, k, v, alpha=None, erase=None, write=None, precond=True,
                         rho_decay=0.99, rho_eps=1e-6, h0=None, nthreads=None,
                         precond_x=2.0, precond_query=False):
    """Preconditioned write key, per-channel decay, erase/write channel gates.

    rho_t = rho_decay rho_{t-1} + k_t (.) k_t and a per-channel factor f(rho_t):
    precond 1 (or True) f = 1/sqrt(rho + eps); 2 f = 1/(rho + eps) (the pages'
    Diag(A_t)^-1); 3 the latter squashed into [1/precond_x, precond_x]; 0 (False)
    none.  ATK (precond_query False): kw = f k_t, read key e = b (.) kw for form 1,
    b (.) k_t for forms 2, 3.  ATQ: kw = k_t, e = b (.) k_t, o_t = S_t (f (.) q_t).
    S_t = S_{t-1}(diag(alpha_t) - e kw^T) + (w_t (.) v_t) kw^T;  o_t = S_t q_t.
    alpha, erase: [B, T, H, d_k]; write: [B, T, H, d_v]; each may be None (ones).
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    alpha, erase, write, h0 = _f64(alpha), _f64(erase), _f64(write), _f64(h0)
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    assert alpha is None or alpha.shape == (B, T, H, dk)
    assert erase is None or erase.shape == (B, T, H, dk)
    assert write is None or write.shape == (B, T, H, dv)
    assert h0 is None or h0.shape == (B, H, dk, dv)
    o = np.zeros((B, T, H, dv))
    hT = np.zeros((B, H, dk, dv))
    _load().oracle_precond_two_gate_fwd(B, T, H, dk, dv, _ptr(q), _ptr(k), _ptr(v),
                                        _ptr(alpha), _ptr(erase), _ptr(write),
                                        int(precond), float(rho_decay), float(rho_eps),
                                        float(precond_x), int(bool(precond_query)),
                                        _ptr(h0), _ptr(o), _ptr(hT), _threads(nthreads))
    return o, hT


def gated_delta_bwd(q, k, v, alpha=None, beta=None, h0=None, do=None, dhT=None,
                    nthreads=None):
    """Gradients of the gated delta rule by the token-by-token adjoint.

    ``do`` [B, T, H, d_v] is dL/do; ``dhT`` [B, H, d_k, d_v] (or None, meaning
    0) is dL/dh_T.  Returns a dict with ``dq``, ``dk`` [B, T, H, d_k], ``dv``
    [B, T, H, d_v], ``dalpha`` and ``dbeta`` [B, T, H] (None when the gate was
    None) and ``dh0`` [B, H, d_k, d_v] (dL/dh_0, also when h0 is None).
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    alpha, beta, h0 = _f64(alpha), _f64(beta), _f64(h0)
    do, dhT = _f64(do), _f64(dhT)
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    assert k.shape == q.shape and v.shape[:3] == q.shape[:3] and do.shape == v.shape
    for a in (alpha, beta):
        assert a is None or a.shape == (B, T, H)
    for s in (h0, dhT):
        assert s is None or s.shape == (B, H, dk, dv)
    out = dict(dq=np.zeros((B, T, H, dk)), dk=np.zeros((B, T, H, dk)),
               dv=np.zeros((B, T, H, dv)),
               dalpha=None if alpha is None else np.zeros((B, T, H)),
               dbeta=None if beta is None else np.zeros((B, T, H)),
               dh0=np.zeros((B, H, dk, dv)))
    _load().oracle_gated_delta_bwd(B, T, H, dk, dv, _ptr(q), _ptr(k), _ptr(v), _ptr(alpha),
                                   _ptr(beta), _ptr(h0), _ptr(do), _ptr(dhT),
                                   _ptr(out["dq"]), _ptr(out["dk"]), _ptr(out["dv"]),
                                   _ptr(out["dalpha"]), _ptr(out["dbeta"]), _ptr(out["dh0"]),
                                   _threads(nthreads))
    return out
