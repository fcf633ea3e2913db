"""The backward kernels' source, compiled for the host and run on CPU threads,
against the fp64 adjoint oracle (CPU only; no GPU and no CUDA toolchain).

This checks the kernels' index arithmetic and algebra before any of it runs on
a GPU: tests/host_sim/ compiles csrc/gdn_bwd_kernels.cuh with g++ against a
small shim for the CUDA keywords it uses, runs every block with one thread per
CUDA thread and a barrier for __syncthreads, fills shared memory and the
workspace with NaN, and checks that no block wrote past its shared memory.
It is test infrastructure: the library never runs its kernels this way, and
the GPU parity tests (tests/test_parity_gpu_bwd.py) remain the parity claim.
The shapes cover every d_k template, chunks 16/32/64, d_v 32/96/128, ragged
tails, T = 1, absent gates and states, and bf16 inputs.
"""
import ctypes
import os
import subprocess

import numpy as np
import pytest
import torch

from oracle import chunk_grad as cg
from oracle import recurrent as rec

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(os.path.dirname(HERE), "chunked_gated_delta_14_b200", "csrc")
SIM = os.path.join(HERE, "host_sim")


@pytest.fixture(scope="module")
def host_lib(tmp_path_factory):
    out = tmp_path_factory.mktemp("host_sim") / "libbwd_host.so"
    subprocess.check_call(["g++", "-O2", "-std=c++20", "-shared", "-fPIC", "-w", "-include",
                           os.path.join(SIM, "cuda_host_shim.h"), "-I", SIM, "-I", CSRC,
                           os.path.join(SIM, "bwd_host_harness.cpp"), "-o", str(out), "-lpthread"])
    return ctypes.CDLL(str(out))


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _bf16(x):
    return x.to(torch.bfloat16)


CASES = [  # B, T, H, dk, dv, C, gates, S0 and dS_T, bf16 inputs
    (1, 70, 2, 16, 32, 16, True, True, False),
    (1, 100, 1, 32, 96, 32, False, True, False),
    (2, 130, 1, 64, 32, 64, True, False, False),
    (1, 77, 1, 128, 128, 64, True, True, True),
    (2, 1, 2, 128, 64, 64, True, True, False),
]


NEUMANN_CASES = [  # ..., N: the masked truncated series of order N as the chunk inverse
    (1, 70, 2, 16, 32, 16, True, True, False, 2),
    (1, 100, 1, 32, 96, 32, True, True, False, 3),
    (1, 77, 1, 128, 128, 64, True, True, True, 4),
    (2, 130, 1, 64, 32, 64, False, False, False, 1),
    (1, 64, 1, 32, 32, 64, True, True, False, 63),
    (1, 9, 1, 16, 32, 16, True, True, False, 2),        # one partial chunk: T < C
]

RESIDUAL_CASES = [  # ..., N, S: the masked series of order N with S correction terms
    (1, 70, 2, 16, 32, 16, True, True, False, 1, 2),
    (1, 77, 1, 128, 128, 64, True, True, True, 3, 8),
    (1, 100, 1, 32, 64, 32, True, False, False, 2, 1),
    (1, 64, 1, 32, 32, 64, True, True, False, 1, 31),
    (1, 5, 1, 16, 32, 32, True, True, False, 1, 1),     # one partial chunk: T < C
    (1, 64, 1, 16, 32, 16, True, True, False, 0, 3),    # N = 0: T0 = I, E = I + L
]


@pytest.mark.parametrize("B,T,H,dk,dv,C,gates,state,bf16", CASES)
def test_backward_kernel_source_on_host(host_lib, B, T, H, dk, dv, C, gates, state, bf16):
    _run_case(host_lib, B, T, H, dk, dv, C, gates, state, bf16, None)


@pytest.mark.parametrize("B,T,H,dk,dv,C,gates,state,bf16,N", NEUMANN_CASES)
def test_backward_kernel_source_on_host_masked_series(host_lib, B, T, H, dk, dv, C, gates, state, bf16, N):
    """The gradient of the forward with the masked truncated series as the chunk
    inverse, against the fp64 autograd of the chunk model (N = C - 1: exact)."""
    _run_case(host_lib, B, T, H, dk, dv, C, gates, state, bf16, N)


@pytest.mark.parametrize("B,T,H,dk,dv,C,gates,state,bf16,N,S", RESIDUAL_CASES)
def test_backward_kernel_source_on_host_residual(host_lib, B, T, H, dk, dv, C, gates, state, bf16, N, S):
    """The gradient of the forward with the residual-corrected series, against the
    fp64 autograd of that chunk model ((N + 1)(S + 1) = C: exact)."""
    _run_case(host_lib, B, T, H, dk, dv, C, gates, state, bf16, N, S)


def _run_case(host_lib, B, T, H, dk, dv, C, gates, state, bf16, N, S=0):
    g = torch.Generator().manual_seed(B * 1000 + T)
    def nrm(*s):
        return torch.randn(*s, generator=g)
    q = torch.nn.functional.normalize(nrm(B, T, H, dk), dim=-1)
    k = torch.nn.functional.normalize(nrm(B, T, H, dk), dim=-1)
    v, do = nrm(B, T, H, dv), nrm(B, T, H, dv)
    alpha = torch.rand(B, T, H, generator=g) * 0.7 + 0.3 if gates else None
    beta = torch.rand(B, T, H, generator=g) * 0.8 + 0.1 if gates else None
    S0 = 0.3 * nrm(B, H, dk, dv) if state else None
    dS = nrm(B, H, dk, dv) if state else None
    if bf16:   # the oracle sees exactly the values the kernels read
        q, k, v, do = (_bf16(t) for t in (q, k, v, do))
    nan = lambda *s: torch.full(s, float("nan"))
    gq, gk, gv, gS0 = nan(B, T, H, dk), nan(B, T, H, dk), nan(B, T, H, dv), nan(B, H, dk, dv)
    ga = nan(B, T, H) if gates else None
    gb = nan(B, T, H) if gates else None
    rc = host_lib.host_bwd(B, T, H, dk, dv, C, int(bf16), int(bf16), _p(q), _p(k), _p(v), _p(alpha),
                           _p(beta), _p(S0), _p(do), _p(dS), _p(gq), _p(gk), _p(gv), _p(ga), _p(gb),
                           _p(gS0), ctypes.c_int(0 if N is None else 1), ctypes.c_int(N or 0), ctypes.c_int(S))
    assert rc == 0, f"a block wrote past its shared memory ({rc - 100} blocks)" if rc >= 100 else rc
    if N is None:
        ref = rec.gated_delta_bwd(q, k, v, alpha, beta, S0, do, dS)
    else:
        ref = cg.neumann_bwd(q, k, v, alpha, beta, S0, do, dS, chunk=C, N=N, S=S if S else None)
    for name, got in (("dq", gq), ("dk", gk), ("dv", gv), ("dalpha", ga), ("dbeta", gb), ("dh0", gS0)):
        if ref[name] is None:
            continue
        got = got.double().numpy()
        assert np.isfinite(got).all(), name
        err = np.abs(got - ref[name]).max() / np.sqrt(np.mean(ref[name] ** 2))
        assert err <= 1e-4, (name, err)
