"""The per-chunk inverse T as the fused tensor-core kernel forms it
(gdn_debug_chunk_T), against the fp64 chunk pieces of the oracle.

For chunk n of sequence (b, h): A = -L with L_ri = beta_r e^{g_r - g_i}
(k_r . k_i) for i < r ("Quando o 'Bom o Suficiente' e Otimo ...", section
"Declaracao do Problema").  Exact mode must give T = (I - A)^-1 (checked
against forward substitution in fp64); Neumann mode the masked truncated
series M^(N) (.) sum_{n<=N} A^n (section "Metodologia", items 1 and 2).
The error of the truncation itself, max |T_N - T|, is reported.  Tolerance:
the kernel works in fp32 from the bf16 keys, so 2e-4 * max(1, max |T|).
"""
import numpy as np
import pytest
import torch

import chunked_gated_delta_14_b200 as gdn
from chunked_gated_delta_14_b200.inputs import make_inputs, workload
from oracle import chunk_forms as cf

from gpu_util import report

pytestmark = pytest.mark.gpu

needs_cuda = pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")


def _chunk_A(x, b, h, n):
    k = x["k"].double().numpy()[b, 64 * n:64 * (n + 1), h]
    C = k.shape[0]
    beta = np.ones(C) if x["beta"] is None else x["beta"].double().numpy()[b, 64 * n:64 * n + C, h]
    la = np.zeros(C) if x["alpha"] is None else np.log(x["alpha"].double().numpy()[b, 64 * n:64 * n + C, h])
    return cf.strictly_lower_A(k, beta, np.cumsum(la))


def _gpu_T(x, b, h, n, mode, N=3):
    d = {k: (None if v is None else v.cuda()) for k, v in x.items()}
    Tg = gdn.debug_chunk_T(d["q"], d["k"], d["v"], d["alpha"], d["beta"], b=b, h=h, n=n, mode=mode, N=N,
                           S0=d["S0"])
    torch.cuda.synchronize()
    gdn.device_check()
    return Tg.double().cpu().numpy()


def _compare(Tg, Tref):
    C = Tref.shape[0]
    tol = 2e-4 * max(1.0, float(np.abs(Tref).max()))
    err = float(np.abs(Tg[:C, :C] - Tref).max())
    assert err <= tol, (err, tol)
    if C < 64:      # rows and columns past the tail chunk: the identity
        pad = Tg.copy()
        pad[:C, :C] = np.eye(C)
        assert np.array_equal(pad, np.eye(64))
    return err


CASES = [("strong", dict(decay="scalar"), 0, 1, 3),
         ("weak", dict(decay="weak"), 1, 2, 5),
         ("unit_decay_beta", dict(decay="none", beta=False), 0, 0, 2),
         ("tail", dict(decay="weak", T=6 * 64 + 17), 1, 1, 6)]


@needs_cuda
@pytest.mark.parametrize("name,over,b,h,n", CASES, ids=[c[0] for c in CASES])
def test_exact_T_matches_forward_substitution(name, over, b, h, n):
    over = dict(over)
    w = workload("gdn_bf16", B=2, H=3, T=over.pop("T", 512), s0_std=0.02, **over)
    x = make_inputs(w, seed=60)
    A = _chunk_A(x, b, h, n)
    Tref = cf.inverse_forward_substitution(A)
    # the oracle's own pin: T (I - A) = I
    assert np.abs(Tref @ (np.eye(A.shape[0]) - A) - np.eye(A.shape[0])).max() < 1e-10
    err = _compare(_gpu_T(x, b, h, n, "exact"), Tref)
    report(f"debug_T_exact_{name}", max_abs_err=err, max_abs_T=float(np.abs(Tref).max()))


@needs_cuda
@pytest.mark.parametrize("N", [2, 3, 4])
@pytest.mark.parametrize("name,over,b,h,n", CASES, ids=[c[0] for c in CASES])
def test_neumann_T_matches_masked_series(name, over, b, h, n, N):
    over = dict(over)
    w = workload("gdn_bf16", B=2, H=3, T=over.pop("T", 512), s0_std=0.02, **over)
    x = make_inputs(w, seed=60)
    A = _chunk_A(x, b, h, n)
    Tn_ref = cf.masked_neumann(A, N)
    Tg = _gpu_T(x, b, h, n, "neumann", N)
    err = _compare(Tg, Tn_ref)
    T_exact = cf.inverse_forward_substitution(A)
    C = A.shape[0]
    trunc = float(np.abs(Tg[:C, :C] - T_exact).max())
    # band identity: inside the band the truncated series is the exact inverse
    band = np.tril(np.triu(np.ones((C, C)), -N))
    assert np.abs((Tg[:C, :C] - T_exact) * band).max() <= 2e-4 * max(1.0, float(np.abs(T_exact).max()))
    report(f"debug_T_neumann_{name}_N{N}", max_abs_err=err, truncation_max_abs=trunc)
