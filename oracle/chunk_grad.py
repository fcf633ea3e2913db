"""Gradient of the chunked gated delta rule with the masked truncated Neumann
inverse, and with that series' residual correction, fp64 PyTorch on the CPU --
TEST INFRASTRUCTURE only.

The pages ("Quando o 'Bom o Suficiente' e Otimo: Aproximacao de Inversao de
Matriz Baseada Apenas em Multiplicacao para Gated DeltaNet Quantizado",
sections "Resumo" and "Declaracao do Problema") use the chunkwise form to make
training parallel, and replace the chunk inverse T = (I - A)^-1 by the masked
series M^(N) (.) sum_{n<=N} A^n ("Metodologia", items 1 and 2), optionally
followed by S terms of the parallel residual correction ("Metodologia", item 3).
With that replacement the model is no longer the token recurrence, so its
gradient is the gradient of the chunk model itself.  This module writes the chunk model
out once more, step by step in the same order as
``oracle.chunk_forms.chunked_gated_delta_fwd`` (whose fp64 numpy forward the
tests hold it to), in plain differentiable PyTorch ops, and takes the
gradient with reverse-mode automatic differentiation (a library primitive).
Nothing here is shared with the CUDA library.
"""
from __future__ import annotations

from typing import Optional

import numpy as np
import torch


def _t(x):
    if x is None:
        return None
    if isinstance(x, torch.Tensor):
        return x.detach().to("cpu", torch.float64).clone()
    return torch.as_tensor(np.asarray(x, dtype=np.float64))


def masked_neumann(A: torch.Tensor, N: int) -> torch.Tensor:
    """M^(N) (.) sum_{n=0}^{N} A^n, M_ij = [i - j <= N] (items 1 and 2)."""
    k = A.shape[0]
    eye = torch.eye(k, dtype=A.dtype)
    term, total = eye, eye
    for _ in range(N):
        term = term @ A
        total = total + term
    i = torch.arange(k)[:, None]
    j = torch.arange(k)[None, :]
    return torch.where(i - j <= N, total, torch.zeros_like(total))


def residual_corrected(A: torch.Tensor, N: int, S: int) -> torch.Tensor:
    """T0 sum_{s=0}^{S} E^s with T0 the masked series and E = I - (I - A) T0
    ("Metodologia", item 3)."""
    k = A.shape[0]
    eye = torch.eye(k, dtype=A.dtype)
    T0 = masked_neumann(A, N)
    E = eye - (eye - A) @ T0
    power, acc = eye, eye
    for _ in range(S):
        power = power @ E
        acc = acc + power
    return T0 @ acc


def chunk_model(q, k, v, log_alpha, beta, h0, chunk: int, N: int, S: Optional[int] = None):
    """o [B, T, H, dv] and h_T [B, H, dk, dv] of the chunked form with the masked
    series of order N as the chunk inverse (with S residual-correction terms when S
    is given); every input a float64 tensor (log_alpha and beta [B, T, H], h0
    [B, H, dk, dv])."""
    B, Tn, H, dk = q.shape
    dv = v.shape[-1]
    outs, finals = [], []
    for b in range(B):
        o_h, f_h = [], []
        for hh in range(H):
            h = h0[b, hh]
            rows = []
            for s in range(0, Tn, chunk):
                e = min(s + chunk, Tn)
                C = e - s
                Q, K, V = q[b, s:e, hh], k[b, s:e, hh], v[b, s:e, hh]
                bet = beta[b, s:e, hh]
                g = torch.cumsum(log_alpha[b, s:e, hh], 0)
                r = torch.arange(C)[:, None]
                i = torch.arange(C)[None, :]
                below, causal = i < r, i <= r
                diff = g[:, None] - g[None, :]
                # A_ri = -beta_r e^{g_r - g_i} (k_r . k_i), i < r
                A = torch.where(below, -bet[:, None] * torch.exp(torch.where(below, diff, 0.0 * diff)) * (K @ K.T),
                                torch.zeros(C, C, dtype=q.dtype))
                Tm = masked_neumann(A, N) if S is None else residual_corrected(A, N, S)
                U = Tm @ (bet[:, None] * V)
                W = Tm @ ((bet * torch.exp(g))[:, None] * K)
                Delta = U - W @ h
                P = torch.where(causal, (Q @ K.T) * torch.exp(torch.where(causal, diff, 0.0 * diff)),
                                torch.zeros(C, C, dtype=q.dtype))
                rows.append(torch.exp(g)[:, None] * (Q @ h) + P @ Delta)
                h = torch.exp(g[-1]) * h + (torch.exp(g[-1] - g)[:, None] * K).T @ Delta
            o_h.append(torch.cat(rows, 0))
            f_h.append(h)
        outs.append(torch.stack(o_h, 1))
        finals.append(torch.stack(f_h, 0))
    return torch.stack(outs, 0), torch.stack(finals, 0)


def neumann_fwd(q, k, v, alpha=None, beta=None, h0=None, chunk: int = 64, N: int = 3, S: Optional[int] = None):
    """(o, h_T) as float64 numpy arrays."""
    q, k, v = _t(q), _t(k), _t(v)
    B, Tn, H, dk = q.shape
    dv = v.shape[-1]
    la = torch.zeros(B, Tn, H, dtype=torch.float64) if alpha is None else torch.log(_t(alpha))
    bt = torch.ones(B, Tn, H, dtype=torch.float64) if beta is None else _t(beta)
    hz = torch.zeros(B, H, dk, dv, dtype=torch.float64) if h0 is None else _t(h0)
    with torch.no_grad():
        o, hT = chunk_model(q, k, v, la, bt, hz, chunk, N, S)
    return o.numpy(), hT.numpy()


def neumann_bwd(q, k, v, alpha=None, beta=None, h0=None, do=None, dhT=None, chunk: int = 64, N: int = 3,
                S: Optional[int] = None):
    """Gradients of L = <o, do> + <h_T, dhT> through the masked-series chunk model
    (with S residual-correction terms when S is given):
    a dict with dq, dk, dv, dalpha, dbeta (None when that gate is None) and dh0,
    float64 numpy arrays in the layouts of the inputs."""
    q, k, v = _t(q), _t(k), _t(v)
    B, Tn, H, dk = q.shape
    dv = v.shape[-1]
    a = None if alpha is None else _t(alpha)
    bt = None if beta is None else _t(beta)
    hz = torch.zeros(B, H, dk, dv, dtype=torch.float64) if h0 is None else _t(h0)
    leaves = [q, k, v, hz] + [x for x in (a, bt) if x is not None]
    for x in leaves:
        x.requires_grad_(True)
    la = torch.zeros(B, Tn, H, dtype=torch.float64) if a is None else torch.log(a)
    bb = torch.ones(B, Tn, H, dtype=torch.float64) if bt is None else bt
    o, hT = chunk_model(q, k, v, la, bb, hz, chunk, N, S)
    loss = (o * _t(do)).sum()
    if dhT is not None:
        loss = loss + (hT * _t(dhT)).sum()
    loss.backward()
    g = lambda x: None if x is None else x.grad.numpy()
    return dict(dq=g(q), dk=g(k), dv=g(v), dalpha=g(a), dbeta=g(bt), dh0=g(hz))
