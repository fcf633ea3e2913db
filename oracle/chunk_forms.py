"""Intra-chunk pieces of the chunkwise gated delta rule, fp64 numpy.

Test infrastructure only (see the package docstring).

The pages (page 4: "Quando o 'Bom o Suficiente' e Otimo: Aproximacao de
Inversao de Matriz Baseada Apenas em Multiplicacao para Gated DeltaNet
Quantizado") define, per chunk of C tokens:

* the triangular inverse T = (I - A)^-1 with A strictly lower triangular, and
  the traditional way to get it, forward substitution with k - 1 sequential
  iterations (section "Declaracao do Problema");
* the truncated Neumann series T0 = sum_{n=0}^{N} A^n (section "Metodologia",
  item 1, with Lemma 3.1: A^n lives on and below the n-th subdiagonal);
* the structural diagonal mask M_ij = 1 if i - j <= N else 0 (item 2);
* the parallel residual correction E = I - (I - A) T0,
  T ~= T0 sum_{s=0}^{S} E^s (item 3).

The chunked forward below is the standard WY/UT rewrite of the token
recurrence (the pages name it but do not print it).  Reading used here: the
chunk system is (I + L) Delta = diag(beta) V - diag(beta e^g) K h with
L_ri = beta_r exp(g_r - g_i) (k_r . k_i) for i < r, so the pages' strictly
lower A is -L and T = (I - A)^-1 = (I + L)^-1.  Decay ratios are always
formed as exp(g_r - g_i) with r >= i (never as a quotient of cumulative
products, which underflow).
"""
from __future__ import annotations

from typing import Callable, Optional

import numpy as np


# ----------------------------------------------------------------- the inverse

def strictly_lower_A(K: np.ndarray, beta: np.ndarray, g: np.ndarray) -> np.ndarray:
    """A_ri = -beta_r exp(g_r - g_i) (k_r . k_i) for i < r, else 0.

    K: [C, d_k]; beta, g: [C] with g the in-chunk cumulative log decay.
    """
    C = K.shape[0]
    gram = K @ K.T
    r = np.arange(C)[:, None]
    i = np.arange(C)[None, :]
    below = i < r
    ratio = np.exp(np.where(below, g[:, None] - g[None, :], 0.0))
    return np.where(below, -beta[:, None] * ratio * gram, 0.0)


def inverse_forward_substitution(A: np.ndarray) -> np.ndarray:
    """T = (I - A)^-1 for strictly lower A by forward substitution.

    (I - A) T = I gives row r of T as e_r + sum_{i<r} A_ri T_i: k - 1
    sequential row iterations for a k x k matrix (page 4, "Declaracao do
    Problema").
    """
    k = A.shape[0]
    T = np.eye(k)
    for r in range(1, k):
        T[r] = T[r] + A[r, :r] @ T[:r]
    return T


def neumann_truncated(A: np.ndarray, N: int) -> np.ndarray:
    """T0 = sum_{n=0}^{N} A^n (page 4, "Metodologia", item 1)."""
    k = A.shape[0]
    term = np.eye(k)
    total = np.eye(k)
    for _ in range(N):
        term = term @ A
        total = total + term
    return total


def structural_mask(k: int, N: int) -> np.ndarray:
    """M_ij = 1 if i - j <= N else 0 (page 4, "Metodologia", item 2)."""
    i = np.arange(k)[:, None]
    j = np.arange(k)[None, :]
    return (i - j <= N).astype(np.float64)


def masked_neumann(A: np.ndarray, N: int) -> np.ndarray:
    """M^(N) (.) sum_{n<=N} A^n: the truncated series with the mask applied."""
    return structural_mask(A.shape[0], N) * neumann_truncated(A, N)


def residual_correction(A: np.ndarray, T0: np.ndarray, S: int) -> np.ndarray:
    """E = I - (I - A) T0;  T ~= T0 sum_{s=0}^{S} E^s (page 4, item 3)."""
    k = A.shape[0]
    I = np.eye(k)
    E = I - (I - A) @ T0
    power = np.eye(k)
    acc = np.eye(k)
    for _ in range(S):
        power = power @ E
        acc = acc + power
    return T0 @ acc


def exact_inverse(A: np.ndarray) -> np.ndarray:
    return inverse_forward_substitution(A)


def neumann_inverse(N: int) -> Callable[[np.ndarray], np.ndarray]:
    return lambda A: masked_neumann(A, N)


def residual_inverse(N: int, S: int, masked: bool = True) -> Callable[[np.ndarray], np.ndarray]:
    def f(A):
        T0 = masked_neumann(A, N) if masked else neumann_truncated(A, N)
        return residual_correction(A, T0, S)
    return f


# ------------------------------------------------------------ chunked forward

def _f64(x):
    if x is None:
        return None
    if hasattr(x, "detach"):
        x = x.detach().to("cpu").double().numpy()
    return np.asarray(x, dtype=np.float64)


def chunked_gated_delta_fwd(q, k, v, alpha=None, beta=None, h0=None, chunk: int = 64,
                            inverse: Callable[[np.ndarray], np.ndarray] = exact_inverse):
    """Chunkwise WY form of the gated delta rule with a pluggable inverse.

    With ``inverse=exact_inverse`` this equals the token recurrence up to
    rounding; with ``neumann_inverse(N)`` it is the exact model of the
    truncated, masked Neumann approximation.  Per chunk (local rows r):

      g_r   = sum_{i<=r} log alpha_i
      A     = strictly_lower_A(K, beta, g);  T = inverse(A)
      U     = T diag(beta) V;  W = T diag(beta e^g) K;  Delta = U - W h
      O     = diag(e^g) Q h + [(Q K^T) (.) exp(g_r - g_i) (.) 1_{i<=r}] Delta
      h    <- e^{g_last} h + (diag(e^{g_last - g}) K)^T Delta

    Shapes as in ``oracle.recurrent.gated_delta_fwd``; returns (o, h_T).
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    alpha, beta, h0 = _f64(alpha), _f64(beta), _f64(h0)
    B, Tn, H, dk = q.shape
    dv = v.shape[-1]
    o = np.zeros((B, Tn, H, dv))
    hT = np.zeros((B, H, dk, dv))
    for b in range(B):
        for hh in range(H):
            h = np.zeros((dk, dv)) if h0 is None else h0[b, hh].copy()
            for s in range(0, Tn, chunk):
                e = min(s + chunk, Tn)
                Q, K, V = q[b, s:e, hh], k[b, s:e, hh], v[b, s:e, hh]
                bet = np.ones(e - s) if beta is None else beta[b, s:e, hh]
                la = np.zeros(e - s) if alpha is None else np.log(alpha[b, s:e, hh])
                g = np.cumsum(la)
                A = strictly_lower_A(K, bet, g)
                Tm = inverse(A)
                U = Tm @ (bet[:, None] * V)
                W = Tm @ ((bet * np.exp(g))[:, None] * K)
                Delta = U - W @ h
                C = e - s
                r = np.arange(C)[:, None]
                i = np.arange(C)[None, :]
                causal = i <= r
                P = np.where(causal, (Q @ K.T) * np.exp(np.where(causal, g[:, None] - g[None, :], 0.0)), 0.0)
                o[b, s:e, hh] = np.exp(g)[:, None] * (Q @ h) + P @ Delta
                h = np.exp(g[-1]) * h + (np.exp(g[-1] - g)[:, None] * K).T @ Delta
            hT[b, hh] = h
    return o, hT


def preconditioned_write_keys(k, rho_decay=0.99, rho_eps=1e-6, precond=True):
    """kw_t = k_t / sqrt(rho_t + eps), rho_t = c rho_{t-1} + k_t (.) k_t, rho_0 = 0.

    k: [B, T, H, d_k].  Running (sequential) evaluation over the full sequence.
    """
    k = _f64(k)
    if not precond:
        return k.copy()
    B, Tn, H, dk = k.shape
    out = np.empty_like(k)
    rho = np.zeros((B, H, dk))
    for t in range(Tn):
        rho = rho_decay * rho + k[:, t] ** 2
        out[:, t] = k[:, t] / np.sqrt(rho + rho_eps)
    return out


def chunked_two_gate_fwd(q, k, v, alpha=None, erase=None, write=None, precond=True,
                         rho_decay=0.99, rho_eps=1e-6, h0=None, chunk: int = 64,
                         inverse: Callable[[np.ndarray], np.ndarray] = exact_inverse):
    """Chunkwise form of the preconditioned two-gate rule (per-channel decay).

    With kw the write key, e = b (.) kw the erase key, u = w (.) v and G_r the
    per-channel cumulative log decay (G_{-1} = 0 at the chunk start):

      A_ri  = -sum_c e_rc kw_ic exp(G_{r-1,c} - G_{i,c})  for i < r
      T     = inverse(A);  Delta = T (U - (E (.) e^{G_{r-1}}) h)
      O     = (Q (.) e^{G_r}) h + P Delta,
              P_ri = sum_c q_rc kw_ic exp(G_{r,c} - G_{i,c}) for i <= r
      h    <- diag(e^{G_last}) h + (kw (.) e^{G_last - G})^T Delta

    The erase acts on the undecayed previous state, as the update
    S_{t-1}(diag(alpha_t) - e_t kw_t^T) is written.
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    alpha, erase, write, h0 = _f64(alpha), _f64(erase), _f64(write), _f64(h0)
    B, Tn, H, dk = q.shape
    dv = v.shape[-1]
    kw_all = preconditioned_write_keys(k, rho_decay, rho_eps, precond)
    o = np.zeros((B, Tn, H, dv))
    hT = np.zeros((B, H, dk, dv))
    for b in range(B):
        for hh in range(H):
            h = np.zeros((dk, dv)) if h0 is None else h0[b, hh].copy()
            for s in range(0, Tn, chunk):
                e_ = min(s + chunk, Tn)
                C = e_ - s
                Q, V = q[b, s:e_, hh], v[b, s:e_, hh]
                KW = kw_all[b, s:e_, hh]
                Eg = KW * (1.0 if erase is None else erase[b, s:e_, hh])
                U = V * (1.0 if write is None else write[b, s:e_, hh])
                la = np.zeros((C, dk)) if alpha is None else np.log(alpha[b, s:e_, hh])
                G = np.cumsum(la, axis=0)                       # G_r
                Gp = np.vstack([np.zeros((1, dk)), G[:-1]])     # G_{r-1}
                A = np.zeros((C, C))
                P = np.zeros((C, C))
                for r in range(C):
                    for i in range(r):
                        A[r, i] = -np.sum(Eg[r] * KW[i] * np.exp(Gp[r] - G[i]))
                    for i in range(r + 1):
                        P[r, i] = np.sum(Q[r] * KW[i] * np.exp(G[r] - G[i]))
                Tm = inverse(A)
                Delta = Tm @ (U - (Eg * np.exp(Gp)) @ h)
                o[b, s:e_, hh] = (Q * np.exp(G)) @ h + P @ Delta
                h = np.exp(G[-1])[:, None] * h + (KW * np.exp(G[-1] - G)).T @ Delta
            hT[b, hh] = h
    return o, hT
