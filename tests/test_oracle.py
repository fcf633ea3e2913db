"""Pins for the fp64 oracle: facts fixed by the pages and by mathematics.

Every check compares the oracle with something computed a different way
(explicit matrix products, closed forms, special cases that reduce to a
textbook result or a library routine, a hand-worked example), so that a
dropped term, a wrong sign or index, or a transposed operand fails one.
"""
import json
import os

import numpy as np
import pytest

from oracle import chunk_forms as cf
from oracle import recurrent as rec
from chunked_gated_delta_14_b200.inputs import make_inputs, workload

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rand(rng, *shape):
    return rng.standard_normal(shape)


def _unit(x):
    return x / np.linalg.norm(x, axis=-1, keepdims=True)


def _small_inputs(rng, B=1, T=5, H=2, dk=3, dv=4, with_h0=True):
    q = _unit(_rand(rng, B, T, H, dk))
    k = _unit(_rand(rng, B, T, H, dk))
    v = _rand(rng, B, T, H, dv)
    alpha = np.exp(-np.logaddexp(0, _rand(rng, B, T, H) + 1))
    beta = 1 / (1 + np.exp(-_rand(rng, B, T, H)))
    h0 = 0.3 * _rand(rng, B, H, dk, dv) if with_h0 else None
    return q, k, v, alpha, beta, h0


# --------------------------------------------------------- hand-worked example

def test_hand_worked_two_tokens():
    g = json.load(open(os.path.join(GOLDEN, "hand_worked_two_tokens.json")))
    x = {kk: np.array(vv, dtype=np.float64) for kk, vv in g["inputs"].items()}
    o, hT = rec.gated_delta_fwd(x["q"], x["k"], x["v"], x["alpha"], x["beta"])
    np.testing.assert_allclose(o, np.array(g["expected"]["o"]), rtol=0, atol=1e-14)
    np.testing.assert_allclose(hT, np.array(g["expected"]["h_T"]), rtol=0, atol=1e-14)


# ------------------------------------------- brute force by transition products

def _brute_force_gdn(q, k, v, alpha, beta, h0):
    """S_t = S_0 M_1..M_t + sum_i beta_i v_i k_i^T M_{i+1}..M_t, M = alpha(I - beta k k^T)."""
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    o = np.zeros((B, T, H, dv))
    hT = np.zeros((B, H, dk, dv))
    I = np.eye(dk)
    for b in range(B):
        for h in range(H):
            M = [alpha[b, t, h] * (I - beta[b, t, h] * np.outer(k[b, t, h], k[b, t, h]))
                 for t in range(T)]
            S0 = h0[b, h].T if h0 is not None else np.zeros((dv, dk))
            for t in range(T):
                prod = lambda a, z: (np.linalg.multi_dot([I] + M[a:z] + [I]))
                S = S0 @ prod(0, t + 1)
                for i in range(t + 1):
                    S = S + beta[b, i, h] * np.outer(v[b, i, h], k[b, i, h]) @ prod(i + 1, t + 1)
                o[b, t, h] = S @ q[b, t, h]
            hT[b, h] = S.T
    return o, hT


@pytest.mark.parametrize("dk,dv,T", [(3, 4, 5), (4, 3, 6), (4, 4, 1)])
def test_gdn_matches_transition_products(dk, dv, T):
    rng = np.random.default_rng(1)
    q, k, v, alpha, beta, h0 = _small_inputs(rng, B=2, T=T, H=2, dk=dk, dv=dv)
    o, hT = rec.gated_delta_fwd(q, k, v, alpha, beta, h0)
    ob, hb = _brute_force_gdn(q, k, v, alpha, beta, h0)
    np.testing.assert_allclose(o, ob, rtol=0, atol=1e-12)
    np.testing.assert_allclose(hT, hb, rtol=0, atol=1e-12)


def test_two_gate_matches_transition_products():
    rng = np.random.default_rng(2)
    B, T, H, dk, dv = 1, 6, 2, 4, 3
    q, k, v, _, _, h0 = _small_inputs(rng, B, T, H, dk, dv)
    alpha = np.exp(-np.logaddexp(0, _rand(rng, B, T, H, dk) + 1))
    erase = 1 / (1 + np.exp(-_rand(rng, B, T, H, dk)))
    write = 1 / (1 + np.exp(-_rand(rng, B, T, H, dv)))
    o, hT = rec.precond_two_gate_fwd(q, k, v, alpha, erase, write, precond=True,
                                     rho_decay=0.9, rho_eps=1e-3, h0=h0)
    # write keys from the closed form rho_t = sum_{i<=t} c^{t-i} k_i^2
    for b in range(B):
        for h in range(H):
            S = h0[b, h].T.copy()
            for t in range(T):
                rho = sum(0.9 ** (t - i) * k[b, i, h] ** 2 for i in range(t + 1))
                kw = k[b, t, h] / np.sqrt(rho + 1e-3)
                M = np.diag(alpha[b, t, h]) - np.outer(erase[b, t, h] * kw, kw)
                S = S @ M + np.outer(write[b, t, h] * v[b, t, h], kw)
                np.testing.assert_allclose(o[b, t, h], S @ q[b, t, h], rtol=0, atol=1e-12)
            np.testing.assert_allclose(hT[b, h], S.T, rtol=0, atol=1e-12)


# ------------------------------------------------------------- special cases

def test_identity_state_when_alpha_one_beta_zero():
    rng = np.random.default_rng(3)
    q, k, v, _, _, h0 = _small_inputs(rng, B=2, T=7, H=3, dk=5, dv=6)
    beta = np.zeros(q.shape[:3])
    o, hT = rec.gated_delta_fwd(q, k, v, None, beta, h0)
    np.testing.assert_allclose(hT, h0, rtol=0, atol=1e-15)
    np.testing.assert_allclose(o, np.einsum("bhkv,bthk->bthv", h0, q), rtol=0, atol=1e-14)
    # same for the two-gate rule: alpha = 1, erase = 0, write = 0
    z = np.zeros_like(q)
    o2, hT2 = rec.precond_two_gate_fwd(q, k, v, None, z, np.zeros_like(v), precond=True, h0=h0)
    np.testing.assert_allclose(hT2, h0, rtol=0, atol=1e-15)
    np.testing.assert_allclose(o2, o, rtol=0, atol=1e-14)


def test_associative_memory_with_orthonormal_keys():
    """alpha = beta = 1 and orthonormal keys: after writing, S k_i = v_i (delta rule)."""
    rng = np.random.default_rng(4)
    d = 8
    Qm, _ = np.linalg.qr(rng.standard_normal((d, d)))
    keys = Qm.T[:5]                        # 5 orthonormal keys
    T = 10
    k = np.zeros((1, T, 1, d))
    q = np.zeros((1, T, 1, d))
    v = rng.standard_normal((1, T, 1, 6))
    k[0, :5, 0] = keys                     # write 5 pairs
    k[0, 5:, 0] = keys[[2, 0, 4, 1, 3]]    # rewrite the same keys with new values
    q[0, :5, 0] = keys
    q[0, 5:, 0] = keys[[2, 0, 4, 1, 3]]
    o, _ = rec.gated_delta_fwd(q, k, v, None, np.ones((1, T, 1)))
    np.testing.assert_allclose(o[0, :, 0], v[0, :, 0], rtol=0, atol=1e-12)


def test_linear_attention_reduction():
    """erase = 0, no preconditioner, alpha = 1: o_t = sum_{i<=t} (w_i v_i)(k_i . q_t)."""
    rng = np.random.default_rng(5)
    q, k, v, _, _, _ = _small_inputs(rng, B=2, T=9, H=2, dk=5, dv=4, with_h0=False)
    w = rng.uniform(size=v.shape)
    o, _ = rec.precond_two_gate_fwd(q, k, v, None, np.zeros_like(k), w, precond=False)
    scores = np.einsum("bthk,bshk->bhts", q, k)
    causal = np.tril(np.ones((9, 9)))
    expect = np.einsum("bhts,bshv->bthv", scores * causal, w * v)
    np.testing.assert_allclose(o, expect, rtol=0, atol=1e-12)


def test_two_gate_reduces_to_gated_delta():
    """alpha_t 1, erase gate alpha_t beta_t, write gate beta_t, no preconditioner == GDN."""
    rng = np.random.default_rng(6)
    q, k, v, alpha, beta, h0 = _small_inputs(rng, B=2, T=11, H=2, dk=6, dv=5)
    o, hT = rec.gated_delta_fwd(q, k, v, alpha, beta, h0)
    a_ch = np.repeat(alpha[..., None], 6, axis=-1)
    er = np.repeat((alpha * beta)[..., None], 6, axis=-1)
    wr = np.repeat(beta[..., None], 5, axis=-1)
    o2, hT2 = rec.precond_two_gate_fwd(q, k, v, a_ch, er, wr, precond=False, h0=h0)
    np.testing.assert_allclose(o2, o, rtol=0, atol=1e-12)
    np.testing.assert_allclose(hT2, hT, rtol=0, atol=1e-12)


def test_preconditioner_scan_closed_form():
    """No erase, alpha = 1, write = 1, one-hot values: row t of S_T is the write key kw_t."""
    rng = np.random.default_rng(7)
    T, dk = 6, 5
    k = rng.standard_normal((1, T, 1, dk))
    q = np.zeros_like(k)
    v = np.eye(T).reshape(1, T, 1, T)
    _, hT = rec.precond_two_gate_fwd(q, k, v, None, np.zeros_like(k), None, precond=True,
                                     rho_decay=0.99, rho_eps=1e-6)
    for t in range(T):
        rho = sum(0.99 ** (t - i) * k[0, i, 0] ** 2 for i in range(t + 1))
        np.testing.assert_allclose(hT[0, 0][:, t], k[0, t, 0] / np.sqrt(rho + 1e-6),
                                   rtol=1e-13, atol=0)


def test_linearity_in_values_and_initial_state():
    rng = np.random.default_rng(8)
    q, k, v1, alpha, beta, h01 = _small_inputs(rng, B=1, T=8, H=2, dk=4, dv=3)
    v2 = _rand(rng, *v1.shape)
    h02 = _rand(rng, *h01.shape)
    a, c = 0.7, -1.3
    o1, s1 = rec.gated_delta_fwd(q, k, v1, alpha, beta, h01)
    o2, s2 = rec.gated_delta_fwd(q, k, v2, alpha, beta, h02)
    o3, s3 = rec.gated_delta_fwd(q, k, a * v1 + c * v2, alpha, beta, a * h01 + c * h02)
    np.testing.assert_allclose(o3, a * o1 + c * o2, rtol=0, atol=1e-12)
    np.testing.assert_allclose(s3, a * s1 + c * s2, rtol=0, atol=1e-12)


# ------------------------------------------------------ intra-chunk inverse

def _chunk_A(rng, C=16, dk=8, alpha_one=False):
    K = _unit(rng.standard_normal((C, dk)))
    beta = 1 / (1 + np.exp(-rng.standard_normal(C)))
    la = np.zeros(C) if alpha_one else -np.logaddexp(0, rng.standard_normal(C) + 2)
    return cf.strictly_lower_A(K, beta, np.cumsum(la)), K, beta, np.cumsum(la)


def test_A_entries_from_definition():
    rng = np.random.default_rng(9)
    A, K, beta, g = _chunk_A(rng, C=7, dk=5)
    for r in range(7):
        for i in range(7):
            want = -beta[r] * np.prod(np.exp(np.diff(g)[i:r])) * K[r] @ K[i] if i < r else 0.0
            assert abs(A[r, i] - want) < 1e-14


@pytest.mark.parametrize("alpha_one", [False, True])
def test_forward_substitution_inverse(alpha_one):
    rng = np.random.default_rng(10)
    A, *_ = _chunk_A(rng, C=64, dk=16, alpha_one=alpha_one)
    T = cf.inverse_forward_substitution(A)
    I = np.eye(64)
    np.testing.assert_allclose(T @ (I - A), I, rtol=0, atol=1e-12)
    np.testing.assert_allclose((I - A) @ T, I, rtol=0, atol=1e-12)
    np.testing.assert_allclose(T, np.linalg.inv(I - A), rtol=0, atol=1e-12)
    assert np.all(np.triu(T, 1) == 0) and np.all(np.diag(T) == 1)


def test_lemma_3_1_banding_and_nilpotency():
    rng = np.random.default_rng(11)
    C = 32
    A, *_ = _chunk_A(rng, C=C, dk=8, alpha_one=True)
    P = np.eye(C)
    for n in range(1, C + 1):
        P = P @ A
        i = np.arange(C)[:, None]
        j = np.arange(C)[None, :]
        assert np.all(P[(i - j) < n] == 0), n
    assert np.all(P == 0)  # A^C = 0


@pytest.mark.parametrize("C", [16, 64])
def test_neumann_exact_at_C_minus_1(C):
    rng = np.random.default_rng(12)
    A, *_ = _chunk_A(rng, C=C, dk=16, alpha_one=True)
    T = cf.inverse_forward_substitution(A)
    np.testing.assert_allclose(cf.neumann_truncated(A, C - 1), T, rtol=0, atol=1e-10)
    # one term short is not exact for a dense strictly lower A
    assert np.abs(cf.neumann_truncated(A, C - 2) - T).max() > 0


def test_structural_mask_definition():
    M = cf.structural_mask(6, 2)
    want = np.array([[1 if i - j <= 2 else 0 for j in range(6)] for i in range(6)])
    np.testing.assert_array_equal(M, want)


@pytest.mark.parametrize("N", [1, 2, 3, 4])
def test_band_identity(N):
    """M (.) sum_{n<=N} A^n equals the exact inverse restricted to band N."""
    rng = np.random.default_rng(13)
    A, *_ = _chunk_A(rng, C=64, dk=16)
    T = cf.inverse_forward_substitution(A)
    band = T * cf.structural_mask(64, N)
    np.testing.assert_allclose(cf.masked_neumann(A, N), band, rtol=0, atol=1e-15)


@pytest.mark.parametrize("N,S", [(1, 2), (3, 8), (2, 3)])
def test_residual_correction_closed_forms(N, S):
    rng = np.random.default_rng(14)
    C = 64
    A, *_ = _chunk_A(rng, C=C, dk=16, alpha_one=True)
    # unmasked: E = A^{N+1}, so T0 sum E^s = sum_{m < (N+1)(S+1)} A^m
    got = cf.residual_correction(A, cf.neumann_truncated(A, N), S)
    want = cf.neumann_truncated(A, (N + 1) * (S + 1) - 1)
    np.testing.assert_allclose(got, want, rtol=1e-10, atol=1e-10)
    # masked: exact once (N+1)(S+1) >= C
    T = cf.inverse_forward_substitution(A)
    masked = cf.residual_correction(A, cf.masked_neumann(A, N), S)
    if (N + 1) * (S + 1) >= C:
        np.testing.assert_allclose(masked, T, rtol=1e-10, atol=1e-10)
    else:
        assert np.abs(masked - T).max() > 1e-12


def test_residual_masked_exactness_threshold():
    rng = np.random.default_rng(15)
    C = 16
    A, *_ = _chunk_A(rng, C=C, dk=8, alpha_one=True)
    T = cf.inverse_forward_substitution(A)
    N, S = 3, 3  # (N+1)(S+1) = 16 = C
    np.testing.assert_allclose(cf.residual_correction(A, cf.masked_neumann(A, N), S), T,
                               rtol=1e-10, atol=1e-10)


# ---------------------------------------------- chunk form vs token recurrence

@pytest.mark.parametrize("chunk,T", [(4, 13), (16, 50), (64, 100), (64, 64)])
def test_chunked_equals_recurrent(chunk, T):
    rng = np.random.default_rng(16)
    q, k, v, alpha, beta, h0 = _small_inputs(rng, B=1, T=T, H=2, dk=8, dv=6)
    o, hT = rec.gated_delta_fwd(q, k, v, alpha, beta, h0)
    oc, hc = cf.chunked_gated_delta_fwd(q, k, v, alpha, beta, h0, chunk=chunk)
    np.testing.assert_allclose(oc, o, rtol=0, atol=1e-12)
    np.testing.assert_allclose(hc, hT, rtol=0, atol=1e-12)


def test_chunked_plain_delta_rule():
    rng = np.random.default_rng(17)
    q, k, v, _, beta, _ = _small_inputs(rng, B=1, T=40, H=1, dk=8, dv=8, with_h0=False)
    o, hT = rec.gated_delta_fwd(q, k, v, None, beta)
    oc, hc = cf.chunked_gated_delta_fwd(q, k, v, None, beta, None, chunk=16)
    np.testing.assert_allclose(oc, o, rtol=0, atol=1e-12)
    np.testing.assert_allclose(hc, hT, rtol=0, atol=1e-12)


def test_chunked_two_gate_equals_recurrent():
    rng = np.random.default_rng(18)
    B, T, H, dk, dv = 1, 37, 2, 6, 5
    q, k, v, _, _, h0 = _small_inputs(rng, B, T, H, dk, dv)
    alpha = np.exp(-np.logaddexp(0, _rand(rng, B, T, H, dk) + 2))
    erase = 1 / (1 + np.exp(-_rand(rng, B, T, H, dk)))
    write = 1 / (1 + np.exp(-_rand(rng, B, T, H, dv)))
    o, hT = rec.precond_two_gate_fwd(q, k, v, alpha, erase, write, True, 0.99, 1e-6, h0)
    oc, hc = cf.chunked_two_gate_fwd(q, k, v, alpha, erase, write, True, 0.99, 1e-6, h0,
                                     chunk=8)
    np.testing.assert_allclose(oc, o, rtol=0, atol=1e-11)
    np.testing.assert_allclose(hc, hT, rtol=0, atol=1e-11)


def test_state_chaining_equals_one_call():
    rng = np.random.default_rng(19)
    q, k, v, alpha, beta, h0 = _small_inputs(rng, B=1, T=30, H=2, dk=5, dv=4)
    o, hT = rec.gated_delta_fwd(q, k, v, alpha, beta, h0)
    oa, ha = rec.gated_delta_fwd(q[:, :11], k[:, :11], v[:, :11], alpha[:, :11], beta[:, :11], h0)
    ob, hb = rec.gated_delta_fwd(q[:, 11:], k[:, 11:], v[:, 11:], alpha[:, 11:], beta[:, 11:], ha)
    np.testing.assert_allclose(np.concatenate([oa, ob], axis=1), o, rtol=0, atol=1e-13)
    np.testing.assert_allclose(hb, hT, rtol=0, atol=1e-13)


def test_neumann_chunk_model_error_shrinks_with_N():
    """Reported, not gated by the pages: the error vs exact falls as N grows."""
    rng = np.random.default_rng(20)
    q, k, v, alpha, beta, _ = _small_inputs(rng, B=1, T=128, H=1, dk=16, dv=8, with_h0=False)
    ox, _ = cf.chunked_gated_delta_fwd(q, k, v, alpha, beta, chunk=64)
    errs = []
    for N in (1, 2, 3, 4):
        on, _ = cf.chunked_gated_delta_fwd(q, k, v, alpha, beta, chunk=64,
                                           inverse=cf.neumann_inverse(N))
        errs.append(np.abs(on - ox).max())
    assert all(errs[i + 1] < errs[i] for i in range(3)), errs
    on, _ = cf.chunked_gated_delta_fwd(q, k, v, alpha, beta, chunk=64,
                                       inverse=cf.neumann_inverse(63))
    np.testing.assert_allclose(on, ox, rtol=0, atol=1e-12)


# --------------------------------------- page-form preconditioners (next row 3)

def _one_hot_stream(T=40, d=6, dv=3, seed=0):
    rng = np.random.default_rng(seed)
    idx = rng.integers(0, d, size=T)
    k = np.zeros((1, T, 1, d))
    k[0, np.arange(T), 0, idx] = 1.0
    v = rng.standard_normal((1, T, 1, dv))
    q = rng.standard_normal((1, T, 1, d))
    return idx, q, k, v


def test_diag_preconditioner_recovers_least_squares_for_one_hot_keys():
    """P_t = Diag(A_t)^-1 with A_t the plain sum of k (.) k: for orthogonal (one-hot)
    keys the Gram matrix is diagonal, so the preconditioned delta rule is the exact
    online least-squares solve: column i of S is the mean of the values written
    with key i (pages: exact preconditioning recovers the least-squares solution)."""
    idx, q, k, v = _one_hot_stream()
    o, hT = rec.precond_two_gate_fwd(q, k, v, precond=2, rho_decay=1.0, rho_eps=1e-12)
    T, d, dv = k.shape[1], k.shape[3], v.shape[3]
    sums, counts = np.zeros((d, dv)), np.zeros(d)
    for t in range(T):
        sums[idx[t]] += v[0, t, 0]
        counts[idx[t]] += 1
        means = np.where(counts[:, None] > 0, sums / np.maximum(counts, 1)[:, None], 0.0)
        np.testing.assert_allclose(o[0, t, 0], means.T @ q[0, t, 0], atol=1e-9)
    np.testing.assert_allclose(hT[0, 0], means, atol=1e-9)


def test_preconditioned_query_linear_attention_equals_preconditioned_key_deltanet():
    """ATQ (linear attention, no erase, preconditioner on the query) and ATK
    (delta rule, preconditioner on the write key) give the same outputs when the
    diagonal preconditioner is exact (one-hot keys)."""
    idx, q, k, v = _one_hot_stream(seed=1)
    zeros = np.zeros_like(k)
    o_atq, _ = rec.precond_two_gate_fwd(q, k, v, erase=zeros, precond=2, rho_decay=1.0,
                                           rho_eps=1e-12, precond_query=True)
    o_atk, _ = rec.precond_two_gate_fwd(q, k, v, precond=2, rho_decay=1.0, rho_eps=1e-12)
    np.testing.assert_allclose(o_atq, o_atk, atol=1e-9)


def test_squashed_preconditioner_bounds_and_monotone():
    """Form 3 keeps the factor in [1/x, x], equals 1 at rho = 1 and decreases with
    rho: read off S = v (f k)^T after one write with no erase (k = c e_0)."""
    x = 2.0
    fs = []
    for c in (0.05, 0.3, 1.0, 3.0, 20.0):
        k = np.zeros((1, 1, 1, 4)); k[0, 0, 0, 0] = c
        v = np.ones((1, 1, 1, 2))
        q = np.zeros((1, 1, 1, 4))
        _, hT = rec.precond_two_gate_fwd(q, k, v, erase=np.zeros_like(k), precond=3, rho_decay=1.0,
                                            rho_eps=0.0, precond_x=x)
        f = hT[0, 0, 0, 0] / c          # S column 0 = v f c
        fs.append(f)
        assert 1.0 / x - 1e-12 <= f <= x + 1e-12
    assert abs(fs[2] - 1.0) < 1e-12
    assert all(a > b for a, b in zip(fs, fs[1:]))


def test_squash_limits():
    """x -> infinity recovers Diag(A)^-1 (form 2); x -> 1 removes the preconditioner.
    eps = 1 keeps form 2's factor in (0, 1], where the log-scale squash with a huge
    x is linear to 1e-4 (with a tiny eps form 2 is the unstable case the squash
    exists for, and the recurrence amplifies any difference)."""
    w = workload("precond_two_gate", B=1, H=1, T=40, dk=8, dv=4)
    x = make_inputs(w, seed=3)
    args = dict(alpha=x["alpha"], erase=x["erase"], write=x["write"], rho_decay=1.0, rho_eps=1.0)
    o2, s2 = rec.precond_two_gate_fwd(x["q"], x["k"], x["v"], precond=2, **args)
    o3, s3 = rec.precond_two_gate_fwd(x["q"], x["k"], x["v"], precond=3, precond_x=1e60, **args)
    np.testing.assert_allclose(o3, o2, rtol=1e-3, atol=1e-6)
    o0, _ = rec.precond_two_gate_fwd(x["q"], x["k"], x["v"], precond=0, **args)
    o1, _ = rec.precond_two_gate_fwd(x["q"], x["k"], x["v"], precond=3, precond_x=1.0 + 1e-9, **args)
    np.testing.assert_allclose(o1, o0, atol=1e-7)
