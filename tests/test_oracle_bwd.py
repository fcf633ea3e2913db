"""Pins for the oracle's gradient of the gated delta rule (CPU only).

The oracle's backward is the token-by-token adjoint written out by hand.  It
is pinned here against two things computed without it:

* central finite differences of the (already pinned) forward oracle, a brute
  force that knows nothing of the adjoint;
* reverse-mode automatic differentiation of a plain fp64 PyTorch loop over the
  tokens, an independent derivation of the same chain rule;

plus closed forms for the degenerate gates.  Together they catch a dropped
term, a wrong sign, a transposed state or a token off by one in any of the six
gradients, and the checkpoint boundary of the reverse sweep (T > 64).
"""
import numpy as np
import pytest
import torch

from oracle import recurrent as rec


def _inputs(rng, B=1, T=6, H=2, dk=3, dv=4, gates=True, h0=True):
    q = rng.standard_normal((B, T, H, dk))
    k = rng.standard_normal((B, T, H, dk))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((B, T, H, dv))
    alpha = rng.uniform(0.4, 1.0, (B, T, H)) if gates else None
    beta = rng.uniform(0.1, 0.95, (B, T, H)) if gates else None
    s0 = 0.5 * rng.standard_normal((B, H, dk, dv)) if h0 else None
    do = rng.standard_normal((B, T, H, dv))
    dhT = rng.standard_normal((B, H, dk, dv))
    return dict(q=q, k=k, v=v, alpha=alpha, beta=beta, h0=s0), do, dhT


def _loss(x, do, dhT):
    o, hT = rec.gated_delta_fwd(**x)
    return float((o * do).sum() + (hT * dhT).sum())


_GRAD = dict(q="dq", k="dk", v="dv", alpha="dalpha", beta="dbeta", h0="dh0")


def _finite_difference(x, do, dhT, name, idx, eps=1e-6):
    xp = dict(x)
    xp[name] = x[name].copy()
    xp[name][idx] += eps
    lp = _loss(xp, do, dhT)
    xp[name][idx] -= 2 * eps
    lm = _loss(xp, do, dhT)
    return (lp - lm) / (2 * eps)


@pytest.mark.parametrize("gates,h0", [(True, True), (True, False), (False, True)])
def test_adjoint_matches_finite_differences(gates, h0):
    rng = np.random.default_rng(3)
    x, do, dhT = _inputs(rng, gates=gates, h0=h0)
    g = rec.gated_delta_bwd(do=do, dhT=dhT, **x)
    if not gates:
        assert g["dalpha"] is None and g["dbeta"] is None
    for name, arr in x.items():
        if arr is None:
            continue
        fd = np.zeros_like(arr)
        for idx in np.ndindex(arr.shape):
            fd[idx] = _finite_difference(x, do, dhT, name, idx)
        np.testing.assert_allclose(g[_GRAD[name]], fd, rtol=0, atol=2e-8 * max(1.0, np.abs(fd).max()),
                                   err_msg=name)
    if not h0:
        # dh0 is still the gradient with respect to a zero initial state
        x0 = dict(x, h0=np.zeros((1, 2, 3, 4)))
        for idx in [(0, 0, 0, 0), (0, 1, 2, 3), (0, 1, 1, 0)]:
            assert abs(g["dh0"][idx] - _finite_difference(x0, do, dhT, "h0", idx)) < 1e-7


def test_adjoint_across_the_checkpoint_boundary_by_finite_differences():
    """T = 131 spans three 64-token segments of the reverse sweep: sampled
    entries of every gradient, on both sides of the segment boundaries."""
    rng = np.random.default_rng(4)
    x, do, dhT = _inputs(rng, T=131, H=1, dk=2, dv=3)
    x["alpha"] = rng.uniform(0.9, 1.0, x["alpha"].shape)   # keep early tokens visible
    g = rec.gated_delta_bwd(do=do, dhT=dhT, **x)
    for name in ("q", "k", "v", "alpha", "beta"):
        for t in (0, 62, 63, 64, 65, 127, 128, 130):
            idx = (0, t, 0) + ((1,) if x[name].ndim == 4 else ())
            fd = _finite_difference(x, do, dhT, name, idx)
            assert abs(g[_GRAD[name]][idx] - fd) < 1e-7 * max(1.0, abs(fd)), (name, t)
    fd = _finite_difference(x, do, dhT, "h0", (0, 0, 1, 2))
    assert abs(g["dh0"][0, 0, 1, 2] - fd) < 1e-7 * max(1.0, abs(fd))


def _torch_loop(q, k, v, alpha, beta, h0):
    """S_t = S_{t-1} alpha_t (I - beta_t k_t k_t^T) + beta_t v_t k_t^T, o_t = S_t q_t,
    one matrix expression per token (state d_v x d_k), for autograd."""
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    I = torch.eye(dk, dtype=torch.float64)
    outs, finals = [], []
    for b in range(B):
        for h in range(H):
            S = h0[b, h].T
            ob = []
            for t in range(T):
                kt = k[b, t, h]
                S = S @ (alpha[b, t, h] * (I - beta[b, t, h] * torch.outer(kt, kt))) \
                    + beta[b, t, h] * torch.outer(v[b, t, h], kt)
                ob.append(S @ q[b, t, h])
            outs.append(torch.stack(ob))
            finals.append(S.T)
    o = torch.stack(outs).reshape(B, H, T, dv).permute(0, 2, 1, 3)
    return o, torch.stack(finals).reshape(B, H, dk, dv)


@pytest.mark.parametrize("T", [1, 9, 70])
def test_adjoint_matches_autograd(T):
    rng = np.random.default_rng(5 + T)
    x, do, dhT = _inputs(rng, B=2, T=T, H=2, dk=4, dv=3)
    g = rec.gated_delta_bwd(do=do, dhT=dhT, **x)
    tx = {n: torch.tensor(a, requires_grad=True) for n, a in x.items()}
    o, hT = _torch_loop(**tx)
    loss = (o * torch.tensor(do)).sum() + (hT * torch.tensor(dhT)).sum()
    grads = torch.autograd.grad(loss, list(tx.values()))
    for (name, _), gr in zip(tx.items(), grads):
        np.testing.assert_allclose(g[_GRAD[name]], gr.numpy(), rtol=0, atol=1e-11, err_msg=name)


def test_zero_beta_is_pure_decay():
    """beta = 0 leaves S_t = (prod alpha) S_0: o_t = g_t h0^T q_t with g_t the
    running product, so dq_t = g_t h0 do_t, dv = dk = 0, dh0 = sum_t g_t q_t do_t^T
    + g_T dhT, and dbeta_t = du . (v_t - g_t h0^T k_t) with du = D_t k_t (the
    write residual against the decayed state)."""
    rng = np.random.default_rng(6)
    x, do, dhT = _inputs(rng, B=1, T=5, H=1, dk=3, dv=2)
    x["beta"] = np.zeros_like(x["beta"])
    g = rec.gated_delta_bwd(do=do, dhT=dhT, **x)
    a = x["alpha"][0, :, 0]
    cum = np.cumprod(a)
    h0 = x["h0"][0, 0]
    np.testing.assert_allclose(g["dv"], 0.0, atol=1e-15)
    np.testing.assert_allclose(g["dk"], 0.0, atol=1e-15)
    for t in range(5):
        np.testing.assert_allclose(g["dq"][0, t, 0], cum[t] * h0 @ do[0, t, 0], atol=1e-13)
    dh0 = sum(cum[t] * np.outer(x["q"][0, t, 0], do[0, t, 0]) for t in range(5)) + cum[-1] * dhT[0, 0]
    np.testing.assert_allclose(g["dh0"][0, 0], dh0, atol=1e-13)
    # D_t (as h-layout d_k x d_v) = sum_{s>=t} (cum_s / cum_t) q_s do_s^T + (cum_T / cum_t) dhT
    for t in range(5):
        D = sum(cum[s] / cum[t] * np.outer(x["q"][0, s, 0], do[0, s, 0]) for s in range(t, 5)) \
            + cum[-1] / cum[t] * dhT[0, 0]
        du = D.T @ x["k"][0, t, 0]
        resid = x["v"][0, t, 0] - cum[t] * h0.T @ x["k"][0, t, 0]
        np.testing.assert_allclose(g["dbeta"][0, t, 0], du @ resid, atol=1e-12)


def test_gradient_is_linear_in_the_cotangents():
    rng = np.random.default_rng(7)
    x, do1, dh1 = _inputs(rng)
    _, do2, dh2 = _inputs(np.random.default_rng(8))
    g1 = rec.gated_delta_bwd(do=do1, dhT=dh1, **x)
    g2 = rec.gated_delta_bwd(do=do2, dhT=dh2, **x)
    g12 = rec.gated_delta_bwd(do=do1 + 2 * do2, dhT=dh1 + 2 * dh2, **x)
    for n in ("dq", "dk", "dv", "dalpha", "dbeta", "dh0"):
        np.testing.assert_allclose(g12[n], g1[n] + 2 * g2[n], atol=1e-12, err_msg=n)


# ------------------------------------------- masked Neumann series (chunk model)

from oracle import chunk_forms as cf  # noqa: E402
from oracle import chunk_grad as cg  # noqa: E402


def test_neumann_chunk_model_forward_matches_numpy_chunk_model():
    """The autograd oracle's forward is the numpy chunk model with the masked
    series, operation for operation."""
    rng = np.random.default_rng(11)
    x, _, _ = _inputs(rng, T=21, dk=6, dv=5)
    o1, s1 = cg.neumann_fwd(chunk=8, N=2, **x)
    o2, s2 = cf.chunked_gated_delta_fwd(chunk=8, inverse=cf.neumann_inverse(2), **x)
    assert np.abs(o1 - o2).max() <= 1e-12 and np.abs(s1 - s2).max() <= 1e-12


@pytest.mark.parametrize("gates", [True, False])
def test_neumann_gradient_at_full_order_is_the_exact_adjoint(gates):
    """At N = C - 1 the masked series is the exact inverse (A is nilpotent), so
    the chunk model's gradient must equal the token-by-token adjoint."""
    rng = np.random.default_rng(12)
    x, do, dhT = _inputs(rng, T=19, dk=5, dv=4, gates=gates)
    C = 8
    g = cg.neumann_bwd(do=do, dhT=dhT, chunk=C, N=C - 1, **x)
    ref = rec.gated_delta_bwd(do=do, dhT=dhT, **x)
    for name, key in (("dq", "dq"), ("dk", "dk"), ("dv", "dv"), ("dalpha", "dalpha"), ("dbeta", "dbeta"),
                      ("dh0", "dh0")):
        if ref[key] is None:
            assert g[name] is None
            continue
        assert np.abs(g[name] - ref[key]).max() <= 1e-9 * max(1.0, np.abs(ref[key]).max()), name


def test_neumann_gradient_matches_finite_differences():
    """N = 2 (the series truncated well below the chunk length): central finite
    differences of the numpy chunk model, element by element on a sample."""
    rng = np.random.default_rng(13)
    x, do, dhT = _inputs(rng, T=13, dk=4, dv=3)
    C, N = 8, 2
    g = cg.neumann_bwd(do=do, dhT=dhT, chunk=C, N=N, **x)

    def loss(xx):
        o, hT = cf.chunked_gated_delta_fwd(chunk=C, inverse=cf.neumann_inverse(N), **xx)
        return float((o * do).sum() + (hT * dhT).sum())

    for name, key in (("q", "dq"), ("k", "dk"), ("v", "dv"), ("alpha", "dalpha"), ("beta", "dbeta"),
                      ("h0", "dh0")):
        arr = x[name]
        for flat in rng.choice(arr.size, size=6, replace=False):
            idx = np.unravel_index(flat, arr.shape)
            xp = dict(x)
            xp[name] = arr.copy()
            xp[name][idx] += 1e-6
            lp = loss(xp)
            xp[name][idx] -= 2e-6
            lm = loss(xp)
            fd = (lp - lm) / 2e-6
            assert abs(g[key][idx] - fd) <= 1e-6 * max(1.0, abs(fd)), (name, idx, g[key][idx], fd)


def test_residual_chunk_model_forward_matches_numpy_chunk_model():
    rng = np.random.default_rng(14)
    x, _, _ = _inputs(rng, T=21, dk=6, dv=5)
    o1, s1 = cg.neumann_fwd(chunk=8, N=2, S=3, **x)
    o2, s2 = cf.chunked_gated_delta_fwd(chunk=8, inverse=cf.residual_inverse(2, 3), **x)
    assert np.abs(o1 - o2).max() <= 1e-12 and np.abs(s1 - s2).max() <= 1e-12


def test_residual_gradient_at_exact_orders_is_the_exact_adjoint():
    """(N + 1)(S + 1) >= C makes the corrected series exact (the residual E
    vanishes within (N + 1)(S + 1) of the diagonal), so the gradient must be the
    token-by-token adjoint."""
    rng = np.random.default_rng(15)
    x, do, dhT = _inputs(rng, T=19, dk=5, dv=4)
    g = cg.neumann_bwd(do=do, dhT=dhT, chunk=8, N=1, S=3, **x)
    ref = rec.gated_delta_bwd(do=do, dhT=dhT, **x)
    for name, key in (("dq", "dq"), ("dk", "dk"), ("dv", "dv"), ("dalpha", "dalpha"), ("dbeta", "dbeta"),
                      ("dh0", "dh0")):
        assert np.abs(g[name] - ref[key]).max() <= 1e-9 * max(1.0, np.abs(ref[key]).max()), name


def test_residual_gradient_matches_finite_differences():
    rng = np.random.default_rng(16)
    x, do, dhT = _inputs(rng, T=13, dk=4, dv=3)
    C, N, S = 8, 1, 1
    g = cg.neumann_bwd(do=do, dhT=dhT, chunk=C, N=N, S=S, **x)

    def loss(xx):
        o, hT = cf.chunked_gated_delta_fwd(chunk=C, inverse=cf.residual_inverse(N, S), **xx)
        return float((o * do).sum() + (hT * dhT).sum())

    for name, key in (("q", "dq"), ("k", "dk"), ("v", "dv"), ("alpha", "dalpha"), ("beta", "dbeta"),
                      ("h0", "dh0")):
        arr = x[name]
        for flat in rng.choice(arr.size, size=6, replace=False):
            idx = np.unravel_index(flat, arr.shape)
            xp = dict(x)
            xp[name] = arr.copy()
            xp[name][idx] += 1e-6
            lp = loss(xp)
            xp[name][idx] -= 2e-6
            lm = loss(xp)
            fd = (lp - lm) / 2e-6
            assert abs(g[key][idx] - fd) <= 1e-6 * max(1.0, abs(fd)), (name, idx, g[key][idx], fd)
