"""A chunked form of the backward pass, restated in float64 numpy and checked against the
oracle's gradients (which are pinned to finite differences): the algebra a GPU backward would
evaluate chunk by chunk.

Forward per chunk (as in the chunk-algebra test; gamma the running gate products, Kg = gamma k^,
Ki = k^ / gamma, Qg = gamma q^):
    A = strict_lower(diag(beta) Kg Ki^T),  T = (I + A)^-1,  W = T diag(beta) Kg,  U = T diag(beta) V
    M = lower(Qg Ki^T),  Q' = Qg - M W,  Kend = gamma_C Ki,  Ac = Diag(gamma_C) - Kend^T W,
    Bc = Kend^T U,  O = scale (Q' S0 + M U),  S1 = Ac S0 + Bc.
Backward: the state gradient runs over the chunks in reverse (dS0 = scale Q'^T dO + Ac^T dS1),
and each chunk's input gradients follow from dO, dS1 and its S0 by reverse-mode through the
formulas above (each step is written out below); gamma = cumprod(alpha) gives
dalpha_r = (sum_{r' >= r} dgamma_r' gamma_r') / alpha_r.  The prologue (rotation, then L2 norm) is
differentiated as in the oracle.
"""
import numpy as np
import pytest

import oracle


def _rot(x, pos, theta, inverse=False):
    """Half-split rotation of rows x[t] by positions pos[t] (the inverse rotates by -pos)."""
    d = x.shape[-1]
    half = d // 2
    w = theta ** (-2.0 * np.arange(half) / d)
    ang = (-1.0 if inverse else 1.0) * pos[:, None] * w[None, :]
    c, s = np.cos(ang), np.sin(ang)
    a, b = x[:, :half], x[:, half:]
    return np.concatenate([a * c - b * s, b * c + a * s], axis=1)


def _chunk_grads(q, k, V, a, b, S0, dO, dS1, scale):
    C = q.shape[0]
    g = np.cumprod(a, axis=0)
    Kg, Ki, Qg = g * k, k / g, g * q
    L = np.tril(np.ones((C, C)), -1)
    Li = np.tril(np.ones((C, C)))
    A = L * (b[:, None] * (Kg @ Ki.T))
    T = np.linalg.inv(np.eye(C) + A)
    bK, bV = b[:, None] * Kg, b[:, None] * V
    W, U = T @ bK, T @ bV
    M = Li * (Qg @ Ki.T)
    Qp = Qg - M @ W
    gC = g[-1]
    Kend = gC * Ki
    Ac = np.diag(gC) - Kend.T @ W
    # read-out and state
    dS0 = scale * Qp.T @ dO + Ac.T @ dS1
    dQp = scale * dO @ S0.T
    dM = scale * dO @ U.T
    dU = scale * M.T @ dO
    dAc = dS1 @ S0.T
    # Bc = Kend^T U
    dKend = U @ dS1.T
    dU += Kend @ dS1
    # Ac = Diag(gC) - Kend^T W
    dgC = np.diag(dAc).copy()
    dKend -= W @ dAc.T
    dW = -Kend @ dAc
    # Q' = Qg - M W
    dQg = dQp.copy()
    dM -= dQp @ W.T
    dW -= M.T @ dQp
    # M = lower(Qg Ki^T)
    dM *= Li
    dQg += dM @ Ki
    dKi = dM.T @ Qg
    # Kend = gC Ki
    dKi += gC * dKend
    dgC += (Ki * dKend).sum(axis=0)
    # W = T bK, U = T bV
    dT = dW @ bK.T + dU @ bV.T
    dbK, dbV = T.T @ dW, T.T @ dU
    db = (dbK * Kg).sum(axis=1) + (dbV * V).sum(axis=1)
    dKg = b[:, None] * dbK
    dV = b[:, None] * dbV
    # T = (I + A)^-1, A = strict_lower(diag(b) Kg Ki^T)
    dA = L * (-T.T @ dT @ T.T)
    P = Kg @ Ki.T
    db += (dA * P).sum(axis=1)
    dKg += (b[:, None] * dA) @ Ki
    dKi += (b[:, None] * dA).T @ Kg
    # Kg = g k, Ki = k / g, Qg = g q
    dk = g * dKg + dKi / g
    dq = g * dQg
    dg = k * dKg - k * dKi / g ** 2 + q * dQg
    dg[-1] += dgC
    # g = cumprod(a)
    da = np.cumsum((dg * g)[::-1], axis=0)[::-1] / a
    return dq, dk, dV, da, db, dS0


def _chunked_bwd(q, k, v, alpha, beta, h0, dout, dhT, C, scale, l2norm, theta, pos0):
    T, dk = q.shape
    pos = pos0 + np.arange(T, dtype=np.float64)
    yq = _rot(q, pos, theta) if theta > 0 else q.copy()
    yk = _rot(k, pos, theta) if theta > 0 else k.copy()
    nq = np.sqrt((yq ** 2).sum(1) + 1e-6)[:, None] if l2norm else np.ones((T, 1))
    nk = np.sqrt((yk ** 2).sum(1) + 1e-6)[:, None] if l2norm else np.ones((T, 1))
    qh, kh = yq / nq, yk / nk
    # forward over chunks, keeping each chunk's entering state
    S = h0.copy()
    S0s = []
    for c0 in range(0, T, C):
        sl = slice(c0, min(T, c0 + C))
        S0s.append(S.copy())
        g = np.cumprod(alpha[sl], axis=0)
        n = sl.stop - sl.start
        Kg, Ki = g * kh[sl], kh[sl] / g
        A = np.tril(np.ones((n, n)), -1) * (beta[sl][:, None] * (Kg @ Ki.T))
        Tm = np.linalg.inv(np.eye(n) + A)
        W, U = Tm @ (beta[sl][:, None] * Kg), Tm @ (beta[sl][:, None] * v[sl])
        Kend = g[-1] * Ki
        S = (np.diag(g[-1]) - Kend.T @ W) @ S + Kend.T @ U
    # backward over chunks in reverse
    dS = dhT.copy()
    dqh, dkh = np.zeros_like(qh), np.zeros_like(kh)
    dv, da, db = np.zeros_like(v), np.zeros_like(alpha), np.zeros_like(beta)
    for ci in reversed(range(len(S0s))):
        sl = slice(ci * C, min(T, ci * C + C))
        gq, gk, gV, ga, gb, dS = _chunk_grads(qh[sl], kh[sl], v[sl], alpha[sl], beta[sl], S0s[ci],
                                              dout[sl], dS, scale)
        dqh[sl], dkh[sl], dv[sl], da[sl], db[sl] = gq, gk, gV, ga, gb
    # prologue: norm, then rotation
    def back(y, n, g):
        if l2norm:
            g = g / n - y * ((y * g).sum(1)[:, None]) / n ** 3
        return _rot(g, pos, theta, inverse=True) if theta > 0 else g
    return back(yq, nq, dqh), back(yk, nk, dkh), dv, da, db, dS


@pytest.mark.parametrize("T,C,theta,l2", [(32, 8, 0.0, True), (29, 8, 100.0, True),
                                          (24, 16, 0.0, False), (40, 16, 1000.0, True)])
def test_chunked_backward_equals_the_oracle(T, C, theta, l2):
    rng = np.random.default_rng(T * 7 + C)
    dk, dv = 6, 4
    q, k = rng.standard_normal((T, dk)), rng.standard_normal((T, dk))
    v = rng.standard_normal((T, dv))
    alpha = rng.choice([-1.0, 1.0], (T, dk)) * rng.uniform(0.4, 1.0, (T, dk))
    beta = rng.uniform(0.0, 2.0, T)
    h0 = rng.standard_normal((dk, dv))
    dout, dhT = rng.standard_normal((T, dv)), rng.standard_normal((dk, dv))
    scale = oracle.default_scale(dk)
    got = _chunked_bwd(q, k, v, alpha, beta, h0, dout, dhT, C, scale, l2, theta, 3)
    ref = oracle.bwd(q[None, :, None], k[None, :, None], v[None, :, None], alpha[None, :, None],
                     beta[None, :, None], h0[None, None], dout[None, :, None], dhT[None, None],
                     l2norm=l2, rope_theta=theta, pos_offset=3)
    want = (ref["dq"][0, :, 0], ref["dk"][0, :, 0], ref["dv"][0, :, 0], ref["dalpha"][0, :, 0],
            ref["dbeta"][0, :, 0], ref["dh0"][0, 0])
    for name, x, y in zip(("dq", "dk", "dv", "dalpha", "dbeta", "dh0"), got, want):
        err = np.abs(x - y).max() / max(np.abs(y).max(), 1e-12)
        assert err < 1e-9, (name, err)
