"""A chunked form of the backward pass, restated in float64 numpy and checked against the
oracle's gradients (which are pinned to finite differences): first in the plain form below, then
in the numerically stable form that the GPU backward (ckda_bwd_chunked) evaluates chunk by chunk
(at the end of this file).

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



# ---- the stable form the GPU backward evaluates -------------------------------------------------
# The form above forms k / gamma, which overflows once the gate products underflow (long runs of
# small gates, exact zeros).  The GPU backward instead keeps the sign of gamma absorbed into q'
# and k' and every ratio as R_rj = |gamma_r| / |gamma_j| = 2^(L_r - L_j) <= 1 (L the running sum
# of log2 max(|alpha|, FLT_MIN)), takes the gradients with respect to R and g = |gamma| directly,
# and reaches the gates without dividing by alpha:
#   dalpha_t = sign(alpha_t) [ g_{t-1} sum_{r>=t} dg_r R_rt + sum_{a>=t} R_at Z_at ],
#   Z_{a,t} = |alpha_{t-1}| Z_{a,t-1} + dR_{a,t-1},  Z_{a,0} = 0.
FLT_MIN = 1.17549435e-38


def _stable_factors(qh, kh, V, a, b):
    C = qh.shape[0]
    sig = np.cumprod(np.where(a < 0, -1.0, 1.0), axis=0)
    L = np.cumsum(np.log2(np.maximum(np.abs(a), FLT_MIN)), axis=0)
    R = 2.0 ** (L[:, None, :] - L[None, :, :]) * np.tril(np.ones((C, C)))[:, :, None]
    g = 2.0 ** L
    kp, qp = sig * kh, sig * qh
    P = np.einsum("rc,jc,rjc->rj", kp, kp, R) * np.tril(np.ones((C, C)), -1)
    M = np.einsum("rc,jc,rjc->rj", qp, kp, R)
    T = np.linalg.inv(np.eye(C) + b[:, None] * P)
    Kg, Qg = g * kp, g * qp
    W, U = T @ (b[:, None] * Kg), T @ (b[:, None] * V)
    return dict(sig=sig, sC=sig[-1], gC=g[-1], R=R, g=g, kp=kp, qp=qp, P=P, M=M, T=T, Kg=Kg,
                Qg=Qg, W=W, U=U, Kend=sig[-1] * R[-1] * kp, Qp=Qg - M @ W)


def _factored_gate_grads(F, a, E, dM, dQp, dKend, dKg, dg, reach=0):
    """dq', dk' and dalpha of a chunk whose decay stays inside the fp32 range, with every ratio
    factored as R_rj = g_r (1/g_j) (the GPU's form for chunks whose decay stays >= 2^-60):
      dk' = g E (K/g) + (E^T K_gamma + dM^T Q_gamma) / g + dK_gamma g + dK_end sigma_C g_C / g
      dq' = g (dM (K/g) + dQ')
      dalpha_t = sign(alpha_t) (g_{t-1} / g_t) [sum_{r>=t} dg_r g_r + S_t],
      S_t = sum_{a>=t} sum_{b<t} D_ab,  D_ab = R_ab dR_ab = (K_gamma,a E_ab + Q_gamma,a dM_ab
            (+ g_C sigma_C dK_end,b at a = C-1)) (K/g)_b.
    reach > 0 widens the staircase to b < t + reach (a planted mistake, for the test below)."""
    g, kp, Kg, Qg, sC = F["g"], F["kp"], F["Kg"], F["Qg"], F["sC"]
    C = g.shape[0]
    Ki = kp / g
    dkp = g * (E @ Ki) + (E.T @ Kg + dM.T @ Qg) / g + dKg * g + dKend * sC * g[-1] / g
    dqp = g * (dM @ Ki + dQp)
    D = (Kg[:, None, :] * E[:, :, None] + Qg[:, None, :] * dM[:, :, None]) * Ki[None, :, :]
    D[-1] += (g[-1] * sC) * dKend * Ki
    D *= np.tril(np.ones((C, C)), -1)[:, :, None]
    da = np.zeros_like(a)
    for t in range(C):
        S_t = D[t:, :t + reach].sum((0, 1))
        gprev = g[t - 1] if t > 0 else 1.0
        da[t] = np.where(a[t] < 0, -1.0, 1.0) * (gprev / g[t]) * ((dg[t:] * g[t:]).sum(0) + S_t)
    return dqp, dkp, da


def _stable_chunk_grads(F, V, a, b, S0, dO, dS1, scale, factored=False, reach=0):
    C = V.shape[0]
    kp, qp, R, g, T, W, U, M, Kend, Kg = (F[x] for x in ("kp", "qp", "R", "g", "T", "W", "U",
                                                         "M", "Kend", "Kg"))
    dQp = scale * dO @ S0.T
    dU = scale * M.T @ dO + Kend @ dS1
    dKend = (U - W @ S0) @ dS1.T
    dW = -(Kend @ dS1) @ S0.T - M.T @ dQp
    dM = np.tril(scale * dO @ U.T - dQp @ W.T)
    dgC = (dS1 * S0).sum(1)
    X, Y = T.T @ dW, T.T @ dU
    dT = dW @ (b[:, None] * Kg).T + dU @ (b[:, None] * V).T
    dA = np.tril(-T.T @ dT @ T.T, -1)
    db = (X * Kg).sum(1) + (Y * V).sum(1) + (dA * F["P"]).sum(1)
    E = b[:, None] * dA
    dKg = b[:, None] * X
    dkp = (np.einsum("rj,jc,rjc->rc", E, kp, R) + np.einsum("rj,rc,rjc->jc", E, kp, R)
           + np.einsum("rj,rc,rjc->jc", dM, qp, R) + dKg * g + dKend * F["sC"] * R[-1])
    dqp = np.einsum("rj,jc,rjc->rc", dM, kp, R) + dQp * g
    dR = np.einsum("rj,rc,jc->rjc", E, kp, kp) + np.einsum("rj,rc,jc->rjc", dM, qp, kp)
    dR[-1] += dKend * F["sC"] * kp
    dg = dKg * kp + dQp * qp
    dg[-1] += dgC * F["sC"]
    am = np.maximum(np.abs(a), FLT_MIN)
    da = np.zeros_like(a)
    Z = np.zeros((C, a.shape[1]))
    for t in range(C):
        if t > 0:
            Z = am[t - 1] * Z + dR[:, t - 1, :]
        gprev = g[t - 1] if t > 0 else 1.0
        da[t] = np.where(a[t] < 0, -1.0, 1.0) * (gprev * (dg[t:] * R[t:, t]).sum(0)
                                                 + (R[t:, t] * Z[t:]).sum(0))
    if factored:
        dqp, dkp, da = _factored_gate_grads(F, a, E, dM, dQp, dKend, dKg, dg, reach)
    dS0 = scale * F["Qp"].T @ dO + (F["sC"] * F["gC"])[:, None] * dS1 - W.T @ (Kend @ dS1)
    return F["sig"] * dqp, F["sig"] * dkp, b[:, None] * Y, da, db, dS0


def _stable_chunked_bwd(q, k, v, alpha, beta, h0, dout, dhT, C, scale, l2norm, theta, pos0,
                        factored=False):
    T, dk = q.shape
    pos = pos0 + np.arange(T, dtype=np.float64)
    yq = _rot(q, pos, theta) if theta > 0 else q.copy()
    yk = _rot(k, pos, theta) if theta > 0 else k.copy()
    nq = np.sqrt((yq ** 2).sum(1) + 1e-6)[:, None] if l2norm else np.ones((T, 1))
    nk = np.sqrt((yk ** 2).sum(1) + 1e-6)[:, None] if l2norm else np.ones((T, 1))
    qh, kh = yq / nq, yk / nk
    S, S0s = h0.copy(), []
    for c0 in range(0, T, C):
        sl = slice(c0, min(T, c0 + C))
        S0s.append(S.copy())
        F = _stable_factors(qh[sl], kh[sl], v[sl], alpha[sl], beta[sl])
        S = (np.diag(F["sC"] * F["gC"]) - F["Kend"].T @ F["W"]) @ S + F["Kend"].T @ F["U"]
    dS = dhT.copy()
    grads = [np.zeros_like(x) for x in (qh, kh, v, alpha, beta)]
    for ci in reversed(range(len(S0s))):
        sl = slice(ci * C, min(T, ci * C + C))
        F = _stable_factors(qh[sl], kh[sl], v[sl], alpha[sl], beta[sl])
        *gs, dS = _stable_chunk_grads(F, v[sl], alpha[sl], beta[sl], S0s[ci], dout[sl], dS,
                                      scale, factored)
        for G_, x in zip(grads, gs):
            G_[sl] = x

    def back(y, n, g):
        if l2norm:
            g = g / n - y * ((y * g).sum(1)[:, None]) / n ** 3
        return _rot(g, pos, theta, inverse=True) if theta > 0 else g
    return back(yq, nq, grads[0]), back(yk, nk, grads[1]), grads[2], grads[3], grads[4], dS


@pytest.mark.parametrize("T,C,theta,l2,amin,zeros", [(32, 8, 0.0, True, 0.4, False),
                                                     (40, 16, 100.0, True, 1e-3, False),
                                                     (48, 16, 0.0, True, 1e-3, True),
                                                     (29, 16, 1000.0, False, 0.05, True)])
def test_stable_chunked_backward_equals_the_oracle(T, C, theta, l2, amin, zeros):
    """Gates down to 1e-3 (their products underflow within a chunk) and exact zeros."""
    rng = np.random.default_rng(T * 7 + C)
    dk, dv = 6, 4
    q, k = rng.standard_normal((T, dk)), rng.standard_normal((T, dk))
    v = rng.standard_normal((T, dv))
    alpha = rng.choice([-1.0, 1.0], (T, dk)) * rng.uniform(amin, 1.0, (T, dk))
    if zeros:
        alpha[rng.random((T, dk)) < 0.1] = 0.0
    beta = rng.uniform(0.0, 2.0, T)
    h0 = rng.standard_normal((dk, dv))
    dout, dhT = rng.standard_normal((T, dv)), rng.standard_normal((dk, dv))
    scale = oracle.default_scale(dk)
    got = _stable_chunked_bwd(q, k, v, alpha, beta, h0, dout, dhT, C, scale, l2, theta, 3)
    ref = oracle.bwd(q[None, :, None], k[None, :, None], v[None, :, None], alpha[None, :, None],
                     beta[None, :, None], h0[None, None], dout[None, :, None], dhT[None, None],
                     l2norm=l2, rope_theta=theta, pos_offset=3)
    want = (ref["dq"][0, :, 0], ref["dk"][0, :, 0], ref["dv"][0, :, 0], ref["dalpha"][0, :, 0],
            ref["dbeta"][0, :, 0], ref["dh0"][0, 0])
    for name, x, y in zip(("dq", "dk", "dv", "dalpha", "dbeta", "dh0"), got, want):
        err = np.abs(x - y).max() / max(np.abs(y).max(), 1e-12)
        assert err < 1e-9, (name, err)


@pytest.mark.parametrize("T,C,theta,l2", [(32, 8, 0.0, True), (45, 16, 1000.0, True),
                                          (40, 16, 0.0, False)])
def test_factored_gate_gradients_equal_the_oracle(T, C, theta, l2):
    """The factored form of the chunk gradients (ratios split into g_r and 1/g_j, the dalpha
    recurrence as a staircase sum) on gates whose chunk decay stays far inside the fp32 range
    (|alpha| >= 0.3: at most 2^-28 over 16 tokens), against the token-by-token oracle."""
    rng = np.random.default_rng(T * 11 + C)
    dk, dv = 6, 4
    q, k = rng.standard_normal((T, dk)), rng.standard_normal((T, dk))
    v = rng.standard_normal((T, dv))
    alpha = rng.choice([-1.0, 1.0], (T, dk)) * rng.uniform(0.3, 1.0, (T, dk))
    beta = rng.uniform(0.0, 2.0, T)
    h0 = rng.standard_normal((dk, dv))
    dout, dhT = rng.standard_normal((T, dv)), rng.standard_normal((dk, dv))
    scale = oracle.default_scale(dk)
    got = _stable_chunked_bwd(q, k, v, alpha, beta, h0, dout, dhT, C, scale, l2, theta, 5,
                              factored=True)
    ref = oracle.bwd(q[None, :, None], k[None, :, None], v[None, :, None], alpha[None, :, None],
                     beta[None, :, None], h0[None, None], dout[None, :, None], dhT[None, None],
                     l2norm=l2, rope_theta=theta, pos_offset=5)
    want = (ref["dq"][0, :, 0], ref["dk"][0, :, 0], ref["dv"][0, :, 0], ref["dalpha"][0, :, 0],
            ref["dbeta"][0, :, 0], ref["dh0"][0, 0])
    for name, x, y in zip(("dq", "dk", "dv", "dalpha", "dbeta", "dh0"), got, want):
        err = np.abs(x - y).max() / max(np.abs(y).max(), 1e-12)
        assert err < 1e-9, (name, err)


def test_factored_staircase_boundary_matters():
    """The factored form equals the exact form chunk by chunk, and the staircase's boundary is
    pinned: widening it to b <= t (one diagonal of D too many) moves dalpha well off."""
    rng = np.random.default_rng(3)
    C, dk, dv = 8, 4, 3
    q, k = rng.standard_normal((C, dk)), rng.standard_normal((C, dk))
    v = rng.standard_normal((C, dv))
    a = rng.choice([-1.0, 1.0], (C, dk)) * rng.uniform(0.5, 1.0, (C, dk))
    b = rng.uniform(0.5, 2.0, C)
    S0, dO, dS1 = (rng.standard_normal(x) for x in ((dk, dv), (C, dv), (dk, dv)))
    F = _stable_factors(q, k, v, a, b)
    exact = _stable_chunk_grads(F, v, a, b, S0, dO, dS1, 0.5)
    fact = _stable_chunk_grads(F, v, a, b, S0, dO, dS1, 0.5, factored=True)
    for x, y in zip(exact, fact):
        assert np.abs(x - y).max() <= 1e-10 * max(np.abs(x).max(), 1.0)
    wide = _stable_chunk_grads(F, v, a, b, S0, dO, dS1, 0.5, factored=True, reach=1)
    assert np.abs(wide[3] - exact[3]).max() > 1e-2 * np.abs(exact[3]).max()
