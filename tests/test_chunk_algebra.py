"""The chunk algebra the CUDA forwards are built on, restated in float64 numpy and checked
against the token-by-token oracle (CPU).

The pages give the recurrence, not a chunked form; the chunked form below is derived from the
transition of the "Complex KDA" paper summary (Background) and is what the tensor-core and SIMT
kernels evaluate.  For a chunk of C tokens with entering state S0, prepared q^, k^ (rotation,
then L2 norm) and per-channel gate products gamma_r = prod_{tau <= r} alpha_tau:

    A_rj = beta_r k^_r . (gamma_r / gamma_j) k^_j  (j < r),   T = (I + A)^-1
    W = T diag(beta) (gamma k^),   U~ = T diag(beta) V
    M_rj = q^_r . (gamma_r / gamma_j) k^_j  (j <= r),   Q' = gamma q^ - M W
    K_end,j = (gamma_C / gamma_j) k^_j,   A_c = Diag(gamma_C) - K_end^T W,   B_c = K_end^T U~
    O = scale (Q' S0 + M U~),   S_C = A_c S0 + B_c

Two forms are checked: with the signed gate products as they stand, and with the signs absorbed
into q and k (q' = sigma q^, k' = sigma k^, sigma_r the running sign product, g = |gamma|), the
form the tensor-core factor role uses ("CKDA summary", Implementation, variant 1).  A sequence
whose length is not a multiple of C is padded with identity steps (alpha = 1, beta = 0, q = k =
v = 0).
"""
import numpy as np
import pytest

import oracle


def _chunked(qh, kh, v, alpha, beta, S0, C, scale, absorb):
    T, dk = qh.shape
    pad = (-T) % C
    if pad:
        qh = np.vstack([qh, np.zeros((pad, dk))])
        kh = np.vstack([kh, np.zeros((pad, dk))])
        v = np.vstack([v, np.zeros((pad, v.shape[1]))])
        alpha = np.vstack([alpha, np.ones((pad, dk))])
        beta = np.concatenate([beta, np.zeros(pad)])
    S = S0.copy()
    out = []
    for c0 in range(0, T + pad, C):
        q, k, V, a, b = (x[c0:c0 + C] for x in (qh, kh, v, alpha, beta))
        gam = np.cumprod(a, axis=0)                       # signed gate products gamma_r
        if absorb:
            sig = np.sign(gam)
            g = np.abs(gam)
            qp, kp = sig * q, sig * k                     # q', k'
            ratio = g[:, None, :] / g[None, :, :]         # g_r / g_j
            Kg, Qg = g * kp, g * qp
            Kend = gam[-1] * kp / g                       # gamma_C k' / g
            qq, kk = qp, kp
        else:
            ratio = gam[:, None, :] / gam[None, :, :]     # gamma_r / gamma_j
            Kg, Qg = gam * k, gam * q
            Kend = gam[-1] / gam * k
            qq, kk = q, k
        A = np.einsum("rc,rjc,jc->rj", kk, ratio, kk) * b[:, None]
        A = np.tril(A, -1)
        Tm = np.linalg.inv(np.eye(C) + A)
        W = Tm @ (b[:, None] * Kg)
        U = Tm @ (b[:, None] * V)
        M = np.tril(np.einsum("rc,rjc,jc->rj", qq, ratio, kk))
        Qp = Qg - M @ W
        Ac = np.diag(gam[-1]) - Kend.T @ W
        Bc = Kend.T @ U
        out.append(scale * (Qp @ S + M @ U))
        S = Ac @ S + Bc
    return np.vstack(out)[:T], S


@pytest.mark.parametrize("absorb", [False, True])
@pytest.mark.parametrize("T,C,rope", [(64, 16, 0.0), (53, 16, 1000.0), (40, 8, 0.0)])
def test_chunked_form_equals_the_recurrence(absorb, T, C, rope):
    rng = np.random.default_rng(T + C)
    dk, dv = 8, 5
    q = rng.standard_normal((1, T, 1, dk))
    k = rng.standard_normal((1, T, 1, dk))
    v = rng.standard_normal((1, T, 1, dv))
    alpha = rng.choice([-1.0, 1.0], (1, T, 1, dk)) * rng.uniform(0.3, 1.0, (1, T, 1, dk))
    beta = rng.uniform(0.0, 2.0, (1, T, 1))
    h0 = rng.standard_normal((1, 1, dk, dv))
    kw = dict(rope_theta=rope, pos_offset=2)
    o_ref, s_ref = oracle.fwd(q, k, v, alpha, beta, h0, **kw)
    qh = oracle.prologue(q, **kw)[0, :, 0]
    kh = oracle.prologue(k, **kw)[0, :, 0]
    o, S = _chunked(qh, kh, v[0, :, 0], alpha[0, :, 0], beta[0, :, 0], h0[0, 0], C,
                    oracle.default_scale(dk), absorb)
    assert np.allclose(o, o_ref[0, :, 0], rtol=0, atol=1e-11)
    assert np.allclose(S, s_ref[0, 0], rtol=0, atol=1e-11)
