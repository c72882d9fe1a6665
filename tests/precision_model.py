"""A float64 model of where the tensor-core forward rounds, for deriving its error bounds.

The tensor-core path evaluates the chunk algebra (derived from the transition of the "Complex
KDA" paper summary, Background; restated in test_chunk_algebra.py) with bf16 operand tiles and
fp32 accumulation.  This module evaluates the same algebra in float64 and rounds exactly the
intermediates the kernel stores as tensor-core operands, to a chosen format:

    L  = [g k'; g q']   R = k'/g   K_end = gamma_C k'/g   M (masked)   T' = T diag(beta)
    W = T' (g k')       U~ = T' V  Q' = g q' - M W        A_c = Diag(gamma_C) - K_end^T W
    S  (the state as the operand of the next chunk's products)

and rounds the output once (its storage type).  Everything else -- the [A | M] product, B_c =
K_end^T U~, the chunk's own output M U~, the state itself between chunks -- stays unrounded, as
the kernel keeps it in fp32 accumulators.  q' = sigma k^, k' = sigma k^ carry the running sign
product of the gates, g = |gamma| (the sign absorption of the summary's Implementation section).

It is a model of rounding placement, not a second oracle: with no rounding it reproduces the
token-by-token oracle to float64 accuracy (checked in test_precision_model.py), and the error it
shows with bf16 operands is the floor that any evaluation with those operand roundings reaches.
"""
from __future__ import annotations

import numpy as np

OPERANDS = ("L", "R", "KE", "M", "Tp", "W", "U", "Qp", "Ac", "S")


def round_bf16(x):
    """float64 -> fp32 -> bf16 (nearest even), back to float64."""
    b = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    b = (b + 0x7FFF + ((b >> 16) & 1)) & 0xFFFF0000
    return b.astype(np.uint32).view(np.float32).astype(np.float64)


def round_tf32(x):
    """float64 -> fp32 -> tf32 (10 explicit mantissa bits, nearest, ties away from zero)."""
    b = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    b = (b + 0x1000) & 0xFFFFE000
    return b.astype(np.uint32).view(np.float32).astype(np.float64)


def chunked_head(q, k, v, alpha, beta, S0, *, rounding=round_bf16, operands=OPERANDS, C=64,
                 round_out=True, l2norm=True, eps=1e-6):
    """One head: q, k, alpha [T, dk]; v [T, dv]; beta [T]; S0 [dk, dv] (float64).  Operands named
    in `operands` are rounded with `rounding`; the output with bf16 when round_out.
    Returns (out [T, dv], S_T [dk, dv])."""
    rnd = lambda name, x: rounding(x) if name in operands else x
    T, dk = q.shape
    dv = v.shape[1]
    if l2norm:
        q = q / np.sqrt((q * q).sum(1, keepdims=True) + eps)
        k = k / np.sqrt((k * k).sum(1, keepdims=True) + eps)
    scale = dk ** -0.5
    S = np.array(S0, dtype=np.float64)
    out = np.zeros((T, dv))
    for c0 in range(0, T, C):
        n = min(C, T - c0)
        a = np.ones((C, dk))
        a[:n] = alpha[c0:c0 + n]
        b = np.zeros(C)
        b[:n] = beta[c0:c0 + n]
        kk, qq, vv = np.zeros((C, dk)), np.zeros((C, dk)), np.zeros((C, dv))
        kk[:n], qq[:n], vv[:n] = k[c0:c0 + n], q[c0:c0 + n], v[c0:c0 + n]
        gam = np.cumprod(a, axis=0)
        sig = np.where(np.signbit(gam), -1.0, 1.0)
        g = np.abs(gam)
        kp, qp = sig * kk, sig * qq
        Lk, Lq, R = rnd("L", g * kp), rnd("L", g * qp), rnd("R", kp / g)
        KE = rnd("KE", gam[-1] * kp / g)
        A = np.tril(b[:, None] * (Lk @ R.T), -1)
        M = rnd("M", np.tril(Lq @ R.T))
        Tp = rnd("Tp", np.linalg.inv(np.eye(C) + A) * b[None, :])
        W = rnd("W", Tp @ Lk)
        U = rnd("U", Tp @ vv)
        Qp = rnd("Qp", Lq - M @ W)
        Ac = rnd("Ac", np.diag(gam[-1]) - KE.T @ W)
        Sb = rnd("S", S)
        o = scale * (Qp @ Sb + M @ U)
        out[c0:c0 + n] = (round_bf16(o) if round_out else o)[:n]
        S = Ac @ Sb + (KE.T @ U)
    return out, S


def chunked(q, k, v, alpha, beta, h0=None, **kw):
    """All (batch, head) pairs of [B, T, H, d] inputs; returns (out [B, T, H, dv], hT)."""
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    out = np.zeros((B, T, H, dv))
    hT = np.zeros((B, H, dk, dv))
    f = lambda x: np.asarray(x, dtype=np.float64)
    for b in range(B):
        for h in range(H):
            S0 = np.zeros((dk, dv)) if h0 is None else f(h0[b, h])
            out[b, :, h], hT[b, h] = chunked_head(f(q[b, :, h]), f(k[b, :, h]), f(v[b, :, h]),
                                                  f(alpha[b, :, h]), f(beta[b, :, h]), S0, **kw)
    return out, hT
