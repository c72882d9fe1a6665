"""Dense-matrix restatement of CKDA for tiny inputs -- TEST INFRASTRUCTURE ONLY.

This is the second, independent statement of the recurrence used to pin the sequential C oracle:
instead of scaling rows and applying a rank-one update in place, it builds every transition
matrix A_t = (I - beta_t k_t k_t^T) Diag(alpha_t) explicitly (the gated delta-rule transition of
the "Complex KDA" paper summary, Background) and evaluates the closed form

    S_t = A_t ... A_1 S_0 + sum_{j<=t} A_t ... A_{j+1} beta_j k_j v_j^T,   o_t = scale * S_t^T q_t

with numpy matrix products.  The rotation is built as a dense block-diagonal matrix R(p) with
angles p * theta^(-2i/d) ("RoPE into the KDA q/k path" review, section 5) and the L2 norm with
numpy.linalg.norm.  Meant for T <= 16 and d <= 8; cost grows as T^2 d^3.
"""
from __future__ import annotations

import numpy as np


def rotation_matrix(d: int, p: float, theta: float, convention: int = 0) -> np.ndarray:
    """Dense R(p): block rotation of coordinate pairs by angle p * theta^(-2i/d)."""
    R = np.eye(d)
    half = d // 2
    for i in range(half):
        ang = p * theta ** (-(2.0 * i) / d)
        a, b = (i, i + half) if convention == 0 else (2 * i, 2 * i + 1)
        R[a, a] = np.cos(ang)
        R[a, b] = -np.sin(ang)
        R[b, a] = np.sin(ang)
        R[b, b] = np.cos(ang)
    return R


def prepare(x: np.ndarray, p: float, l2norm: bool, theta: float, convention: int) -> np.ndarray:
    y = np.array(x, dtype=np.float64)
    if theta > 0:
        y = rotation_matrix(len(y), p, theta, convention) @ y
    if l2norm:
        y = y / np.sqrt(np.dot(y, y) + 1e-6)
    return y


def transition(k: np.ndarray, alpha: np.ndarray, beta: float) -> np.ndarray:
    """A = (I - beta k k^T) Diag(alpha)."""
    n = len(k)
    return (np.eye(n) - beta * np.outer(k, k)) @ np.diag(alpha)


def fwd_one_head(q, k, v, alpha, beta, h0=None, *, l2norm=True, rope_theta=0.0,
                 rope_convention=0, scale=None, pos_offset=0):
    """q, k, alpha: [T, dk]; v: [T, dv]; beta: [T]; h0: [dk, dv].  Returns (o [T, dv], S_T)."""
    T, dk = q.shape
    dv = v.shape[1]
    if scale is None:
        scale = 1.0 / np.sqrt(dk)
    S0 = np.zeros((dk, dv)) if h0 is None else np.array(h0, dtype=np.float64)
    qs = [prepare(q[t], pos_offset + t, l2norm, rope_theta, rope_convention) for t in range(T)]
    ks = [prepare(k[t], pos_offset + t, l2norm, rope_theta, rope_convention) for t in range(T)]
    A = [transition(ks[t], np.asarray(alpha[t], np.float64), float(beta[t])) for t in range(T)]
    outs = np.zeros((T, dv))
    S_t = None
    for t in range(T):
        # product A_t ... A_1 applied to S_0
        P = np.eye(dk)
        for j in range(t, -1, -1):
            P = P @ A[j]
        S_t = P @ S0
        for j in range(t + 1):
            Pj = np.eye(dk)
            for m in range(t, j, -1):
                Pj = Pj @ A[m]
            S_t = S_t + Pj @ (float(beta[j]) * np.outer(ks[j], v[j]))
        outs[t] = scale * (S_t.T @ qs[t])
    if S_t is None:
        S_t = S0
    return outs, S_t
