"""Checks that pin the float64 oracle to facts fixed outside itself.

Each ``pin_*`` function raises AssertionError when the oracle (optionally a build with a planted
mistake, ``mutant=n``) disagrees with the pages' closed forms, with a mathematical invariant, or
with the independent dense restatement in ``oracle.dense``.  ``test_oracle_pins`` runs them on the
real oracle; ``test_oracle_mutants`` runs them on every planted mistake and requires that at least
one fails for each.
"""
from __future__ import annotations

import math
import os

import numpy as np

import oracle
from oracle import dense

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _closed_forms():
    forms = {}
    with open(os.path.join(GOLDEN, "ckda_closed_forms.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            name, expr, _src = (s.strip() for s in line.split("|"))
            forms[name] = expr
    return forms


def _eval(expr, **env):
    ns = {"cos": math.cos, "sin": math.sin, "__builtins__": {}}
    ns.update(env)
    return float(eval(expr, ns))  # expressions come from the committed fixture only


def extract_transition(k, alpha, beta, mutant=0):
    """Run the oracle one step from S_0 = I with v = 0 and no L2 norm: S_1 = A_1."""
    n = len(k)
    q = np.zeros((1, 1, 1, n))
    kk = np.asarray(k, np.float64).reshape(1, 1, 1, n)
    al = np.asarray(alpha, np.float64).reshape(1, 1, 1, n)
    v = np.zeros((1, 1, 1, n))
    b = np.full((1, 1, 1), float(beta))
    h0 = np.eye(n).reshape(1, 1, n, n)
    _, hT = oracle.fwd(q, kk, v, al, b, h0, l2norm=False, mutant=mutant)
    return hT[0, 0]


def _unit(rng, n):
    x = rng.standard_normal(n)
    return x / np.linalg.norm(x)


# --- the transition matrix and its closed forms -------------------------------------------------

def pin_commutator(mutant=0):
    """(H_k D - D H_k)_ij = beta k_i k_j (alpha_i - alpha_j); with H, D symmetric, H D - D H = A - A^T."""
    rng = np.random.default_rng(11)
    for n in (2, 3, 6):
        k = _unit(rng, n)
        alpha = rng.uniform(-1, 1, n)
        beta = rng.uniform(0, 2)
        A = extract_transition(k, alpha, beta, mutant)
        expect = beta * np.outer(k, k) * (alpha[:, None] - alpha[None, :])
        assert np.allclose(A - A.T, expect, atol=1e-13), "commutator identity violated"


def pin_2d_construction(mutant=0):
    """beta = 2, k = (cos t, sin t), alpha = (a, 1) gives the printed A_{alpha,theta};
    a = -1 is the rotation by 2 theta, n steps give the rotation by 2 n theta."""
    f = _closed_forms()
    for a in (-1.0, -0.5, 0.3, 1.0):
        for theta in (0.1, 0.7, 1.9):
            k = np.array([math.cos(theta), math.sin(theta)])
            A = extract_transition(k, [a, 1.0], 2.0, mutant)
            want = np.array([[_eval(f["A2d_00"], a=a, theta=theta), _eval(f["A2d_01"], a=a, theta=theta)],
                             [_eval(f["A2d_10"], a=a, theta=theta), _eval(f["A2d_11"], a=a, theta=theta)]])
            assert np.allclose(A, want, atol=1e-13), f"2D construction wrong at a={a}, theta={theta}"
            # spectrum: trace (1-a) cos 2t, det -a, complex pair iff the printed discriminant < 0
            ev = np.linalg.eigvals(A)
            disc = _eval(f["disc2d"], a=a, theta=theta)
            assert (abs(ev.imag).max() > 1e-9) == (disc < -1e-9), "discriminant does not predict spectrum"
    # a = -1: composition of two reflections = rotation by 2 theta; T steps rotate by 2 T theta
    theta, T = 0.37, 9
    k = np.array([math.cos(theta), math.sin(theta)])
    q = np.zeros((1, T, 1, 2))
    kk = np.tile(k, (1, T, 1, 1)).reshape(1, T, 1, 2)
    al = np.tile([-1.0, 1.0], (1, T, 1, 1)).reshape(1, T, 1, 2)
    v = np.zeros((1, T, 1, 2))
    b = np.full((1, T, 1), 2.0)
    _, hT = oracle.fwd(q, kk, v, al, b, np.eye(2).reshape(1, 1, 2, 2), l2norm=False, mutant=mutant)
    ang = 2 * T * theta
    R = np.array([[math.cos(ang), -math.sin(ang)], [math.sin(ang), math.cos(ang)]])
    assert np.allclose(hT[0, 0], R, atol=1e-12), "alpha=-1, beta=2 is not a rotation by 2 theta per step"


def pin_prop2_block(mutant=0):
    """alpha in {+-1}, k = cos t e_- + sin t e_+: the transition restricted to span{e_-, e_+} is
    the printed block B(beta, theta), with trace beta cos 2t, det beta - 1, and non-real
    eigenvalues exactly when beta^2 cos^2 2t < 4 (beta - 1)."""
    f = _closed_forms()
    n, i_minus, i_plus = 5, 1, 3
    alpha = np.array([1.0, -1.0, -1.0, 1.0, 1.0])
    for beta in (0.0, 0.5, 1.0, 1.5, 1.9, 2.0):
        for theta in (0.2, 0.6, 1.1, 2.5):
            k = np.zeros(n)
            k[i_minus], k[i_plus] = math.cos(theta), math.sin(theta)
            A = extract_transition(k, alpha, beta, mutant)
            blk = A[np.ix_([i_minus, i_plus], [i_minus, i_plus])]
            want = np.array([[_eval(f[f"B_{r}{c}"], beta=beta, theta=theta) for c in (0, 1)] for r in (0, 1)])
            assert np.allclose(blk, want, atol=1e-13), f"Prop. 2 block wrong at beta={beta}, theta={theta}"
            assert abs(np.trace(blk) - beta * math.cos(2 * theta)) < 1e-12
            assert abs(np.linalg.det(blk) - (beta - 1)) < 1e-12
            nonreal = _eval(f["B_nonreal"], beta=beta, theta=theta) < -1e-9
            ev = np.linalg.eigvals(blk)
            assert (abs(ev.imag).max() > 1e-9) == nonreal
            # the block is invariant: the other coordinates are untouched (pure sign flips)
            rest = [i for i in range(n) if i not in (i_minus, i_plus)]
            assert np.allclose(A[np.ix_(rest, rest)], np.diag(alpha[rest]), atol=1e-13)


def pin_orthogonal_norm(mutant=0):
    """|alpha_i| = 1, beta in {0, 2}, unit k (Theorem 1: (I - 2kk^T) Diag(s) is orthogonal):
    with v = 0 the Frobenius norm of the state is preserved over any number of steps."""
    rng = np.random.default_rng(5)
    for T in (1, 7, 64):
        B, H, dk, dv = 1, 2, 8, 5
        k = rng.standard_normal((B, T, H, dk))
        k /= np.linalg.norm(k, axis=-1, keepdims=True)
        alpha = rng.choice([-1.0, 1.0], size=(B, T, H, dk))
        beta = rng.choice([0.0, 2.0], size=(B, T, H))
        v = np.zeros((B, T, H, dv))
        q = rng.standard_normal((B, T, H, dk))
        h0 = rng.standard_normal((B, H, dk, dv))
        _, hT = oracle.fwd(q, k, v, alpha, beta, h0, l2norm=False, mutant=mutant)
        n0 = np.linalg.norm(h0.reshape(B * H, -1), axis=1)
        n1 = np.linalg.norm(hT.reshape(B * H, -1), axis=1)
        assert np.allclose(n0, n1, rtol=1e-12), "state norm not preserved by orthogonal transitions"
    # and the single-step transition is orthogonal and equals a reflection times signs
    k = _unit(rng, 6)
    s = rng.choice([-1.0, 1.0], 6)
    A = extract_transition(k, s, 2.0, mutant)
    assert np.allclose(A @ A.T, np.eye(6), atol=1e-13)


def pin_delta_write(mutant=0):
    """beta = 1 and a unit key make the write exact: S_t^T k_t = v_t, so with q_t = k_t the
    read-out is dk^-1/2 v_t whatever the gates and the history."""
    rng = np.random.default_rng(3)
    B, T, H, dk, dv = 2, 9, 3, 8, 6
    k = rng.standard_normal((B, T, H, dk))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((B, T, H, dv))
    alpha = rng.uniform(-1, 1, (B, T, H, dk))
    beta = np.ones((B, T, H))
    h0 = rng.standard_normal((B, H, dk, dv))
    out, _ = oracle.fwd(k, k, v, alpha, beta, h0, l2norm=False, mutant=mutant)
    assert np.allclose(out, v / math.sqrt(dk), atol=1e-12), "delta-rule write identity violated"


def pin_identity_gates(mutant=0):
    """beta = 0 and alpha = 1 leave the state unchanged: hT = h0 and o_t = scale h0^T q_t."""
    rng = np.random.default_rng(8)
    B, T, H, dk, dv = 1, 5, 2, 4, 3
    q = rng.standard_normal((B, T, H, dk))
    k = rng.standard_normal((B, T, H, dk))
    v = rng.standard_normal((B, T, H, dv))
    h0 = rng.standard_normal((B, H, dk, dv))
    out, hT = oracle.fwd(q, k, v, np.ones((B, T, H, dk)), np.zeros((B, T, H)), h0, l2norm=False,
                         mutant=mutant)
    assert np.allclose(hT, h0, atol=1e-14)
    want = np.einsum("bhcj,bthc->bthj", h0, q) / math.sqrt(dk)
    assert np.allclose(out, want, atol=1e-13)


def pin_gdn_and_kda_spectra(mutant=0):
    """A scalar gate commutes with H (GDN: symmetric transition); positive channel-wise gates
    give a real spectrum (KDA: similar to a symmetric matrix); only signed gates with beta > 1
    and a key spanning opposite-sign coordinates can give a complex pair."""
    rng = np.random.default_rng(21)
    n = 6
    for _ in range(20):
        k = _unit(rng, n)
        a = rng.uniform(-1, 1)
        A = extract_transition(k, np.full(n, a), rng.uniform(0, 2), mutant)
        assert np.allclose(A, A.T, atol=1e-13), "scalar-gate transition is not symmetric"
        A = extract_transition(k, rng.uniform(0.01, 1, n), rng.uniform(0, 2), mutant)
        assert abs(np.linalg.eigvals(A).imag).max() < 1e-9, "positive gates gave a complex spectrum"
        A = extract_transition(k, rng.uniform(-1, 1, n), rng.uniform(0, 1), mutant)
        assert abs(np.linalg.eigvals(A).imag).max() < 1e-9, "beta <= 1 gave a complex spectrum"


def pin_sign_absorption(mutant=0):
    """Sign absorption (the paper's compiled-PyTorch variant): CKDA(q, k, v, alpha, beta) equals
    KDA(P q, P k, v, |alpha|, beta) with P_t the running product of sign(alpha) per channel,
    and the final state is P_T applied to the rows of the KDA state."""
    rng = np.random.default_rng(4)
    B, T, H, dk, dv = 2, 23, 2, 8, 4
    q = rng.standard_normal((B, T, H, dk))
    k = rng.standard_normal((B, T, H, dk))
    v = rng.standard_normal((B, T, H, dv))
    alpha = rng.uniform(-1, 1, (B, T, H, dk))
    beta = rng.uniform(0, 2, (B, T, H))
    h0 = rng.standard_normal((B, H, dk, dv))
    P = np.cumprod(np.sign(alpha), axis=1)
    o1, s1 = oracle.fwd(q, k, v, alpha, beta, h0, mutant=mutant)
    o2, s2 = oracle.fwd(P * q, P * k, v, np.abs(alpha), beta, h0, mutant=mutant)
    assert np.allclose(o1, o2, atol=1e-12), "sign absorption changes the output"
    assert np.allclose(s1, P[:, -1][..., None] * s2, atol=1e-12), "sign absorption changes the state"


def pin_brute_force(mutant=0):
    """Explicit dense products of the transition matrices on tiny inputs (oracle.dense)."""
    rng = np.random.default_rng(17)
    cases = [dict(T=1, dk=2, dv=2), dict(T=5, dk=3, dv=4), dict(T=8, dk=4, dv=4),
             dict(T=6, dk=4, dv=3, rope=10000.0, conv=0, pos=3),
             dict(T=7, dk=6, dv=2, rope=10000.0, conv=1, pos=11),
             dict(T=4, dk=4, dv=4, rope=50.0, conv=0, pos=40000),
             dict(T=6, dk=4, dv=2, l2=False)]
    for c in cases:
        T, dk, dv = c["T"], c["dk"], c["dv"]
        B, H = 1, 2
        q = rng.standard_normal((B, T, H, dk))
        k = rng.standard_normal((B, T, H, dk))
        v = rng.standard_normal((B, T, H, dv))
        alpha = rng.uniform(-1, 1, (B, T, H, dk))
        beta = rng.uniform(0, 2, (B, T, H))
        h0 = rng.standard_normal((B, H, dk, dv))
        kw = dict(l2norm=c.get("l2", True), rope_theta=c.get("rope", 0.0),
                  rope_convention=c.get("conv", 0), pos_offset=c.get("pos", 0))
        out, hT = oracle.fwd(q, k, v, alpha, beta, h0, mutant=mutant, **kw)
        for h in range(H):
            o_d, s_d = dense.fwd_one_head(q[0, :, h], k[0, :, h], v[0, :, h], alpha[0, :, h],
                                          beta[0, :, h], h0[0, h], **kw)
            assert np.allclose(out[0, :, h], o_d, atol=1e-11, rtol=1e-11), f"brute force output mismatch {c}"
            assert np.allclose(hT[0, h], s_d, atol=1e-11, rtol=1e-11), f"brute force state mismatch {c}"


# --- the q/k prologue --------------------------------------------------------------------------

def _rope_cases():
    with open(os.path.join(GOLDEN, "rope_closed_forms.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            conv, pos, idx, vec, _src = (s.strip() for s in line.split("|"))
            yield (0 if conv == "half" else 1), int(pos), int(idx), [_eval(e) for e in vec.split(",")]


def pin_rope_closed_form(mutant=0):
    """Basis vectors rotated by the printed frequency rule at theta = 10000, d = 4."""
    for conv, pos, idx, want in _rope_cases():
        x = np.zeros((1, 1, 1, 4))
        x[..., idx] = 1.0
        y = oracle.prologue(x, l2norm=False, rope_theta=10000.0, rope_convention=conv,
                            pos_offset=pos, mutant=mutant)
        assert np.allclose(y[0, 0, 0], want, atol=1e-14), f"rotation wrong: conv={conv} pos={pos} e{idx}"


def pin_rope_both_q_and_k(mutant=0):
    """The rotation reaches q and k alike: <R_m q, R_n k> depends only on m - n, so the read-out
    of a one-token-back key is invariant to shifting every position."""
    rng = np.random.default_rng(2)
    B, T, H, dk, dv = 1, 2, 1, 8, 3
    q = rng.standard_normal((B, T, H, dk))
    k = rng.standard_normal((B, T, H, dk))
    v = rng.standard_normal((B, T, H, dv))
    alpha = np.ones((B, T, H, dk))
    beta = np.array([[[1.0], [0.0]]])
    outs = []
    for pos in (0, 5, 1234):
        o, _ = oracle.fwd(q, k, v, alpha, beta, None, l2norm=True, rope_theta=10000.0,
                          pos_offset=pos, mutant=mutant)
        outs.append(o)
    assert np.allclose(outs[0], outs[1], atol=1e-12) and np.allclose(outs[0], outs[2], atol=1e-12), \
        "read-out depends on absolute position: q and k are not rotated alike"


def pin_rope_properties(mutant=0):
    """Rotation at p = 0 is the identity, preserves the per-head norm, commutes with the L2 norm
    at full fraction, moves q/k by >= 1e-2 (vacuity) and moves the forward output."""
    rng = np.random.default_rng(9)
    x = rng.standard_normal((2, 6, 3, 16))
    y = oracle.prologue(x, l2norm=False, rope_theta=10000.0, pos_offset=0, mutant=mutant)
    assert np.allclose(y[:, 0], x[:, 0], atol=1e-15), "rotation at p = 0 is not the identity"
    assert np.allclose(np.linalg.norm(y, axis=-1), np.linalg.norm(x, axis=-1), rtol=1e-13)
    assert np.abs(y[:, 1:] - x[:, 1:]).max() > 1e-2, "rotation does not move q/k"
    a = oracle.prologue(x, l2norm=True, rope_theta=10000.0, pos_offset=7, mutant=mutant)
    n = oracle.prologue(x, l2norm=True, rope_theta=0.0, mutant=mutant)
    b = oracle.prologue(n, l2norm=False, rope_theta=10000.0, pos_offset=7, mutant=mutant)
    assert np.allclose(a, b, atol=1e-14), "l2norm(rope(x)) != rope(l2norm(x))"
    B, T, H, dk, dv = 1, 12, 2, 8, 4
    q = rng.standard_normal((B, T, H, dk))
    k = rng.standard_normal((B, T, H, dk))
    v = rng.standard_normal((B, T, H, dv))
    al = rng.uniform(-1, 1, (B, T, H, dk))
    be = rng.uniform(0, 2, (B, T, H))
    o0, _ = oracle.fwd(q, k, v, al, be, l2norm=True, rope_theta=0.0, mutant=mutant)
    o1, _ = oracle.fwd(q, k, v, al, be, l2norm=True, rope_theta=10000.0, mutant=mutant)
    assert np.abs(o1 - o0).max() / np.abs(o0).max() > 1e-2, "rotation does not move the output"


def pin_l2norm(mutant=0):
    """x / sqrt(sum x^2 + 1e-6) per head: norm sqrt(s/(s+1e-6)); each of q and k normalised alone
    (checked through the decode read-out with beta = 1, where o = scale (k.q) v)."""
    rng = np.random.default_rng(6)
    x = rng.standard_normal((1, 4, 3, 8)) * rng.uniform(0.1, 10, (1, 4, 3, 1))
    y = oracle.prologue(x, l2norm=True, mutant=mutant)
    s = (x * x).sum(-1)
    assert np.allclose(np.linalg.norm(y, axis=-1), np.sqrt(s / (s + 1e-6)), rtol=1e-13)
    assert np.allclose(y / np.linalg.norm(y, axis=-1, keepdims=True),
                       x / np.linalg.norm(x, axis=-1, keepdims=True), atol=1e-14)
    z = oracle.prologue(np.zeros((1, 1, 1, 8)), l2norm=True, mutant=mutant)
    assert np.all(z == 0.0)
    # one decode step from a zero state: o = scale * beta * (k_hat . q_hat) * v
    N, H, dk, dv = 3, 2, 8, 5
    q = rng.standard_normal((N, H, dk)) * 3.0
    k = rng.standard_normal((N, H, dk)) * 0.2
    v = rng.standard_normal((N, H, dv))
    o, _ = oracle.decode(q, k, v, np.ones((N, H, dk)), np.ones((N, H)), np.zeros((N, H, dk, dv)),
                         l2norm=True, mutant=mutant)
    qh = q / np.sqrt((q * q).sum(-1, keepdims=True) + 1e-6)
    kh = k / np.sqrt((k * k).sum(-1, keepdims=True) + 1e-6)
    want = (qh * kh).sum(-1)[..., None] * v / math.sqrt(dk)
    assert np.allclose(o, want, atol=1e-13), "q and k are not each L2-normalised per head"


# --- consistency of the entry points -----------------------------------------------------------

def pin_decode_matches_fwd(mutant=0):
    """T decode steps (positions pos_offset + t) reproduce the forward over T tokens, and a forward
    resumed from hT at the right position offset reproduces one long forward."""
    rng = np.random.default_rng(12)
    B, T, H, dk, dv = 2, 10, 2, 6, 4
    q = rng.standard_normal((B, T, H, dk))
    k = rng.standard_normal((B, T, H, dk))
    v = rng.standard_normal((B, T, H, dv))
    al = rng.uniform(-1, 1, (B, T, H, dk))
    be = rng.uniform(0, 2, (B, T, H))
    h0 = rng.standard_normal((B, H, dk, dv))
    kw = dict(l2norm=True, rope_theta=10000.0, rope_convention=0)
    o, hT = oracle.fwd(q, k, v, al, be, h0, pos_offset=3, mutant=mutant, **kw)
    st = h0.copy()
    for t in range(T):
        od, st = oracle.decode(q[:, t], k[:, t], v[:, t], al[:, t], be[:, t], st,
                               pos=np.full(B, 3 + t), mutant=mutant, **kw)
        assert np.allclose(od, o[:, t], atol=1e-13)
    assert np.allclose(st, hT, atol=1e-13)
    t1 = 4
    o1, s1 = oracle.fwd(q[:, :t1], k[:, :t1], v[:, :t1], al[:, :t1], be[:, :t1], h0, pos_offset=3,
                        mutant=mutant, **kw)
    o2, s2 = oracle.fwd(q[:, t1:], k[:, t1:], v[:, t1:], al[:, t1:], be[:, t1:], s1,
                        pos_offset=3 + t1, mutant=mutant, **kw)
    assert np.allclose(np.concatenate([o1, o2], axis=1), o, atol=1e-13)
    assert np.allclose(s2, hT, atol=1e-13)


def pin_gate_activation(mutant=0):
    """Gates from logits ("Complex KDA" paper summary, Methodology, CKDA Definition: beta = 2 sigma(b),
    signed alpha = 2 sigma(a) - 1), against facts outside the oracle: the identities
    2 sigma(x) - 1 = tanh(x / 2) and 2 sigma(x) = 1 + tanh(x / 2) (numpy's tanh, another formula),
    the values at 0, the odd / complementary symmetries and the ranges [-1, 1] and [0, 2] at the
    ends."""
    rng = np.random.default_rng(5)
    a = np.concatenate([rng.normal(0.0, 3.0, 500), [0.0, -0.0, 1e-8, -1e-8, 40.0, -40.0, 745.0, -745.0]])
    b = rng.normal(0.0, 3.0, 200)
    al, be = oracle.gates(a, b, mutant=mutant)
    assert np.allclose(al, np.tanh(a / 2.0), rtol=1e-14, atol=1e-15), "alpha = tanh(a/2)"
    assert np.allclose(be, 1.0 + np.tanh(b / 2.0), rtol=1e-14, atol=1e-15), "beta = 1 + tanh(b/2)"
    a0, b0 = oracle.gates(np.zeros(3), np.zeros(3), mutant=mutant)
    assert np.all(a0 == 0.0) and np.all(b0 == 1.0), "alpha(0) = 0, beta(0) = 1"
    am, bm = oracle.gates(-a, -b, mutant=mutant)
    assert np.allclose(am, -al, rtol=0, atol=1e-15), "alpha odd"
    assert np.allclose(bm + be, 2.0, rtol=0, atol=1e-15), "beta(b) + beta(-b) = 2"
    ends, bends = oracle.gates(np.array([800.0, -800.0]), np.array([800.0, -800.0]), mutant=mutant)
    assert ends[0] == 1.0 and ends[1] == -1.0, "alpha spans [-1, 1]"
    assert bends[0] == 2.0 and bends[1] == 0.0, "beta spans [0, 2]"


ALL_PINS = [pin_commutator, pin_2d_construction, pin_prop2_block, pin_orthogonal_norm,
            pin_delta_write, pin_identity_gates, pin_gdn_and_kda_spectra, pin_sign_absorption,
            pin_brute_force, pin_rope_closed_form, pin_rope_both_q_and_k, pin_rope_properties,
            pin_l2norm, pin_decode_matches_fwd, pin_gate_activation]
