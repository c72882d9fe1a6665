"""The segment decomposition the segment-parallel forward is built on, checked with the float64
oracle alone (CPU).

The recurrence S_t = A_t S_{t-1} + beta_t k_t v_t^T (A_t = (I - beta_t k_t k_t^T) Diag(alpha_t),
the transition of the "Complex KDA" paper summary, Background) is affine in the state, so over a
segment of tokens the end state is F S_in + E: F the product of the segment's transitions (the
same run entered with the identity and with v = 0) and E the end state entered with zero.  The
state entering segment s + 1 is then S_{s+1} = F_s S_s + E_s, and a segment run from its entering
state gives the outputs of the whole run on its tokens.  Every quantity below is an oracle run on
a slice of the inputs (rotary positions offset to the slice's first token); nothing of the GPU
code is involved.
"""
import numpy as np
import pytest

import oracle
import synth


def _case(T, H, d, seed, kind="ckda"):
    x = synth.fwd_inputs(1, T, H, d, d, kind=kind, dtype="f32", h0_std=0.1, seed=seed)
    return x["q"], x["k"], x["v"], x["alpha"], x["beta"], x["h0"]


def _segments(T, L):
    return [(t0, min(T, t0 + L)) for t0 in range(0, T, L)]


def _summaries(q, k, v, a, b, h0, segs, kw):
    """E_s (entered with h0 for s = 0, zero otherwise) and F_s of every segment."""
    H, d = v.shape[2], v.shape[3]
    eye = np.broadcast_to(np.eye(d), (1, H, d, d)).copy()
    E, F = [], []
    for s, (t0, t1) in enumerate(segs):
        sl = slice(t0, t1)
        args = (q[:, sl], k[:, sl])
        _, e = oracle.fwd(*args, v[:, sl], a[:, sl], b[:, sl], h0 if s == 0 else None,
                          pos_offset=t0, **kw)
        _, f = oracle.fwd(*args, np.zeros_like(v[:, sl]), a[:, sl], b[:, sl], eye,
                          pos_offset=t0, **kw)
        E.append(e)
        F.append(f)
    return E, F


def _scan(E, F, h0, transpose=False):
    """States entering every segment: S_0 = h0, S_1 = E_0, S_{s+1} = F_s S_s + E_s."""
    S = [h0] + ([E[0]] if len(E) > 1 else [])
    for s in range(1, len(E) - 1):
        Fs = np.swapaxes(F[s], -1, -2) if transpose else F[s]
        S.append(np.einsum("bhij,bhjn->bhin", Fs, S[s]) + E[s])
    return S


@pytest.mark.parametrize("T,L,rope", [(200, 64, 0.0), (300, 37, 1e4), (128, 128, 0.0)])
def test_segments_reproduce_the_run(T, L, rope):
    q, k, v, a, b, h0 = _case(T, 2, 8, seed=T + L)
    kw = dict(rope_theta=rope)
    out, hT = oracle.fwd(q, k, v, a, b, h0, **kw)
    segs = _segments(T, L)
    E, F = _summaries(q, k, v, a, b, h0, segs, kw)
    S = _scan(E, F, h0)
    assert len(S) == len(segs)
    for s, (t0, t1) in enumerate(segs):
        sl = slice(t0, t1)
        o_s, h_s = oracle.fwd(q[:, sl], k[:, sl], v[:, sl], a[:, sl], b[:, sl], S[s],
                              pos_offset=t0, **kw)
        np.testing.assert_allclose(o_s, out[:, sl], rtol=0, atol=1e-11 * np.abs(out).max())
        if s + 1 == len(segs):
            np.testing.assert_allclose(h_s, hT, rtol=0, atol=1e-11 * np.abs(hT).max())


def test_transition_is_the_product_of_the_token_transitions():
    """F of a segment (the oracle entered with the identity, v = 0) equals A_T ... A_1 built
    densely, token by token, by the separate dense restatement (prepared k, then
    (I - beta k k^T) Diag(alpha))."""
    from oracle import dense
    T, d, t0 = 24, 4, 7
    q, k, v, a, b, h0 = _case(T, 1, d, seed=5)
    eye = np.eye(d)[None, None]
    _, Fo = oracle.fwd(q, k, np.zeros_like(v), a, b, eye, rope_theta=1e4, pos_offset=t0)
    P = np.eye(d)
    for t in range(T):
        kt = dense.prepare(np.asarray(k[0, t, 0], np.float64), t0 + t, True, 1e4, 0)
        P = dense.transition(kt, np.asarray(a[0, t, 0], np.float64), float(b[0, t, 0])) @ P
    np.testing.assert_allclose(Fo[0, 0], P, rtol=0, atol=1e-12)


def test_a_transposed_composition_fails():
    """The composition order matters: F_s^T in place of F_s misses the run (long memory, so the
    entering states carry weight)."""
    T, L = 192, 48
    q, k, v, a, b, h0 = _case(T, 2, 8, seed=9, kind="longmem")
    _, hT = oracle.fwd(q, k, v, a, b, h0)
    segs = _segments(T, L)
    E, F = _summaries(q, k, v, a, b, h0, segs, {})
    S_bad = _scan(E, F, h0, transpose=True)
    _, h_bad = oracle.fwd(q[:, segs[-1][0]:], k[:, segs[-1][0]:], v[:, segs[-1][0]:],
                          a[:, segs[-1][0]:], b[:, segs[-1][0]:], S_bad[-1],
                          pos_offset=segs[-1][0])
    assert np.abs(h_bad - hT).max() > 1e-3 * np.abs(hT).max()
