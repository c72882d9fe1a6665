"""Gradients of the float64 oracle (the backward pass, backpropagation through the token loop),
pinned to central finite differences of the oracle's own forward (which is pinned by the closed
forms, the brute-force products and the other pins) and to a closed form.

L = <dout, out> + <dhT, hT> with random dout, dhT; every element of q, k, v, alpha, beta and h0
is perturbed by +-1e-6.  The cases cover the L2 norm on and off, the rotation (half-split, and
interleaved over half the channels), a read-out scale, and grouped value heads (a q/k head's
gradient is the sum over the value heads it serves).
"""
import numpy as np
import pytest

import oracle


def _inputs(B, T, H, Hk, dk, dv, seed):
    rng = np.random.default_rng(seed)
    return dict(q=rng.standard_normal((B, T, Hk, dk)), k=rng.standard_normal((B, T, Hk, dk)),
                v=rng.standard_normal((B, T, H, dv)),
                alpha=rng.choice([-1.0, 1.0], (B, T, H, dk)) * rng.uniform(0.2, 1.0, (B, T, H, dk)),
                beta=rng.uniform(0.0, 2.0, (B, T, H)), h0=0.5 * rng.standard_normal((B, H, dk, dv)))


CASES = [
    dict(name="plain", H=2, Hk=2, dk=4, dv=3, kw=dict()),
    dict(name="rope-half", H=1, Hk=1, dk=6, dv=3, kw=dict(rope_theta=100.0, pos_offset=5)),
    dict(name="rope-partial-interleaved-no-norm", H=1, Hk=1, dk=8, dv=2,
         kw=dict(rope_theta=50.0, rope_convention=1, rope_dims=4, l2norm=False, scale=0.7)),
    dict(name="grouped-heads", H=4, Hk=2, dk=4, dv=2, kw=dict(rope_theta=10.0)),
]


@pytest.mark.parametrize("case", CASES, ids=[c["name"] for c in CASES])
def test_gradients_match_finite_differences(case):
    B, T = 1, 5
    x = _inputs(B, T, case["H"], case["Hk"], case["dk"], case["dv"], seed=10 + [c["name"] for c in CASES].index(case["name"]))
    rng = np.random.default_rng(99)
    dout = rng.standard_normal((B, T, case["H"], case["dv"]))
    dhT = rng.standard_normal((B, case["H"], case["dk"], case["dv"]))
    kw = case["kw"]

    def loss(**over):
        a = dict(x)
        a.update(over)
        o, hT = oracle.fwd(a["q"], a["k"], a["v"], a["alpha"], a["beta"], a["h0"], nthreads=1, **kw)
        return float((o * dout).sum() + (hT * dhT).sum())

    g = oracle.bwd(x["q"], x["k"], x["v"], x["alpha"], x["beta"], x["h0"], dout, dhT, **kw)
    eps = 1e-6
    for name, gname in (("q", "dq"), ("k", "dk"), ("v", "dv"), ("alpha", "dalpha"),
                        ("beta", "dbeta"), ("h0", "dh0")):
        fd = np.zeros_like(x[name])
        for idx in np.ndindex(x[name].shape):
            xp = x[name].copy()
            xm = x[name].copy()
            xp[idx] += eps
            xm[idx] -= eps
            fd[idx] = (loss(**{name: xp}) - loss(**{name: xm})) / (2 * eps)
        assert g[gname].shape == fd.shape
        err = np.abs(g[gname] - fd).max() / max(np.abs(fd).max(), 1e-12)
        assert err < 1e-6, (name, err)


def test_identity_gates_closed_form():
    # beta = 0, alpha = 1: S_t = h0 for every t, out_t = scale h0^T q^_t, so
    # dh0 = dhT + scale sum_t q^_t dout_t^T and dv = 0
    B, T, H, dk, dv = 1, 7, 2, 8, 4
    x = _inputs(B, T, H, H, dk, dv, seed=3)
    x["alpha"][:] = 1.0
    x["beta"][:] = 0.0
    rng = np.random.default_rng(4)
    dout = rng.standard_normal((B, T, H, dv))
    dhT = rng.standard_normal((B, H, dk, dv))
    g = oracle.bwd(x["q"], x["k"], x["v"], x["alpha"], x["beta"], x["h0"], dout, dhT)
    qh = oracle.prologue(x["q"])                         # L2-normalised q
    want = dhT + np.einsum("bthi,bthj->bhij", qh, dout) / np.sqrt(dk)
    assert np.allclose(g["dh0"], want, rtol=0, atol=1e-12)
    assert np.array_equal(g["dv"], np.zeros_like(g["dv"]))
