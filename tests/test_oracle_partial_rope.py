"""Partial rotation (rope_dims = dk / 2) in the float64 oracle.

The "RoPE review" (section 3) describes FLA's reference for a partial rotation: the leading
ro_dim channels are rotated as a vector of their own (ro_dim / 2 frequencies, half-split or
interleaved pairs among those channels) and the channels after them pass through unchanged; it
names the fractions 0.5 and 1.0 as the ones accepted.
Pins: the partial rotation equals the full rotation of the first dk / 2 channels as a head of
dk / 2 channels (whose frequencies and pairings the full-rotation pins already fix), with the
other half untouched; it differs from the full rotation; the inner product of a rotated q at
position m and a rotated k at position n depends only on m - n; and the L2 norm commutes with it.

On that last point the review claims that the two orders give different results once the norm
runs over the whole head.  The arithmetic decides otherwise: a partial rotation is linear and
orthogonal (a rotation on the leading channels, the identity on the rest), so it keeps the norm and
commutes with a scaling of the whole head.  The oracle rotates first, then normalises; the test
shows the order is free.
"""
import numpy as np
import pytest

import oracle


def _x(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


@pytest.mark.parametrize("conv", [0, 1])
def test_partial_rotation_is_a_full_rotation_of_the_first_half(conv):
    x = _x((2, 9, 3, 64), 5)
    kw = dict(l2norm=False, rope_theta=10000.0, rope_convention=conv, pos_offset=17)
    y = oracle.prologue(x, rope_dims=32, **kw)
    head = oracle.prologue(np.ascontiguousarray(x[..., :32]), **kw)
    assert np.allclose(y[..., :32], head, rtol=0, atol=1e-13)
    assert np.array_equal(y[..., 32:], x[..., 32:])
    full = oracle.prologue(x, **kw)
    assert not np.allclose(y, full)
    # the rotation happened (positions > 0)
    assert not np.allclose(y[..., :32], x[..., :32])


@pytest.mark.parametrize("conv", [0, 1])
def test_partial_rotation_is_relative(conv):
    rng = np.random.default_rng(9)
    q = rng.standard_normal((1, 1, 1, 64))
    k = rng.standard_normal((1, 1, 1, 64))
    kw = dict(l2norm=False, rope_theta=500.0, rope_convention=conv, rope_dims=32)
    def dot(m, n):
        return float(np.sum(oracle.prologue(q, pos_offset=m, **kw) * oracle.prologue(k, pos_offset=n, **kw)))
    assert dot(7, 3) == pytest.approx(dot(104, 100), abs=1e-12)
    assert dot(0, 0) == pytest.approx(float(np.sum(q * k)), abs=1e-12)


@pytest.mark.parametrize("conv", [0, 1])
def test_l2_norm_commutes_with_the_partial_rotation(conv):
    x = _x((1, 12, 2, 128), 7)
    kw = dict(rope_theta=10000.0, rope_convention=conv, rope_dims=64, pos_offset=3)
    rot_then_norm = oracle.prologue(x, l2norm=True, **kw)
    norm_then_rot = oracle.prologue(oracle.prologue(x, l2norm=True), l2norm=False, **kw)
    assert np.allclose(rot_then_norm, norm_then_rot, rtol=0, atol=1e-12)
    # the rotation keeps each head's norm
    r = oracle.prologue(x, l2norm=False, **kw)
    assert np.allclose(np.linalg.norm(r, axis=-1), np.linalg.norm(x, axis=-1), rtol=1e-13)


def test_forward_uses_the_partial_rotation():
    import synth
    d = synth.fwd_inputs(1, 20, 2, 32, 16, kind="ckda", dtype="f32", h0_std=0.02, seed=33)
    kw = dict(rope_theta=10000.0, rope_convention=0)
    o_part, _ = oracle.fwd(d["q"], d["k"], d["v"], d["alpha"], d["beta"], d["h0"], rope_dims=16, **kw)
    # the same forward on q, k rotated beforehand by the partial prologue (no norm), norm after
    qr = oracle.prologue(d["q"], l2norm=False, rope_dims=16, **kw)
    kr = oracle.prologue(d["k"], l2norm=False, rope_dims=16, **kw)
    o_pre, _ = oracle.fwd(qr, kr, d["v"], d["alpha"], d["beta"], d["h0"])
    assert np.allclose(o_part, o_pre, rtol=0, atol=1e-12)
    o_full, _ = oracle.fwd(d["q"], d["k"], d["v"], d["alpha"], d["beta"], d["h0"], **kw)
    assert not np.allclose(o_part, o_full)
