"""Packed sequences of different lengths (cu_seqlens) in the float64 oracle.

The "RoPE review" (section 4) shows FLA's attention layer rotating packed sequences described by
cu_seqlens: token offsets [n + 1], sequence s owning tokens cu[s] .. cu[s+1] - 1 of one token
axis.  Read with the recurrence, each packed sequence is an independent sequence: it starts from
its own initial state, ends in its own final state, and its rotary positions start again at the
packing offset.  Pins: agreement with the batched oracle run on each sequence cut out on its own
(another indexing path of the C code) and on equal-length packs reshaped to a batch; no state and
no position crossing a boundary (two equal sequences packed side by side give equal results;
changing one sequence leaves the others bit for bit); an empty sequence hands h0 back as hT; bad
offsets are refused.
"""
import numpy as np
import pytest

import oracle


def _pack(lens, H, dk, dv, seed, Hk=None):
    rng = np.random.default_rng(seed)
    Hk = Hk or H
    T = int(sum(lens))
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    d = dict(q=rng.standard_normal((T, Hk, dk)), k=rng.standard_normal((T, Hk, dk)),
             v=rng.standard_normal((T, H, dv)),
             alpha=rng.choice([-1.0, 1.0], (T, H, dk)) * rng.uniform(0.05, 1.0, (T, H, dk)),
             beta=rng.uniform(0.0, 2.0, (T, H)),
             h0=0.3 * rng.standard_normal((len(lens), H, dk, dv)))
    return cu, d


@pytest.mark.parametrize("rope", [(0.0, 0, 0), (1000.0, 0, 0), (1000.0, 1, 4)])
def test_each_sequence_is_an_independent_run(rope):
    theta, conv, rd = rope
    lens = [7, 0, 13, 1, 20]
    cu, d = _pack(lens, 3, 8, 5, seed=1)
    kw = dict(rope_theta=theta, rope_convention=conv, rope_dims=rd, pos_offset=3)
    out, hT = oracle.fwd_varlen(d["q"], d["k"], d["v"], d["alpha"], d["beta"], cu, d["h0"], **kw)
    for s, n in enumerate(lens):
        sl = slice(cu[s], cu[s + 1])
        if n == 0:
            assert np.array_equal(hT[s], d["h0"][s])
            continue
        o1, h1 = oracle.fwd(*(d[x][None, sl] for x in ("q", "k", "v", "alpha", "beta")),
                            d["h0"][s:s + 1], **kw)
        assert np.allclose(out[sl], o1[0], rtol=0, atol=1e-13)
        assert np.allclose(hT[s], h1[0], rtol=0, atol=1e-13)


def test_equal_lengths_match_the_batched_layout():
    B, T, H, Hk = 3, 11, 4, 2
    cu, d = _pack([T] * B, H, 16, 8, seed=2, Hk=Hk)
    out, hT = oracle.fwd_varlen(d["q"], d["k"], d["v"], d["alpha"], d["beta"], cu, d["h0"],
                                rope_theta=500.0)
    bat = {x: d[x].reshape((B, T) + d[x].shape[1:]) for x in ("q", "k", "v", "alpha", "beta")}
    ob, hb = oracle.fwd(bat["q"], bat["k"], bat["v"], bat["alpha"], bat["beta"], d["h0"],
                        rope_theta=500.0)
    assert np.allclose(out.reshape(ob.shape), ob, rtol=0, atol=1e-13)
    assert np.allclose(hT, hb, rtol=0, atol=1e-13)


def test_no_state_or_position_crosses_a_boundary():
    # the same sequence packed twice (same h0): equal outputs and final states, RoPE on
    cu, d = _pack([9], 2, 8, 4, seed=3)
    two = {x: np.concatenate([d[x], d[x]]) for x in ("q", "k", "v", "alpha", "beta")}
    h0 = np.concatenate([d["h0"], d["h0"]])
    out, hT = oracle.fwd_varlen(two["q"], two["k"], two["v"], two["alpha"], two["beta"],
                                [0, 9, 18], h0, rope_theta=100.0)
    assert np.array_equal(out[:9], out[9:]) and np.array_equal(hT[0], hT[1])
    # changing the first sequence leaves the second one bit for bit
    cu, d = _pack([6, 10], 2, 8, 4, seed=4)
    o1, h1 = oracle.fwd_varlen(d["q"], d["k"], d["v"], d["alpha"], d["beta"], cu, d["h0"])
    d["v"][:6] += 1.0
    d["alpha"][:6] *= -1.0
    o2, h2 = oracle.fwd_varlen(d["q"], d["k"], d["v"], d["alpha"], d["beta"], cu, d["h0"])
    assert np.array_equal(o1[6:], o2[6:]) and np.array_equal(h1[1], h2[1])
    assert not np.allclose(o1[:6], o2[:6])


def test_bad_offsets_are_refused():
    cu, d = _pack([4, 4], 1, 4, 4, seed=5)
    args = (d["q"], d["k"], d["v"], d["alpha"], d["beta"])
    for bad in ([1, 4, 8], [0, 6, 5, 8], [0, 4, 7]):
        with pytest.raises((RuntimeError, AssertionError)):
            oracle.fwd_varlen(*args, bad)
