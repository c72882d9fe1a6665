"""Grouped value heads (GVA) in the float64 oracle.

The pages describe GVA as a repeat of q and k on the head axis, with the L2 norm (and the
rotation) applied on the key-head axis above the repeat ("RoPE review", section 7).  Pins: every
value head h of a grouped run equals a single-head run on q/k head h // G with value head h's v,
gates and state, selected here with explicit index arithmetic (a tiled mapping h % Hk, or a repeat
on the wrong axis, fails); and the grouped decode step agrees with the forward on one token.
"""
import numpy as np

import oracle
import synth


def _case(B, T, H, G, seed, h0_std=0.02):
    d = synth.fwd_inputs(B, T, H, 16, 16, kind="ckda", dtype="f32", h0_std=h0_std, seed=seed)
    Hk = H // G
    # the first Hk heads of the generated q, k serve as the q/k heads
    return d["q"][:, :, :Hk].copy(), d["k"][:, :, :Hk].copy(), d


def test_grouped_forward_is_per_head_with_the_interleaved_mapping():
    B, T, H, G = 2, 40, 6, 3
    qk, kk, d = _case(B, T, H, G, seed=71)
    kw = dict(rope_theta=10000.0, rope_convention=1, pos_offset=5)
    out, hT = oracle.fwd(qk, kk, d["v"], d["alpha"], d["beta"], d["h0"], **kw)
    assert out.shape == (B, T, H, 16) and hT.shape == (B, H, 16, 16)
    for h in range(H):
        g = h // G
        o1, s1 = oracle.fwd(qk[:, :, g:g + 1], kk[:, :, g:g + 1], d["v"][:, :, h:h + 1],
                            d["alpha"][:, :, h:h + 1], d["beta"][:, :, h:h + 1],
                            d["h0"][:, h:h + 1], **kw)
        assert np.array_equal(out[:, :, h:h + 1], o1)
        assert np.array_equal(hT[:, h:h + 1], s1)
    # the tiled mapping h % Hk would read different q/k heads for h >= Hk
    Hk = H // G
    assert not np.allclose(qk[:, :, 1], qk[:, :, 0])
    h = 1
    o_tiled, _ = oracle.fwd(qk[:, :, h % Hk:h % Hk + 1], kk[:, :, h % Hk:h % Hk + 1],
                            d["v"][:, :, h:h + 1], d["alpha"][:, :, h:h + 1],
                            d["beta"][:, :, h:h + 1], d["h0"][:, h:h + 1], **kw)
    assert not np.allclose(out[:, :, h:h + 1], o_tiled)


def test_grouped_decode_equals_grouped_forward_on_one_token():
    N, H, G = 3, 4, 2
    qk, kk, d = _case(N, 1, H, G, seed=72)
    st0 = d["h0"]
    o_fwd, s_fwd = oracle.fwd(qk, kk, d["v"], d["alpha"], d["beta"], st0)
    o_dec, s_dec = oracle.decode(qk[:, 0], kk[:, 0], d["v"][:, 0], d["alpha"][:, 0],
                                 d["beta"][:, 0], st0)
    assert np.allclose(o_dec, o_fwd[:, 0], rtol=1e-12, atol=1e-14)
    assert np.allclose(s_dec, s_fwd, rtol=1e-12, atol=1e-14)
