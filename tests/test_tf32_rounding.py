"""Integer forms of tf32 operand preparation (CPU): the rounding of the fused forward's T-merge
operands, and the head/tail split of the CUDA-core paths' fp32-grade warp tiles.

The fused kernel rounds an fp32 value to tf32 (10 stored mantissa bits, round to nearest, ties
away from zero -- the rounding of cvt.rna.tf32.f32 in the PTX ISA) by integer arithmetic on its
bit pattern: (bits + 0x1000) & 0xffffe000.  This checks that expression against the rounding
computed independently in float64 (frexp / ldexp, the significand scaled to 11 bits and rounded
half away from zero) over a spread of normal floats of both signs, including every tie.
"""
import numpy as np


def _integer_form(x):
    u = x.view(np.uint32)
    return ((u + np.uint32(0x1000)) & np.uint32(0xffffe000)).view(np.float32)


def _reference(x):
    m, e = np.frexp(np.abs(x.astype(np.float64)))          # |x| = m 2^e, m in [0.5, 1)
    s = np.ldexp(m, 11)
    r = np.floor(s + 0.5)                                     # half away from zero on |x|
    return (np.sign(x) * np.ldexp(r, e - 11)).astype(np.float32)


def test_integer_tf32_rounding_matches_round_half_away():
    rng = np.random.default_rng(0)
    bits = rng.integers(0x00800000, 0x7f000000, size=4_000_000, dtype=np.uint32)
    bits[: 1 << 20] = (bits[: 1 << 20] & np.uint32(0xffffe000)) | np.uint32(0x1000)   # ties
    bits[::2] |= np.uint32(0x80000000)                                               # negatives
    x = bits.view(np.float32)
    got, want = _integer_form(x), _reference(x)
    assert np.array_equal(got.view(np.uint32), want.view(np.uint32))


def test_a_truncating_form_differs():
    """Clearing the low bits without the half-unit increment (truncation) is a different
    rounding: it misses on every value whose dropped bits are at least half a unit."""
    x = np.array([1.0 + 2.0 ** -11, -3.0 - 2.0 ** -10 - 2.0 ** -11], dtype=np.float32)
    trunc = (x.view(np.uint32) & np.uint32(0xffffe000)).view(np.float32)
    assert not np.array_equal(trunc, _reference(x))
    assert np.array_equal(_integer_form(x), _reference(x))


def _mask_split(x):
    """Head and tail of the warp tiles' split-tf32 operands: the head is x with its 13 low
    mantissa bits cleared, the tail the remainder x - head (exact in fp32) cut the same way."""
    m = np.uint32(0xffffe000)
    hi = (x.view(np.uint32) & m).view(np.float32)
    lo = ((x - hi).view(np.uint32) & m).view(np.float32)
    return hi.astype(np.float64), lo.astype(np.float64)


def test_mask_split_products_hold_three_units_of_2_pow_minus_20():
    """a b = a_hi b_hi + a_hi b_lo + a_lo b_hi (the three tensor-core products; each tf32 product
    is exact in fp32 accumulation terms, here in float64) within 3 * 2^-20 of |a b|, and the
    split loses at most 2^-20 of each operand."""
    rng = np.random.default_rng(1)
    a = (rng.standard_normal(2_000_000) * 10.0 ** rng.uniform(-6, 6, 2_000_000)).astype(np.float32)
    b = (rng.standard_normal(2_000_000) * 10.0 ** rng.uniform(-6, 6, 2_000_000)).astype(np.float32)
    ah, al = _mask_split(a)
    bh, bl = _mask_split(b)
    a64, b64 = a.astype(np.float64), b.astype(np.float64)
    assert np.all(np.abs(a64 - (ah + al)) <= 2.0 ** -20 * np.abs(a64))
    prod = ah * bh + ah * bl + al * bh
    assert np.all(np.abs(prod - a64 * b64) <= 3 * 2.0 ** -20 * np.abs(a64 * b64))
    # a single tf32 product (no tails) is only good to about 2^-10
    assert np.max(np.abs(ah * bh - a64 * b64) / np.abs(a64 * b64)) > 2.0 ** -12
