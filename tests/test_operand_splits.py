"""The operand splits the tensor-core flush relies on, pinned on the CPU.

The tensor-core flush feeds fp32 values to tf32 and bf16 MMAs and recovers
fp32 accuracy by splitting operands (paper §4.1 needs fp32 state arithmetic;
the parity bar is 1e-4):

* bf16 in three parts (GDN's Gram products): p1 = bf16(x), p2 = bf16(x - p1),
  p3 = bf16(x - p1 - p2), each rounded to nearest even; p1 + p2 + p3 = x
  exactly for every fp32 x in the normal range, and every bf16 x bf16 product
  is exact in fp32, so sum_i p_i k against a bf16 key k is x k up to the
  accumulation's rounding.
* tf32 hi / lo (the pass and the update): hi = x with the 13 low mantissa
  bits cleared (the tensor core's own conversion of an fp32 operand), lo =
  x - hi exact in fp32; with b exact in tf32 the product hi b + tf32(lo) b
  is within 2^-21 |x b|, and with both split, hi hi + hi lo + lo hi is within
  2^-19 |x y| (each lo half loses up to 2^-20 |x| to its own truncation).
These are properties of the arithmetic the kernel performs, checked by
emulating its roundings bit for bit in numpy.
"""
import numpy as np


def bf16_rn(x):
    """fp32 -> bf16 (round to nearest, ties to even), returned as fp32."""
    b = np.asarray(x, np.float32).view(np.uint32).astype(np.uint64)
    b = (b + 0x7FFF + ((b >> 16) & 1)) & 0xFFFF0000
    return b.astype(np.uint32).view(np.float32)


def tf32_trunc(x):
    """fp32 with its 13 low mantissa bits cleared."""
    return (np.asarray(x, np.float32).view(np.uint32) & np.uint32(0xFFFFE000)).view(np.float32)


def three_parts(x):
    x = np.asarray(x, np.float32)
    p1 = bf16_rn(x)
    r1 = (x - p1).astype(np.float32)
    p2 = bf16_rn(r1)
    r2 = (r1 - p2).astype(np.float32)
    p3 = bf16_rn(r2)
    return p1, p2, p3, r1, r2


def _samples(rng, n=200_000):
    mant = rng.uniform(1.0, 2.0, n)
    exp = rng.integers(-100, 100, n)
    sign = rng.choice([-1.0, 1.0], n)
    x = (sign * mant * np.exp2(exp)).astype(np.float32)
    # halfway cases of the first rounding: low 16 bits 0x8000 exactly, and its neighbours
    bits = x[:4096].view(np.uint32) & np.uint32(0xFFFF0000)
    half = np.concatenate([bits | np.uint32(0x8000), bits | np.uint32(0x7FFF), bits | np.uint32(0x8001)])
    return np.concatenate([x, half.view(np.float32), np.float32([1.0, -1.0, 3.0, 1.0 + 2 ** -23])])


def test_bf16_three_parts_sum_exactly():
    x = _samples(np.random.default_rng(1))
    p1, p2, p3, r1, r2 = three_parts(x)
    # the remainders are exact in fp32 (no rounding in x - p1 and r1 - p2)
    assert np.array_equal(r1.astype(np.float64), x.astype(np.float64) - p1.astype(np.float64))
    assert np.array_equal(r2.astype(np.float64), r1.astype(np.float64) - p2.astype(np.float64))
    # and the last part takes what is left without rounding
    assert np.array_equal(p3, r2)
    total = p1.astype(np.float64) + p2.astype(np.float64) + p3.astype(np.float64)
    assert np.array_equal(total, x.astype(np.float64))


def test_bf16_products_are_exact_in_fp32():
    rng = np.random.default_rng(2)
    a = bf16_rn(rng.standard_normal(100_000).astype(np.float32))
    b = bf16_rn(rng.standard_normal(100_000).astype(np.float32))
    exact = a.astype(np.float64) * b.astype(np.float64)
    assert np.array_equal((a * b).astype(np.float64), exact)


def test_three_part_dot_against_bf16_keys_is_the_fp32_dot():
    rng = np.random.default_rng(3)
    x = rng.standard_normal((64, 128)).astype(np.float32)          # probes
    k = bf16_rn(rng.standard_normal((16, 128)).astype(np.float32))  # keys, exact in bf16
    p1, p2, p3, _, _ = three_parts(x)
    parts = sum(p.astype(np.float64) @ k.T.astype(np.float64) for p in (p1, p2, p3))
    assert np.array_equal(parts, x.astype(np.float64) @ k.T.astype(np.float64))
    # without the third part the error is of order 2^-16: the split needs it
    two = (p1.astype(np.float64) + p2.astype(np.float64)) @ k.T.astype(np.float64)
    ref = x.astype(np.float64) @ k.T.astype(np.float64)
    assert np.abs(two - ref).max() > 1e-7 * np.abs(ref).max()


def test_tf32_hi_lo_products():
    rng = np.random.default_rng(4)
    x = rng.standard_normal(100_000).astype(np.float32)
    y = rng.standard_normal(100_000).astype(np.float32)
    hx = tf32_trunc(x)
    lx = (x - hx).astype(np.float32)
    assert np.array_equal(lx.astype(np.float64), x.astype(np.float64) - hx.astype(np.float64))
    # against a value exact in tf32 (a bf16 key): hi b + tf32(lo) b
    b = bf16_rn(y)
    prod = hx.astype(np.float64) * b + tf32_trunc(lx).astype(np.float64) * b
    ref = x.astype(np.float64) * b.astype(np.float64)
    assert np.all(np.abs(prod - ref) <= 2.0 ** -21 * np.abs(ref) + 1e-300)
    # both split: hi hi + hi lo + lo hi, each operand truncated to tf32
    hy = tf32_trunc(y)
    ly = (y - hy).astype(np.float32)
    t = lambda v: tf32_trunc(v).astype(np.float64)
    prod3 = t(hx) * t(hy) + t(hx) * t(ly) + t(lx) * t(hy)
    ref3 = x.astype(np.float64) * y.astype(np.float64)
    assert np.all(np.abs(prod3 - ref3) <= 2.0 ** -19 * np.abs(ref3) + 1e-300)
    # one product alone is only tf32-accurate: beyond the 1e-4 parity bar
    assert np.max(np.abs(t(hx) * t(hy) - ref3) / np.abs(ref3)) > 1e-4
