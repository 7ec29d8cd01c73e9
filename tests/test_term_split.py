"""The arithmetic the fp32 mode rests on, checked on the CPU with exact
rounding: an fp32 value x carried as bf16 terms x_0 = bf16(x),
x_1 = bf16(x - x_0), x_2 = bf16(x - x_0 - x_1) (round to nearest even, every
remainder exact in fp32).

- Each rounding to bf16 (8 significant bits) leaves at most 2^-8 of its
  input, so |x_1| <= 2^-8 |x| and |x_2| <= 2^-16 |x|.
- Two terms keep x to 2^-17 relative (measured bound over a wide sample).
- Three terms keep every normal fp32 value exactly (whose bf16 rounding does
  not overflow, |x| < 3.39e38, and whose remainders stay normal): 24
  significant bits fit in 8 + 8 + 8, and each remainder is a multiple of x's
  last-place unit.
- The dropped term products: two terms drop a_1 b_1, at most 2^-16 |a b|
  and typically ~2^-18; three terms drop a_1 b_2, a_2 b_1, a_2 b_2, at most
  ~2^-23 |a b| and typically ~2^-27.
"""
import numpy as np

from oracle import vggt_oracle as O


def terms(x: np.ndarray, n: int):
    """The n bf16 terms of float32 x, as float64 values."""
    out = []
    r = x.astype(np.float32)
    for _ in range(n):
        t = O.bf16_bits_to_f32(O.f32_to_bf16_bits(r))
        out.append(t.astype(np.float64))
        r = (r - t).astype(np.float32)
    return out


def sample(n=200_000, seed=0):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal(n) * np.exp2(rng.integers(-60, 60, n))
    x = x.astype(np.float32)
    return x[(x != 0) & np.isfinite(x)]


def test_remainders_are_exact_in_fp32():
    x = sample()
    t0 = O.bf16_bits_to_f32(O.f32_to_bf16_bits(x))
    r = (x - t0).astype(np.float32)
    assert np.array_equal(r.astype(np.float64), x.astype(np.float64) - t0.astype(np.float64))


def test_two_terms_keep_x_to_2_pow_minus_17():
    x = sample()
    t = terms(x, 2)
    err = np.abs(x.astype(np.float64) - t[0] - t[1]) / np.abs(x.astype(np.float64))
    assert err.max() <= 2.0 ** -17
    assert err.max() > 2.0 ** -19  # the bound is nearly reached: the two terms are not exact


def test_three_terms_are_exact():
    x = sample()
    t = terms(x, 3)
    assert np.array_equal(t[0] + t[1] + t[2], x.astype(np.float64))


def test_three_terms_exact_on_hard_values():
    # values whose 24 bits alternate, and values next to powers of two
    bits = np.array([0x3F555555, 0x3FAAAAAB, 0x3F7FFFFF, 0x3F800001, 0x4B7FFFFF, 0x0B800001, 0x7F7F7FFF,
                     0xBF555555], dtype=np.uint32)
    x = bits.view(np.float32)
    t = terms(x, 3)
    assert np.array_equal(t[0] + t[1] + t[2], x.astype(np.float64))


def test_dropped_products_are_small():
    a, b = sample(seed=1), sample(seed=2)
    n = min(len(a), len(b))
    a, b = a[:n], b[:n]
    exact = a.astype(np.float64) * b.astype(np.float64)
    ab = np.abs(exact)
    ta2, tb2 = terms(a, 2), terms(b, 2)
    d2 = np.abs(ta2[1] * tb2[1]) / ab
    assert d2.max() <= 2.0 ** -16 and np.median(d2[d2 > 0]) < 2.0 ** -17
    ta3, tb3 = terms(a, 3), terms(b, 3)
    d3 = sum(np.abs(ta3[i] * tb3[j]) for i in range(3) for j in range(3) if i + j >= 3) / ab
    assert d3.max() <= 2.0 ** -23 and np.median(d3[d3 > 0]) < 2.0 ** -26
    # what the kept products miss, against the exact product
    kept2 = ta2[0] * tb2[0] + ta2[0] * tb2[1] + ta2[1] * tb2[0]
    assert (np.abs(kept2 - exact) <= 2.0 ** -15 * ab).all()
    kept3 = sum(ta3[i] * tb3[j] for i in range(3) for j in range(3) if i + j < 3)
    assert (np.abs(kept3 - exact) <= 2.0 ** -23 * ab).all()
