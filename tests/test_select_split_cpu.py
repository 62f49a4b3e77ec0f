"""The error bound of the tensor-core selection scores, on the host.

The selection kernel multiplies fp32 pooled means on the tensor cores in
tf32 by splitting every operand x into hi (x with its low 13 mantissa bits
cleared, exactly a tf32 value) and lo = x - hi, and summing qh*kh + qh*kl +
ql*kh.  The tensor cores read lo as tf32 too.  Emulated here in fp64 with lo
truncated to tf32 (the worst case; rounding halves it), each channel's
product must stay within 3 * 2^-20 |q_c||k_c| of the exact one, and a full
score within 3 * 2^-20 sum_c |q_c||k_c| (plus fp32 accumulation rounding on
the device, not modelled here).  A split that kept only qh*kh, or forgot the
truncation of lo, must break the bound it claims.
"""
import numpy as np


def tf32_trunc(x):
    """fp32 values with the low 13 mantissa bits cleared (exact tf32)."""
    u = np.asarray(x, dtype=np.float32).view(np.uint32) & np.uint32(0xFFFFE000)
    return u.view(np.float32)


def split_products(q, k, drop_lo=False):
    qh, kh = tf32_trunc(q), tf32_trunc(k)
    ql = (q.astype(np.float32) - qh).astype(np.float32)   # exact in fp32
    kl = (k.astype(np.float32) - kh).astype(np.float32)
    qlt, klt = tf32_trunc(ql), tf32_trunc(kl)             # what the MMA reads
    p = qh.astype(np.float64) * kh.astype(np.float64)
    if not drop_lo:
        p += qh.astype(np.float64) * klt.astype(np.float64)
        p += qlt.astype(np.float64) * kh.astype(np.float64)
    return p


def draw(rng, shape):
    # pooled means: block averages of unit-scale tokens, with a spread of
    # magnitudes (exponents) to exercise the split at every binade
    x = rng.standard_normal(shape) * np.exp2(rng.integers(-12, 4, size=shape))
    return x.astype(np.float32)


def test_hi_lo_split_is_exact():
    rng = np.random.default_rng(7)
    x = draw(rng, (4096,))
    hi = tf32_trunc(x)
    lo = (x - hi).astype(np.float32)
    assert np.array_equal((hi.astype(np.float64) + lo.astype(np.float64)), x.astype(np.float64))
    # hi carries at most 10 explicit mantissa bits
    assert np.all((hi.view(np.uint32) & np.uint32(0x1FFF)) == 0)


def test_channel_products_within_three_times_2_pow_minus_20():
    rng = np.random.default_rng(11)
    q, k = draw(rng, (200000,)), draw(rng, (200000,))
    exact = q.astype(np.float64) * k.astype(np.float64)
    err = np.abs(split_products(q, k) - exact)
    bound = 3.0 * 2.0 ** -20 * np.abs(exact)
    assert np.all(err <= bound)
    # the bound is not loose by orders of magnitude
    assert err.max() > 2.0 ** -24 * np.abs(exact).max() * 1e-3


def test_scores_within_bound_and_single_product_fails_it():
    rng = np.random.default_rng(13)
    q, k = draw(rng, (512, 128)), draw(rng, (512, 128))
    exact = (q.astype(np.float64) * k.astype(np.float64)).sum(axis=1)
    scale = (np.abs(q.astype(np.float64)) * np.abs(k.astype(np.float64))).sum(axis=1)
    got = split_products(q, k).sum(axis=1)
    assert np.all(np.abs(got - exact) <= 3.0 * 2.0 ** -20 * scale)
    # a planted mistake: hi products only (no split) misses the bound
    bad = split_products(q, k, drop_lo=True).sum(axis=1)
    assert np.any(np.abs(bad - exact) > 3.0 * 2.0 ** -20 * scale)
