"""The accuracy argument of the tensor-core pooled logits, checked in numpy:
each block mean m is split as hi = tf32(m), lo = tf32(m - hi) (round to
nearest), and a product is taken as lo_q hi_k + hi_q lo_k + hi_q hi_k.  The
dropped lo_q lo_k term and the rounding of lo stay below 3 * 2^-22 (under
2^-20) of |q| |k| per channel, the size of fp32 rounding."""

import numpy as np


def tf32_rna(x):
    """fp32 -> tf32, round to nearest (ties away from zero), as fp32."""
    b = np.asarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    b = ((b + 0x1000) & 0xFFFFE000).astype(np.uint32)
    return b.view(np.float32)


def test_tf32_rounding_keeps_ten_mantissa_bits():
    # ulp 2^-10 on [1, 2) and 2^-9 on [2, 4): exact, tie (away from zero),
    # below half an ulp, negative tie
    x = np.float32([1.0 + 2.0 ** -10, 1.0 + 2.0 ** -11, 1.0 + 2.0 ** -12, -3.0 - 2.0 ** -10])
    np.testing.assert_array_equal(tf32_rna(x), np.float32([1.0 + 2.0 ** -10, 1.0 + 2.0 ** -10,
                                                           1.0, -3.0 - 2.0 ** -9]))


def test_split_product_error_bound():
    rng = np.random.default_rng(11)
    for scale in (1e-3, 1.0, 1e3):
        q = (rng.standard_normal((4000, 128)) * scale).astype(np.float32)
        k = (rng.standard_normal((4000, 128)) * scale).astype(np.float32)
        # a wide dynamic range inside a vector too
        q[:, ::7] *= np.float32(1e-4)
        qh, kh = tf32_rna(q), tf32_rna(k)
        ql = tf32_rna(q - qh)                     # q - hi is exact in fp32
        kl = tf32_rna(k - kh)
        assert np.all(np.abs(q.astype(np.float64) - qh) <= 2.0 ** -11 * np.abs(q))
        split = (ql.astype(np.float64) * kh + qh.astype(np.float64) * kl +
                 qh.astype(np.float64) * kh)
        exact = q.astype(np.float64) * k
        err = np.abs(split - exact)
        bound = 3.0 * 2.0 ** -22 * (1 + 2.0 ** -10) * np.abs(exact)
        assert np.all(err <= bound)
        # per dot product: under 2^-20 of sum |q_c| |k_c|
        derr = np.abs(split.sum(axis=1) - exact.sum(axis=1))
        assert np.all(derr <= 2.0 ** -20 * np.abs(exact).sum(axis=1))


def test_single_tf32_product_would_not_do():
    # without the lo terms the error is ~2^-11 relative: far above fp32
    rng = np.random.default_rng(12)
    q = rng.standard_normal((1000, 128)).astype(np.float32)
    k = rng.standard_normal((1000, 128)).astype(np.float32)
    one = tf32_rna(q).astype(np.float64) * tf32_rna(k)
    exact = q.astype(np.float64) * k
    assert np.max(np.abs(one - exact) / np.abs(exact)) > 2.0 ** -13
