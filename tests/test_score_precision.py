"""The tf32 split behind the tensor-core centroid scores, emulated on the
host: the split is exact, the three-product form stays inside the tolerance
the GPU score test allows, and the one-product (plain tf32) form does not --
so that tolerance tells the two apart.  No GPU needed.

x = hi + lo with hi = x with its 13 low mantissa bits cleared (a tf32 value)
and lo = x - hi; the product x*y is taken as hi_x*hi_y + hi_x*lo_y + lo_x*hi_y
with lo itself cut to tf32 by the tensor core (truncation is the worst case).
"""
import numpy as np
import pytest

RNG = np.random.default_rng(20240531)


def tf32_trunc(x):
    x = np.asarray(x, dtype=np.float32)
    return (x.view(np.uint32) & np.uint32(0xFFFFE000)).view(np.float32)


def split(x):
    x = np.asarray(x, dtype=np.float32)
    hi = tf32_trunc(x)
    return hi, (x - hi).astype(np.float32)


def dot_three_products(q, c):
    """Each tf32 product is exact in fp32 (11 x 11 significant bits); the
    terms are accumulated one by one in fp32, the order least kind to
    rounding among those a tensor core might use."""
    qh, ql = split(q)
    ch, cl = split(c)
    ql, cl = tf32_trunc(ql), tf32_trunc(cl)
    acc = np.float32(0.0)
    for d in range(len(q)):
        for term in (ql[d] * ch[d], qh[d] * cl[d], qh[d] * ch[d]):
            acc = np.float32(acc + np.float32(term))
    return acc


def dot_one_product(q, c):
    acc = np.float32(0.0)
    for a, b in zip(tf32_trunc(q), tf32_trunc(c)):
        acc = np.float32(acc + np.float32(a * b))
    return acc


def tolerance(q, c, exact, scale):
    """The GPU test's bound: 2^-16 sum|q_d c_d| scale + 2^-23 |s|."""
    mag = float(np.abs(q.astype(np.float64)) @ np.abs(c.astype(np.float64))) * scale
    return 2.0 ** -16 * mag + 2.0 ** -23 * abs(exact)


def test_split_is_exact_and_the_remainder_is_small():
    x = (RNG.standard_normal(4096) * np.exp(RNG.uniform(-20, 20, 4096))).astype(np.float32)
    hi, lo = split(x)
    np.testing.assert_array_equal(hi.astype(np.float64) + lo.astype(np.float64),
                                  x.astype(np.float64))
    assert np.all(np.abs(lo) < 2.0 ** -10 * np.abs(x))
    # hi is a tf32 value: its 13 low mantissa bits are clear
    assert np.all((hi.view(np.uint32) & np.uint32(0x1FFF)) == 0)


@pytest.mark.parametrize("ds", [64, 128])
def test_three_products_stay_within_the_gpu_tolerance(ds):
    scale = float(np.float32(1.0) / np.sqrt(np.float32(ds)))
    worst = 0.0
    for trial in range(200):
        q = RNG.standard_normal(ds).astype(np.float32)
        c = RNG.standard_normal(ds).astype(np.float32)
        if trial % 4 == 0:
            # heavy cancellation: c nearly orthogonal to q
            c = (c - (c @ q) / (q @ q) * q).astype(np.float32)
        exact = float(q.astype(np.float64) @ c.astype(np.float64)) * scale
        got = float(np.float32(dot_three_products(q, c) * np.float32(scale)))
        tol = tolerance(q, c, exact, scale)
        assert abs(got - exact) <= tol, (trial, got, exact, tol)
        worst = max(worst, abs(got - exact) / tol)
    assert worst < 0.5  # the bound holds with room to spare


def test_plain_tf32_would_break_the_tolerance():
    """The check is sharp enough to catch a kernel that dropped the hi*lo
    products: plain tf32 errors exceed the bound on typical rows."""
    ds, scale = 128, float(np.float32(1.0) / np.sqrt(np.float32(128)))
    broken = 0
    for _ in range(50):
        q = RNG.standard_normal(ds).astype(np.float32)
        c = RNG.standard_normal(ds).astype(np.float32)
        exact = float(q.astype(np.float64) @ c.astype(np.float64)) * scale
        got = float(np.float32(dot_one_product(q, c) * np.float32(scale)))
        broken += abs(got - exact) > tolerance(q, c, exact, scale)
    assert broken >= 40
