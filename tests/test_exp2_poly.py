"""The FMA-pipe 2^x of the tensor-core kernel (ptx.cuh, exp2_poly_x2), on the
CPU: its coefficients are the ones the committed Remez fit produces, and the
whole function (round-to-nearest range reduction, Horner polynomial, exponent
add), emulated in fp32 with fused multiply-adds, stays within the stated
relative-error bound of 2^x over the range the kernel feeds it."""

import os
import re
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "tiled_attention_13_b200", "csrc")
sys.path.insert(0, CSRC)

import gen_exp2_poly  # noqa: E402

BOUND = 7.5e-5  # the bound ptx.cuh states for exp2_poly_x2


def _kernel_coefficients():
    src = open(os.path.join(CSRC, "ptx.cuh")).read()
    m = re.search(r"constexpr float C0 = ([-+0-9.e]+)f, C1 = ([-+0-9.e]+)f, C2 = ([-+0-9.e]+)f, "
                  r"C3 = ([-+0-9.e]+)f;", src)
    assert m, "exp2_poly_x2's coefficient line not found"
    return np.array([float(x) for x in m.groups()], dtype=np.float32)


def test_coefficients_are_the_fit():
    fitted = gen_exp2_poly.fit(3).astype(np.float32)
    got = _kernel_coefficients()
    # the committed constants print 10 significant digits: the same fp32 values
    assert np.array_equal(got, fitted), (got, fitted)
    assert gen_exp2_poly.fp32_error(fitted.astype(np.float64)) <= BOUND


def _fma32(a, b, c):
    # fp32 fused multiply-add: the product of two fp32 values is exact in fp64
    return (a.astype(np.float64) * b.astype(np.float64) + c.astype(np.float64)).astype(np.float32)


def _exp2_poly(x):
    c0, c1, c2, c3 = _kernel_coefficients()
    magic = np.float32(12582912.0)  # 1.5 * 2^23
    xx = np.maximum(x.astype(np.float32), np.float32(-125.0))
    t = (xx + magic).astype(np.float32)
    r = (t - magic).astype(np.float32)
    f = _fma32(r, np.full_like(r, -1.0), xx)
    q = _fma32(np.full_like(f, c3), f, np.full_like(f, c2))
    q = _fma32(q, f, np.full_like(f, c1))
    q = _fma32(q, f, np.full_like(f, c0))
    # n = round(x) sits in the low mantissa bits of t; add it to q's exponent
    n = t.view(np.int32) - magic.view(np.int32)
    return (q.view(np.int32) + (n << 23)).view(np.float32), n


def test_whole_function_error_bound():
    rng = np.random.default_rng(7)
    x = np.concatenate([np.linspace(-124.0, 127.0, 400001), rng.uniform(-30.0, 0.0, 200000),
                        np.arange(-124, 128, dtype=np.float64) + 0.5, np.arange(-124, 128, dtype=np.float64)])
    x = x.astype(np.float32)
    y, n = _exp2_poly(x)
    assert np.array_equal(n, np.rint(x).astype(np.int32))  # the magic-number rounding is round-to-nearest
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(y.astype(np.float64) - ref) / ref
    assert rel.max() <= BOUND * 1.01, rel.max()
    # exact powers of two come out within the polynomial's error at f = 0
    assert np.all(np.abs(y[-252:].astype(np.float64) / ref[-252:] - 1.0) <= BOUND)
