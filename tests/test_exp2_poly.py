"""The FMA-pipe exponential of the tensor-core kernels, checked on the CPU.

The forward and backward kernels compute one pair of exponentials in four as
2^x = 2^n * p(f), x = n + f, n = round(x), with a fitted cubic p and n added
to the exponent field of p(f) (csrc/lvx_ptx.cuh).  These tests read the cubic's
coefficients and the argument clamp out of that header and emulate the whole
evaluation in fp32, bit for bit (the magic-number rounding, the Horner steps,
the integer add into the exponent field).  They check it against 2^x over
the full range the kernels can pass: no NaN or negative value anywhere, the
fitted accuracy where 2^x is a normal number, and a negligible value below.
"""

import os
import re

import numpy as np

from blockwise_long_context_b200 import fit_exp2

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                      "blockwise_long_context_b200", "csrc", "lvx_ptx.cuh")


def _header():
    with open(HEADER) as f:
        return f.read()


def _scalar_body():
    src = _header()
    start = src.index("float exp2_poly(float x)")
    return src[start:src.index("}", start)]


def _coefficients():
    """(c0, c1, c2, c3) of the scalar version, from its nested fmaf calls."""
    nums = [float(v.rstrip("f")) for v in re.findall(r"-?\d\.\d+e[-+]\d+f", _scalar_body())]
    assert len(nums) == 4, nums
    c3, c2, c1, c0 = nums
    return np.array([c0, c1, c2, c3], dtype=np.float32)


def _clamp():
    m = re.search(r"fmaxf\(x, (-\d+)\.f\)", _scalar_body())
    assert m, "clamp not found"
    return float(m.group(1))


def _emulate(x, c, lo):
    """The kernel's evaluation in fp32, as integer and float operations."""
    f32 = np.float32
    x = np.maximum(np.asarray(x, dtype=f32), f32(lo))
    magic = f32(12582912.0)                   # 1.5 * 2^23
    t = (x + magic).astype(f32)
    f = (x - (t - magic).astype(f32)).astype(f32)
    p = ((c[3] * f + c[2]).astype(f32) * f + c[1]).astype(f32)
    p = (p * f + c[0]).astype(f32)
    bits = (p.view(np.int32).astype(np.int64) + (t.view(np.int32).astype(np.int64) << 23)) & 0xFFFFFFFF
    return bits.astype(np.uint32).view(np.float32)


def test_header_coefficients_are_the_fit():
    c = _coefficients()
    ref = fit_exp2.fit()
    assert np.allclose(c, ref, rtol=1e-6, atol=0), (c, ref)
    # the documented accuracy of the fp32 Horner evaluation on [-1/2, 1/2]
    assert fit_exp2.max_rel_error(c) < 8e-5


def test_every_argument_gives_a_finite_nonnegative_value():
    c, lo = _coefficients(), _clamp()
    x = np.concatenate([np.linspace(-1e4, 127.0, 400001, dtype=np.float32),
                        np.float32([-np.inf, -3e38, -127.0, -126.5, -126.0, -125.5]),
                        # every fp32 value around the clamp, where the exponent add is tightest
                        np.arange(-130.0, -122.0, 2.0 ** -16, dtype=np.float32)])
    y = _emulate(x, c, lo)
    assert np.all(np.isfinite(y)), x[~np.isfinite(y)][:8]
    assert np.all(y >= 0), x[y < 0][:8]


def test_accuracy_where_the_result_is_normal():
    c, lo = _coefficients(), _clamp()
    x = np.linspace(-125.0, 127.0, 1000001, dtype=np.float32)
    y = _emulate(x, c, lo).astype(np.float64)
    rel = np.abs(y / np.exp2(x.astype(np.float64)) - 1)
    assert rel.max() < 1e-4, (rel.max(), x[rel.argmax()])


def test_below_the_normal_range_the_value_is_negligible():
    # at most about 2^-125: relative to the row's largest term (2^0 in the
    # kernels' arguments) it vanishes in the fp32 row sum and in bf16 P
    c, lo = _coefficients(), _clamp()
    x = np.linspace(-1e4, -125.0, 100001, dtype=np.float32)
    assert float(_emulate(x, c, lo).max()) <= 2.0 ** -125


def test_packed_version_uses_the_same_clamp_and_coefficients():
    src = _header()
    start = src.index("uint64_t exp2_poly2(uint64_t x2)")
    body = src[start:src.index("\n}\n", start)]
    lo = _clamp()
    assert f"fmaxf(x0, {lo:.0f}.f)" in body and f"fmaxf(x1, {lo:.0f}.f)" in body
    nums = sorted({np.float32(v.rstrip("f")) for v in re.findall(r"-?\d\.\d+e[-+]\d+f", body)})
    assert np.array_equal(np.sort(_coefficients()), np.array(nums, dtype=np.float32))
