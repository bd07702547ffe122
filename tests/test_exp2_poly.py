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


def _accept(x, c, lo, poly_every=4, factor=256.0, threshold=8.0):
    """The forward kernel's steady-state acceptance of one row's 128 arguments
    x (log2 units, relative to the running maximum): pair i of each 32-key chunk
    goes through the FMA-pipe exponential when i % poly_every == poly_every - 1,
    the others through the SFU (exact 2^x here; ex2.approx is within 2 ulp).
    Accepted iff the sum of the exponentials is <= 2^threshold and every
    FMA-pipe argument is <= threshold."""
    x = np.asarray(x, dtype=np.float32)
    pair = (np.arange(128) % 32) // 2
    on_poly = pair % poly_every == poly_every - 1
    with np.errstate(invalid="ignore", over="ignore"):     # 2^x overflows to inf, as on the SFU
        e = np.where(on_poly, _emulate(x, c, lo), np.exp2(x.astype(np.float64)).astype(np.float32))
        total = np.float32(e.astype(np.float32).sum(dtype=np.float32))
        xp = np.max(np.where(on_poly, x, -np.inf))
        return bool(total <= factor and xp <= threshold)


def test_steady_state_acceptance_never_admits_an_exponential_above_the_threshold():
    c, lo = _coefficients(), _clamp()
    rng = np.random.default_rng(5)
    pair = (np.arange(128) % 32) // 2
    poly_keys = np.nonzero(pair % 4 == 3)[0]
    sfu_keys = np.nonzero(pair % 4 != 3)[0]
    rows = []
    for _ in range(3000):                                   # ordinary rows around the maximum
        rows.append(rng.normal(-3.0, 2.0, 128))
    for big in (8.5, 20.0, 127.0, 128.7, 150.0, 1e4):       # one large argument on each pipe
        for keys in (poly_keys, sfu_keys):
            r = rng.normal(-5.0, 1.0, 128)
            r[rng.choice(keys)] = big
            rows.append(r)
    rows.append(np.full(128, 7.9))                           # all just under the threshold
    r = rng.normal(-5.0, 1.0, 128); r[3] = np.nan; rows.append(r)
    accepted = 0
    for r in rows:
        if _accept(r, c, lo):
            accepted += 1
            assert np.nanmax(r) <= 8.0, r[np.argmax(r)]     # no exponential above 2^8
    assert accepted >= 2900                                  # the ordinary rows pass
    # a row the sum rejects although every argument is below the threshold falls
    # back to the exact path (never a wrong accept, only a slower tile)
    assert not _accept(np.full(128, 7.9), c, lo)
