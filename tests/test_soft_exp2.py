"""The scoring kernels' software 2^t (FMA pipe instead of the SFU).

The kernel header states its construction: t = n + f with n = round(t) and
f in [-1/2, 1/2], and 2^f by the degree-5 polynomial interpolating 2^f at the
six Chebyshev nodes of [-1/2, 1/2], coefficients rounded to fp32. This test
derives that interpolant independently (numpy, float64), checks that the fp32
constants in the header are its coefficients, and bounds the error of the whole
construction as the kernel evaluates it (fp32 Horner with fused multiply-adds,
round-to-nearest split, exponent-field insert), emulated here in numpy.
"""
import os
import re

import numpy as np

HEADER = os.path.join(os.path.dirname(__file__), "..", "speculative_decoding_draft_07_b200",
                      "csrc", "umma.cuh")


def _header_coefficients():
    src = open(HEADER).read()
    vals = {}
    for name, v in re.findall(r"kExp2C(\d)\s*=\s*([0-9.eE+-]+)f", src):
        vals[int(name)] = np.float32(float(v))
    assert sorted(vals) == list(range(6)), vals
    return np.array([vals[i] for i in range(6)], dtype=np.float32)


def _chebyshev_interpolant(deg=5):
    k = np.arange(deg + 1)
    nodes = 0.5 * np.cos((2 * k + 1) * np.pi / (2 * (deg + 1)))
    V = np.vander(nodes, deg + 1, increasing=True)
    return np.linalg.solve(V, 2.0 ** nodes)


def _fma32(a, b, c):
    return (a.astype(np.float64) * b.astype(np.float64) + c.astype(np.float64)).astype(np.float32)


def _soft_exp2(t, c):
    """numpy emulation of the kernel's soft_exp2x2 on one lane."""
    t = np.maximum(t.astype(np.float32), np.float32(-125.0))
    R = np.float32(12582912.0)
    r = (t + R).astype(np.float32)
    n = (r - R).astype(np.float32)
    f = _fma32(n, np.float32(-1.0) * np.ones_like(n), t)
    q = np.full_like(f, c[5])
    for j in range(4, -1, -1):
        q = _fma32(q, f, np.full_like(f, c[j]))
    bits = q.view(np.uint32).astype(np.uint64) + (r.view(np.uint32).astype(np.uint64) << np.uint64(23))
    return (bits & np.uint64(0xFFFFFFFF)).astype(np.uint32).view(np.float32)


def test_constants_are_the_chebyshev_interpolant():
    c64 = _chebyshev_interpolant()
    np.testing.assert_array_equal(_header_coefficients(), c64.astype(np.float32))


def test_interpolant_error_bound():
    c64 = _chebyshev_interpolant()
    f = np.linspace(-0.5, 0.5, 200001)
    rel = np.abs(np.polyval(c64[::-1], f) / 2.0 ** f - 1.0)
    # interpolation error of degree 5 at Chebyshev nodes: (ln 2)^6 2^(1/2) / (2^5 6!) (1/2)^6 / 2^(-1/2)
    bound = np.log(2.0) ** 6 * 2 ** 0.5 / (2 ** 5 * 720) / 2 ** 6 / 2 ** -0.5
    assert rel.max() <= bound
    assert rel.max() < 1.1e-7


def test_full_construction_in_fp32():
    c = _header_coefficients()
    rng = np.random.default_rng(5)
    t = np.concatenate([rng.uniform(-125.0, 92.0, 400000), np.arange(-125, 93, 0.25),
                        np.array([0.0, -0.5, 0.5, 1e-7, -1e-7, 91.999])]).astype(np.float32)
    got = _soft_exp2(t, c).astype(np.float64)
    want = 2.0 ** t.astype(np.float64)
    rel = np.abs(got / want - 1.0)
    assert rel.max() < 3e-7, rel.max()
    # below the clamp the result is 2^-125 (negligible next to a softmax sum >= 1)
    low = _soft_exp2(np.array([-130.0, -1e30, -np.inf], dtype=np.float32), c)
    np.testing.assert_allclose(low.astype(np.float64), 2.0 ** -125, rtol=3e-7)
