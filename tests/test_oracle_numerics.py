"""Pins of the oracle's numeric helpers against library routines and closed forms."""
import math

import numpy as np
import torch

import oracle


def test_decode_bf16_known_patterns():
    # sign | 8-bit exponent | 7-bit fraction: values fixed by the IEEE layout
    cases = {0x3F80: 1.0, 0xC000: -2.0, 0x4049: 3.140625, 0x0000: 0.0, 0x8000: -0.0,
             0x7F80: math.inf, 0xFF80: -math.inf, 0x0001: 2.0 ** -133, 0x7F7F: 3.3895313892515355e38}
    bits = np.array(list(cases), dtype=np.uint16)
    got = oracle.decode_bf16(bits)
    for g, want in zip(got, cases.values()):
        assert g == want and math.copysign(1, g) == math.copysign(1, want)


def test_decode_bf16_matches_torch_widening():
    g = torch.Generator().manual_seed(5)
    x = (torch.randn(4096, generator=g) * 50).to(torch.bfloat16)
    ref = x.to(torch.float64).numpy()
    got = oracle.decode_bf16(x.view(torch.int16).numpy())
    np.testing.assert_array_equal(got, ref)


def test_row_log_softmax_matches_library():
    rng = np.random.default_rng(1)
    Z = rng.normal(0, 3, size=(7, 513))
    Z[3, 5] = -np.inf
    got, lse = oracle.row_log_softmax(Z)
    ref = torch.log_softmax(torch.from_numpy(Z), dim=-1).numpy()
    np.testing.assert_allclose(got, ref, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, torch.logsumexp(torch.from_numpy(Z), -1).numpy(), atol=1e-12)


def test_row_log_softmax_closed_forms():
    V = 1000
    got, lse = oracle.row_log_softmax(np.full((1, V), 7.25))
    np.testing.assert_allclose(got, -math.log(V), atol=1e-12)
    assert abs(lse[0] - (7.25 + math.log(V))) < 1e-12
    # two-point row: softmax of (x, 0) is the logistic function
    x = 1.7
    got, _ = oracle.row_log_softmax(np.array([[x, 0.0]]))
    assert abs(got[0, 0] - math.log(1 / (1 + math.exp(-x)))) < 1e-12
    # large offsets do not overflow
    got, lse = oracle.row_log_softmax(np.array([[1000.0, 1000.0]]))
    np.testing.assert_allclose(got, -math.log(2), atol=1e-12)
