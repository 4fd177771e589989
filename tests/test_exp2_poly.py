"""The sparse kernel's FMA-pipe exponential (2^x by range reduction and a
cubic) against the definition 2^x.

The cubic's float32 coefficients come from the committed minimax fit
(block_sparse_attention_15_b200/exp2_fit.py); these CPU tests check that the
kernel header holds exactly the fit's coefficients and that the routine's
float32 steps (modelled in exp2_fit.exp2_model) stay within the stated
relative error bound against numpy's float64 2^x over the whole range the
softmax uses, including the points where the rounding of x to an integer
switches and the clamp at -120.
"""
import os
import re

import numpy as np

from block_sparse_attention_15_b200 import exp2_fit as E

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "block_sparse_attention_15_b200", "csrc", "vsa_device.cuh")
BOUND = 7.5e-5  # the routine's stated maximum relative error


def _header_coefficients():
    text = open(HEADER).read()
    body = text[text.index("exp2_fma2"):]
    body = body[:body.index("\n}\n")]
    lits = re.findall(r"pk2\((-?0x1\.[0-9a-f]+p-?\d+)f,", body)
    assert len(lits) == 4, lits
    # the header evaluates c3 first (Horner), then c2 (same line), c1, c0
    c3, c2, c1, c0 = (np.float32(float.fromhex(x)) for x in lits)
    return np.array([c0, c1, c2, c3], dtype=np.float32)


def test_header_holds_the_fitted_coefficients():
    assert np.array_equal(_header_coefficients(), E.coefficients_f32())


def test_fit_equioscillates():
    """A minimax fit of degree 3 touches its error bound at 5 alternating
    points (Chebyshev's theorem); a wrong fit does not."""
    c = E.remez()
    x = np.linspace(E.LO, E.HI, 200001)
    e = E.rel_error(c, x)
    m = np.abs(e).max()
    s = np.sign(e)
    runs = np.split(np.arange(x.size), np.flatnonzero(np.diff(s)) + 1)
    peaks = [np.abs(e[r]).max() for r in runs]
    assert len(runs) == 5
    assert min(peaks) > 0.999 * m


def test_relative_error_over_the_softmax_range():
    rng = np.random.default_rng(7)
    x = np.concatenate([
        np.linspace(-120.0, 32.0, 3_000_001),
        rng.uniform(-120.0, 32.0, 1_000_000),
        np.arange(-120, 33) + 0.5,                   # f = +-1/2: rounding to even switches
        np.nextafter(np.arange(-120, 33) + 0.5, -np.inf),
        np.nextafter(np.arange(-120, 33) + 0.5, np.inf),
        np.arange(-120, 33, dtype=np.float64),       # exact powers of two
        [0.0, -0.0, 1e-30, -1e-30],
    ]).astype(np.float32)
    y = E.exp2_model(x).astype(np.float64)
    rel = np.abs(y / np.exp2(x.astype(np.float64)) - 1.0)
    assert rel.max() <= BOUND, rel.max()
    # integers give 2^j times p(0) = c0
    ints = np.arange(-120, 33).astype(np.float32)
    assert np.allclose(E.exp2_model(ints) / np.exp2(ints.astype(np.float64)),
                       E.coefficients_f32()[0], rtol=0, atol=1e-7)


def test_clamp_below_minus_120():
    x = np.array([-120.0, -120.5, -150.0, -1e30, -np.inf], dtype=np.float32)
    y = E.exp2_model(x).astype(np.float64)
    assert np.all(y <= 2.0 ** -119) and np.all(y >= 2.0 ** -121)


def test_a_planted_coefficient_error_is_caught():
    """The bound test is sensitive: a one-percent change of c3 breaks it."""
    c = E.coefficients_f32().copy()
    c[3] *= np.float32(1.01)
    x = np.linspace(-3, 3, 100001).astype(np.float32)
    rel = np.abs(E.exp2_model(x, c) / np.exp2(x.astype(np.float64)) - 1.0)
    assert rel.max() > BOUND
