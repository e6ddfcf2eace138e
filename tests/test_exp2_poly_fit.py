"""The cubic of exp2_poly_x2 (csrc/frt_device.cuh) is the one the committed
Remez fit produces (CPU only): its fp32 literals equal the fit's coefficients
to fp32 precision, and the fit's relative error is the bound the comment
states."""
import os
import re

import numpy as np
import pytest

from flash_attention_tiled_b200 import fit_exp2_poly

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "flash_attention_tiled_b200", "csrc", "frt_device.cuh")


def _literals():
    text = open(SRC).read()
    body = text[text.index("uint64_t exp2_poly_x2("):]
    body = body[:body.index("\n}\n")]
    # the four coefficients, highest degree first, in the Horner steps
    vals = [float(v) for v in re.findall(r"f2_pack\(([0-9.]+)f, \1f\)", body)]
    vals = [v for v in vals if v < 2.0]          # drop the rounding constant 1.5 * 2^23
    assert len(vals) == 4, vals
    return np.array(vals[::-1])                   # c0..c3


@pytest.fixture(scope="module")
def remez():
    return fit_exp2_poly.fit()


def test_literals_are_the_remez_fit(remez):
    c, err = remez
    lit = _literals()
    np.testing.assert_allclose(lit, c, rtol=2.0 ** -23, atol=0)
    assert err < 7.5e-5


def test_fit_error_equioscillates(remez):
    # a minimax cubic's error reaches its largest magnitude at deg + 2 = 5
    # points, with alternating signs (the two ends among them)
    c, err = remez
    x = np.linspace(-0.5, 0.5, 20001)
    r = np.polyval(c[::-1], x) / 2.0 ** x - 1.0
    ext = [0] + [k for k in range(1, len(x) - 1)
                 if (r[k] - r[k - 1]) * (r[k + 1] - r[k]) < 0] + [len(x) - 1]
    peaks = [k for k in ext if abs(r[k]) > 0.99 * err]
    assert len(peaks) == 5, [(x[k], r[k]) for k in ext]
    assert all(np.sign(r[a]) != np.sign(r[b]) for a, b in zip(peaks, peaks[1:]))
