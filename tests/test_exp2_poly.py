"""The FMA-pipe exponential the attention kernel uses for a share of the
softmax weights: its coefficients are the documented Remez fit, and the
evaluation scheme (floor split, degree-3 polynomial, exponent add) stays
within the stated relative error over the whole input range the kernel feeds
it (x in [-126, 8]; smaller x is clamped)."""
import os
import re
import subprocess
import sys

import numpy as np

CSRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                    "attention_forward_17_b200", "csrc")


def kernel_coeffs():
    text = open(os.path.join(CSRC, "fa_fwd_kernel.cuh")).read()
    return [float(re.search(rf"kExp2A{i} = ([0-9.e+-]+)f;", text).group(1)) for i in (1, 2, 3)]


def emulate(x, a):
    """fp32 re-statement of the kernel's scheme (the kernel fuses the FMAs,
    numpy rounds twice; both stay inside the bound)."""
    x = np.maximum(x.astype(np.float32), np.float32(-126.0))
    j = np.floor(x)                       # the magic-constant add rounded toward -inf
    f = (x - j).astype(np.float32)        # exact
    a1, a2, a3 = (np.float32(c) for c in a)
    q = (a3 * f + a2).astype(np.float32)
    q = (q * f + a1).astype(np.float32)
    p = (q * f + np.float32(1.0)).astype(np.float32)
    bits = p.view(np.uint32).astype(np.int64) + (j.astype(np.int64) << 23)
    return (bits & 0xFFFFFFFF).astype(np.uint32).view(np.float32)


def test_relative_error_bound():
    a = kernel_coeffs()
    x = np.linspace(-126.0, 8.0, 4_000_001, dtype=np.float64).astype(np.float32)
    y = emulate(x, a).astype(np.float64)
    rel = np.abs(y / np.exp2(x.astype(np.float64)) - 1)
    assert rel.max() < 1.0e-4, rel.max()


def test_integers_exact_and_clamp():
    a = kernel_coeffs()
    x = np.arange(-126, 9, dtype=np.float32)
    np.testing.assert_array_equal(emulate(x, a), np.exp2(x.astype(np.float64)).astype(np.float32))
    # -inf and very negative inputs clamp to 2^-126 (a normal number, no NaN)
    y = emulate(np.array([-np.inf, -1000.0, -127.5], dtype=np.float32), a)
    assert np.all(y == np.float32(2.0 ** -126))


def test_fit_reproduces_kernel_constants():
    out = subprocess.run([sys.executable, os.path.join(CSRC, "fit_exp2_poly.py")],
                         capture_output=True, text=True, check=True).stdout
    fitted = [float(m) for m in re.findall(r"a\d = +([0-9.e+-]+)f", out)]
    np.testing.assert_allclose(fitted, kernel_coeffs(), rtol=1e-6)
