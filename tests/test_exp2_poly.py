"""CPU pin of the forward kernel's exp2 polynomial: the constants compiled into
the CUDA source reproduce the derivation's relative error bound, and the
derivation itself (Remez, relative error) equioscillates as it should."""
import os
import re

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "sparse_attention_attn_b200", "csrc", "s2_fwd.cu")


def _kernel_coeffs():
    text = open(SRC).read()
    return np.array([float(re.search(rf"kExp2C{i} = ([0-9.e+-]+)f", text).group(1)) for i in range(4)],
                    dtype=np.float32)


def _eval32(c, f):
    p = np.zeros_like(f)
    for ci in c[::-1]:
        p = (p * f + ci).astype(np.float32)
    return p


def test_kernel_polynomial_error_bound():
    c = _kernel_coeffs()
    f = np.linspace(-0.5, 0.5, 200001).astype(np.float32)
    rel = np.abs(_eval32(c, f).astype(np.float64) - 2.0 ** f.astype(np.float64)) / 2.0 ** f
    assert rel.max() < 7.6e-5
    # minimax: the error reaches its bound with alternating sign at deg+2 = 5 points
    err = (_eval32(c, f).astype(np.float64) - 2.0 ** f) / 2.0 ** f
    peaks = np.sum(np.abs(err) > 0.95 * np.abs(err).max())
    assert peaks >= 5


def test_cody_waite_reconstruction_in_numpy():
    """Same split as the kernel, evaluated bit for bit in numpy float32."""
    c = _kernel_coeffs()
    x = np.linspace(-125.0, 8.0, 500001).astype(np.float32)
    t = (x + np.float32(12582912.0)).astype(np.float32)
    f = (x - (t - np.float32(12582912.0))).astype(np.float32)
    p = _eval32(c, f)
    bits = (p.view(np.int32) + (t.view(np.int32) << 23)).astype(np.int32)
    y = bits.view(np.float32).astype(np.float64)
    rel = np.abs(y - 2.0 ** x.astype(np.float64)) / 2.0 ** x.astype(np.float64)
    assert rel.max() < 8e-5
