"""The FMA-pipe exponential of the forward kernel, checked on the CPU.

The kernel computes part of its 2^x as 2^round(x) * p(x - round(x)) with a cubic p
fitted by fit_exp2_poly.py.  These tests pin (1) the constants in fwd_kernel.cuh to
the fit and to its error bound, and (2) the kernel's sequence of fp32 steps, emulated
here with NumPy, to exp2 over the clamped range the kernel accepts."""
import os
import re

import numpy as np

from exact_attention_108_b200 import fit_exp2_poly

HERE = os.path.dirname(os.path.abspath(__file__))
KERNEL = os.path.join(HERE, "..", "exact_attention_108_b200", "csrc", "fwd_kernel.cuh")


def _kernel_constants():
    text = open(KERNEL).read()
    vals = [float(re.search(rf"kExpC{i} = ([0-9.e+-]+)f", text).group(1)) for i in (1, 2, 3)]
    return np.float32(vals)


def test_kernel_constants_are_the_minimax_fit():
    c, t = fit_exp2_poly.fit()
    k = _kernel_constants()
    assert np.allclose(k, np.float32(c), rtol=1e-6, atol=0)
    assert t < 1.02e-4
    assert fit_exp2_poly.max_rel_error(k) < 1.02e-4


def test_fitted_cubic_beats_taylor():
    # the fit must improve on the plain Taylor cubic (a dropped or wrong coefficient would not)
    ln2 = np.log(2.0)
    taylor = [ln2, ln2 ** 2 / 2, ln2 ** 3 / 6]
    assert fit_exp2_poly.max_rel_error(_kernel_constants()) < 0.2 * fit_exp2_poly.max_rel_error(taylor)


def _kernel_exp2(x, c):
    """The kernel's steps in fp32: saturated y, magic-number rounding, cubic, exponent add."""
    f32 = np.float32
    x = x.astype(np.float32)
    m_ref = f32(0.0)
    sl2 = f32(1.0)  # x = s * sl2 - m_ref with s = x
    pa, pb = f32(sl2 * f32(1.0 / 256.0)), f32((f32(124.0) - m_ref) * f32(1.0 / 256.0))
    y = np.clip(np.fma(x, pa, pb) if hasattr(np, "fma") else (x.astype(np.float64) * pa + pb).astype(f32), 0, 1).astype(f32)
    magic = f32(12582912.0 - 124.0)
    t = (y.astype(np.float64) * 256.0 + magic).astype(f32)
    w = (t.astype(np.float64) * -1.0 + magic).astype(f32)
    fr = (y.astype(np.float64) * 256.0 + w).astype(f32)
    q = (fr.astype(np.float64) * c[2] + c[1]).astype(f32)
    q = (q.astype(np.float64) * fr + c[0]).astype(f32)
    q = (q.astype(np.float64) * fr + 1.0).astype(f32)
    bits = (q.view(np.uint32).astype(np.uint64) + (t.view(np.uint32).astype(np.uint64) << np.uint64(23))) & 0xFFFFFFFF
    return bits.astype(np.uint32).view(np.float32)


def test_kernel_steps_match_exp2_over_the_clamped_range():
    c = _kernel_constants()
    x = np.concatenate([np.linspace(-124.0, 8.0, 200001), np.array([-0.5, 0.0, 0.5, 1.0, -1.0, 7.99])])
    got = _kernel_exp2(x.astype(np.float32), c).astype(np.float64)
    ref = np.exp2(x.astype(np.float32).astype(np.float64))
    rel = np.abs(got / ref - 1)
    # the cubic's 1.01e-4, plus the fp32 rounding of y (2^-16 in x at most: 1.1e-5 relative)
    assert rel.max() < 1.2e-4, rel.max()
    # below the clamp every weight becomes 2^-124, never garbage or zero
    low = _kernel_exp2(np.array([-124.4, -200.0, -1e4], dtype=np.float32), c).astype(np.float64)
    assert np.all(np.abs(low / 2.0 ** -124 - 1) < 1.2e-4)
