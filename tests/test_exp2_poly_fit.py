"""The FMA-pipe exp2 of the softmax kernels (exp2_fma2 in csrc/sm100.cuh) uses the float32
coefficients printed by exact_tiled_attention_41_b200/fit_exp2_poly.py: re-run the Remez fit
here and compare with the constants written in the header, and check the fitted polynomial's
accuracy in a float32 model of the kernel's evaluation (rint by the 1.5 * 2^23 trick, Horner,
exponent add)."""

import os
import re

import numpy as np

from exact_tiled_attention_41_b200 import fit_exp2_poly as F
from tests.conftest import ROOT


def _header_coefficients():
    src = open(os.path.join(ROOT, "exact_tiled_attention_41_b200", "csrc", "sm100.cuh")).read()
    body = src[src.index("float2 exp2_fma2(float2 x)"):]
    body = body[: body.index("\n}\n")]
    # every float literal after the rounding constant and the clamp, in Horner order
    lits = re.findall(r"make_float2\(([-0-9.e]+)f, \1f\)", body)
    return [np.float32(float(x)) for x in lits if float(x) not in (12582912.0,)]


def test_header_constants_are_the_fit():
    fit = F.coefficients_f32()
    hdr = _header_coefficients()
    assert len(hdr) == F.DEG + 1 == len(fit)
    for a, b in zip(hdr, fit):
        assert a == b, (a, b)


def test_fitted_polynomial_error_in_float32():
    err = F.fp32_horner_error(F.remez())
    assert err <= 2.5e-7          # about 2 ulp, the bound the GPU self-test also applies


def _model(x, c):
    """float32 model of exp2_fma2: clamp, rint via 1.5 * 2^23, Horner with one rounding per step,
    exponent add on the bit patterns."""
    x = np.maximum(x.astype(np.float32), np.float32(-126.0))
    t = (x + np.float32(12582912.0)).astype(np.float32)
    f = (x - (t - np.float32(12582912.0))).astype(np.float32)
    p = np.full_like(f, c[0])
    for a in c[1:]:
        p = (p * f + a).astype(np.float32)
    bits = (p.view(np.uint32).astype(np.uint64) + (t.view(np.uint32).astype(np.uint64) << 23)) & 0xFFFFFFFF
    return bits.astype(np.uint32).view(np.float32)


def test_kernel_model_is_accurate_and_never_negative():
    c = F.coefficients_f32()
    x = np.linspace(-125.0, 8.0, 2_000_001).astype(np.float32)
    y = _model(x, c).astype(np.float64)
    rel = np.abs(y / np.exp2(x.astype(np.float64)) - 1.0)
    assert rel.max() <= 2.5e-7
    # below the accurate range the value stays a tiny non-negative number
    z = _model(np.array([-125.5, -126.0, -200.0, -1e30, -np.inf], dtype=np.float32), c)
    assert np.all(z >= 0) and np.all(z <= 2.0 ** -125)
