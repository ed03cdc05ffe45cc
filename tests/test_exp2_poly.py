"""The exp2 the attention kernels evaluate on the FMA pipe (Cody-Waite
reduction + the fitted degree-3 polynomial of csrc/fp2_exp2_poly.h), replayed
step by step in float32 and checked against 2^x in float64: relative error
within the fit's bound (plus float32 rounding of the few operations) over the
whole range the softmax feeds it, and the clamp that turns -inf / NaN / very
negative inputs into a zero weight."""
import os
import re
import subprocess
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "block_sparse_long_blockmean_b200", "csrc")


def coeffs():
    txt = open(os.path.join(CSRC, "fp2_exp2_poly.h")).read()
    c = [float(re.search(rf"FP2_EXP2_C{i} ([-0-9.e]+)f", txt).group(1)) for i in range(4)]
    rel = float(re.search(r"FP2_EXP2_REL_ERR ([-0-9.e]+)", txt).group(1))
    return [np.float32(v) for v in c], rel


def exp2_poly_f32(x):
    c, _ = coeffs()
    f32 = np.float32
    magic = f32(12582912.0)
    x = np.fmax(x.astype(np.float32), f32(-126.0))  # fmaxf: a NaN operand loses
    t = (x + magic).astype(np.float32)
    j = (t - magic).astype(np.float32)
    f = (x - j).astype(np.float32)
    p = (f * c[3] + c[2]).astype(np.float32)
    p = (p * f + c[1]).astype(np.float32)
    p = (p * f + c[0]).astype(np.float32)
    bits = p.view(np.uint32) + (t.view(np.uint32) << np.uint32(23))
    return bits.astype(np.uint32).view(np.float32)


def test_relative_error_within_bound():
    _, rel = coeffs()
    x = np.linspace(-120.0, 8.0, 2_000_003).astype(np.float32)
    got = exp2_poly_f32(x).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    err = np.abs(got / ref - 1.0).max()
    assert err <= rel + 8 * 2.0 ** -24, err


def test_integers_and_halves():
    x = np.array([-3, -2, -1, 0, 1, 2, 5, -0.5, 0.5, 7.5], dtype=np.float32)
    got = exp2_poly_f32(x)
    np.testing.assert_allclose(got, np.exp2(x.astype(np.float64)), rtol=1e-4)


def test_clamp_gives_zero_weight():
    x = np.array([-np.inf, np.nan, -1e30, -200.0, -126.5], dtype=np.float32)
    with np.errstate(invalid="ignore"):
        got = exp2_poly_f32(x)
    assert np.isfinite(got).all() and (got >= 0).all() and (got <= 2.0 ** -125).all()


def test_header_is_what_the_fit_script_writes(tmp_path):
    """The committed header is reproducible from fit_exp2_poly.py."""
    import importlib.util
    spec = importlib.util.spec_from_file_location("fitexp2", os.path.join(CSRC, "fit_exp2_poly.py"))
    m = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(m)
    c, rel = m.fit()
    cc, hrel = coeffs()
    np.testing.assert_allclose([float(v) for v in cc], c.astype(np.float32), rtol=0, atol=0)
    assert abs(rel - hrel) / rel < 1e-3
