"""The exp2 the attention kernels evaluate on the FMA pipe (Cody-Waite
reduction + the fitted degree-3 or degree-2 polynomial of
csrc/fp2_exp2_poly.h), replayed step by step in float32 and checked against
2^x in float64: relative error within the fit's bound (plus float32 rounding
of the few operations) over the whole range the softmax feeds it, and the
clamp that turns -inf / NaN / very negative inputs into a zero weight.  The
degree-2 form feeds probabilities that are rounded to e4m3 (3 mantissa bits),
so its bound must stay far below half of e4m3's relative step, 2^-4."""
import os
import re
import subprocess
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "block_sparse_long_blockmean_b200", "csrc")


def coeffs(deg: int = 3):
    txt = open(os.path.join(CSRC, "fp2_exp2_poly.h")).read()
    name, err = ("C", "REL_ERR") if deg == 3 else ("Q", "Q_REL_ERR")
    c = [float(re.search(rf"FP2_EXP2_{name}{i} ([-0-9.e]+)f", txt).group(1))
         for i in range(deg + 1)]
    rel = float(re.search(rf"FP2_EXP2_{err} ([-0-9.e]+)", txt).group(1))
    return [np.float32(v) for v in c], rel


def exp2_poly_f32(x, deg: int = 3):
    c, _ = coeffs(deg)
    f32 = np.float32
    magic = f32(12582912.0)
    x = np.fmax(x.astype(np.float32), f32(-126.0))  # fmaxf: a NaN operand loses
    t = (x + magic).astype(np.float32)
    j = (t - magic).astype(np.float32)
    f = (x - j).astype(np.float32)
    p = (f * c[deg] + c[deg - 1]).astype(np.float32)
    for k in range(deg - 2, -1, -1):
        p = (p * f + c[k]).astype(np.float32)
    bits = p.view(np.uint32) + (t.view(np.uint32) << np.uint32(23))
    return bits.astype(np.uint32).view(np.float32)


@pytest.mark.parametrize("deg", [3, 2])
def test_relative_error_within_bound(deg):
    _, rel = coeffs(deg)
    x = np.linspace(-120.0, 8.0, 2_000_003).astype(np.float32)
    got = exp2_poly_f32(x, deg).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    err = np.abs(got / ref - 1.0).max()
    assert err <= rel + 8 * 2.0 ** -24, err


def test_degree2_is_far_inside_e4m3_rounding():
    """e4m3 rounds to nearest with a relative step between 2^-4 and 2^-3, so
    half a step is at least 2^-5; the degree-2 bound is under a tenth of it."""
    _, rel = coeffs(2)
    assert rel < 0.1 * 2.0 ** -5


@pytest.mark.parametrize("deg", [3, 2])
def test_integers_and_halves(deg):
    x = np.array([-3, -2, -1, 0, 1, 2, 5, -0.5, 0.5, 7.5], dtype=np.float32)
    got = exp2_poly_f32(x, deg)
    np.testing.assert_allclose(got, np.exp2(x.astype(np.float64)), rtol=2e-3 if deg == 2 else 1e-4)


@pytest.mark.parametrize("deg", [3, 2])
def test_clamp_gives_zero_weight(deg):
    x = np.array([-np.inf, np.nan, -1e30, -200.0, -126.5], dtype=np.float32)
    with np.errstate(invalid="ignore"):
        got = exp2_poly_f32(x, deg)
    assert np.isfinite(got).all() and (got >= 0).all() and (got <= 2.0 ** -125).all()


def test_header_is_what_the_fit_script_writes(tmp_path):
    """The committed header is reproducible from fit_exp2_poly.py."""
    import importlib.util
    spec = importlib.util.spec_from_file_location("fitexp2", os.path.join(CSRC, "fit_exp2_poly.py"))
    m = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(m)
    for deg in (3, 2):
        c, rel = m.fit(deg)
        cc, hrel = coeffs(deg)
        np.testing.assert_allclose([float(v) for v in cc], c.astype(np.float32), rtol=0, atol=0)
        assert abs(rel - hrel) / rel < 1e-3


def exp2_sat_poly_f32(x, k, c, deg: int = 3):
    """exp2_sat_poly2 replayed in float32: e = x*k + c, clamp folded into a
    saturating FMA y = sat(x*(k/128) + (c+120)/128)."""
    cc, _ = coeffs(deg)
    f32 = np.float32
    K = f32(12582792.0)
    k128, c128 = f32(k) * f32(1 / 128), (f32(c) + f32(120.0)) * f32(1 / 128)
    # one rounding of the exact x*k128 + c128 (an FMA), then saturation to [0, 1]
    y = (x.astype(np.float64) * np.float64(k128) + np.float64(c128)).astype(np.float32)
    y = np.where(np.isnan(y), f32(0), np.clip(y, f32(0), f32(1))).astype(np.float32)
    t = (y.astype(np.float64) * 128 + np.float64(K)).astype(np.float32)
    nu = (K - t).astype(np.float32)
    f = (y.astype(np.float64) * 128 + nu.astype(np.float64)).astype(np.float32)
    p = (f.astype(np.float64) * cc[deg] + cc[deg - 1]).astype(np.float32)
    for j in range(deg - 2, -1, -1):
        p = (p.astype(np.float64) * f + cc[j]).astype(np.float32)
    bits = p.view(np.uint32) + (t.view(np.uint32) << np.uint32(23))
    return bits.astype(np.uint32).view(np.float32)


@pytest.mark.parametrize("deg", [3, 2])
@pytest.mark.parametrize("k,c", [(1.0, 0.0), (0.127, -37.5), (0.0884, 3.25)])
def test_saturating_form_within_bound(deg, k, c):
    """Over the range the lazy rescale allows (e = x*k + c in [-120, 8]) the
    saturating form is as accurate as the plain one; below -120 it returns
    2^-120, a weight that vanishes next to the row maximum (>= 1)."""
    _, rel = coeffs(deg)
    e = np.linspace(-119.5, 8.0, 1_000_003)
    x = ((e - c) / k).astype(np.float32)
    got = exp2_sat_poly_f32(x, k, c, deg).astype(np.float64)
    ref = np.exp2(x.astype(np.float64) * np.float32(k) + np.float32(c))
    err = np.abs(got / ref - 1.0).max()
    # e is rebuilt from y with |e| <= 128 at 2^-24 relative: 2^-17 absolute
    assert err <= rel + 2.0 ** -17 * np.log(2) + 8 * 2.0 ** -24, err
    low = exp2_sat_poly_f32(np.array([-1e30, -np.inf, np.nan], dtype=np.float32), k, c, deg)
    assert np.isfinite(low).all() and (low >= 0).all() and (low <= 2.0 ** -119).all()
