"""The FMA-pipe exponential of the forward's softmax (ex2_poly2 in sm100_ptx.cuh).

The softmax of the FlashAttention wiki notes (section Tiling) needs 2^x for
every score; the kernel evaluates part of them with a degree-3 polynomial for
2^f on [-1/2, 1/2] and puts 2^round(x) into the exponent field.  These tests
pin it:

* CPU: the constants in the header are the ones fit_exp2_poly.fit() produces
  (minimax with constant term 1), and their max relative error on [-1/2, 1/2]
  is the stated 1.013e-4;
* CPU: the same steps in float32 arithmetic (NumPy) meet the bounds over
  x in [-140, 127] and give exactly +0 at -inf and at x <= -127;
* GPU: attn_selftest_ex2 runs the device function itself on such a sweep.
"""
import importlib.util
import os
import re

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "exact_io_aware_102_b200", "csrc")
REL_BOUND = 1.02e-4  # minimax 1.013e-4 plus float32 evaluation


def load_fit():
    spec = importlib.util.spec_from_file_location("fit_exp2_poly", os.path.join(CSRC, "fit_exp2_poly.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def header_constants():
    text = open(os.path.join(CSRC, "sm100_ptx.cuh")).read()
    body = text[text.index("float2 ex2_poly2(float2 x)"):]
    body = body[:body.index("\n}\n")]
    c = {k: np.float32(float(v)) for k, v in re.findall(r"\b(kC[123])\s*=\s*([0-9.eE+-]+)f", body)}
    # the last Horner step adds exactly 1 (the constant term)
    assert re.search(r"__ffma2_rn\(q, f, make_float2\(1\.0f, 1\.0f\)\)", body)
    assert "fmaxf(x.x, -127.0f)" in body and "fmaxf(x.y, -127.0f)" in body
    return np.array([1.0, c["kC1"], c["kC2"], c["kC3"]], dtype=np.float32)


def test_header_constants_are_the_fit():
    fit = load_fit()
    c_fit = fit.fit()
    c_hdr = header_constants()
    assert c_fit[0] == np.float32(1.0)
    # same float32 values (a last-bit difference between solver versions is tolerated)
    np.testing.assert_allclose(c_hdr, c_fit, rtol=4e-7, atol=0)
    err = fit.max_rel_error(c_hdr)
    assert err <= 1.014e-4, err


def emulate(x):
    """The device steps in float32: clamp at -127, round to an integer with
    the 1.5 * 2^23 trick, Horner in fused multiply-adds, then j * 2^23 added
    to the bits of the polynomial (an integer multiply-add, mod 2^32)."""
    c = header_constants().astype(np.float64)
    x = np.maximum(np.asarray(x, np.float32), np.float32(-127.0))
    r = np.float32(12582912.0)
    t = (x + r).astype(np.float32)
    j = (t - r).astype(np.float32)
    f = (x.astype(np.float64) - j.astype(np.float64)).astype(np.float32)  # exact
    # fused multiply-add: exact product and sum in extended precision, one rounding to float32
    fma = lambda a, b, d: (a.astype(np.longdouble) * b.astype(np.longdouble) + np.longdouble(d)).astype(np.float32)
    q = fma(np.full_like(f, c[3], dtype=np.float32), f, c[2])
    q = fma(q, f, c[1])
    q = fma(q, f, c[0])
    bits = (t.view(np.uint32).astype(np.uint64) * (1 << 23) + q.view(np.uint32).astype(np.uint64)) % (1 << 32)
    return bits.astype(np.uint32).view(np.float32)


def sweep():
    x = np.concatenate([np.linspace(-140.0, 127.0, 400001), np.arange(-140, 128, dtype=np.float64),
                        np.arange(-140, 127) + 0.5, [-np.inf]]).astype(np.float32)
    return x


def check_bounds(x, y):
    x = x.astype(np.float64)
    y = y.astype(np.float64)
    assert np.all(np.isfinite(y)) and np.all(y >= 0)
    ok = x >= -126
    rel = np.abs(y[ok] / np.exp2(x[ok]) - 1)
    assert rel.max() <= REL_BOUND, rel.max()
    assert np.all(y[x <= -127] == 0.0)          # -inf (a masked score) included
    mid = (x > -127) & (x < -126)
    assert np.all(y[mid] < 2.0 ** -126)
    # exact at integers: the polynomial is exactly 1 at f = 0
    ints = (x == np.round(x)) & (x >= -126)
    assert np.all(y[ints] == np.exp2(x[ints]))


def test_algorithm_bounds_in_float32():
    x = sweep()
    check_bounds(x, emulate(x))


@pytest.mark.gpu
def test_device_exp2_matches_2_pow_x():
    import torch
    import exact_io_aware_102_b200 as pkg
    x = sweep()
    n = x.size
    xd = torch.from_numpy(x).cuda()
    yd = torch.full((n,), float("nan"), dtype=torch.float32, device="cuda")
    assert pkg.attn_selftest_ex2(xd.data_ptr(), yd.data_ptr(), n) == pkg.ATTN_OK
    y = yd.cpu().numpy()
    check_bounds(x, y)
    # and bit for bit what the float32 steps give
    np.testing.assert_array_equal(y.view(np.uint32), emulate(x).view(np.uint32))
    # odd length: the last element is paired with itself
    assert pkg.attn_selftest_ex2(xd.data_ptr(), yd.data_ptr(), 7) == pkg.ATTN_OK
    np.testing.assert_array_equal(yd[:7].cpu().numpy().view(np.uint32), emulate(x[:7]).view(np.uint32))
    # argument checks
    assert pkg.attn_selftest_ex2(xd.data_ptr(), xd.data_ptr() + 4, 16) == pkg.ATTN_ERR_INVALID_ARG
    assert pkg.attn_selftest_ex2(xd.data_ptr(), yd.data_ptr(), 0) == pkg.ATTN_ERR_INVALID_ARG
