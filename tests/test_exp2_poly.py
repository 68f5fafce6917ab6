"""The software exp2 the dK/dV kernel uses for part of its keys (exp2_poly2 in
usp_ptx.cuh): its coefficients are the Remez minimax ones the derivation script
produces, and the fp32 evaluation, step by step as the kernel does it, stays
within the stated relative error of 2^x over the range the kernel feeds it."""
import importlib.util
import pathlib
import re

import numpy as np

CSRC = pathlib.Path(__file__).resolve().parents[1] / "long_context_exact_tma_b200" / "csrc"


def _header_coeffs():
    text = (CSRC / "usp_ptx.cuh").read_text()
    m = re.search(r"kC0 = ([0-9.e+-]+)f, kC1 = ([0-9.e+-]+)f, kC2 = ([0-9.e+-]+)f, kC3 = ([0-9.e+-]+)f", text)
    assert m, "coefficient line not found"
    return np.array([float(v) for v in m.groups()], dtype=np.float32)


def _derived():
    spec = importlib.util.spec_from_file_location("exp2_poly_coeffs", CSRC / "exp2_poly_coeffs.py")
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod.remez_exp2()


def _emulate(x, c):
    """fp32 emulation of exp2_poly2: clamp, round-to-nearest split, Horner (fma in
    fp64 then rounded to fp32, which is what a fused multiply-add gives), exponent add."""
    f32 = np.float32
    x = np.maximum(x.astype(f32), f32(-125.0))
    t = (x + f32(12582912.0)).astype(f32)
    n = (t - f32(12582912.0)).astype(f32)
    f = (x - n).astype(f32)
    fma = lambda a, b, d: (a.astype(np.float64) * b + d).astype(f32)  # noqa: E731
    p = fma(np.full_like(f, c[3]), f, np.full_like(f, c[2]))
    p = fma(p, f, np.full_like(f, c[1]))
    p = fma(p, f, np.full_like(f, c[0]))
    bits = p.view(np.uint32) + (t.view(np.uint32) << np.uint32(23))
    return bits.view(f32)


def test_header_coefficients_are_the_derived_minimax_ones():
    c, err = _derived()
    assert err < 7.6e-5
    np.testing.assert_array_equal(_header_coeffs(), c)


def test_fp32_evaluation_error_bound():
    c = _header_coeffs()
    rng = np.random.default_rng(0)
    x = np.concatenate([np.linspace(-124.0, 8.0, 200001), rng.uniform(-30.0, 8.0, 200000),
                        np.arange(-124, 9, dtype=np.float64), np.arange(-124, 8) + 0.5]).astype(np.float32)
    y = _emulate(x, c).astype(np.float64)
    rel = np.abs(y / np.exp2(x.astype(np.float64)) - 1.0)
    # minimax bound 7.5e-5 plus a few fp32 roundings
    assert rel.max() < 8.0e-5, rel.max()
    assert (y > 0).all()


def test_clamp_keeps_tiny_positive_weights():
    c = _header_coeffs()
    x = np.array([-np.inf, -1e30, -400.0, -126.0, -125.0], dtype=np.float32)
    y = _emulate(x, c)
    assert np.all(y > 0) and np.all(y <= np.float32(2.0 ** -124))
