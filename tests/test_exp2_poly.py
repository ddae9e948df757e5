"""The FMA-pipe exponential of the kernels (lard_exp2.cuh): its coefficients
are the Remez minimax fit the committed generator produces, and the fp32
evaluation (range reduction included) stays within 3e-7 relative of 2^x."""
import importlib.util
import os
import re

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "linear_memory_attention_b200", "csrc")


def _gen():
    spec = importlib.util.spec_from_file_location("gen_exp2_poly", os.path.join(CSRC, "gen_exp2_poly.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _header_coeffs():
    text = open(os.path.join(CSRC, "lard_exp2.cuh")).read()
    m = re.search(r"#define LARD_EXP2_POLY \{([^}]*)\}", text)
    return np.array([float(v.strip().rstrip("f")) for v in m.group(1).split(",")])


def test_coefficients_are_the_remez_fit():
    c, err = _gen().remez_exp2(5)
    h = _header_coeffs()
    assert len(h) == 6
    np.testing.assert_allclose(h, c, rtol=1e-8, atol=0)
    assert err < 1e-7


def _fma32(a, b, c):
    return np.float32(np.float64(a) * np.float64(b) + np.float64(c))


def exp2_fma_emulated(x):
    """float32 emulation of exp2_fma (vectorised)."""
    c = _header_coeffs().astype(np.float32)
    x = np.maximum(np.asarray(x, dtype=np.float32), np.float32(-125.0))
    t = (x + np.float32(12582912.0)).astype(np.float32)
    n = (t - np.float32(12582912.0)).astype(np.float32)
    f = (x - n).astype(np.float32)
    p = np.full_like(f, c[5])
    for k in (4, 3, 2, 1, 0):
        p = _fma32(p, f, c[k])
    bits = (p.view(np.int32).astype(np.int64) + (t.view(np.int32).astype(np.int64) << 23)) & 0xFFFFFFFF
    return bits.astype(np.uint32).view(np.float32)


def test_relative_error_bound():
    x = np.concatenate([np.linspace(-125.0, 8.0, 2_000_001, dtype=np.float32),
                        np.float32([-0.5, 0.5, 0.0, -1e-8, 1e-8, -124.99, 7.5])])
    got = exp2_fma_emulated(x).astype(np.float64)
    want = np.exp2(x.astype(np.float64))
    rel = np.abs(got / want - 1.0)
    assert rel.max() < 3e-7, rel.max()


def test_clamps_far_negative_inputs_to_a_tiny_normal():
    got = exp2_fma_emulated(np.float32([-1e30, -200.0, -126.0]))
    assert np.all(got > 0) and np.all(got < 3e-38)
    assert np.all(np.isfinite(got))
