"""Error bound of the FMA-pipe 2^x used for part of bsa_fwd's softmax weights.

The constants are read from the CUDA header, and the same steps (round to nearest
by adding 1.5 * 2^23, degree-3 polynomial on the remainder, exponent-field add)
are replayed in IEEE fp32 with numpy, against exp2 in fp64.  The bound needed is
far below the 2^-9 relative rounding the weights then get as bf16."""
import os
import re

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _coeffs():
    src = open(os.path.join(ROOT, "block_sparse_attention_poem_b200", "csrc", "sm100.cuh")).read()
    return [np.float32(float(re.search(rf"kExp2C{i} = ([0-9.e+-]+)f;", src).group(1))) for i in range(4)]


def _exp2_poly_f32(x):
    c0, c1, c2, c3 = _coeffs()
    x = np.maximum(x.astype(np.float32), np.float32(-126.0))
    magic = np.float32(12582912.0)
    t = (x + magic).astype(np.float32)
    j = (t - magic).astype(np.float32)
    f = (x - j).astype(np.float32)
    p = np.float32(c3) * f + c2
    p = (p * f + c1).astype(np.float32)
    p = (p * f + c0).astype(np.float32)
    bits = (p.view(np.uint32) + (t.view(np.uint32) << np.uint32(23))).astype(np.uint32)
    return bits.view(np.float32)


def test_polynomial_relative_error_on_reduced_range():
    f = np.linspace(-0.5, 0.5, 200001, dtype=np.float32)
    y = _exp2_poly_f32(f).astype(np.float64)
    rel = np.abs(y - np.exp2(f.astype(np.float64))) / np.exp2(f.astype(np.float64))
    assert rel.max() < 8e-5


def test_full_range_reconstruction():
    x = np.concatenate([np.linspace(-125.5, 8.0, 400001), -np.random.default_rng(0).random(100000) * 30]).astype(np.float32)
    y = _exp2_poly_f32(x).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(y - ref) / ref
    assert rel.max() < 1e-4
    # clamped tail stays tiny and non-negative
    tail = _exp2_poly_f32(np.array([-200.0, -1e30, -np.inf], dtype=np.float32))
    assert np.all(tail >= 0) and np.all(tail < 1e-37)
