"""The kernel's FMA-pipe exp2 (range reduction + degree-3 minimax polynomial),
re-evaluated step by step in fp32 on the CPU from the constants in the CUDA
header, against exp2 in fp64.  The kernel feeds bf16 P (relative rounding
2^-9), so the bound that matters is a relative error far below that."""

import os
import re

import numpy as np

HDR = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "tiled_attention_12_b200", "csrc", "ptx.cuh")


def _coeffs():
    text = open(HDR).read()
    body = text[text.index("exp2_poly2("):]
    body = body[: body.index("return pack2")]
    vals = [float(v) for v in re.findall(r"pack2\((-?\d+\.\d+)f, -?\d+\.\d+f\)", body)]
    # order of appearance: magic, -magic, -1, c3, c2, c1, c0
    return vals[3], vals[4], vals[5], vals[6]


def _emulate(x):
    f32 = np.float32
    c3, c2, c1, c0 = (f32(c) for c in _coeffs())
    xc = np.maximum(x.astype(f32), f32(-126.0))
    r = (xc + f32(12582912.0)).astype(f32)
    n = (r - f32(12582912.0)).astype(f32)
    f = (xc - n).astype(f32)
    p = ((c3 * f).astype(f32) + c2).astype(f32)        # fp32 products/sums, no fma:
    p = ((p * f).astype(f32) + c1).astype(f32)         # a slightly worse rounding
    p = ((p * f).astype(f32) + c0).astype(f32)         # than the kernel's fma
    bits = p.view(np.uint32) + (r.view(np.uint32) << np.uint32(23))
    return bits.astype(np.uint32).view(np.float32)


def test_coefficients_parse():
    c3, c2, c1, c0 = _coeffs()
    assert abs(c0 - 1) < 1e-3 and abs(c1 - np.log(2)) < 1e-3


def test_relative_error_bound_over_the_used_range():
    # results are normal floats for x >= -125 (below that they shade into
    # subnormals, which only ever stand for p ~ 0)
    x = np.concatenate([np.linspace(-125, 9, 3_000_001, dtype=np.float32),
                        np.arange(-20, 9, dtype=np.float32),            # integers: f = 0
                        np.arange(-20, 9, dtype=np.float32) + 0.5])     # ties of the rounding
    y = _emulate(x).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(y - ref) / ref
    assert rel.max() < 1.0e-4, rel.max()


def test_clamps_far_negative_inputs_to_tiny_positive_values():
    x = np.array([-np.inf, -1e30, -1000.0, -127.0, -126.5], dtype=np.float32)
    y = _emulate(x)
    assert np.all(np.isfinite(y)) and np.all(y >= 0) and np.all(y < 2.0 ** -124)
