"""Host-side pins of the decode GEMM's NF4 table (no GPU): the fp16 table
scale fixed in csrc/decode_gemm.cu bounds the rounding error of every code
value, and the up rows' remainder part restores the scaled value to well
within fp32 precision. The NF4 values come from the oracle (the pages'
table); the scale is read from the kernel source as text."""
import os
import re

import numpy as np

import oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "grouped_nf4_w4a16_b200", "csrc", "decode_gemm.cu")


def table_scale() -> float:
    m = re.search(r"constexpr float kTableScale = ([0-9.]+)f;", open(SRC).read())
    assert m, "kTableScale not found"
    return float(np.float32(m.group(1)))


def worst_code_error(s: float) -> float:
    """max over the 16 codes of |fp16(fp32(NF4[c] * s)) / s - NF4[c]|."""
    v = oracle.nf4_table().astype(np.float32)
    scaled = (v * np.float32(s)).astype(np.float32)
    hi = scaled.astype(np.float16).astype(np.float64)
    return float(np.max(np.abs(hi - scaled.astype(np.float64)) / s))


def test_table_scale_bounds_the_code_error():
    s = table_scale()
    assert 1.0 <= s < 2.0
    plain = worst_code_error(1.0)
    scaled = worst_code_error(s)
    assert scaled <= 6.1e-5            # of the code range [-1, 1]
    assert plain >= 1.8e-4             # the plain fp16 rounding, for comparison
    assert plain / scaled >= 3.0


def test_table_scale_is_a_local_best():
    # no scale within +-1e-3 of the chosen one (2001 points) does better than
    # 0.1% of its error
    s = table_scale()
    best = worst_code_error(s)
    for t in np.linspace(s - 1e-3, s + 1e-3, 2001):
        assert worst_code_error(float(t)) >= best * 0.999


def test_up_row_remainder_restores_the_scaled_value():
    s = np.float32(table_scale())
    v = (oracle.nf4_table().astype(np.float32) * s).astype(np.float32)
    hi = v.astype(np.float16).astype(np.float32)
    rem = (v - hi).astype(np.float32)                      # exact in fp32
    assert np.array_equal(rem.astype(np.float64), v.astype(np.float64) - hi.astype(np.float64))
    lo = (rem * np.float32(8192.0)).astype(np.float16).astype(np.float64)
    back = hi.astype(np.float64) + lo / 8192.0
    nz = v != 0
    rel = np.abs(back[nz] - v[nz].astype(np.float64)) / np.abs(v[nz].astype(np.float64))
    assert rel.max() <= 2.0 ** -21
