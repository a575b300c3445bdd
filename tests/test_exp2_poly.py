"""The FMA-pipe 2^x of the prefill kernels (a compile-time option, off by
default): its coefficients are the ones derive_exp2_poly.py fits, the scalar
and the packed copies in jl_prefill_common.cuh agree, and the floor-plus-cubic
evaluation, emulated here in fp32 steps, stays within the stated relative
error over the range the softmax feeds it (x <= 0 after the row maximum is
subtracted).  CPU only."""
import importlib.util
import os
import re

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "long_context_attention_bifocal_b200", "csrc")


def _derive():
    spec = importlib.util.spec_from_file_location("derive_exp2_poly",
                                                  os.path.join(CSRC, "derive_exp2_poly.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _header_coefficients():
    src = open(os.path.join(CSRC, "jl_prefill_common.cuh")).read()
    scalar = src[src.index("float exp2_poly(float x)"):src.index("uint64_t exp2_poly2(")]
    packed = src[src.index("uint64_t exp2_poly2("):]
    c3, c2 = (np.float32(v) for v in
              re.search(r"fmaf\(([0-9.]+)f, f, ([0-9.]+)f\)", scalar).groups())
    c1 = np.float32(re.search(r"fmaf\(p, f, ([0-9.]+)f\)", scalar).group(1))
    words = re.findall(r"0x([0-9A-F]{8})([0-9A-F]{8})ull", packed)
    return (c1, c2, c3), words


def _exp2_emulated(x, c):
    """2^x as the kernels evaluate it: clamp, floor, cubic by three fp32 FMAs,
    exponent added to the bits."""
    c0, c1, c2, c3 = (np.float64(v) for v in c)
    x = np.maximum(x.astype(np.float32), np.float32(-127.0))
    fl = np.floor(x.astype(np.float64))
    f = (x.astype(np.float64) - fl).astype(np.float32).astype(np.float64)
    p = (c3 * f + c2).astype(np.float32).astype(np.float64)
    p = (p * f + c1).astype(np.float32).astype(np.float64)
    p = (p * f + c0).astype(np.float32).astype(np.float64)
    return np.ldexp(p, fl.astype(np.int64))


def test_coefficients_match_the_fit():
    c, rel = _derive().fit()
    assert c[0] == np.float32(1.0)
    (c1, c2, c3), words = _header_coefficients()
    assert (c1, c2, c3) == (c[1], c[2], c[3])
    assert rel < 1.2e-4
    # the packed copy holds the same fp32 bit patterns in both halves
    bits = {f"{np.float32(v).view(np.uint32):08X}" for v in c[1:]} | {"3F800000"}
    for hi, lo in words:
        assert hi == lo
    assert bits <= {hi for hi, _ in words}


def test_relative_error_over_softmax_range():
    c, _ = _derive().fit()
    x = np.concatenate([np.linspace(-126.0, 0.0, 400001),
                        -np.arange(0, 127, dtype=np.float64),          # integers
                        -np.arange(0, 126, dtype=np.float64) - 0.5])
    got = _exp2_emulated(x, c)
    rel = np.abs(got / np.exp2(x.astype(np.float32).astype(np.float64)) - 1.0)
    assert rel.max() < 1.2e-4
    # exact at the integers, where the cubic is pinned to p(0) = 1
    ints = -np.arange(0, 126, dtype=np.float64)
    assert np.array_equal(_exp2_emulated(ints, c), np.exp2(ints))
