"""The FMA-pipe exp2 used by part of the prefill softmax, checked on the CPU:
its constants are the ones the derivation produces, the cubic's relative error
is below 1e-4 on the reduced range, and a bit-level emulation of the whole
routine (range reduction, cubic, exponent add) matches 2^x over the range the
softmax feeds it."""
import os
import re

import numpy as np

from sequence_expanded_attention_b200.csrc import exp2_poly

PTX = os.path.join(os.path.dirname(exp2_poly.__file__), "hd_ptx.cuh")


def _constants_in_source():
    src = open(PTX).read()
    body = src[src.index("float ex2_poly(float x)"):]
    body = body[: body.index("}")]
    return [float(v) for v in re.findall(r"([0-9]\.[0-9]+e[-+][0-9]+)f", body)]


def test_source_constants_are_the_derived_ones():
    got = _constants_in_source()
    # order in the source: c3, c2 (first fmaf), c1, c0
    c3, c2, c1, c0 = got
    want = np.asarray(exp2_poly.fit(), dtype=np.float32)
    assert np.allclose([c0, c1, c2, c3], want, rtol=1e-7, atol=0)


def test_cubic_relative_error_bound():
    assert exp2_poly.max_rel_error(exp2_poly.fit()) < 1e-4


def _emulate(x):
    """fp32 emulation of ex2_poly step by step."""
    x = np.maximum(np.asarray(x, dtype=np.float32), np.float32(-125.0))
    shifter = np.float32(12582912.0)
    t = (x + shifter).astype(np.float32)
    j = (t - shifter).astype(np.float32)
    f = (x - j).astype(np.float32)
    c0, c1, c2, c3 = np.asarray(exp2_poly.fit(), dtype=np.float32)
    p = exp2_poly.horner_f32([c0, c1, c2, c3], f)
    bits = p.view(np.int32).astype(np.int64) + (t.view(np.int32).astype(np.int64) << 23)
    return (bits & 0xFFFFFFFF).astype(np.uint32).view(np.int32).view(np.float32)


def test_full_routine_matches_exp2():
    x = np.concatenate([np.linspace(-120.0, 8.0, 400001, dtype=np.float32),
                        np.array([0.0, -0.5, 0.5, 1.0, -1.0, 7.999, -119.5], dtype=np.float32)])
    y = _emulate(x).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    assert np.max(np.abs(y / ref - 1.0)) < 1e-4


def test_underflow_is_tiny_and_positive():
    y = _emulate(np.array([-126.0, -200.0, -np.inf], dtype=np.float32))
    assert np.all(y >= 0) and np.all(y <= 2.0 ** -124)
