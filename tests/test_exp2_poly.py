"""The kernel's polynomial 2^x (exp2_poly_pair in attn_fwd_sm100.cu), re-evaluated
on the CPU step by step in fp32 from the constants in the source file: its
relative error stays below the stated 7.5e-5 over the inputs the softmax can
pass (x <= the lazy-rescale threshold, clamped below at -125), far below the
bf16 rounding (2^-9) that P gets anyway."""
import os
import re

import numpy as np

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "exact_attention_127_b200", "csrc", "attn_fwd_sm100.cu")


def constants():
    text = open(SRC).read()
    vals = {}
    for name in ("EXP2_ROUND", "EXP2_C0", "EXP2_C1", "EXP2_C2", "EXP2_C3"):
        m = re.search(rf"constexpr float {name} = ([0-9.e+-]+)f;", text)
        assert m, name
        vals[name] = np.float32(float(m.group(1)))
    return vals


def f32(x):
    return np.asarray(x, dtype=np.float32)


def fma32(a, b, c):
    # a*b is exact in fp64 for fp32 a, b; one rounding to fp32 after the add
    # (the double rounding through fp64 is below the bound's precision)
    return f32(a.astype(np.float64) * b.astype(np.float64) + c.astype(np.float64))


def exp2_poly(x, k):
    x = np.maximum(f32(x), np.float32(-125.0))
    t = f32(x + k["EXP2_ROUND"])                  # fp32 add: rounds x to an integer
    n = f32(t - k["EXP2_ROUND"])
    f = f32(x - n)
    q = fma32(np.full_like(f, k["EXP2_C3"]), f, np.full_like(f, k["EXP2_C2"]))
    q = fma32(q, f, np.full_like(f, k["EXP2_C1"]))
    q = fma32(q, f, np.full_like(f, k["EXP2_C0"]))
    bits = q.view(np.int32) + (t.view(np.int32) << 23)
    return bits.astype(np.int32).view(np.float32)


def test_relative_error_bound():
    k = constants()
    x = f32(np.linspace(-125.0, 16.0, 2_000_001))
    got = exp2_poly(x, k).astype(np.float64)
    want = np.exp2(x.astype(np.float64))
    rel = np.abs(got - want) / want
    assert rel.max() <= 7.6e-5, rel.max()
    assert rel.max() >= 1e-5          # a real degree-3 fit, not an exact routine


def test_integer_arguments_are_nearly_exact_and_clamp():
    k = constants()
    x = f32(np.arange(-125, 17))
    got = exp2_poly(x, k).astype(np.float64)
    assert np.allclose(got, np.exp2(x.astype(np.float64)), rtol=1e-4, atol=0)
    # below the clamp the result is 2^-125 (tiny, finite, positive), never garbage
    low = exp2_poly(f32([-126.0, -300.0, -1e30]), k)
    assert np.all(low == exp2_poly(f32([-125.0]), k)[0])
