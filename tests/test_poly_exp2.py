"""Error bound of the library's own FMA-pipe 2^x (``poly_exp2`` in bsa_common.cuh).

The function is an option of the attention kernel (off by default): a
Cody-Waite style reduction x = n + f with n = round(x) taken by adding and
subtracting 1.5 * 2^23, a cubic fitted on f in [-0.5, 0.5], and n added to the
exponent field.  This test reads the constants out of the CUDA source, replays
the same float32 steps in NumPy (integer arithmetic on the bit patterns for the
exponent step) and checks the relative error the source states against 2^x in
float64, over the whole input range the kernel feeds it.  CPU only.
"""
import os
import re

import numpy as np

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "block_sparse_attention_tokens_b200", "csrc", "bsa_common.cuh")
STATED_MAX_REL = 7.8e-5


def _constants():
    text = open(SRC).read()
    body = re.search(r"float poly_exp2\(float x\) \{(.*?)\n\}", text, re.S).group(1)
    clamp = float(re.search(r"fmaxf\(x, (-?[\d.]+)f\)", body).group(1))
    rc = float(re.search(r"round_const = ([\d.]+)f", body).group(1))
    c3, c2 = (float(v) for v in re.search(r"fmaf\(([\d.]+)f, f, ([\d.]+)f\)", body).groups())
    c1 = float(re.search(r"fmaf\(p, f, ([\d.]+)f\);\n\s*p = fmaf", body).group(1))
    c0 = float(re.findall(r"fmaf\(p, f, ([\d.]+)f\)", body)[-1])
    return clamp, rc, (c3, c2, c1, c0)


def _f32(v):
    return np.asarray(v, dtype=np.float64).astype(np.float32)


def _fma32(a, b, c):
    # float32 a*b is exact in float64; one rounding to float64, one to float32
    return (a.astype(np.float64) * b.astype(np.float64) + c.astype(np.float64)).astype(np.float32)


def poly_exp2_f32(x):
    clamp, rc, (c3, c2, c1, c0) = _constants()
    x = np.maximum(_f32(x), np.float32(clamp))
    r = np.float32(rc)
    t = (x + r).astype(np.float32)
    f = (x - (t - r).astype(np.float32)).astype(np.float32)
    p = _fma32(np.full_like(f, c3, dtype=np.float32), f, np.full_like(f, c2, dtype=np.float32))
    p = _fma32(p, f, np.full_like(f, c1, dtype=np.float32))
    p = _fma32(p, f, np.full_like(f, c0, dtype=np.float32))
    bits = (p.view(np.uint32).astype(np.uint64) + (t.view(np.uint32).astype(np.uint64) << 23)) \
        & 0xFFFFFFFF
    return bits.astype(np.uint32).view(np.float32), f


def test_constants_are_the_documented_ones():
    clamp, rc, coeffs = _constants()
    assert clamp == -125.0 and rc == 1.5 * 2 ** 23
    assert len(coeffs) == 4 and abs(coeffs[3] - 1.0) < 1e-3 and abs(coeffs[2] - np.log(2)) < 1e-3


def test_cubic_relative_error_on_the_reduced_range():
    _, _, (c3, c2, c1, c0) = _constants()
    f = np.linspace(-0.5, 0.5, 200001)
    rel = np.abs((((c3 * f + c2) * f + c1) * f + c0) / np.exp2(f) - 1.0)
    assert rel.max() <= STATED_MAX_REL
    # a minimax fit spreads its error: both ends and the interior come near the maximum
    assert rel[0] > 0.5 * rel.max() and rel[-1] > 0.5 * rel.max()


def test_float32_replay_over_the_input_range():
    x = np.concatenate([np.linspace(-125.0, 64.0, 400001), np.arange(-125, 65, dtype=np.float64),
                        np.arange(-125, 64, dtype=np.float64) + 0.5])
    y, f = poly_exp2_f32(x)
    x32 = _f32(np.maximum(x, -125.0)).astype(np.float64)
    ref = np.exp2(x32)
    assert np.all(np.abs(f) <= 0.5)                       # round-to-nearest reduction
    rel = np.abs(y.astype(np.float64) / ref - 1.0)
    # the cubic's error plus a few float32 roundings (2^-24 each)
    assert rel.max() <= STATED_MAX_REL + 4 * 2.0 ** -24, rel.max()
    # exact powers of two come out within the cubic's error at f = 0
    ints = np.arange(-125, 65)
    yi, _ = poly_exp2_f32(ints.astype(np.float64))
    assert np.all(np.abs(yi.astype(np.float64) / np.exp2(ints) - 1.0) <= STATED_MAX_REL)


def test_below_the_clamp_the_result_is_two_to_the_minus_125():
    y, _ = poly_exp2_f32(np.array([-126.0, -1000.0, -np.inf]))
    assert np.all(np.abs(y.astype(np.float64) / 2.0 ** -125 - 1.0) <= STATED_MAX_REL)
