"""The attention kernel computes part of its softmax exponentials on the FMA pipe
(exp2_poly_pair in csrc/attn_tc05.cu): a Cody-Waite split v = j + f with
j = rint(v) by magic-number rounding, a degree-3 polynomial for 2^f on
[-1/2, 1/2], and 2^j added to the exponent bits.  This CPU test replays that
exact float32 sequence in numpy, with the coefficients read from the kernel
source, and checks its error against 2^v over the whole input range the
kernel sees: relative error below 1e-4 for v in [-125, 8] (far below the bf16
rounding, 2^-9, that P gets next) and absolute error below 1e-41 for
v in [-126, -125).  The GPU parity tests check the kernel's
outputs end to end.
"""
import os
import re

import numpy as np

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "ar_decoding_b200", "csrc", "attn_tc05.cu")


def _coeffs():
    text = open(SRC).read()
    body = text[text.index("exp2_poly_pair(float v0"):]
    body = body[:body.index("f2_split(p, p0, p1)")]
    magic = float(re.search(r"kMagic = ([0-9.e]+)f", body).group(1))
    vals = re.findall(r"f2_make\(([-0-9.e]+)f, \1f\)", body)
    nums = [float(v) for v in vals]
    # literal pairs in the source order: -1 (for f = v - rint(v)), c3, c2, c1, c0
    assert nums[0] == -1.0 and len(nums) == 5
    return np.float32(magic), [np.float32(v) for v in nums[1:5]]


def _emulate(v):
    magic, (c3, c2, c1, c0) = _coeffs()
    v = np.maximum(v.astype(np.float32), np.float32(-126.0))
    t = (v + magic).astype(np.float32)
    tf = (t - magic).astype(np.float32)
    f = (v - tf).astype(np.float32)
    p = (c3 * f + c2).astype(np.float32)         # the kernel fuses these (fma); rounding
    p = (p * f + c1).astype(np.float32)          # differences are ~1e-7, far below the bound
    p = (p * f + c0).astype(np.float32)
    bits = (t.view(np.uint32).astype(np.uint64) * 8388608 + p.view(np.uint32)) & 0xFFFFFFFF
    return bits.astype(np.uint32).view(np.float32)


def test_magic_rounding_split_is_exact():
    v = np.linspace(-126, 8, 200001).astype(np.float32)
    magic, _ = _coeffs()
    t = (v + magic).astype(np.float32)
    j = (t - magic).astype(np.float32)
    np.testing.assert_array_equal(j, np.rint(v))
    f = v - j
    assert np.abs(f).max() <= 0.5


def test_relative_error_bound():
    v = np.concatenate([np.linspace(-126, 8, 2_000_001), np.random.default_rng(0).uniform(-20, 0, 10**6)])
    got = _emulate(v).astype(np.float64)
    want = np.exp2(np.maximum(v.astype(np.float32), -126.0).astype(np.float64))
    rel = np.abs(got - want) / want
    normal = v >= -125.0          # below, results are ~1e-38 (at the edge of fp32 normals)
    assert rel[normal].max() < 1e-4, rel[normal].max()
    assert np.abs(got - want)[~normal].max() < 1e-41
    # and it is monotone enough for a softmax: never off by a power of two
    assert np.all(got > 0)
