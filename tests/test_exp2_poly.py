"""The FMA-pipe exponential of the attention kernel (Cody-Waite reduction + degree-3
polynomial): its constants equal the committed fit, and a float32 emulation of its exact
steps is within the stated relative error of 2^x, with masked (-inf) inputs giving 0."""

import os
import re

import numpy as np

from prefix_shared_attention_b200.csrc import fit_exp2_poly

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "prefix_shared_attention_b200", "csrc", "bat_attn_tc.cu")


def kernel_coefficients():
    text = open(SRC).read()
    return np.array([float(re.search(rf"kExp2C{i} = ([-0-9.e+]+)f", text).group(1)) for i in range(4)], np.float32)


def emulate(x):
    """The kernel's steps in float32 (fmaf on the packed path rounds once, like these ops)."""
    c = kernel_coefficients()
    x = np.maximum(np.asarray(x, np.float32), np.float32(-125.0))
    shift = np.float32(12582912.0)
    t = (x + shift).astype(np.float32)
    j = (t - shift).astype(np.float32)
    f = (x - j).astype(np.float32)
    p = (f * c[3] + c[2]).astype(np.float32)
    p = (p * f + c[1]).astype(np.float32)
    p = (p * f + c[0]).astype(np.float32)
    bits = p.view(np.int32) + (t.view(np.int32) << 23)
    return bits.astype(np.int32).view(np.float32)


def test_constants_match_the_fit():
    np.testing.assert_array_equal(kernel_coefficients(), fit_exp2_poly.fit())


def test_relative_error_bound():
    x = np.concatenate([np.linspace(-120.0, 10.0, 400001, dtype=np.float32),
                        np.array([0.0, -0.5, 0.5, -1.5, 7.999, -0.49999], np.float32)])
    got = emulate(x).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(got / ref - 1.0)
    assert rel.max() < 1.2e-4, rel.max()
    assert fit_exp2_poly.max_rel_error(kernel_coefficients()) < 1e-4


def test_masked_inputs_give_zero_contribution():
    got = emulate(np.array([-np.inf, -1e30, -200.0], np.float32))
    assert np.all(np.isfinite(got)) and np.all(got >= 0) and np.all(got < 1e-37)
