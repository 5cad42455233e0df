"""Pins of the oracle's temperature softmax (CPU only).

Checked against closed forms worked out by hand, scipy's logsumexp (a
library routine), shift/scale invariances and normalisation."""
import json
import os
from decimal import Decimal

import numpy as np
import pytest
from scipy.special import logsumexp

import oracle
from speculative_decoding_block_spec_b200.synth import f32_to_bf16_bits, bf16_bits_to_f32


def test_golden_closed_forms(golden_dir):
    with open(os.path.join(golden_dir, "softmax_closed_form.json")) as f:
        cases = json.load(f)["cases"]
    for c in cases:
        if c["dtype"] == "f32":
            x = np.array([c["x"]], np.float32)
        else:
            x = np.array([c["bits"]], np.uint16)
            assert list(bf16_bits_to_f32(x[0])) == c["decoded"]
        m, lse, p = oracle.softmax_T(x, c["T"], probs=True)
        assert m[0] == c["row_max"], c["name"]
        assert abs(Decimal(repr(float(lse[0]))) - Decimal(c["row_lse"])) < Decimal("1e-14"), c["name"]
        assert abs(p.sum() - 1.0) < 1e-15


def test_matches_library_logsumexp():
    rng = np.random.default_rng(1)
    x = (rng.standard_normal((7, 1001)) * 3).astype(np.float32)
    for T in (1.0, 1.5, 0.7):
        m, lse = oracle.softmax_T(x, T)
        z = x.astype(np.float64) / T
        np.testing.assert_array_equal(m, z.max(axis=1))
        np.testing.assert_allclose(lse, logsumexp(z, axis=1), rtol=1e-14, atol=0)


def test_shift_and_scale_invariance():
    rng = np.random.default_rng(2)
    # integers keep x + c and x * T exact in fp32
    x = rng.integers(-20, 20, size=(5, 333)).astype(np.float32)
    m0, l0, p0 = oracle.softmax_T(x, 1.0, probs=True)
    m1, l1, p1 = oracle.softmax_T(x + np.float32(16), 1.0, probs=True)
    np.testing.assert_allclose(l1 - l0, 16.0, rtol=0, atol=1e-12)
    np.testing.assert_allclose(p1, p0, rtol=1e-12, atol=1e-300)
    m2, l2, p2 = oracle.softmax_T(x * np.float32(4), 4.0, probs=True)
    np.testing.assert_allclose(l2, l0, rtol=1e-15, atol=1e-14)
    np.testing.assert_allclose(p2, p0, rtol=1e-13, atol=1e-300)


def test_probs_are_exp_z_minus_lse_and_normalised():
    rng = np.random.default_rng(3)
    h = f32_to_bf16_bits(rng.standard_normal((4, 4097)).astype(np.float32) * 2)
    m, lse, p = oracle.softmax_T(h, 1.5, probs=True)
    np.testing.assert_allclose(p.sum(axis=1), 1.0, rtol=0, atol=1e-13)
    assert np.all(p > 0)
    z = bf16_bits_to_f32(h).astype(np.float64) / 1.5
    np.testing.assert_allclose(np.log(p), z - lse[:, None], rtol=0, atol=1e-12)


def test_single_column_row():
    x = np.array([[3.5], [-2.0]], np.float32)
    m, lse, p = oracle.softmax_T(x, 2.0, probs=True)
    np.testing.assert_array_equal(lse, [1.75, -1.0])
    np.testing.assert_array_equal(p, [[1.0], [1.0]])


def test_rejects_bad_arguments():
    with pytest.raises(ValueError):
        oracle.softmax_T(np.zeros((1, 4), np.float32), 0.0)
    with pytest.raises(TypeError):
        oracle.softmax_T(np.zeros((1, 4), np.float64), 1.0)
