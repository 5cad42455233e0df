"""exp2_fma (csrc/exp2_fma.cuh), the FMA-pipe base-2 exponential that the
row-statistics kernels use for a share of their exponentials, checked on
the CPU against its error bound. The header compiles as plain C++; the host
build uses the same IEEE float operations and fused multiply-adds as the
device build, so the bits measured here are the kernel's.

Bound: the polynomial's relative error with float32 coefficients (1.55e-7,
printed by csrc/exp2_poly.py) plus the float32 rounding of five Horner
steps (at most 2^-24 relative each, times the steps' gain of at most
about 1.5), so below 4e-7 relative over the whole domain y in [-125, 0]."""
import os
import shutil
import subprocess

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "speculative_decoding_block_spec_b200", "csrc")

PROGRAM = r"""
#include <cstdio>
#include <cstdlib>
#include "exp2_fma.cuh"
int main(int argc, char** argv) {
  // reads float32 arguments from stdin (binary), writes float32 results to stdout
  float y;
  while (std::fread(&y, sizeof y, 1, stdin) == 1) {
    const float r = specv::exp2_fma(y);
    std::fwrite(&r, sizeof r, 1, stdout);
  }
  return 0;
}
"""


@pytest.fixture(scope="module")
def exp2_fma(tmp_path_factory):
    gxx = shutil.which("g++")
    if gxx is None:
        pytest.skip("no C++ compiler")
    d = tmp_path_factory.mktemp("exp2")
    src = d / "e.cpp"
    src.write_text(PROGRAM)
    exe = d / "e"
    subprocess.run([gxx, "-std=c++17", "-O2", "-ffp-contract=off", "-I", CSRC, str(src), "-o", str(exe)], check=True)

    def run(y):
        y = np.ascontiguousarray(y, np.float32)
        out = subprocess.run([str(exe)], input=y.tobytes(), capture_output=True, check=True).stdout
        return np.frombuffer(out, np.float32)

    return run


def test_relative_error_over_the_domain(exp2_fma):
    rng = np.random.default_rng(0)
    y = np.concatenate([
        -rng.random(2_000_000, dtype=np.float32) * 125.0,       # the whole domain
        -rng.random(500_000, dtype=np.float32),                # near 0, where most terms live
        -np.arange(0, 126, dtype=np.float32),                  # integers (f = 0)
        -np.arange(0, 125, dtype=np.float32) - 0.5,            # round-half cases (f = +-1/2)
        np.nextafter(-np.arange(0, 125, dtype=np.float32) - 0.5, np.float32(0)),
        np.float32([0.0, -0.0, -1e-30, -124.99999]),
    ]).astype(np.float32)
    r = exp2_fma(y).astype(np.float64)
    rel = np.abs(r / np.exp2(y.astype(np.float64)) - 1.0)
    assert rel.max() < 4e-7, (rel.max(), y[np.argmax(rel)])
    # no systematic bias beyond the polynomial's (a normaliser sums many terms)
    assert abs(np.mean(r / np.exp2(y.astype(np.float64)) - 1.0)) < 1e-7


def test_special_arguments(exp2_fma):
    y = np.float32([np.nan, -np.inf, -1000.0, -125.0, -126.0])
    r = exp2_fma(y)
    assert np.isnan(r[0])
    # clamped to 2^-125 (within the bound: p(0) = c0 is 1 + 1.2e-7), a term below 1e-37 of the row's largest
    np.testing.assert_allclose(r[1:], 2.0 ** -125, rtol=4e-7, atol=0)
    assert r[1] == r[2] == r[3] == r[4]


def test_monotone_on_a_fine_grid(exp2_fma):
    """Sums of exponentials do not need monotonicity, but a non-monotone step
    would show a broken range reduction at the half-integer seams."""
    y = np.linspace(-3.0, 0.0, 300001).astype(np.float32)
    r = exp2_fma(y)
    assert np.all(np.diff(r.astype(np.float64)) >= -4e-7 * r[1:])
