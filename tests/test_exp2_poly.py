"""The attention kernel's FMA-pipe exponential (csrc/exp2_poly.h), compiled for the
host with g++ and checked against the C library's exp2 in double precision: the
relative error bound of the minimax cubic over the whole range the softmax uses,
exact powers of two at integers, the clamp for very negative (and -inf) inputs, and
monotonicity.  CPU only."""
import os
import shutil
import subprocess

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "flow_matching_mmdit_b200", "csrc")

PROGRAM = r"""
#include <stdio.h>
#include <stdlib.h>
#include "exp2_poly.h"
int main(int argc, char** argv) {
  // x from argv[1] to argv[2] in steps of 2^-12, then a few special inputs
  const double lo = atof(argv[1]), hi = atof(argv[2]);
  double worst = 0, worst_x = 0, prev = 0;
  long long n = 0, nonmono = 0;
  for (double xd = lo; xd <= hi; xd += 1.0 / 4096.0, ++n) {
    const float x = (float)xd;
    const double y = lens::exp2_poly(x), r = exp2((double)x);
    const double e = fabs(y / r - 1.0);
    if (e > worst) { worst = e; worst_x = x; }
    if (n > 0 && y < prev) ++nonmono;
    prev = y;
  }
  printf("%.9g %.9g %lld %lld\n", worst, worst_x, n, nonmono);
  const float specials[] = {-INFINITY, -1e30f, -200.f, -126.f, -125.f, -1.f, 0.f, 1.f, 7.f, 8.f};
  for (float s : specials) printf("%.9g\n", (double)lens::exp2_poly(s));
  return 0;
}
"""


@pytest.fixture(scope="module")
def exe(tmp_path_factory):
    if shutil.which("g++") is None:
        pytest.skip("no host C++ compiler")
    d = tmp_path_factory.mktemp("exp2")
    src, out = d / "t.cpp", d / "t"
    src.write_text(PROGRAM)
    subprocess.run(["g++", "-O2", "-std=c++17", "-ffp-contract=off", "-I", CSRC, str(src), "-o", str(out), "-lm"],
                   check=True)
    return str(out)


def _run(exe, lo, hi):
    lines = subprocess.run([exe, str(lo), str(hi)], capture_output=True, text=True, check=True).stdout.split("\n")
    worst, worst_x, n, nonmono = lines[0].split()
    return float(worst), float(worst_x), int(n), int(nonmono), [float(v) for v in lines[1:11]]


def test_relative_error_bound_over_the_softmax_range(exe):
    worst, worst_x, n, nonmono, _ = _run(exe, -125.0, 8.0)
    assert n > 500_000
    assert worst < 7.6e-5, (worst, worst_x)        # the Remez bound of the cubic, 7.48e-5
    assert nonmono == 0                            # never decreasing: larger scores never weigh less


def test_special_inputs(exe):
    *_, sp = _run(exe, 0.0, 0.0)
    tiny = 2.0 ** -125
    for v in sp[:5]:                               # -inf, -1e30, -200, -126 and -125 all clamp to 2^-125 (+-7.5e-5)
        assert abs(v / tiny - 1) < 7.6e-5
    for x, v in zip([-1, 0, 1, 7, 8], sp[5:]):
        assert abs(v / 2.0 ** x - 1) < 7.6e-5      # at integers f = 0, so only p(0) = c0 errs
    ratios = [v / 2.0 ** x for x, v in zip([-1, 0, 1, 7, 8], sp[5:])]
    assert max(ratios) - min(ratios) < 1e-8 * ratios[0]   # c0 * 2^j exactly (printed to 9 digits)


def test_the_cubic_is_the_relative_minimax():
    """Equioscillation: the relative error of the committed coefficients reaches its
    bound with alternating signs at five points of [-1/2, 1/2] (degree 3 + 2), which
    is what characterises the minimax polynomial."""
    src = open(os.path.join(CSRC, "exp2_poly.h")).read()
    c = [float(src.split(f"kExp2C{i} = ")[1].split("f;")[0]) for i in range(4)]
    f = np.linspace(-0.5, 0.5, 400001)
    err = (c[0] + f * (c[1] + f * (c[2] + f * c[3]))) / 2.0 ** f - 1
    E = np.max(np.abs(err))
    assert 7.4e-5 < E < 7.6e-5
    # local extrema of |err| within 2 % of the bound, signs alternating
    peaks = [i for i in range(1, len(f) - 1) if abs(err[i]) >= abs(err[i - 1]) and abs(err[i]) >= abs(err[i + 1])]
    peaks = [0] + peaks + [len(f) - 1]
    big = [i for i in peaks if abs(err[i]) > 0.98 * E]
    assert len(big) == 5
    assert all(np.sign(err[a]) != np.sign(err[b]) for a, b in zip(big, big[1:]))
