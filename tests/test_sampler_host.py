"""Host logic of the sampler variants, no GPU: the library's time grid and mu(n)
against the oracle, the option defaults and the argument errors."""
import math
import os

import numpy as np
import pytest

from flow_matching_mmdit_b200 import binding
from oracle import lens_oracle as o


@pytest.fixture(scope="module")
def lib():
    if not os.path.exists(binding.LIB_PATH):
        from flow_matching_mmdit_b200 import build
        build.build()
    return binding.load_library()


def test_uniform_grid_is_bit_identical(lib):
    for S in (1, 2, 3, 4, 7, 20, 50):
        assert np.array_equal(binding.lens_time_grid(S, False, 0.0), o.time_grid(S))


@pytest.mark.parametrize("mu", [-0.7, 0.5, 1.06, 2.0, math.log(3.0)])
def test_shifted_grid_matches_oracle(lib, mu):
    for S in (1, 2, 4, 20, 50):
        g = binding.lens_time_grid(S, True, mu)
        assert g[0] == 1.0 and g[-1] == 0.0
        assert np.allclose(g, o.time_grid(S, mu), rtol=0, atol=1e-15)


def test_shift_mu_matches_oracle(lib):
    for n in (256, 1024, 4096, 8100, 8192):
        assert binding.lens_shift_mu(n, 1024, 1.06, 4096, 1.5) == pytest.approx(
            o.shift_mu(n, 1024, 1.06, 4096, 1.5), rel=0, abs=1e-14)
    assert math.isnan(binding.lens_shift_mu(5, 7, 1.0, 7, 2.0))    # degenerate anchors


def test_options_and_argument_errors(lib):
    opt = binding.lens_sampler_default_options()
    assert (opt.guidance, opt.cfg_rescale, opt.time_shift, opt.shift_mu) == (1.0, 0.0, 0, 0.0)
    for steps, mu in ((0, 0.0), (4, float("nan")), (4, 51.0), (4, -60.0)):
        with pytest.raises(binding.LensError) as e:
            binding.lens_time_grid(steps, True, mu)
        assert e.value.status == 1
