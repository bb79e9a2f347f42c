"""B200 (sm_100a) Lens MMDiT denoiser and flow-matching Euler sampler.

The compute lives in liblens_dit.so (CUDA kernels behind the C ABI of
include/lens_dit.h); this package is its ctypes binding.
"""
from .binding import *  # noqa: F401,F403
from .binding import EXPORTS, LensDit, LensError, lens_dit_config, lens_weight, load_library  # noqa: F401
