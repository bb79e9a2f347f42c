"""The C-ABI library loads without a GPU and exports every declared symbol."""
import ctypes
import os
import re
import subprocess

import pytest

from flow_matching_mmdit_b200 import binding

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "lens_dit.h")


def declared_symbols():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"LENS_API\s+[\w\s\*]+?\b(lens_\w+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib():
    if not os.path.exists(binding.LIB_PATH):
        from flow_matching_mmdit_b200 import build
        build.build()
    return binding.load_library()


def test_header_declares_the_boundary():
    syms = declared_symbols()
    for s in ("lens_dit_create", "lens_dit_forward", "lens_sample_euler", "lens_dit_debug_blocks",
              "lens_dit_destroy", "lens_status_string"):
        assert s in syms
    assert sorted(binding.EXPORTS) == syms


def test_library_exports_every_declared_symbol(lib):
    out = subprocess.run(["nm", "-D", "--defined-only", binding.LIB_PATH], capture_output=True, text=True,
                         check=True).stdout
    exported = set(re.findall(r"\bT (lens_\w+)", out))
    missing = [s for s in declared_symbols() if s not in exported]
    assert not missing, missing
    for s in declared_symbols():
        assert hasattr(lib, s)


def test_no_driver_or_runtime_link_dependency():
    out = subprocess.run(["ldd", binding.LIB_PATH], capture_output=True, text=True).stdout
    assert "libcuda.so" not in out and "libcudart.so" not in out


def test_default_config_and_status_strings(lib):
    c = binding.lens_dit_default_config()
    assert (c.num_blocks, c.hidden, c.heads, c.head_dim, c.mlp_hidden) == (48, 1536, 24, 64, 4096)
    assert (c.in_channels, c.latent_channels, c.patch, c.txt_layers, c.txt_dim) == (128, 32, 2, 4, 2880)
    assert list(c.rope_axes) == [8, 28, 28] and c.rope_theta == 10000.0 and c.freq_dim == 256
    assert binding.lens_status_string(0) == "ok"
    assert binding.lens_status_string(5) == "device wait timed out"
    assert binding.lens_status_string(99) == "unknown status"


def test_argument_errors_return_synchronously(lib):
    """Null handles and bad sizes are rejected before any CUDA call."""
    assert lib.lens_dit_default_config(None) == 1
    assert lib.lens_dit_create(None, None, 0, None, None) == 1
    assert lib.lens_dit_forward(None, None, 1, 1, 1, None, 0, None, None, None) == 1
    assert lib.lens_sample_euler(None, None, None, 1, 1, 16, 16, 1, 1.0, 0, None, None) == 1
    assert lib.lens_op_patchify(None, 1, 1, 1, None, None) == 1
    assert lib.lens_op_gemm_bf16(ctypes.c_void_p(16), ctypes.c_void_p(16), None, ctypes.c_void_p(16), 10, 48, 64,
                                 None) == 2   # N not a multiple of 32
    assert lib.lens_op_attention(ctypes.c_void_p(16), ctypes.c_void_p(16), ctypes.c_void_p(16), 1, 0, 0, None, None,
                                 None) == 2   # empty sequence
    assert lib.lens_op_euler_cfg(ctypes.c_void_p(16), ctypes.c_void_p(16), None, 0, 0.1, 1.0, None) == 2
    assert lib.lens_op_rmsnorm_modulate(ctypes.c_void_p(16), 0, 1, ctypes.c_void_p(16), ctypes.c_void_p(16), 0,
                                        1e-6, ctypes.c_void_p(16), None) == 2


def test_attention_with_no_key_is_refused(lib):
    """A batch row with no image token and no valid text token has no key to attend,
    so its softmax is undefined: the masked attention op refuses it (SHAPE) before
    touching the device.  A row that keeps one text key is accepted as far as the
    size checks go (it then fails on the misaligned fake pointer, INVALID_ARG)."""
    P = lambda a: ctypes.c_void_p(a)
    lens = (ctypes.c_int * 2)(3, 0)
    assert lib.lens_op_attention_masked(P(16), P(16), P(16), 2, 4, 0, lens, P(16), None, None) == 2
    lens_ok = (ctypes.c_int * 2)(3, 1)
    assert lib.lens_op_attention_masked(P(8), P(16), P(16), 2, 4, 0, lens_ok, P(16), None, None) == 1
