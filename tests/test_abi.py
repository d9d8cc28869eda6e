"""The C-ABI library loads and exports every entry point include/bltdec.h declares (no GPU needed)."""

import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    names = []
    for fn in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if fn.endswith(".h"):
            src = open(os.path.join(ROOT, "include", fn)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            names += re.findall(r"^\s*(?:const\s+)?[a-z_0-9]+\s*\*?\s*(blt_[a-z_0-9]+)\s*\(", src, flags=re.M)
    return sorted(set(names))


@pytest.fixture(scope="module")
def lib():
    from block_diffusion_byte_b200 import _build

    path = _build.build()
    return ctypes.CDLL(path)


def test_header_declares_the_boundary():
    names = _declared()
    for n in ("blt_dec_init", "blt_dec_prefill", "blt_dec_diffuse_block", "blt_dec_draft", "blt_dec_verify_accept"):
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    for n in _declared():
        assert hasattr(lib, n), n


def test_binding_covers_every_export(lib):
    from block_diffusion_byte_b200 import binding

    assert sorted(binding.EXPORTS) == sorted(_declared())
    binding.load_library()


def test_struct_layouts_match_header():
    from block_diffusion_byte_b200 import binding as B

    assert ctypes.sizeof(B.blt_dec_config) == 18 * 4
    assert ctypes.sizeof(B.blt_dec_weights) == 4 * 8
    assert ctypes.sizeof(B.blt_rows_in) == 5 * 8
    assert ctypes.sizeof(B.blt_dec_counters) == 11 * 8


def test_init_rejects_bad_config_without_touching_the_gpu(lib):
    from block_diffusion_byte_b200 import binding as B

    cfg = B.blt_dec_config(n_layers=2, d_model=100, n_heads=4, d_ffn=512, d_global=256, vocab=257, weight_dtype=0,
                           rope_theta=1e4, norm_eps=1e-5, max_batch=1, max_ctx=64, max_latents=64, max_rows=64, max_block=4,
                           page_tokens=64)
    out = ctypes.c_void_p()
    w = B.blt_dec_weights()
    L = B.load_library()
    assert L.blt_dec_init(ctypes.byref(cfg), ctypes.byref(w), None, ctypes.byref(out)) == B.BLT_ERR_INVALID_ARG
    assert L.blt_dec_prefill(None, 1, None, None) == B.BLT_ERR_INVALID_ARG
