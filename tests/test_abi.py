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


def test_struct_layouts_match_header(tmp_path):
    """The binding's ctypes structs have the sizes and field offsets a C compiler gives the
    header's structs (checked by compiling the header with gcc)."""
    import subprocess

    from block_diffusion_byte_b200 import binding as B

    structs = {"blt_dec_config": B.blt_dec_config, "blt_dec_weights": B.blt_dec_weights, "blt_rows_in": B.blt_rows_in,
               "blt_dec_counters": B.blt_dec_counters}
    lines = ['#include <stddef.h>', '#include <stdio.h>', '#include "bltdec.h"', "int main(void) {"]
    for name, cls in structs.items():
        lines.append(f'  printf("{name} %zu\\n", sizeof({name}));')
        for f, _ in cls._fields_:
            lines.append(f'  printf("{name}.{f} %zu\\n", offsetof({name}, {f}));')
    lines.append("  return 0; }")
    src = tmp_path / "layout.c"
    src.write_text("\n".join(lines))
    exe = tmp_path / "layout"
    inc = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include")
    subprocess.run(["gcc", "-I", inc, "-o", str(exe), str(src)], check=True)
    got = dict(line.split() for line in subprocess.run([str(exe)], capture_output=True, text=True, check=True).stdout.splitlines())
    for name, cls in structs.items():
        assert int(got[name]) == ctypes.sizeof(cls), name
        for f, _ in cls._fields_:
            assert int(got[f"{name}.{f}"]) == getattr(cls, f).offset, (name, f)


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
