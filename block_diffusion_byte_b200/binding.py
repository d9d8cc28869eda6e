"""ctypes binding of the bltdec C ABI (include/bltdec.h): argument marshalling only.

Every function keeps the C name and signature; device pointers are passed as
torch CUDA tensors (or raw integers), host arrays as sequences of ints.  No
decoder arithmetic happens here.  The library must exist: there is no
fallback, and loading fails loudly when it is missing.
"""

from __future__ import annotations

import ctypes as C
import os
from typing import Optional, Sequence

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libbltdec.so")

BLT_OK = 0
BLT_ERR_INVALID_ARG = -1
BLT_ERR_NO_SPACE = -2
BLT_ERR_STATE = -3
BLT_ERR_CUDA = -4
BLT_ERR_STEP_LIMIT = -5
BLT_ERR_DEVICE = -6
BLT_W_F32 = 0
BLT_W_BF16 = 1
BLT_DRAFT_AR = 0
BLT_DRAFT_DIFFUSION = 1
BLT_FLAG_TIME_PASSES = 1
BLT_FLAG_PERSISTENT = 2
BLT_FLAG_TEST_STALL = 4  # test only: the persistent kernel's bounded waits must run out
BLT_FLAG_TENSOR_CORES = 8  # passes of >= 128 rows: projections on the tcgen05 GEMM
BLT_UNMASK_CONFIDENCE = 0
BLT_UNMASK_EB = 1
BLT_LAYER_NT = 12
LAYER_ORDER = ("wq_c", "wk_c", "wv_c", "wo_c", "norm_c", "attn_norm", "wqkv", "wo", "ffn_norm", "w1", "w3", "w2")

EXPORTS = (
    "blt_dec_init",
    "blt_dec_prefill",
    "blt_dec_prefill_noalloc",
    "blt_dec_diffuse_block",
    "blt_dec_diffuse_block_eb",
    "blt_dec_draft",
    "blt_dec_verify_accept",
    "blt_dec_diffuse_block_sampled",
    "blt_dec_draft_sampled",
    "blt_dec_verify_sampled",
    "blt_dec_rewind",
    "blt_dec_stats",
    "blt_dec_upload",
    "blt_dec_download",
    "blt_dec_sync",
    "blt_dec_last_error",
    "blt_dec_free",
)


class blt_dec_config(C.Structure):
    _fields_ = [
        ("n_layers", C.c_int32),
        ("d_model", C.c_int32),
        ("n_heads", C.c_int32),
        ("d_ffn", C.c_int32),
        ("d_global", C.c_int32),
        ("vocab", C.c_int32),
        ("weight_dtype", C.c_int32),
        ("rope_theta", C.c_float),
        ("norm_eps", C.c_float),
        ("max_batch", C.c_int32),
        ("max_ctx", C.c_int32),
        ("max_latents", C.c_int32),
        ("max_rows", C.c_int32),
        ("max_block", C.c_int32),
        ("page_tokens", C.c_int32),
        ("kv_pages", C.c_int32),
        ("attn_chunk", C.c_int32),
        ("flags", C.c_int32),
    ]


class blt_dec_weights(C.Structure):
    _fields_ = [
        ("embed", C.c_void_p),
        ("head", C.c_void_p),
        ("final_norm", C.c_void_p),
        ("layer", C.POINTER(C.c_void_p)),
    ]


class blt_rows_in(C.Structure):
    _fields_ = [
        ("bytes", C.c_void_p),
        ("row_latent", C.c_void_p),
        ("row_offsets", C.POINTER(C.c_int32)),
        ("new_latents", C.c_void_p),
        ("latent_offsets", C.POINTER(C.c_int32)),
    ]


class blt_sampling(C.Structure):
    _fields_ = [("temperature", C.c_float), ("top_p", C.c_float), ("uniforms", C.c_void_p)]


class blt_dec_counters(C.Structure):
    _fields_ = [
        ("passes", C.c_uint64),
        ("rows", C.c_uint64),
        ("prefill_rows", C.c_uint64),
        ("latents", C.c_uint64),
        ("calls", C.c_uint64),
        ("weight_bytes", C.c_uint64),
        ("kv_read_bytes", C.c_uint64),
        ("kernel_launches", C.c_uint64),
        ("timed_passes", C.c_uint64),
        ("pass_ns", C.c_uint64),
        ("persistent_calls", C.c_uint64),
        ("prefill_kv_read_bytes", C.c_uint64),
        ("tc_gemms", C.c_uint64),
    ]

    def as_dict(self):
        return {k: int(getattr(self, k)) for k, _ in self._fields_}


_lib = None


def load_library(path: str = LIB_PATH) -> C.CDLL:
    """Load libbltdec.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise ImportError(f"bltdec engine library not built: {path} (run block_diffusion_byte_b200._build.build())")
    lib = C.CDLL(path)
    P, I, F, V = C.c_void_p, C.c_int, C.c_float, None
    lib.blt_dec_init.argtypes = [C.POINTER(blt_dec_config), C.POINTER(blt_dec_weights), P, C.POINTER(P)]
    lib.blt_dec_prefill.argtypes = [P, I, C.POINTER(blt_rows_in), P]
    lib.blt_dec_prefill_noalloc.argtypes = [P, I, C.POINTER(blt_rows_in), P]
    lib.blt_dec_diffuse_block.argtypes = [P, I, C.POINTER(blt_rows_in), I, F, I, P, P, P]
    lib.blt_dec_diffuse_block_eb.argtypes = [P, I, C.POINTER(blt_rows_in), I, F, I, P, P, P]
    lib.blt_dec_draft.argtypes = [P, I, C.POINTER(blt_rows_in), I, I, F, I, P, P]
    lib.blt_dec_verify_accept.argtypes = [P, P, P, C.POINTER(C.c_int32), P, P, P]
    SP = C.POINTER(blt_sampling)
    lib.blt_dec_diffuse_block_sampled.argtypes = [P, I, C.POINTER(blt_rows_in), I, F, I, I, SP, P, P, P]
    lib.blt_dec_draft_sampled.argtypes = [P, I, C.POINTER(blt_rows_in), I, I, F, I, SP, P, P]
    lib.blt_dec_verify_sampled.argtypes = [P, P, P, C.POINTER(C.c_int32), SP, P, P, P]
    lib.blt_dec_rewind.argtypes = [P, I, C.POINTER(C.c_int32), C.POINTER(C.c_int32)]
    lib.blt_dec_stats.argtypes = [P, C.POINTER(blt_dec_counters)]
    lib.blt_dec_upload.argtypes = [P, P, P, C.c_size_t]
    lib.blt_dec_download.argtypes = [P, P, P, C.c_size_t]
    lib.blt_dec_sync.argtypes = [P]
    lib.blt_dec_last_error.argtypes = [P]
    lib.blt_dec_last_error.restype = C.c_char_p
    lib.blt_dec_free.argtypes = [P]
    lib.blt_dec_free.restype = V
    for name in EXPORTS:
        if name not in ("blt_dec_last_error", "blt_dec_free"):
            getattr(lib, name).restype = C.c_int
    _lib = lib
    return lib


class BltError(RuntimeError):
    def __init__(self, code: int, where: str, msg: str):
        super().__init__(f"{where} -> {code}: {msg}")
        self.code = code


def _ptr(t) -> Optional[int]:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _i32(seq: Optional[Sequence[int]]):
    if seq is None:
        return None
    arr = (C.c_int32 * len(seq))(*[int(v) for v in seq])
    return arr


def _check(h, rc: int, where: str) -> None:
    if rc != BLT_OK:
        msg = load_library().blt_dec_last_error(h).decode() if h else ""
        raise BltError(rc, where, msg)


def rows_in(bytes_dev=None, row_latent_dev=None, row_offsets=None, new_latents_dev=None, latent_offsets=None):
    """Build a blt_rows_in; returns (struct, keepalive)."""
    ro = _i32(row_offsets)
    lo = _i32(latent_offsets)
    r = blt_rows_in(_ptr(bytes_dev), _ptr(row_latent_dev), ro, _ptr(new_latents_dev), lo)
    return r, (ro, lo, bytes_dev, row_latent_dev, new_latents_dev)


# ----------------------------------------------------------------------------- thin wrappers, C names
def blt_dec_init(cfg: blt_dec_config, embed, head, final_norm, layers, stream: Optional[int] = None) -> int:
    """``embed``, ``head``, ``final_norm``: float32 C-contiguous numpy arrays;
    ``layers``: per layer a list of BLT_LAYER_NT arrays (or None for unused ones)."""
    lib = load_library()
    keep = [embed, head, final_norm]
    ptrs = (C.c_void_p * (len(layers) * BLT_LAYER_NT))()
    for l, tensors in enumerate(layers):
        for t, arr in enumerate(tensors):
            if arr is not None:
                keep.append(arr)
                ptrs[l * BLT_LAYER_NT + t] = arr.ctypes.data
    w = blt_dec_weights(embed.ctypes.data, head.ctypes.data, final_norm.ctypes.data, ptrs)
    out = C.c_void_p()
    rc = lib.blt_dec_init(C.byref(cfg), C.byref(w), stream, C.byref(out))
    if rc != BLT_OK:
        raise BltError(rc, "blt_dec_init", "see stderr")
    return out.value


def blt_dec_prefill(h: int, batch: int, rows: blt_rows_in, out_logits=None) -> None:
    _check(h, load_library().blt_dec_prefill(h, batch, C.byref(rows), _ptr(out_logits)), "blt_dec_prefill")


def blt_dec_prefill_noalloc(h: int, batch: int, rows: blt_rows_in, out_logits=None) -> None:
    _check(h, load_library().blt_dec_prefill_noalloc(h, batch, C.byref(rows), _ptr(out_logits)), "blt_dec_prefill_noalloc")


def blt_dec_diffuse_block(h, batch, pending, k, alpha, max_steps, out_block, out_steps=None, out_logits=None) -> None:
    rc = load_library().blt_dec_diffuse_block(
        h, batch, C.byref(pending), k, float(alpha), max_steps, _ptr(out_block), _ptr(out_steps), _ptr(out_logits)
    )
    _check(h, rc, "blt_dec_diffuse_block")


def blt_dec_diffuse_block_eb(h, batch, pending, k, gamma, max_steps, out_block, out_steps=None, out_logits=None) -> None:
    rc = load_library().blt_dec_diffuse_block_eb(
        h, batch, C.byref(pending), k, float(gamma), max_steps, _ptr(out_block), _ptr(out_steps), _ptr(out_logits)
    )
    _check(h, rc, "blt_dec_diffuse_block_eb")


def blt_dec_draft(h, batch, pending, mode, k, alpha, max_steps, out_draft, out_logits=None) -> None:
    rc = load_library().blt_dec_draft(h, batch, C.byref(pending), mode, k, float(alpha), max_steps, _ptr(out_draft), _ptr(out_logits))
    _check(h, rc, "blt_dec_draft")


def blt_dec_verify_accept(h, draft_row_latent, new_latents, latent_offsets, out_accepted, out_next, out_logits=None) -> None:
    lo = _i32(latent_offsets)
    rc = load_library().blt_dec_verify_accept(
        h, _ptr(draft_row_latent), _ptr(new_latents), lo, _ptr(out_accepted), _ptr(out_next), _ptr(out_logits)
    )
    _check(h, rc, "blt_dec_verify_accept")


def sampling(temperature: float, top_p: float, uniforms_dev) -> blt_sampling:
    """Sampling parameters; uniforms_dev: device float32 [batch][2 k + 1] in [0, 1)."""
    return blt_sampling(float(temperature), float(top_p), _ptr(uniforms_dev))


def blt_dec_diffuse_block_sampled(h, batch, pending, k, threshold, unmask, max_steps, samp, out_block, out_steps=None,
                                  out_logits=None) -> None:
    rc = load_library().blt_dec_diffuse_block_sampled(h, batch, C.byref(pending), k, float(threshold), unmask, max_steps,
                                                      C.byref(samp), _ptr(out_block), _ptr(out_steps), _ptr(out_logits))
    _check(h, rc, "blt_dec_diffuse_block_sampled")


def blt_dec_draft_sampled(h, batch, pending, mode, k, alpha, max_steps, samp, out_draft, out_logits=None) -> None:
    rc = load_library().blt_dec_draft_sampled(h, batch, C.byref(pending), mode, k, float(alpha), max_steps, C.byref(samp),
                                              _ptr(out_draft), _ptr(out_logits))
    _check(h, rc, "blt_dec_draft_sampled")


def blt_dec_verify_sampled(h, draft_row_latent, new_latents, latent_offsets, samp, out_accepted, out_next, out_logits=None) -> None:
    lo = _i32(latent_offsets)
    rc = load_library().blt_dec_verify_sampled(h, _ptr(draft_row_latent), _ptr(new_latents), lo, C.byref(samp),
                                               _ptr(out_accepted), _ptr(out_next), _ptr(out_logits))
    _check(h, rc, "blt_dec_verify_sampled")


def blt_dec_rewind(h, batch, kv_len=None, n_latents=None) -> None:
    _check(h, load_library().blt_dec_rewind(h, batch, _i32(kv_len), _i32(n_latents)), "blt_dec_rewind")


def blt_dec_stats(h) -> dict:
    c = blt_dec_counters()
    _check(h, load_library().blt_dec_stats(h, C.byref(c)), "blt_dec_stats")
    return c.as_dict()


def blt_dec_upload(h, dst_device, src_host: int, n: int) -> None:
    """Host -> device copy of n bytes on the handle's stream (src_host: an address; reusable at once)."""
    _check(h, load_library().blt_dec_upload(h, _ptr(dst_device), src_host, n), "blt_dec_upload")


def blt_dec_download(h, dst_host: int, src_device, n: int) -> None:
    """Device -> host copy of n bytes after the handle's queued work (dst_host: an address)."""
    _check(h, load_library().blt_dec_download(h, dst_host, _ptr(src_device), n), "blt_dec_download")


def blt_dec_sync(h) -> int:
    """Returns the device status (0, BLT_ERR_STEP_LIMIT or BLT_ERR_DEVICE)."""
    rc = load_library().blt_dec_sync(h)
    if rc == BLT_ERR_CUDA:
        _check(h, rc, "blt_dec_sync")
    return rc


def blt_dec_last_error(h) -> str:
    return load_library().blt_dec_last_error(h).decode()


def blt_dec_free(h) -> None:
    if h:
        load_library().blt_dec_free(h)
