"""blt_dec_prefill_noalloc: the prefill entry point that allocates nothing.

Some callers cannot allocate device memory once the engine is set up (a server
whose device-memory budget is spent, or that sized the handle's scratch small;
a host thread that must not allocate after start-up).  For them the per-call
scratch of this entry point lives in a static device arena of fixed size.
Through the C ABI it must give the same logits and the same engine state as
blt_dec_prefill on a handle without BLT_FLAG_TENSOR_CORES, bit for bit (a row's
arithmetic does not depend on which rows share its pass, so chunking the rows
differently changes no bit; the flag would send blt_dec_prefill's chunks of 128
rows and more to the tcgen05 GEMM, which agrees to rounding only), on two calls
in a row; it must also serve a handle whose own scratch holds a single row, and
leave the device's free memory unchanged.  This file runs alone in a fresh
process or after the other tests.
"""

from dataclasses import replace

import numpy as np
import pytest
import torch

from workload import CONFIGS, Patcher, WeightSet, prefix_bytes

pytestmark = pytest.mark.gpu


def _rows(eng, wl, seq):
    from block_diffusion_byte_b200.driver import SeqHost

    s = SeqHost(Patcher(wl.patch_kind, wl.seed, wl.cfg_index, seq), wl.seed, wl.cfg_index, seq, wl.shape.d_global)
    s.commit([int(b) for b in prefix_bytes(wl.seed, wl.cfg_index, seq, wl.prefix_len)])
    b, sl, l = s.take_pending()
    return eng.rows([b[:-1]], [sl[:-1]], [l]), (b[-1:], sl[-1:])


def _block(eng, pb, ps, k=4):
    """One BLT-D block from the cache the prefill left: its bytes and every pass's logits."""
    from block_diffusion_byte_b200 import binding as B

    rp, keep = eng.rows([pb], [ps], [[]])
    logits = torch.full((k, 1, k, 256), float("nan"), dtype=torch.float32, device="cuda")
    torch.cuda.synchronize()  # filled before the engine's stream writes it
    B.blt_dec_diffuse_block(eng.h, 1, rp, k, 0.7, 0, eng.d_out, eng.d_steps, logits)
    assert B.blt_dec_sync(eng.h) == 0
    steps = int(eng._get(eng.d_steps[:1])[0])
    return eng._get(eng.out_view(1, k)).copy(), steps, logits.cpu().numpy()[:steps]


@pytest.mark.parametrize("name,max_rows", [("tiny_d4", 256), ("tiny_d4", 1), ("d4_b1", 256), ("d4_b1", 8)])
def test_prefill_noalloc_matches_prefill_twice(name, max_rows):
    """max_rows 1 and 8: the handle's own scratch is far smaller than the arena's 32-row chunks
    and than the prefix (a block of 4 after a pending row needs 5 rows, so the one-row handle
    checks the logits only)."""
    from block_diffusion_byte_b200 import _build
    from block_diffusion_byte_b200 import binding as B
    from block_diffusion_byte_b200.driver import Engine

    _build.build()
    wl = CONFIGS[name]
    ws = WeightSet(wl.shape).materialize()
    n = wl.prefix_len - 1
    # the reference: the regular prefill on a handle with room for 256 rows per pass
    eng = Engine(wl.shape, ws, max_batch=1, max_ctx=wl.prefix_len + 32, max_block=8, max_rows=256, tensor_cores=False)
    try:
        (r, keep), (pb, ps) = _rows(eng, wl, 0)
        ref = torch.zeros((n, 256), dtype=torch.float32, device="cuda")
        torch.cuda.synchronize()
        B.blt_dec_prefill(eng.h, 1, r, ref)
        assert B.blt_dec_sync(eng.h) == 0
        ref_np = ref.cpu().numpy()
        ref_block, ref_steps, ref_blk_logits = _block(eng, pb, ps)
    finally:
        eng.close()
    # the entry point under test, on a handle whose own scratch holds max_rows rows
    eng = Engine(wl.shape, ws, max_batch=1, max_ctx=wl.prefix_len + 32, max_block=8, max_rows=max_rows, tensor_cores=False)
    try:
        for call in range(2):
            B.blt_dec_rewind(eng.h, 1, [0], [0])
            (r, keep), _ = _rows(eng, wl, 0)  # staged before the call: the call itself must allocate nothing
            out = torch.full((n, 256), float("nan"), dtype=torch.float32, device="cuda")
            torch.cuda.synchronize()
            free0 = torch.cuda.mem_get_info()[0]
            B.blt_dec_prefill_noalloc(eng.h, 1, r, out)
            assert B.blt_dec_sync(eng.h) == 0
            free1 = torch.cuda.mem_get_info()[0]
            if call == 1:
                assert free1 == free0, (free0, free1)
            got = out.cpu().numpy()
            assert np.array_equal(got, ref_np), (call, np.abs(got - ref_np).max())
            # the cache it wrote serves the next call exactly as the regular prefill's does
            if max_rows < 5:
                continue
            blk, steps, blk_logits = _block(eng, pb, ps)
            assert np.array_equal(blk, ref_block) and steps == ref_steps, call
            assert np.array_equal(blk_logits, ref_blk_logits), call
    finally:
        eng.close()


def test_prefill_noalloc_rejects_oversized_sequences():
    from block_diffusion_byte_b200 import _build
    from block_diffusion_byte_b200 import binding as B
    from block_diffusion_byte_b200.driver import Engine

    _build.build()
    wl = CONFIGS["tiny_d4"]
    eng = Engine(wl.shape, WeightSet(wl.shape).materialize(), max_batch=1, max_ctx=8192, max_block=8, max_rows=64)
    try:
        rows = [[1] * 4097]
        r, keep = eng.rows(rows, [[0] * 4097], [[np.zeros(wl.shape.d_global, np.float32)]])
        with pytest.raises(B.BltError) as ei:
            B.blt_dec_prefill_noalloc(eng.h, 1, r)
        assert ei.value.code == B.BLT_ERR_INVALID_ARG
    finally:
        eng.close()


class _ZeroWeights:
    """Zero weights of any shape (the rejection below happens before any pass runs)."""

    def __init__(self, shape):
        from workload.gen import tensor_shape

        self.shape = shape
        self._t = tensor_shape
        self._c = {}

    def get(self, name, layer=-1):
        if name not in self._c:
            self._c[name] = np.zeros(self._t(self.shape, name), np.float32)
        return self._c[name]

    def layer(self, l):
        from workload import LAYER_TENSORS

        return {n: self.get(n, l) for n in LAYER_TENSORS}


def test_prefill_noalloc_rejects_too_many_layers():
    """n_layers * d_model above 32768 would overflow the arena's latent-projection
    temporary: the call refuses before any work."""
    from block_diffusion_byte_b200 import _build
    from block_diffusion_byte_b200 import binding as B
    from block_diffusion_byte_b200.driver import Engine

    _build.build()
    wl = CONFIGS["tiny_d4"]
    shape = replace(wl.shape, n_layers=32768 // wl.shape.d_model + 1, weight_dtype="bf16")
    eng = Engine(shape, _ZeroWeights(shape), max_batch=1, max_ctx=128, max_block=8, max_rows=16)
    try:
        r, keep = eng.rows([[1, 2, 3]], [[0, 0, 0]], [[np.zeros(shape.d_global, np.float32)]])
        with pytest.raises(B.BltError) as ei:
            B.blt_dec_prefill_noalloc(eng.h, 1, r)
        assert ei.value.code == B.BLT_ERR_INVALID_ARG
        assert "n_layers" in B.blt_dec_last_error(eng.h)
    finally:
        eng.close()
