"""blt_dec_prefill_noalloc: the prefill entry point that allocates nothing.

Its per-call scratch lives in a static device arena, for callers that cannot
allocate device memory once the engine is set up.  Through the C ABI it must
give the same logits and the same engine state as blt_dec_prefill (within the
2e-2 logit tolerance of the other parity tests), on two calls in a row.  Runs
alone in a fresh process or after the other tests.
"""

import numpy as np
import pytest
import torch

from workload import CONFIGS, Patcher, WeightSet, prefix_bytes

pytestmark = pytest.mark.gpu

TOL = 2e-2


def _rows(eng, wl, seq):
    from block_diffusion_byte_b200.driver import SeqHost

    s = SeqHost(Patcher(wl.patch_kind, wl.seed, wl.cfg_index, seq), wl.seed, wl.cfg_index, seq, wl.shape.d_global)
    s.commit([int(b) for b in prefix_bytes(wl.seed, wl.cfg_index, seq, wl.prefix_len)])
    b, sl, l = s.take_pending()
    return eng.rows([b[:-1]], [sl[:-1]], [l]), (b[-1:], sl[-1:])


@pytest.mark.parametrize("name", ["tiny_d4", "d4_b1"])
def test_prefill_noalloc_matches_prefill_twice(name):
    from block_diffusion_byte_b200 import _build
    from block_diffusion_byte_b200 import binding as B
    from block_diffusion_byte_b200.driver import Engine

    _build.build()
    wl = CONFIGS[name]
    ws = WeightSet(wl.shape).materialize()
    n = wl.prefix_len - 1
    eng = Engine(wl.shape, ws, max_batch=1, max_ctx=wl.prefix_len + 32, max_block=8, max_rows=256)
    try:
        (r, keep), (pb, ps) = _rows(eng, wl, 0)
        ref = torch.zeros((n, 256), dtype=torch.float32, device="cuda")
        B.blt_dec_prefill(eng.h, 1, r, ref)
        assert B.blt_dec_sync(eng.h) == 0
        # what the cache then produces: one block of the next call
        rp, keep2 = eng.rows([pb], [ps], [[]])
        blk_ref = torch.zeros((4, 1, 4, 256), dtype=torch.float32, device="cuda")
        B.blt_dec_diffuse_block(eng.h, 1, rp, 4, 0.7, 0, eng.d_out, None, blk_ref)
        ref_block = eng._get(eng.out_view(1, 4)).copy()
        ref_np, blk_ref_np = ref.cpu().numpy(), blk_ref.cpu().numpy()
        for call in range(2):
            B.blt_dec_rewind(eng.h, 1, [0], [0])
            (r, keep), _ = _rows(eng, wl, 0)  # re-stage: the diffuse call reused the staging buffers
            out = torch.full((n, 256), float("nan"), dtype=torch.float32, device="cuda")
            B.blt_dec_prefill_noalloc(eng.h, 1, r, out)
            assert B.blt_dec_sync(eng.h) == 0
            got = out.cpu().numpy()
            assert np.isfinite(got).all()
            assert np.abs(got - ref_np).max() < TOL, (call, np.abs(got - ref_np).max())
            # the cache it wrote serves the next call exactly as the regular prefill's does
            blk = torch.zeros((4, 1, 4, 256), dtype=torch.float32, device="cuda")
            rp, keep2 = eng.rows([pb], [ps], [[]])
            B.blt_dec_diffuse_block(eng.h, 1, rp, 4, 0.7, 0, eng.d_out, None, blk)
            assert np.array_equal(eng._get(eng.out_view(1, 4)), ref_block), call
            steps = 4
            assert np.abs(np.nan_to_num(blk.cpu().numpy()[:steps]) - np.nan_to_num(blk_ref_np[:steps])).max() < TOL
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
