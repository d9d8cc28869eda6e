"""Error paths of the C ABI: host checks and bounded device checks (no GPU fault is provoked)."""

import numpy as np
import pytest
import torch

from workload import CONFIGS, WeightSet, prefix_bytes

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def eng():
    from block_diffusion_byte_b200 import _build
    from block_diffusion_byte_b200.driver import Engine

    _build.build()
    wl = CONFIGS["tiny_d4"]
    e = Engine(wl.shape, WeightSet(wl.shape).materialize(), max_batch=2, max_ctx=160, max_block=8, max_rows=64)
    yield wl, e
    e.close()


def _prefill(wl, e, seq=0):
    from block_diffusion_byte_b200 import binding as B
    from block_diffusion_byte_b200.driver import SeqHost
    from workload import Patcher

    B.blt_dec_rewind(e.h, 2, [0, 0], [0, 0])
    s = SeqHost(Patcher(wl.patch_kind, wl.seed, wl.cfg_index, seq), wl.seed, wl.cfg_index, seq, wl.shape.d_global)
    s.commit([int(b) for b in prefix_bytes(wl.seed, wl.cfg_index, seq, wl.prefix_len)])
    b, sl, l = s.take_pending()
    r, keep = e.rows([b[:-1]], [sl[:-1]], [l])
    B.blt_dec_prefill(e.h, 1, r)
    return s, b[-1:], sl[-1:]


def test_verify_without_draft_is_state_error(eng):
    from block_diffusion_byte_b200 import binding as B

    wl, e = eng
    _prefill(wl, e)
    with pytest.raises(B.BltError) as ei:
        B.blt_dec_verify_accept(e.h, e.d_vslots, None, None, e.d_acc, e.d_next)
    assert ei.value.code == B.BLT_ERR_STATE


def test_bad_arguments(eng):
    from block_diffusion_byte_b200 import binding as B

    wl, e = eng
    s, pb, ps = _prefill(wl, e)
    r, keep = e.rows([pb], [ps], [[]])
    for k in (0, 9, 33):
        with pytest.raises(B.BltError) as ei:
            B.blt_dec_diffuse_block(e.h, 1, r, k, 0.7, 0, e.d_out)
        assert ei.value.code == B.BLT_ERR_INVALID_ARG
    with pytest.raises(B.BltError) as ei:
        B.blt_dec_diffuse_block(e.h, 3, r, 4, 0.7, 0, e.d_out)  # batch > max_batch
    assert ei.value.code == B.BLT_ERR_INVALID_ARG
    with pytest.raises(B.BltError) as ei:
        B.blt_dec_diffuse_block(e.h, 1, r, 4, float("nan"), 0, e.d_out)
    assert ei.value.code == B.BLT_ERR_INVALID_ARG
    r0, keep0 = e.rows([[]], [[]], [[]])
    with pytest.raises(B.BltError) as ei:
        B.blt_dec_draft(e.h, 1, r0, B.BLT_DRAFT_AR, 4, 0.0, 0, e.d_out)  # no pending row: no y_l
    assert ei.value.code == B.BLT_ERR_INVALID_ARG


def test_step_limit_reported_by_device(eng):
    from block_diffusion_byte_b200 import binding as B

    wl, e = eng
    s, pb, ps = _prefill(wl, e)
    r, keep = e.rows([pb], [ps], [[]])
    # alpha > 1 commits one position per pass: 4 positions need 4 passes, 2 are allowed
    B.blt_dec_diffuse_block(e.h, 1, r, 4, 1.5, 2, e.d_out)
    assert B.blt_dec_sync(e.h) == B.BLT_ERR_STEP_LIMIT
    assert B.blt_dec_sync(e.h) == 0  # the status word is cleared


def test_bad_latent_slot_caught_on_device(eng):
    from block_diffusion_byte_b200 import binding as B

    wl, e = eng
    s, pb, ps = _prefill(wl, e)
    r, keep = e.rows([pb], [[10_000]], [[]])  # slot far beyond the sequence's latents
    B.blt_dec_diffuse_block(e.h, 1, r, 4, 0.7, 0, e.d_out)
    assert B.blt_dec_sync(e.h) == B.BLT_ERR_DEVICE


def test_context_capacity_is_no_space(eng):
    from block_diffusion_byte_b200 import binding as B

    wl, e = eng
    s, pb, ps = _prefill(wl, e)
    rows = [pb + [1] * 100]
    r, keep = e.rows(rows, [ps + [0] * 100], [[]])
    with pytest.raises(B.BltError) as ei:
        B.blt_dec_diffuse_block(e.h, 1, r, 4, 0.7, 0, e.d_out)
    assert ei.value.code == B.BLT_ERR_NO_SPACE


def test_persistent_kernel_wait_runs_out():
    """A bounded wait of the persistent pass kernel that runs out ends the call with
    BLT_ERR_DEVICE instead of hanging: under the test-only flag one output of the first
    O projection is never published, so every consumer of it waits about a millisecond and
    gives up, and all CTAs leave.  A fresh handle then decodes normally."""
    import time

    from block_diffusion_byte_b200 import binding as B
    from block_diffusion_byte_b200.driver import Engine, generate

    wl = CONFIGS["tiny_d4"]
    ws = WeightSet(wl.shape).materialize()
    prefix = [int(b) for b in prefix_bytes(wl.seed, wl.cfg_index, 0, wl.prefix_len)]
    e = Engine(wl.shape, ws, max_batch=1, max_ctx=160, max_block=8, max_rows=64, persistent=True, extra_flags=B.BLT_FLAG_TEST_STALL)
    try:
        t0 = time.perf_counter()
        with pytest.raises(B.BltError) as ei:
            generate(e, wl, [prefix], 4)
        assert ei.value.code == B.BLT_ERR_DEVICE
        assert time.perf_counter() - t0 < 30.0
        assert B.blt_dec_stats(e.h)["persistent_calls"] >= 1
    finally:
        e.close()
    f = Engine(wl.shape, ws, max_batch=1, max_ctx=160, max_block=8, max_rows=64, persistent=True)
    try:
        res = generate(f, wl, [prefix], 8)
        assert B.blt_dec_sync(f.h) == 0 and len(res.out[0]) == 8
    finally:
        f.close()
