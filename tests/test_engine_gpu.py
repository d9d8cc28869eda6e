"""Parity of the CUDA engine (through the C ABI) with the fp64 oracle.

Tolerances (stated by the workload definition): logits max-abs 2e-2; decoded
bytes, pass counts and accept lengths identical, except for a divergence exactly
at a position the oracle flags as a near-tie (top-2 logit gap < 0.05,
|conf - alpha| < 0.03, a fallback choice between confidences within 0.03, or an
EB cut within 0.05 nats), after which the comparison re-syncs on the oracle's
bytes and goes on (``_parity.compare_generation``).
"""

from dataclasses import replace

import numpy as np
import pytest
import torch

from oracle.model import BLOCK, CAUSAL, OracleModel, Row, decoder_pass
from oracle.policies import OracleSequence
from workload import CONFIGS, WeightSet, prefix_bytes

from _parity import compare_generation, engine_gen_factory

pytestmark = pytest.mark.gpu

LOGIT_TOL = 2e-2


@pytest.fixture(scope="module")
def tiny_setup():
    from block_diffusion_byte_b200 import _build

    _build.build()
    wl = CONFIGS["tiny_d4"]
    ws = WeightSet(wl.shape, gain_std=0.1).materialize()
    return wl, ws, OracleModel(wl.shape, ws)


def _engine(wl, ws, batch=1, G=64, max_block=16, max_rows=256):
    from block_diffusion_byte_b200.driver import Engine

    return Engine(wl.shape, ws, max_batch=batch, max_ctx=wl.prefix_len + G + 2 * max_block + 8, max_block=max_block, max_rows=max_rows)


def _prefix(wl, seq):
    return [int(b) for b in prefix_bytes(wl.seed, wl.cfg_index, seq, wl.prefix_len)]


def test_prefill_and_first_block_logits(tiny_setup):
    from block_diffusion_byte_b200 import binding as B

    wl, ws, om = tiny_setup
    pre = _prefix(wl, 0)
    eng = _engine(wl, ws)
    try:
        # engine: prefill every byte but the last with logits, then one block with logits
        from block_diffusion_byte_b200.driver import SeqHost
        from workload import Patcher

        s = SeqHost(Patcher(wl.patch_kind, wl.seed, wl.cfg_index, 0), wl.seed, wl.cfg_index, 0, wl.shape.d_global)
        s.commit(pre)
        b, sl, l = s.take_pending()
        r, keep = eng.rows([b[:-1]], [sl[:-1]], [l])
        pl = torch.zeros((len(pre) - 1, 256), dtype=torch.float32, device="cuda")
        torch.cuda.synchronize()  # filled before the engine's stream writes it
        B.blt_dec_prefill(eng.h, 1, r, pl)
        k = wl.block
        r, keep = eng.rows([b[-1:]], [sl[-1:]], [[]])
        logits = torch.zeros((k, 1, k, 256), dtype=torch.float32, device="cuda")
        torch.cuda.synchronize()  # filled before the engine's stream writes it
        B.blt_dec_diffuse_block(eng.h, 1, r, k, wl.alpha, 0, eng.d_out, eng.d_steps, logits)
        assert B.blt_dec_sync(eng.h) == 0
        gl = pl.cpu().numpy()
        gb = logits.cpu().numpy()[0, 0]
    finally:
        eng.close()
    o = OracleSequence(om, wl, 0, pre)
    rows = [Row(o.bytes[p], p, o.lat[p], CAUSAL) for p in range(len(pre) - 1)]
    zp = decoder_pass(om, o.st, rows)
    o.cached = len(pre) - 1
    N = len(pre)
    zb = decoder_pass(om, o.st, o._pending() + [Row(256, N + i, o.n_closed - 1, BLOCK, N + k) for i in range(k)])[1:]
    assert np.abs(gl - zp).max() < LOGIT_TOL, np.abs(gl - zp).max()
    assert np.abs(gb - zb).max() < LOGIT_TOL, np.abs(gb - zb).max()


@pytest.mark.parametrize("persistent", [False, True], ids=["phased", "persistent"])
@pytest.mark.parametrize("mode,k,alpha", [("D", 4, 0.7), ("D", 8, 0.0), ("AR", 1, 0.0), ("S", 8, 0.0), ("DV", 8, 0.0), ("DV", 4, 0.7)])
def test_tiny_generation_matches_oracle(tiny_setup, mode, k, alpha, persistent):
    wl, ws, om = tiny_setup
    w = replace(wl, mode=mode, block=k, alpha=alpha)
    gen = engine_gen_factory(w.shape, ws, w, [0], persistent=persistent, max_rows=256)
    compare_generation(f"tiny {mode}-{k} alpha {alpha} {'persistent' if persistent else 'phased'}", w, om, 0, _prefix(wl, 0), 32, gen)


def test_blt_s_equals_ar_on_engine(tiny_setup):
    from block_diffusion_byte_b200.driver import generate

    wl, ws, om = tiny_setup
    outs = {}
    for mode, k in (("AR", 1), ("S", 5), ("S", 8), ("DV", 6)):
        w = replace(wl, mode=mode, block=k, alpha=0.0)
        eng = _engine(w, ws, batch=3)
        try:
            outs[(mode, k)] = generate(eng, w, [_prefix(wl, s) for s in range(3)], 40).out
        finally:
            eng.close()
    for key, v in outs.items():
        assert v == outs[("AR", 1)], key


def test_batch_invariance(tiny_setup):
    """A sequence decodes to the same bytes alone and inside a batch."""
    from block_diffusion_byte_b200.driver import generate

    wl, ws, om = tiny_setup
    pres = [_prefix(wl, s) for s in range(4)]
    eng = _engine(wl, ws, batch=4)
    try:
        batched = generate(eng, wl, pres, 24).out
    finally:
        eng.close()
    for s in range(4):
        eng = _engine(wl, ws, batch=1)
        try:
            solo = generate(eng, wl, [pres[s]], 24, seq_ids=[s]).out[0]
        finally:
            eng.close()
        assert solo == batched[s]


@pytest.fixture(scope="module")
def d4_setup():
    from block_diffusion_byte_b200 import _build

    _build.build()
    wl = CONFIGS["d4_b1"]
    ws = WeightSet(wl.shape).materialize()
    return wl, ws, OracleModel(wl.shape, ws)


def _call_logits(wl, ws, persistent, mode, k, alpha, G=24, batch=2, **wkw):
    """Logits of every engine call of a short generation (diffuse / draft / verify), via out_logits."""
    import ctypes

    from block_diffusion_byte_b200 import binding as B
    from block_diffusion_byte_b200.driver import Engine, generate

    eng = Engine(wl.shape, ws, max_batch=batch, max_ctx=wl.prefix_len + G + 64, max_block=16, max_rows=256, persistent=persistent)
    try:
        w = replace(wl, mode=mode, block=k, alpha=alpha, **wkw)
        res = generate(eng, w, [_prefix(wl, s) for s in range(batch)], G, record=True)
        st = B.blt_dec_stats(eng.h)
    finally:
        eng.close()
    return res, st


@pytest.mark.parametrize("mode,k,alpha,batch", [("D", 4, 0.7, 2), ("D", 8, 0.5, 1), ("AR", 1, 0.0, 2), ("S", 6, 0.0, 2), ("DV", 4, 0.0, 2)])
def test_persistent_kernel_matches_per_phase_bitwise(tiny_setup, mode, k, alpha, batch):
    """The persistent pass kernel and the per-phase kernels share every arithmetic step
    (every pass of these calls has at most 16 rows, so the persistent kernel runs them)."""
    wl, ws, om = tiny_setup
    a, sa = _call_logits(wl, ws, True, mode, k, alpha, batch=batch)
    b, sb = _call_logits(wl, ws, False, mode, k, alpha, batch=batch)
    assert a.out == b.out
    assert sa["passes"] == sb["passes"]
    assert sa["kernel_launches"] < sb["kernel_launches"]  # the persistent path ran
    for ra, rb in zip(a.rounds, b.rounds):
        for key in ra:
            assert np.array_equal(ra[key], rb[key]), key


def _block_logits(wl, ws, persistent, k=4, alpha=0.7):
    from block_diffusion_byte_b200 import binding as B
    from block_diffusion_byte_b200.driver import Engine, SeqHost
    from workload import Patcher

    pre = _prefix(wl, 0)
    eng = Engine(wl.shape, ws, max_batch=1, max_ctx=wl.prefix_len + 64, max_block=16, max_rows=1024, persistent=persistent)
    try:
        s = SeqHost(Patcher(wl.patch_kind, wl.seed, wl.cfg_index, 0), wl.seed, wl.cfg_index, 0, wl.shape.d_global)
        s.commit(pre)
        b, sl, l = s.take_pending()
        r, keep = eng.rows([b[:-1]], [sl[:-1]], [l])
        B.blt_dec_prefill(eng.h, 1, r)
        r, keep = eng.rows([b[-1:]], [sl[-1:]], [[]])
        logits = torch.full((k, 1, k, 256), float("nan"), dtype=torch.float32, device="cuda")
        torch.cuda.synchronize()  # filled before the engine's stream writes it
        B.blt_dec_diffuse_block(eng.h, 1, r, k, alpha, 0, eng.d_out, eng.d_steps, logits)
        assert B.blt_dec_sync(eng.h) == 0
        return logits.cpu().numpy(), eng._get(eng.d_steps[:1])[0]
    finally:
        eng.close()


@pytest.mark.parametrize("which", ["tiny", "d4"])
def test_persistent_block_logits_bitwise(tiny_setup, d4_setup, which):
    wl, ws, om = tiny_setup if which == "tiny" else d4_setup
    a, sa = _block_logits(wl, ws, True)
    b, sb = _block_logits(wl, ws, False)
    assert sa == sb
    n = int(sa)
    assert np.array_equal(a[:n], b[:n])


# ------------------------------------------------------------------ entropy-bounded (EB) sampling
@pytest.mark.parametrize("k,gamma", [(4, 4.0), (8, 6.0), (6, 0.0)])
def test_tiny_eb_generation_matches_oracle(tiny_setup, k, gamma):
    """BLT-D with EB sampling (blt_dec_diffuse_block_eb) against the oracle's EB rule,
    block by block (bytes and pass counts)."""
    wl, ws, om = tiny_setup
    w = replace(wl, mode="D", block=k, alpha=0.0, unmask="entropy", gamma=gamma)
    gen = engine_gen_factory(w.shape, ws, w, [0], persistent=False, max_rows=256)
    compare_generation(f"tiny EB-{k} gamma {gamma}", w, om, 0, _prefix(wl, 0), 32, gen)


@pytest.mark.parametrize("k,gamma,batch", [(4, 4.0, 2), (8, 6.0, 1)])
def test_persistent_eb_matches_per_phase_bitwise(tiny_setup, k, gamma, batch):
    """EB sampling runs in the persistent kernel's bookkeeping and in the per-phase
    unmask kernel with the same arithmetic: bytes, pass counts and logits agree bitwise."""
    wl, ws, om = tiny_setup
    a, sa = _call_logits(wl, ws, True, "D", k, 0.0, batch=batch, unmask="entropy", gamma=gamma)
    b, sb = _call_logits(wl, ws, False, "D", k, 0.0, batch=batch, unmask="entropy", gamma=gamma)
    assert a.out == b.out
    assert sa["passes"] == sb["passes"]
    assert sa["persistent_calls"] > 0 and sb["persistent_calls"] == 0
    for ra, rb in zip(a.rounds, b.rounds):
        for key in ra:
            assert np.array_equal(ra[key], rb[key]), key


def test_eb_rejects_bad_gamma(tiny_setup):
    from block_diffusion_byte_b200 import binding as B

    wl, ws, om = tiny_setup
    eng = _engine(wl, ws)
    try:
        r, keep = eng.rows([[1, 2, 3]], [[0, 0, 0]], [[]])
        for bad in (float("nan"), -1.0, float("inf")):
            with pytest.raises(B.BltError):
                B.blt_dec_diffuse_block_eb(eng.h, 1, r, 4, bad, 0, eng.d_out)
    finally:
        eng.close()


def test_upload_download_round_trip(tiny_setup):
    """blt_dec_upload / blt_dec_download: bytes survive a round trip through device
    memory at small, bounce-ring and large sizes; the source may be reused at once;
    n = 0 copies nothing; NULL pointers are INVALID_ARG."""
    from block_diffusion_byte_b200 import binding as B

    wl, ws, _ = tiny_setup
    eng = _engine(wl, ws)
    try:
        dev = torch.empty(3 << 20, dtype=torch.uint8, device="cuda")
        rng = np.random.default_rng(5)
        for n in (1, 4096, 300_000, 3 << 20):
            src = rng.integers(0, 256, n, dtype=np.uint8)
            want = src.copy()
            B.blt_dec_upload(eng.h, dev.data_ptr(), src.ctypes.data, n)
            src[:] = 0  # reused at once: the upload took its bytes before returning
            got = np.empty(n, dtype=np.uint8)
            B.blt_dec_download(eng.h, got.ctypes.data, dev.data_ptr(), n)
            assert np.array_equal(got, want), n
        B.blt_dec_upload(eng.h, dev.data_ptr(), 0, 0)
        B.blt_dec_download(eng.h, 0, dev.data_ptr(), 0)
        with pytest.raises(B.BltError):
            B.blt_dec_upload(eng.h, None, src.ctypes.data, 16)
        with pytest.raises(B.BltError):
            B.blt_dec_download(eng.h, 0, dev.data_ptr(), 16)
    finally:
        eng.close()
