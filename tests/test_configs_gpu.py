"""Engine parity at the workload configurations' real shapes and batches.

The oracle (fp64, CPU) decodes sampled sequences of each configuration; the
engine decodes the whole batch.  Bytes must agree except at positions the
oracle flags as near-ties.  Full generation lengths are checked where the
oracle finishes in about a minute; otherwise a prefix of the generation.
"""

from dataclasses import replace

import numpy as np
import pytest

from oracle.model import OracleModel
from oracle.policies import OracleSequence
from workload import CONFIGS, SWEEP, WeightSet, prefix_bytes

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dec9():
    from block_diffusion_byte_b200 import _build

    _build.build()
    wl = CONFIGS["d4_b1"]
    ws = WeightSet(wl.shape).materialize()
    return ws, OracleModel(wl.shape, ws)


def _prefix(wl, seq):
    return [int(b) for b in prefix_bytes(wl.seed, wl.cfg_index, seq, wl.prefix_len)]


def _engine_run(wl, ws, G, seqs, **kw):
    from block_diffusion_byte_b200.driver import Engine, generate

    eng = Engine(wl.shape, ws, max_batch=len(seqs), max_ctx=wl.prefix_len + G + 4 * wl.block + 16, max_block=max(16, wl.block),
                 max_rows=kw.pop("max_rows", 1024), **kw)
    try:
        return generate(eng, wl, [_prefix(wl, s) for s in seqs], G, seq_ids=seqs)
    finally:
        eng.close()


def _oracle_run(wl, om, seq, G):
    o = OracleSequence(om, wl, seq, _prefix(wl, seq))
    o.prefill()
    return o.generate(G), o


def _check(got, want, o, wl, what):
    if got == want:
        return
    i = next(j for j in range(min(len(got), len(want))) if got[j] != want[j])
    near = [f for f in o.flags if abs(f.pos - (wl.prefix_len + i)) <= 2 * wl.block + 2]
    assert near, f"{what}: differs at byte {i} without a flagged near-tie"


@pytest.mark.parametrize("persistent", [True, False], ids=["persistent", "phased"])
def test_config2_full_job(dec9, persistent):
    """BLT-D-4, prefix 1024, all 512 bytes: the configuration bench.py times (persistent kernel by default)."""
    from block_diffusion_byte_b200.driver import Engine, generate

    ws, om = dec9
    wl = CONFIGS["d4_b1"]
    eng = Engine(wl.shape, ws, max_batch=1, max_ctx=wl.prefix_len + wl.gen_bytes + 4 * wl.block + 16, max_block=16,
                 max_rows=1024, persistent=persistent)
    try:
        res = generate(eng, wl, [_prefix(wl, 0)], wl.gen_bytes, seq_ids=[0])
        from block_diffusion_byte_b200 import binding as B

        assert (B.blt_dec_stats(eng.h)["persistent_calls"] > 0) == persistent
    finally:
        eng.close()
    want, o = _oracle_run(wl, om, 0, wl.gen_bytes)
    _check(res.out[0], want, o, wl, "config 2")


def test_config3_dv16_batch8(dec9):
    """BLT-DV-16 one-step drafts + verification, prefix 2048, batch 8 (two sequences checked)."""
    ws, om = dec9
    wl = CONFIGS["dv16_b8"]
    G = 48
    res = _engine_run(wl, ws, G, list(range(8)))
    for s in (0, 5):
        want, o = _oracle_run(wl, om, s, G)
        _check(res.out[s], want, o, wl, f"config 3 seq {s}")
    # DV is lossless against greedy AR on the same weights
    ar = _engine_run(replace(wl, mode="AR", block=1), ws, G, list(range(8)))
    assert ar.out == res.out


@pytest.mark.parametrize("persistent", [False, True], ids=["phased", "persistent"])
def test_config4_s8_batch16(dec9, persistent):
    """BLT-S k=8, prefix 4096, batch 16: byte-identical to AR greedy on the engine; oracle on one sequence.
    With the persistent kernel the 16-row drafting passes run in it (two row groups)."""
    ws, om = dec9
    wl = CONFIGS["s8_b16"]
    G = 48
    res = _engine_run(wl, ws, G, list(range(16)), persistent=persistent)
    ar = _engine_run(replace(wl, mode="AR", block=1), ws, G, list(range(16)))
    assert res.out == ar.out
    want, o = _oracle_run(replace(wl, mode="AR", block=1), om, 3, G)
    _check(res.out[3], want, o, wl, "config 4 seq 3")


@pytest.mark.parametrize("name", ["sweep_b4_k8_p512", "sweep_b64_k16_p512", "sweep_b1_k16_p8192"])
def test_config5_sweep_points(name):
    """Sweep points (d_global 4096): sequence 0 against the oracle; batched == solo."""
    from block_diffusion_byte_b200 import _build

    _build.build()
    wl = next(w for w in SWEEP if w.name == name)
    ws = WeightSet(wl.shape).materialize()
    G = 2 * wl.block
    res = _engine_run(wl, ws, G, list(range(wl.batch)), max_rows=2048)
    if wl.batch > 1:
        solo = _engine_run(wl, ws, G, [wl.batch - 1])
        assert solo.out[0] == res.out[wl.batch - 1]
    if wl.prefix_len <= 2048:
        om = OracleModel(wl.shape, ws)
        want, o = _oracle_run(wl, om, 0, G)
        _check(res.out[0], want, o, wl, name)


def test_config2_eb_sampling(dec9):
    """BLT-D-4 with EB sampling (gamma 4.5), prefix 1024, 64 bytes, persistent kernel."""
    from block_diffusion_byte_b200 import binding as B
    from block_diffusion_byte_b200.driver import Engine, generate

    ws, om = dec9
    wl = CONFIGS["d4eb_b1"]
    G = 64
    eng = Engine(wl.shape, ws, max_batch=1, max_ctx=wl.prefix_len + G + 4 * wl.block + 16, max_block=16, max_rows=1024,
                 persistent=True)
    try:
        res = generate(eng, wl, [_prefix(wl, 0)], G, seq_ids=[0])
        assert B.blt_dec_stats(eng.h)["persistent_calls"] > 0
    finally:
        eng.close()
    want, o = _oracle_run(wl, om, 0, G)
    _check(res.out[0], want, o, wl, "config 2, EB")
