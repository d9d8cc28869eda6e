"""Engine parity at the workload configurations' full sizes, strictly.

The fp64 oracle's generation records of these jobs (decoded bytes, the pass
count of every BLT-D block, the accept length of every BLT-S / BLT-DV round,
every near-tie flag) are stored in ``tests/golden/oracle_records`` by
``tests/golden/make_oracle_records.py``, which calls only the oracle: its
longest jobs take minutes on a CPU.  The engine decodes the whole batch of
each configuration; the sequence under test is compared round by round with
the rule of ``_parity.compare_generation`` (identical, or a divergence exactly
at a flagged position followed by a re-sync on the oracle's bytes), and every
flagged position is listed in the session summary.
"""

import json
import os
from dataclasses import replace

import pytest

from workload import CONFIGS, SWEEP, WeightSet, prefix_bytes

from _parity import compare_generation, engine_gen_factory

pytestmark = pytest.mark.gpu

REC = os.path.join(os.path.dirname(__file__), "golden", "oracle_records")


class StoredOracle:
    """Duck-typed stand-in for an oracle run, read from a stored record."""

    def __init__(self, name):
        with open(os.path.join(REC, name + ".json")) as f:
            self.r = json.load(f)


def _stored_compare(name, wl, seq, s_index, engine_gen):
    """compare_generation against a stored oracle record (no oracle work at test time)."""
    import _parity
    from oracle.policies import Flag

    st = StoredOracle(name).r
    assert st["workload"] == wl.name and st["seq"] == seq
    G = st["gen_bytes"]

    class _O:
        flags = [Flag(f["pos"], f["what"], f["value"]) for f in st["flags"]]

    def fake_oracle_run(model, wl_, seq_, prefix, G_):
        # re-syncs restart the engine only; the oracle's trajectory is the stored one
        assert G_ == G
        return st["bytes"], st["rounds"], _O()

    real = _parity.oracle_run
    _parity.oracle_run = fake_oracle_run
    try:
        prefix = [int(b) for b in prefix_bytes(wl.seed, wl.cfg_index, seq, wl.prefix_len)]
        return compare_generation(name, wl, None, seq, prefix, G, engine_gen, s_index=s_index)
    finally:
        _parity.oracle_run = real


@pytest.fixture(scope="module")
def dec9():
    from block_diffusion_byte_b200 import _build

    _build.build()
    wl = CONFIGS["d4_b1"]
    return WeightSet(wl.shape).materialize()


@pytest.fixture(scope="module")
def dec9_g4096():
    wl = SWEEP[0]
    return WeightSet(wl.shape).materialize()


@pytest.mark.parametrize("persistent", [True, False], ids=["persistent", "phased"])
def test_config2_full_job(dec9, persistent):
    """BLT-D-4, prefix 1024, all 512 bytes (the job bench.py times)."""
    wl = CONFIGS["d4_b1"]
    gen = engine_gen_factory(wl.shape, dec9, wl, [0], persistent=persistent)
    _stored_compare("d4_b1_seq0", wl, 0, 0, gen)


def test_config2_eb_full_job(dec9):
    """BLT-D-4 with EB sampling (gamma 4.5), prefix 1024, 512 bytes, persistent kernel."""
    wl = CONFIGS["d4eb_b1"]
    gen = engine_gen_factory(wl.shape, dec9, wl, [0], persistent=True)
    _stored_compare("d4eb_b1_seq0", wl, 0, 0, gen)


@pytest.mark.parametrize("tensor_cores", [False, True], ids=["gemv", "tcgen05"])
def test_config3_dv16_batch8_full(dec9, tensor_cores):
    """BLT-DV-16 one-step drafts + verification, prefix 2048, batch 8, sequence 0 for all
    1024 bytes (accept lengths compared round by round).  Its passes hold 8 x 16 = 128 rows:
    the projections run on the GEMV kernels, or with BLT_FLAG_TENSOR_CORES on the tcgen05 GEMM."""
    wl = CONFIGS["dv16_b8"]
    gen = engine_gen_factory(wl.shape, dec9, wl, list(range(8)), s_index=0, persistent=True, tensor_cores=tensor_cores)
    _stored_compare("dv16_b8_seq0", wl, 0, 0, gen)


@pytest.mark.parametrize("persistent", [True, False], ids=["persistent", "phased"])
def test_config4_s8_batch1_full(dec9, persistent):
    """BLT-S k=8, prefix 4096, batch 1, all 512 bytes."""
    wl = CONFIGS["s8_b1"]
    gen = engine_gen_factory(wl.shape, dec9, wl, [0], persistent=persistent)
    _stored_compare("s8_b1_seq0", wl, 0, 0, gen)


def test_config4_s8_batch16_full(dec9):
    """BLT-S k=8, prefix 4096, batch 16: sequence 3 for all 512 bytes inside the batch, and
    the whole batch byte-identical to greedy AR decoding on the engine.  (For the exact
    identity both jobs run on the GEMV kernels: the verification passes' 128 rows would
    otherwise take the tcgen05 GEMM, whose fp32 sums differ in order from the AR passes'.)"""
    from block_diffusion_byte_b200.driver import Engine, generate

    wl = CONFIGS["s8_b16"]
    gen = engine_gen_factory(wl.shape, dec9, wl, list(range(16)), s_index=3, persistent=True)
    res = _stored_compare("s8_b16_seq3", wl, 3, 3, gen)
    if not res.divergences:  # without a near-tie the whole batch must equal greedy AR
        prefs = [[int(b) for b in prefix_bytes(wl.seed, wl.cfg_index, s, wl.prefix_len)] for s in range(16)]
        outs = {}
        for mode, k in (("S", 8), ("AR", 1)):
            w = replace(wl, mode=mode, block=k)
            eng = Engine(wl.shape, dec9, max_batch=16, max_ctx=wl.prefix_len + 2 * 128 + 64, max_block=16, max_rows=1024, persistent=True,
                         tensor_cores=False)
            try:
                outs[mode] = generate(eng, w, prefs, 128).out
            finally:
                eng.close()
        assert outs["S"] == outs["AR"]


@pytest.mark.parametrize("p", [512, 2048, 8192])
@pytest.mark.parametrize("k", [4, 8, 16])
def test_config5_sweep_against_oracle(dec9_g4096, k, p):
    """Sweep shape (d_global 4096): sequence 0 decoded alone, two blocks, against the oracle."""
    wl = next(w for w in SWEEP if w.prefix_len == p and w.block == k and w.batch == 1)
    gen = engine_gen_factory(wl.shape, dec9_g4096, wl, [0], persistent=True)
    _stored_compare(f"sweep_k{k}_p{p}_seq0", wl, 0, 0, gen)


@pytest.mark.parametrize("b", [4, 16, 64])
def test_config5_sweep_every_batch(dec9_g4096, b):
    """Every sweep point runs on the engine: for this batch size, every block size and prefix,
    two blocks per sequence; sequence 0 inside the batch decodes exactly as alone (the rows of a
    pass do not change one another's arithmetic), which the oracle checks above."""
    from block_diffusion_byte_b200.driver import Engine, generate

    for p in (512, 2048, 8192):
        for k in (4, 8, 16):
            wl = next(w for w in SWEEP if w.prefix_len == p and w.block == k and w.batch == b)
            prefs = [[int(x) for x in prefix_bytes(wl.seed, wl.cfg_index, s, p)] for s in range(b)]
            G = 2 * k
            eng = Engine(wl.shape, dec9_g4096, max_batch=b, max_ctx=p + G + 4 * k + 16, max_block=16, max_rows=2048, persistent=True)
            try:
                res = generate(eng, wl, prefs, G, record=True)
            finally:
                eng.close()
            with open(os.path.join(REC, f"sweep_k{k}_p{p}_seq0.json")) as f:
                st = json.load(f)
            flagged = {f["pos"] for f in st["flags"]}
            if not flagged:
                assert res.out[0] == st["bytes"], (b, k, p)
            assert all(len(o) == G for o in res.out)
