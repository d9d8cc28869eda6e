"""The tcgen05 projection GEMM (BLT_FLAG_TENSOR_CORES) against the fp64 oracle and the GEMV path.

The sweep's largest corner: batch 64 x block 16 (1024 rows per pass, past the
128 rows from which the projections run on the tensor cores), prefix 512, one
BLT-D-16 block (alpha 0.7) for the whole batch.

* The oracle decodes sequence 0 alone (the rows of a pass do not touch one
  another), pass by pass.  The engine's logits of sequence 0's block rows must
  match at max-abs 2e-2 in every pass both take, and the block's bytes and pass
  count must be equal unless the oracle flags a near-tie inside the block.
* The same batch with the flag off (mma.sync GEMV kernels): the first pass's
  logits of all 64 sequences must agree with the tensor-core path's within
  1e-2 (the same products, summed in another fp32 order).
* The counters must show that the projections ran on the tensor cores.
"""

import numpy as np
import pytest
import torch

from workload import SWEEP, Patcher, WeightSet, prefix_bytes

pytestmark = pytest.mark.gpu

TOL = 2e-2


@pytest.fixture(scope="module")
def corner():
    from block_diffusion_byte_b200 import _build

    _build.build()
    wl = next(w for w in SWEEP if w.batch == 64 and w.block == 16 and w.prefix_len == 512)
    return wl, WeightSet(wl.shape).materialize()


def _out(shape):
    t = torch.full(shape, float("nan"), dtype=torch.float32, device="cuda")
    torch.cuda.synchronize()  # filled before the engine's stream writes it
    return t


def _block(wl, ws, tensor_cores):
    """Prefill the 64 prefixes, then one BLT-D-16 block: (bytes, passes, logits, counters)."""
    from block_diffusion_byte_b200 import binding as B
    from block_diffusion_byte_b200.driver import Engine, SeqHost

    b, k = wl.batch, wl.block
    eng = Engine(wl.shape, ws, max_batch=b, max_ctx=wl.prefix_len + 64, max_block=16, max_rows=2048, tensor_cores=tensor_cores)
    try:
        hosts = []
        for s in range(b):
            sh = SeqHost(Patcher(wl.patch_kind, wl.seed, wl.cfg_index, s), wl.seed, wl.cfg_index, s, wl.shape.d_global)
            sh.commit([int(x) for x in prefix_bytes(wl.seed, wl.cfg_index, s, wl.prefix_len)])
            hosts.append(sh)
        pend = [sh.take_pending() for sh in hosts]
        r, keep = eng.rows([p[0][:-1] for p in pend], [p[1][:-1] for p in pend], [p[2] for p in pend])
        B.blt_dec_prefill(eng.h, b, r)
        assert B.blt_dec_sync(eng.h) == 0
        for sh, p in zip(hosts, pend):
            sh.pend_bytes, sh.pend_slots = p[0][-1:], p[1][-1:]
        pend = [sh.take_pending() for sh in hosts]
        r, keep = eng.rows([p[0] for p in pend], [p[1] for p in pend], [p[2] for p in pend])
        lg = _out((k, b, k, 256))
        B.blt_dec_diffuse_block(eng.h, b, r, k, wl.alpha, 0, eng.d_out, eng.d_steps, lg)
        assert B.blt_dec_sync(eng.h) == 0
        blocks = eng._get(eng.out_view(b, k)).copy()
        steps = eng._get(eng.d_steps[:b]).copy()
        return blocks, steps, lg.cpu().numpy(), B.blt_dec_stats(eng.h)
    finally:
        eng.close()


def test_tensor_core_block_matches_oracle_and_gemv(corner):
    from oracle.model import OracleModel
    from oracle.policies import OracleSequence

    wl, ws = corner
    k = wl.block
    blocks, steps, lg, st = _block(wl, ws, True)
    assert st["tc_gemms"] > 0, st
    # sequence 0 against the oracle, pass by pass
    o = OracleSequence(OracleModel(wl.shape, ws), wl, 0, [int(x) for x in prefix_bytes(wl.seed, wl.cfg_index, 0, wl.prefix_len)])
    zs = []
    real = o._pass

    def rec(rows):
        z = real(rows)
        zs.append(z)
        return z

    o._pass = rec
    blk_o, steps_o, _ = o.diffuse(k, wl.alpha)
    n = min(int(steps[0]), steps_o)
    err = max(float(np.abs(lg[t, 0] - np.asarray(zs[t])[-k:]).max()) for t in range(n))
    flagged = [f for f in o.flags if len(o.bytes) <= f.pos < len(o.bytes) + k]  # diffuse does not commit
    print(f"tcgen05 GEMM, batch 64 x block 16: seq 0 logits max-abs error vs fp64 oracle {err:.3g} over {n} passes; "
          f"flags in the block: {[(f.pos, f.what) for f in flagged]}")
    assert err < TOL, err
    if not flagged:
        assert [int(x) for x in blocks[0]] == list(blk_o) and int(steps[0]) == steps_o
    # the GEMV path on the same batch: first-pass logits of every sequence
    blocks_g, steps_g, lg_g, st_g = _block(wl, ws, False)
    assert st_g["tc_gemms"] == 0
    d = float(np.abs(lg[0] - lg_g[0]).max())
    print(f"tcgen05 vs GEMV, first pass, 64 sequences: max-abs difference {d:.3g}")
    assert d < 1e-2, d
