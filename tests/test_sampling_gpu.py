"""Stochastic decoding on the engine against the fp64 oracle, with the same uniforms.

Temperature / top-p draws (BLT-D with confidence or EB selection, BLT-S and
BLT-DV drafts) and rejection-sampling verification: blt_dec_diffuse_block_sampled,
blt_dec_draft_sampled and blt_dec_verify_sampled, driven by
driver.generate_sampled; the oracle runs oracle.sampling's definitions on its
fp64 passes with the uniforms of workload.sampling_uniforms.

Rule: the decoded bytes must be identical, except that a divergence is excused
when the oracle flags a near-tie (a uniform within 2e-3 of a CDF boundary or of
an acceptance ratio, or a top-p cut within 2e-3) in the round where it occurs;
the comparison stops there.  Every case must agree on at least its first 16
bytes.  Two configurations: the tiny fp32 decoder (sequence 0 alone) and the
9-layer bf16 decoder at batch 2 (prefix 256).
"""

from dataclasses import replace

import numpy as np
import pytest

from workload import CONFIGS, WeightSet, prefix_bytes, sampling_uniforms

pytestmark = pytest.mark.gpu

T, TOP_P = 0.8, 0.9


def _oracle(wl, ws, seq, prefix, G):
    from oracle.model import OracleModel
    from oracle.policies import OracleSequence

    o = OracleSequence(OracleModel(wl.shape, ws), wl, seq, prefix)
    o.prefill()
    k = wl.block
    out, starts = [], []
    rnd = 0
    while len(out) < G:
        u_d = [float(v) for v in sampling_uniforms(wl.seed, wl.cfg_index, seq, 2 * rnd, 2 * k + 1)]
        u_v = [float(v) for v in sampling_uniforms(wl.seed, wl.cfg_index, seq, 2 * rnd + 1, 2 * k + 1)]
        start = len(o.bytes)
        if wl.mode == "D":
            new, _, _ = o.diffuse(k, wl.alpha, unmask=wl.unmask, gamma=wl.gamma, samp=(T, TOP_P, u_d))
        elif wl.mode == "S":
            draft, a, nxt = o.blt_s_round_sampled(k, T, TOP_P, u_d, u_v)
            new = draft[:a] + [nxt]
        else:
            draft, a, nxt, _ = o.blt_dv_round_sampled(k, wl.alpha, T, TOP_P, u_d, u_v)
            new = draft[:a] + [nxt]
        o.commit(new)
        o.cached = min(o.cached, len(o.bytes))
        starts.append(start)
        out += new
        rnd += 1
    return out[:G], starts, o.flags, len(prefix)


def _compare(name, eng_out, orc):
    out, starts, flags, n0 = orc
    G = len(out)
    div = next((i for i in range(G) if eng_out[i] != out[i]), None)
    fl = sorted({(f.pos, f.what) for f in flags})
    print(f"{name}: {G} bytes, first divergence {div}, oracle flags {fl[:12]}{' ...' if len(fl) > 12 else ''}")
    if div is None:
        return
    pos = n0 + div
    rstart = max(s for s in starts if s <= pos)
    assert any(rstart <= f.pos <= pos for f in flags), (name, div, eng_out[div], out[div])
    assert div >= 16, (name, div)


@pytest.mark.parametrize(
    "mode,block,alpha,unmask,gamma",
    [("S", 8, 0.0, "confidence", 0.0), ("DV", 8, 0.0, "confidence", 0.0), ("D", 4, 0.7, "confidence", 0.0), ("D", 4, 0.0, "entropy", 3.0)],
    ids=["S8", "DV8", "D4", "D4-EB"],
)
def test_tiny_sampled_matches_oracle(mode, block, alpha, unmask, gamma):
    from block_diffusion_byte_b200 import _build
    from block_diffusion_byte_b200.driver import Engine, generate_sampled

    _build.build()
    wl = replace(CONFIGS["tiny_d4"], mode=mode, block=block, alpha=alpha, unmask=unmask, gamma=gamma)
    ws = WeightSet(wl.shape).materialize()
    G = 48
    pre = [int(b) for b in prefix_bytes(wl.seed, wl.cfg_index, 0, wl.prefix_len)]
    eng = Engine(wl.shape, ws, max_batch=1, max_ctx=wl.prefix_len + 3 * G + 64, max_block=16, max_rows=256, persistent=True)
    try:
        res = generate_sampled(eng, wl, [pre], G, T, TOP_P)
        assert res.stats["persistent_calls"] == 0  # sampled calls take the per-phase kernels
    finally:
        eng.close()
    _compare(f"tiny {mode}{block} {unmask}", res.out[0], _oracle(wl, ws, 0, pre, G))


@pytest.mark.parametrize("mode", ["S", "DV"])
def test_bf16_sampled_batch2_matches_oracle(mode):
    from block_diffusion_byte_b200 import _build
    from block_diffusion_byte_b200.driver import Engine, generate_sampled

    _build.build()
    base = CONFIGS["s8_b1"] if mode == "S" else CONFIGS["dv16_b8"]
    wl = replace(base, prefix_len=256, block=8, batch=2)
    ws = WeightSet(wl.shape).materialize()
    G = 32
    prefs = [[int(b) for b in prefix_bytes(wl.seed, wl.cfg_index, s, wl.prefix_len)] for s in range(2)]
    eng = Engine(wl.shape, ws, max_batch=2, max_ctx=wl.prefix_len + 3 * G + 64, max_block=16, max_rows=512)
    try:
        res = generate_sampled(eng, wl, prefs, G, T, TOP_P)
    finally:
        eng.close()
    for s in range(2):
        _compare(f"bf16 {mode}8 seq {s}", res.out[s], _oracle(wl, ws, s, prefs[s], G))
