"""Strict engine-versus-oracle comparison of whole generations (test helper).

Rule (the workloads' parity bar): decoded bytes, per-block pass counts and
accept lengths must be identical round by round, except where the oracle flags
a near-tie, and a divergence is excused only by a flag that can cause it:

* a byte that differs is excused by an ``argmax`` flag at that very position
  (top-2 logit gap below 0.05);
* in a BLT-D block, a commit-order flag inside the block (``threshold``,
  ``fallback``, ``eb_bound``, ``eb_order``) excuses any difference in that
  block: committing the block's positions in another order changes the inputs
  of every later pass of the block;
* in a BLT-S / BLT-DV round, a flag on the round's draft or verification
  positions excuses a different accept length or next byte (the bytes of both
  sides are greedy AR bytes up to their own accept length).

After an excused divergence both sides are re-synchronised on the oracle's
bytes: the engine is restarted with the oracle's output up to the end of the
diverging round appended to the prefix, and the comparison goes on to the end
of the generation.  Every flagged position of the oracle and every divergence
is listed in the report.
"""

from __future__ import annotations

from dataclasses import dataclass, field, replace
from typing import Callable, List, Optional, Sequence

from oracle.policies import OracleSequence

REPORT: List[str] = []  # printed at the end of the session (conftest)


@dataclass
class ParityResult:
    name: str
    bytes_compared: int = 0
    rounds_compared: int = 0
    divergences: List[dict] = field(default_factory=list)
    flagged: List[tuple] = field(default_factory=list)  # (position, kind, value)
    resyncs: int = 0

    def line(self) -> str:
        fl = ", ".join(f"{p}:{k}" for p, k, _ in self.flagged) or "none"
        dv = "; ".join(f"pos {d['pos']} ({d['what']}, flag {d['flag']})" for d in self.divergences) or "none"
        return (f"{self.name}: {self.bytes_compared} bytes, {self.rounds_compared} rounds identical or excused; "
                f"divergences: {dv}; re-syncs {self.resyncs}; flagged positions: {fl}")


def oracle_run(model, wl, seq: int, prefix: Sequence[int], G: int):
    """The oracle's generation of G bytes after ``prefix`` with its per-round record."""
    o = OracleSequence(model, wl, seq, list(prefix))
    o.prefill()
    rec: list = []
    out = o.generate(G, rec)
    return out, rec, o


def _engine_rounds(res, wl, s_index: int, G: int, P: int):
    """The engine's rounds for sequence s_index as (start, bytes, steps, accepted) records."""
    out, pos = [], P
    for r in res.rounds:
        if wl.mode == "D":
            blk = [int(v) for v in r["block"][s_index]]
            new = blk[: G - (pos - P)]
            out.append(dict(start=pos, bytes=new, steps=int(r["steps"][s_index]), accepted=None))
        elif wl.mode == "AR":
            new = [int(r["next"][s_index])]
            out.append(dict(start=pos, bytes=new, steps=None, accepted=None))
        else:
            a = int(r["accepted"][s_index])
            new = [int(v) for v in r["draft"][s_index][:a]] + [int(r["next"][s_index])]
            new = new[: G - (pos - P)]
            out.append(dict(start=pos, bytes=new, steps=None, accepted=a))
        pos += len(new)
        if pos - P >= G:
            break
    return out


def compare_generation(name: str, wl, model, seq: int, prefix: Sequence[int], G: int,
                       engine_gen: Callable[[List[int], int], object], s_index: int = 0,
                       max_resyncs: int = 32) -> ParityResult:
    """Compare the engine's generation of sequence ``seq`` with the oracle's, strictly.

    ``engine_gen(prefix, G)`` runs the engine from ``prefix`` for G bytes with
    ``record=True`` and returns the driver's GenResult; the sequence under test
    is entry ``s_index`` of its batch.
    """
    res_p = ParityResult(name)
    want, rec, o = oracle_run(model, wl, seq, prefix, G)
    flags = {}
    for f in o.flags:
        flags.setdefault(f.pos, []).append(f.what)
        res_p.flagged.append((f.pos, f.what, f.value))
    P0 = len(prefix)
    cur_prefix = list(prefix)
    done = 0  # oracle bytes already confirmed (relative to the original prefix)
    ri = 0  # next oracle round
    while done < G:
        eng = engine_gen(cur_prefix, G - done)
        got = eng.out[s_index]
        er = _engine_rounds(eng, wl, s_index, G - done, len(cur_prefix))
        diverged = False
        for k, r in enumerate(er):
            orr = rec[ri + k]
            assert r["start"] == orr["start"], (name, r["start"], orr["start"])
            same_bytes = r["bytes"] == orr["bytes"]
            same_steps = wl.mode == "S" or r["steps"] is None or r["steps"] == orr.get("steps")
            same_acc = r["accepted"] is None or r["accepted"] == orr.get("accepted")
            if same_bytes and same_steps and same_acc:
                res_p.rounds_compared += 1
                res_p.bytes_compared += len(r["bytes"])
                continue
            lo, hi = orr["start"], orr["start"] + len(orr["bytes"])
            eb, ob = r["bytes"], orr["bytes"]
            diff = [j for j in range(min(len(eb), len(ob))) if eb[j] != ob[j]]
            if diff or len(eb) != len(ob):
                pos = lo + (diff[0] if diff else min(len(eb), len(ob)))
                what = "byte"
            else:
                pos = lo
                what = "steps" if not same_steps else "accepted"
            span = range(lo, lo + max(len(ob), len(eb), wl.block + 1))
            if wl.mode == "D":
                order = [p for p in span if p < lo + wl.block and any(kind != "argmax" for kind in flags.get(p, []))]
                ok = (what == "byte" and "argmax" in flags.get(pos, [])) or bool(order)
                used = pos if (what == "byte" and "argmax" in flags.get(pos, [])) else (order[0] if order else None)
            elif wl.mode == "AR":
                ok = "argmax" in flags.get(pos, [])
                used = pos if ok else None
            else:
                near = [p for p in span if p in flags]
                ok = bool(near)
                used = near[0] if near else None
            div = dict(pos=pos, what=what, flag=(f"{used}:" + ",".join(flags[used])) if used is not None else "-", engine=r, oracle=orr)
            res_p.divergences.append(div)
            assert ok, (f"{name}: unflagged divergence ({what}) at position {pos}: engine {r} vs oracle {orr}; "
                        f"flagged positions {sorted(flags)}")
            # re-sync on the oracle's bytes through the end of this round
            end = hi - P0
            cur_prefix = list(prefix) + want[:end]
            done = end
            ri = ri + k + 1
            res_p.resyncs += 1
            res_p.rounds_compared += 1
            diverged = True
            break
        if not diverged:
            assert got[: G - done] == want[done:], (name, "rounds agree but bytes differ")
            done = G
        assert res_p.resyncs <= max_resyncs, f"{name}: too many re-syncs"
    REPORT.append(res_p.line())
    print(res_p.line())
    return res_p


def engine_gen_factory(shape, ws, wl, seq_ids: Sequence[int], prefixes_other: Optional[dict] = None, s_index: int = 0,
                       persistent: bool = False, max_rows: int = 1024, extra_ctx: int = 0, tensor_cores: bool = True):
    """An ``engine_gen`` for compare_generation: a fresh engine per call, the sequence under
    test at batch index s_index and the other sequences with their own prefixes."""
    from block_diffusion_byte_b200.driver import Engine, generate
    from workload import prefix_bytes

    def run(prefix: List[int], G: int):
        prefs = []
        for i, s in enumerate(seq_ids):
            if i == s_index:
                prefs.append(list(prefix))
            else:
                prefs.append([int(b) for b in prefix_bytes(wl.seed, wl.cfg_index, s, wl.prefix_len)])
        # in a batch every sequence decodes until the slowest has G bytes: room for the faster ones' extra rounds
        max_ctx = max(len(p) for p in prefs) + (2 * G if len(prefs) > 1 else G) + 4 * wl.block + 32 + extra_ctx
        eng = Engine(shape, ws, max_batch=len(seq_ids), max_ctx=max_ctx, max_block=max(16, wl.block), max_rows=max_rows,
                     persistent=persistent, tensor_cores=tensor_cores)
        try:
            return generate(eng, wl, prefs, G, record=True, seq_ids=list(seq_ids))
        finally:
            eng.close()

    return run
