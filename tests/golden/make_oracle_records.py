#!/usr/bin/env python
"""Write the oracle's generation records used by the full-size GPU parity tests.

Every value in ``tests/golden/oracle_records/*.json`` comes from this script,
which calls only the fp64 oracle (``oracle/``) and the seeded input generators
(``workload/``): decoded bytes, the per-round record (round start, bytes,
decoder passes of each BLT-D block, accept length of each BLT-S / BLT-DV
round) and every near-tie flag.  The engine never contributes to them.

The oracle of the longest jobs (prefix 8192, or 1024 BLT-DV bytes after a
2048-byte prefix) takes minutes on a CPU, longer than a GPU test run should
hold a GPU; storing its records lets the GPU tests compare the engine at the
full sizes.  Run:  python tests/golden/make_oracle_records.py [name ...]
"""

from __future__ import annotations

import json
import os
import sys
import time
from dataclasses import replace

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(os.path.dirname(HERE))
sys.path.insert(0, ROOT)

from oracle.model import OracleModel  # noqa: E402
from oracle.policies import OracleSequence  # noqa: E402
from workload import CONFIGS, SWEEP, WeightSet, prefix_bytes  # noqa: E402

OUT = os.path.join(HERE, "oracle_records")


def cases():
    """(record name, workload, sequence id, bytes generated)."""
    out = [
        ("d4_b1_seq0", CONFIGS["d4_b1"], 0, 512),
        ("d4eb_b1_seq0", CONFIGS["d4eb_b1"], 0, 512),
        ("dv16_b8_seq0", CONFIGS["dv16_b8"], 0, 1024),
        ("s8_b1_seq0", CONFIGS["s8_b1"], 0, 512),
        ("s8_b16_seq3", CONFIGS["s8_b16"], 3, 512),
    ]
    for p in (512, 2048, 8192):
        for k in (4, 8, 16):
            wl = next(w for w in SWEEP if w.prefix_len == p and w.block == k and w.batch == 1)
            out.append((f"sweep_k{k}_p{p}_seq0", wl, 0, 2 * k))
    return out


def record(name, wl, seq, G, model):
    prefix = [int(b) for b in prefix_bytes(wl.seed, wl.cfg_index, seq, wl.prefix_len)]
    t0 = time.time()
    o = OracleSequence(model, wl, seq, prefix)
    o.prefill()
    t1 = time.time()
    rec = []
    out = o.generate(G, rec)
    t2 = time.time()
    rounds = []
    for r in rec:
        rounds.append({k: (int(v) if isinstance(v, (int,)) else v) for k, v in r.items() if k in ("start", "bytes", "steps", "accepted", "draft")})
    return {
        "name": name,
        "workload": wl.name,
        "mode": wl.mode,
        "block": wl.block,
        "alpha": wl.alpha,
        "unmask": wl.unmask,
        "gamma": wl.gamma,
        "seq": seq,
        "prefix_len": wl.prefix_len,
        "gen_bytes": G,
        "bytes": [int(b) for b in out],
        "rounds": rounds,
        "flags": [{"pos": int(f.pos), "what": f.what, "value": float(f.value)} for f in o.flags],
        "decoder_passes": int(o.c.passes),
        "oracle_seconds": {"prefill": round(t1 - t0, 1), "generate": round(t2 - t1, 1)},
        "source": "tests/golden/make_oracle_records.py (fp64 oracle only)",
    }


def main(names):
    os.makedirs(OUT, exist_ok=True)
    models = {}
    for name, wl, seq, G in cases():
        if names and name not in names:
            continue
        key = (wl.shape, wl.seed)
        if key not in models:
            models[key] = OracleModel(wl.shape, WeightSet(wl.shape, seed=wl.seed).materialize())
        t = time.time()
        r = record(name, wl, seq, G, models[key])
        with open(os.path.join(OUT, name + ".json"), "w") as f:
            json.dump(r, f, indent=0)
        print(f"{name}: {len(r['bytes'])} bytes, {len(r['flags'])} flags, {time.time() - t:.0f} s", flush=True)


if __name__ == "__main__":
    main(sys.argv[1:])
