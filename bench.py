#!/usr/bin/env python
"""Benchmark of the Fast-BLT local-decoder engine on B200.

One step = one whole job of the workload: prefill the prefix, then decode
``gen_bytes`` bytes per sequence with the workload's decoding rule (default:
BLT-D-4, 9 layers d=1024 bf16, prefix 1024, 512 bytes, batch 1, alpha 0.7).
Between blocks the host re-patches the committed bytes and supplies the
latents of newly closed patches (the synthetic stand-in for the entropy
patcher + encoder + global model), as in BLT-D inference.

value  decoded bytes/s over all ranks, prefix inputs already on the device
e2e    the same job through the public API from pinned host buffers
       (prefix H2D and result D2H inside the timed region)
roofline  the decoder pass (all kernels of one pass) against measured HBM
       bandwidth: algorithmic bytes per pass / mean pass time (CUDA events)

Multi-GPU: replicas only (sequences are independent; no collective on the
data path).  Each rank decodes its own batch; value = all ranks' bytes / the
slowest rank's time.
"""

from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

from workload import CONFIGS, WeightSet, prefix_bytes  # noqa: E402

PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0}


def measured_traffic(workload: str, persistent: bool):
    """DRAM bytes per decoder pass from the committed ncu record of the persistent
    kernel, or None when the record is for another workload or path, or the kernel
    sources changed since it was taken."""
    import hashlib

    path = os.path.join(ROOT, "profiles", f"k_mega_{workload}_dram.json")
    if not persistent or not os.path.exists(path):
        return None
    with open(path) as f:
        rec = json.load(f)
    h = hashlib.sha256()
    for rel in rec["source_files"]:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return rec["dram_bytes_per_pass"] if h.hexdigest() == rec["source_sha256"] else None


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return PEAKS_FALLBACK, "fallback"


class Clocks:
    """nvidia-smi sampling of SM clocks and throttle reasons during the timed region."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
         "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.f = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        self.p = None

    def __enter__(self):
        try:
            self.p = subprocess.Popen(["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                                       "-lms", "200"], stdout=self.f, stderr=subprocess.DEVNULL)
        except OSError:
            self.p = None
        return self

    def __exit__(self, *a):
        if self.p:
            self.p.terminate()
            self.p.wait()

    def summary(self):
        self.f.flush()
        self.f.seek(0)
        sm, mx, reasons = [], [], set()
        for line in self.f:
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx.append(float(parts[2]))
            except ValueError:
                continue
            names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
            for n, v in zip(names, parts[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        os.unlink(self.f.name)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons), "samples": len(sm)}


def oracle_rate(wl, seconds_cap: float = 25.0):
    """The fp64 oracle, as it stands, on a bounded sample of the workload.

    Sample: the full prefill of sequence 0's prefix plus the first blocks
    (rounds) of decoding until ``seconds_cap`` is reached; the rate is
    extrapolated to the whole job: gen_bytes / (t_prefill + t_per_byte * gen_bytes).
    """
    from oracle.model import OracleModel
    from oracle.policies import OracleSequence

    try:
        from threadpoolctl import threadpool_info

        blas_threads = max((i.get("num_threads", 1) for i in threadpool_info()), default=1)
    except Exception:
        blas_threads = os.cpu_count() or 1
    ws = WeightSet(wl.shape, seed=wl.seed).materialize()
    m = OracleModel(wl.shape, ws)
    pre = [int(b) for b in prefix_bytes(wl.seed, wl.cfg_index, 0, wl.prefix_len)]
    o = OracleSequence(m, wl, 0, pre)
    t0 = time.perf_counter()
    o.prefill()
    t_pre = time.perf_counter() - t0
    t1 = time.perf_counter()
    made = 0
    while made < wl.gen_bytes and (time.perf_counter() - t0) < seconds_cap:
        made += len(o.generate(min(wl.block if wl.mode != "AR" else 1, wl.gen_bytes - made)))
    t_dec = time.perf_counter() - t1
    per_byte = t_dec / max(made, 1)
    rate = wl.gen_bytes * wl.batch / (wl.batch * (t_pre + per_byte * wl.gen_bytes))
    return {
        "value": rate,
        "unit": "bytes/s",
        "cores": int(blas_threads),
        "host_cpus": os.cpu_count(),
        "kind": "oracle",
        "sample": f"seq 0: full prefill of {wl.prefix_len} bytes ({t_pre:.1f} s) + {made} decoded bytes ({t_dec:.1f} s), "
        f"extrapolated to {wl.gen_bytes} bytes x batch {wl.batch}",
    }


def run_reference(args, wl):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    steps = []
    for i in range(args.warmup + args.steps):
        r = oracle_rate(wl, seconds_cap=args.ref_seconds)
        if i >= args.warmup:
            steps.append(r)
    v = statistics.mean(s["value"] for s in steps)
    line = {
        "impl": "reference",
        "metric": "decoded bytes/s",
        "value": v,
        "unit": "bytes/s",
        "n_gpus": args.gpus,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": 1000.0 * wl.gen_bytes * wl.batch / v,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f64",
        "data": "synthetic",
        "config": workload_config(wl),
        "cpu_baseline": {k: steps[-1][k] for k in ("kind", "cores", "sample")} | {"value": v, "unit": "bytes/s"},
        "e2e": {"value": v, "unit": "bytes/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def workload_config(wl):
    return {
        "workload": wl.name,
        "mode": {"D": "BLT-D", "S": "BLT-S", "DV": "BLT-DV", "AR": "AR greedy"}[wl.mode],
        "layers": wl.shape.n_layers,
        "d_model": wl.shape.d_model,
        "d_ffn": wl.shape.d_ffn,
        "d_global": wl.shape.d_global,
        "block": wl.block,
        "alpha": wl.alpha,
        "batch": wl.batch,
        "prefix": wl.prefix_len,
        "gen_bytes": wl.gen_bytes,
        "weights": wl.shape.weight_dtype,
        "l2": "no flush: every pass streams 302 MB of weights (> 126 MB L2)",
        "parallelism": "replicas",
    }


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="engine", choices=["engine", "reference"])
    ap.add_argument("--workload", default="d4_b1", choices=sorted(CONFIGS))
    ap.add_argument("--ref-seconds", type=float, default=25.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-ar-baseline", action="store_true", help="skip the greedy AR decoding of the same job")
    ap.add_argument("--path", default="persistent", choices=["persistent", "phased"],
                    help="decoder passes in the persistent kernel (one launch per call) or as per-phase kernels")
    args = ap.parse_args()
    wl = CONFIGS[args.workload]
    if args.impl == "reference":
        return run_reference(args, wl)

    import torch

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dist = None
    if world > 1:
        import datetime

        import torch.distributed as dist

        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))

    from block_diffusion_byte_b200 import binding as B
    from block_diffusion_byte_b200._build import build
    from block_diffusion_byte_b200.driver import Engine, generate
    from block_diffusion_byte_b200.replicas import max_over_ranks, shard_ids

    if rank == 0:
        build()
    if dist:
        dist.barrier()
    ws = WeightSet(wl.shape, seed=wl.seed).materialize()
    nb = wl.batch
    max_ctx = wl.prefix_len + wl.gen_bytes + 4 * wl.block + 16
    eng = Engine(wl.shape, ws, max_batch=nb, max_ctx=max_ctx, max_block=max(wl.block, 16), max_rows=1024, time_passes=True,
                 persistent=args.path == "persistent")
    seq_ids = shard_ids(rank, world, nb)
    prefixes = [[int(b) for b in prefix_bytes(wl.seed, wl.cfg_index, s, wl.prefix_len)] for s in seq_ids]

    def one_step():
        B.blt_dec_rewind(eng.h, nb, [0] * nb, [0] * nb)
        return generate(eng, wl, prefixes, seq_ids=seq_ids)

    def barrier():
        torch.cuda.synchronize()
        if dist:
            dist.barrier()

    for _ in range(args.warmup):
        one_step()
    st0 = B.blt_dec_stats(eng.h)
    barrier()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    h2d = d2h = 0
    with Clocks(local) as clk:
        ev0.record(eng.stream)
        for _ in range(args.steps):
            r = one_step()
            h2d += r.h2d_bytes
            d2h += r.d2h_bytes
        ev1.record(eng.stream)
        barrier()
    ms = ev0.elapsed_time(ev1)
    st1 = B.blt_dec_stats(eng.h)
    clocks = clk.summary()
    d = {k: st1[k] - st0[k] for k in st1}
    ms = max_over_ranks(ms, "cuda")
    total_bytes = wl.gen_bytes * nb * world * args.steps
    value = total_bytes / (ms / 1000.0)

    # e2e: the public API from host buffers (prefix bytes from pinned memory; the
    # generated bytes read back every step) -- generate() stages all inputs from the host
    barrier()
    t0 = time.perf_counter()
    e2e_steps = max(1, min(args.steps, 3))
    for _ in range(e2e_steps):
        r = one_step()
    barrier()
    e2e_s = max_over_ranks((time.perf_counter() - t0) / e2e_steps, "cuda")
    e2e_value = wl.gen_bytes * nb * world / e2e_s

    pk, pk_kind = peaks()
    passes = d["passes"]
    pass_ms = d["pass_ns"] / 1e6 / max(d["timed_passes"], 1)
    weight_b = d["weight_bytes"] / max(passes, 1)
    kv_b = d["kv_read_bytes"] / max(d["timed_passes"], 1)
    rows_per_pass = d["rows"] / max(d["timed_passes"], 1)
    alg_bytes = weight_b + kv_b
    achieved = alg_bytes / (pass_ms / 1000.0) / 1e9 if pass_ms > 0 else 0.0
    peak = float(pk["hbm_gbs"])
    line = {
        "metric": "decoded bytes/s",
        "value": value,
        "unit": "bytes/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": ms / args.steps,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic",
        "config": workload_config(wl),
        "e2e": {"value": e2e_value, "unit": "bytes/s", "h2d_bytes_per_step": h2d // args.steps, "d2h_bytes_per_step": d2h // args.steps},
        "gpu_launches": d["kernel_launches"],
        "roofline": {
            "bound": "hbm",
            "achieved": achieved,
            "peak": peak,
            "peak_kind": pk_kind,
            "unit": "GB/s",
            "frac": achieved / peak,
            "frac_of_8tbs": achieved / 8000.0,
            "traffic": measured_traffic(wl.name, bool(d["persistent_calls"])),
            "traffic_unit": "bytes per pass (dram__bytes_read.sum + dram__bytes_write.sum)",
            "kernel": "k_mega (persistent decoder pass)" if d["persistent_calls"] else "decoder pass (all kernels of one pass)",
            "alg_bytes_per_pass": alg_bytes,
            "pass_ms": pass_ms,
        },
        "decoder": {
            "passes_per_step": passes / args.steps,
            "passes_per_s": passes / (ms / 1000.0),
            "rows_per_pass": rows_per_pass,
            "weight_bytes_per_pass": weight_b,
            "kv_bytes_per_pass": kv_b,
            "launches_per_step": d["kernel_launches"] / args.steps,
            "path": args.path,
            "persistent_calls_per_step": d["persistent_calls"] / args.steps,
        },
        "clocks": clocks,
    }
    if world == 1 and not args.no_ar_baseline and wl.mode != "AR":
        # the same job decoded one byte per pass (plain greedy AR BLT) on the same
        # engine: wall-clock speedup beside the decoder-NFE ratio (the pages' proxy)
        from dataclasses import replace

        wl_ar = replace(wl, mode="AR", block=1, alpha=0.0)

        def ar_step():
            B.blt_dec_rewind(eng.h, nb, [0] * nb, [0] * nb)
            return generate(eng, wl_ar, prefixes, seq_ids=seq_ids)

        ar_step()
        sa0 = B.blt_dec_stats(eng.h)
        barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(eng.stream)
        ar_step()
        e1.record(eng.stream)
        barrier()
        ar_ms = e0.elapsed_time(e1)
        sa1 = B.blt_dec_stats(eng.h)
        ar_passes = sa1["passes"] - sa0["passes"]
        ar_value = wl.gen_bytes * nb / (ar_ms / 1000.0)
        line["ar_baseline"] = {
            "value": ar_value,
            "unit": "bytes/s",
            "ms_per_step": ar_ms,
            "passes_per_step": ar_passes,
            "speedup_wallclock": value / ar_value,
            "decoder_nfe_ratio": ar_passes / (passes / args.steps),
            "note": "same engine, prefix and length; greedy AR decoding (one byte per decoder pass); "
            "decoder_nfe_ratio = AR passes / this mode's passes, the decoder term of the pages' proxy",
        }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = oracle_rate(wl, seconds_cap=args.ref_seconds)
    eng.close()
    if dist:
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
