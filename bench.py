#!/usr/bin/env python
"""Benchmark of the Fast-BLT local-decoder engine on B200.

One step = one whole job of the workload: prefill the prefix, then decode
``gen_bytes`` bytes per sequence with the workload's decoding rule (default:
BLT-D-4, 9 layers d=1024 bf16, prefix 1024, 512 bytes, batch 1, alpha 0.7).
Between blocks the host re-patches the committed bytes and supplies the
latents of newly closed patches (the synthetic stand-in for the entropy
patcher + encoder + global model), as in BLT-D inference.

value     decoded bytes/s over all ranks, prefix inputs already on the device
e2e       the same job through the public API from pinned host buffers
          (prefix H2D and result D2H inside the timed region)
roofline  the decoder pass (all kernels of one pass) against measured HBM
          bandwidth: algorithmic bytes per pass / mean pass time (CUDA events)
batch16   the BLT-S k=8 job at batch 16 (prefix 4096, 512 bytes per sequence),
          timed the same way
modes     BLT-S k=8, BLT-DV-16 (one step) and greedy AR on the default job's
          prefix and length, with the decoder-NFE ratio and the pages' proxy
          memory bandwidth recomputed from counted passes

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


class OracleTimer:
    """The fp64 oracle, as it stands, timed on a bounded sample of the workload.

    The prefill of sequence 0's prefix runs once (timed); every ``step()`` then
    decodes a few rounds from a copy of the prefilled state (timed), and the
    rate is extrapolated to the whole job:
    gen_bytes / (t_prefill + t_per_byte * gen_bytes), per sequence.
    """

    def __init__(self, wl, min_bytes: int = 8):
        import copy

        from oracle.model import OracleModel
        from oracle.policies import OracleSequence

        self.copy = copy
        self.wl = wl
        try:
            from threadpoolctl import threadpool_info

            self.cores = max((i.get("num_threads", 1) for i in threadpool_info()), default=1)
        except Exception:
            self.cores = os.cpu_count() or 1
        ws = WeightSet(wl.shape, seed=wl.seed).materialize()
        pre = [int(b) for b in prefix_bytes(wl.seed, wl.cfg_index, 0, wl.prefix_len)]
        t0 = time.perf_counter()
        self.o = OracleSequence(OracleModel(wl.shape, ws), wl, 0, pre)
        self.o.prefill()
        self.t_pre = time.perf_counter() - t0
        self.min_bytes = min_bytes

    def step(self):
        o = self.copy.deepcopy(self.o)
        t0 = time.perf_counter()
        made = 0
        unit = self.wl.block if self.wl.mode != "AR" else 1
        while made < self.min_bytes:
            made += len(o.generate(unit))
        dt = time.perf_counter() - t0
        self.last_dt = dt
        per_byte = dt / made
        wl = self.wl
        rate = wl.gen_bytes / (self.t_pre + per_byte * wl.gen_bytes)
        return {
            "value": rate,
            "unit": "bytes/s",
            "cores": int(self.cores),
            "host_cpus": os.cpu_count(),
            "kind": "oracle",
            "sample": f"seq 0: prefill of {wl.prefix_len} bytes once ({self.t_pre:.1f} s), then {made} decoded bytes "
            f"({dt:.2f} s) from a copy of the prefilled state, extrapolated to {wl.gen_bytes} bytes per sequence",
        }


def oracle_rate(wl, seconds_cap: float = 20.0):
    """cpu_baseline of the engine arm: the prefill once, then decoded rounds doubling
    until the sample would pass about seconds_cap of CPU time."""
    t = OracleTimer(wl, min_bytes=max(8, int(wl.block)))
    r = t.step()
    while t.t_pre + 3 * t.last_dt < seconds_cap and t.min_bytes < wl.gen_bytes:
        t.min_bytes *= 2
        r = t.step()
    return r


def run_reference(args, wl):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    timer = OracleTimer(wl)
    steps = []
    for i in range(args.warmup + args.steps):
        r = timer.step()
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


def proxy_gb_counted(passes: int, latents: int, p_dec: float) -> float:
    """The pages' proxy memory bandwidth, GB = 2 [N_dec P_dec + N_enc (P_enc + P_global)] / 1e9,
    from counted decoder passes and global-model calls (one per latent consumed), with the
    1B model's encoder and global sizes (19M, 1.28B) and this decoder's streamed parameters."""
    return 2.0 * (passes * p_dec + latents * (19e6 + 1.28e9)) / 1e9


def time_job(eng, wl, prefixes, seq_ids, steps, warmup, barrier, generate, B):
    """Warm-up, then `steps` whole jobs bracketed by CUDA events on the engine's stream."""
    import torch

    nb = len(prefixes)

    def one():
        B.blt_dec_rewind(eng.h, nb, [0] * nb, [0] * nb)
        return generate(eng, wl, prefixes, seq_ids=seq_ids)

    for _ in range(warmup):
        one()
    st0 = B.blt_dec_stats(eng.h)
    barrier()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    h2d = d2h = 0
    ev0.record(eng.stream)
    for _ in range(steps):
        r = one()
        h2d += r.h2d_bytes
        d2h += r.d2h_bytes
    ev1.record(eng.stream)
    barrier()
    ms = ev0.elapsed_time(ev1)
    st1 = B.blt_dec_stats(eng.h)
    d = {k: st1[k] - st0[k] for k in st1}
    return ms, d, h2d, d2h, one


def pass_figures(d, steps, ms, peak, pk_kind):
    """Per-pass figures of the decoder passes in d (prefill excluded)."""
    passes = d["passes"]
    tp = max(d["timed_passes"], 1)
    pass_ms = d["pass_ns"] / 1e6 / tp
    weight_b = d["weight_bytes"] / max(passes, 1)
    kv_b = d["kv_read_bytes"] / tp
    alg_bytes = weight_b + kv_b
    achieved = alg_bytes / (pass_ms / 1000.0) / 1e9 if pass_ms > 0 else 0.0
    roof = {
        "bound": "hbm",
        "achieved": achieved,
        "peak": peak,
        "peak_kind": pk_kind,
        "unit": "GB/s",
        "frac": achieved / peak,
        "frac_of_8tbs": achieved / 8000.0,
        "alg_bytes_per_pass": alg_bytes,
        "pass_ms": pass_ms,
    }
    dec = {
        "passes_per_step": passes / steps,
        "passes_per_s": passes / (ms / 1000.0),
        "rows_per_pass": (d["rows"] - d["prefill_rows"]) / tp,
        "weight_bytes_per_pass": weight_b,
        "kv_bytes_per_pass": kv_b,
        "launches_per_step": d["kernel_launches"] / steps,
        "persistent_calls_per_step": d["persistent_calls"] / steps,
    }
    return roof, dec


class _TimingWeights:
    """Weights of a given shape for timing only: one random set of layer tensors, shared by
    every layer (the engine copies each layer separately), so a 1.2B-parameter model costs
    one layer's worth of host memory and generation time.  Values do not change the time."""

    def __init__(self, shape, seed=0):
        from workload.gen import GLOBAL_TENSORS, LAYER_TENSORS, tensor_shape

        rng = np.random.default_rng(seed)
        self.shape = shape
        self._layer = {}
        for n in LAYER_TENSORS:
            dims = tensor_shape(shape, n)
            if n.endswith("norm") or n == "norm_c":
                self._layer[n] = np.ones(dims, np.float32)
            else:
                self._layer[n] = (rng.standard_normal(dims, dtype=np.float32) / np.sqrt(shape.d_model)).astype(np.float32)
        self._glob = {n: (rng.standard_normal(tensor_shape(shape, n), dtype=np.float32) / np.sqrt(shape.d_model)).astype(np.float32)
                      for n in GLOBAL_TENSORS}
        self._glob["final_norm"] = np.ones(shape.d_model, np.float32)

    def get(self, name, layer=-1):
        return self._glob[name] if layer < 0 else self._layer[name]

    def layer(self, l):
        return dict(self._layer)


# decoder-step sweep points timed by the bench (batch, block, prefix): the sample rows of the
# sweep's roofline table, from one row per pass up to 1024 rows per pass
SWEEP_POINTS = ((1, 4, 512), (1, 4, 2048), (1, 16, 8192), (16, 8, 2048), (16, 16, 8192), (64, 16, 512))


def sweep_timing(barrier, generate, B, Engine, persistent, peak, pk_kind, points=SWEEP_POINTS):
    """Decoder-pass time at points of the decoder-step sweep (d_global 4096, BLT-D with
    alpha 0.7, two blocks per sequence): per point one warm-up job, then one job whose
    decoder passes are timed with CUDA events; the same per-pass figures as the main line."""
    from workload import SWEEP

    by = {(w.batch, w.block, w.prefix_len): w for w in SWEEP}
    ws_s = WeightSet(SWEEP[0].shape, seed=SWEEP[0].seed).materialize()
    out = []
    for b, k, p in points:
        w = by[(b, k, p)]
        ids = list(range(b))
        pres = [[int(x) for x in prefix_bytes(w.seed, w.cfg_index, s, p)] for s in ids]
        # a call's rows: the previous block (now causal) and the new block of every sequence
        eng = Engine(w.shape, ws_s, max_batch=b, max_ctx=p + 4 * w.gen_bytes + 4 * max(k, 16) + 16, max_block=max(k, 16),
                     max_rows=max(1024, 2 * b * (k + 1)), time_passes=True, persistent=persistent)
        try:
            ms, d, _, _, _ = time_job(eng, w, pres, ids, 1, 1, barrier, generate, B)
        finally:
            eng.close()
        roof, dec = pass_figures(d, 1, ms, peak, pk_kind)
        out.append(
            {
                "batch": b,
                "block": k,
                "prefix": p,
                "rows_per_pass": dec["rows_per_pass"],
                "decoder_passes": d["passes"],
                "pass_ms": roof["pass_ms"],
                "alg_mb_per_pass": roof["alg_bytes_per_pass"] / 1e6,
                "achieved_gbs": roof["achieved"],
                "frac": roof["frac"],
                "path": "persistent" if d["persistent_calls"] else "per-phase",
            }
        )
    return out


def global_step_timing(barrier, generate, B, Engine, peak, tokens: int = 256, steps: int = 48):
    """One step of a global transformer at the pages' 1B size on the device, so the
    N_enc (P_enc + P_global) term of the proxy can be timed: 24 layers, d 2048, 16 heads,
    FFN 5632 (1.23B parameters per step, bf16), one new token per step after `tokens`
    cached ones (the global model sees one latent per patch), run through this engine's
    own per-phase kernels (greedy AR steps of one row)."""
    import torch
    from dataclasses import replace

    from workload import ModelShape, Workload

    shape = ModelShape(n_layers=24, d_model=2048, n_heads=16, d_ffn=5632, d_global=128, weight_dtype="bf16")
    wl = Workload("global_1b_step", shape, "AR", 1, 0.0, steps, 1, tokens, "uniform8", 0, 9)
    ws = _TimingWeights(shape)
    eng = Engine(shape, ws, max_batch=1, max_ctx=tokens + steps + 32, max_block=16, max_rows=1024, time_passes=True,
                 persistent=False)
    try:
        pre = [[int(b) for b in prefix_bytes(0, 9, 0, tokens)]]
        generate(eng, wl, pre, 4)  # warm-up
        B.blt_dec_rewind(eng.h, 1, [0], [0])
        st0 = B.blt_dec_stats(eng.h)
        generate(eng, wl, pre, steps)
        st1 = B.blt_dec_stats(eng.h)
    finally:
        eng.close()
    d = {k: st1[k] - st0[k] for k in st1}
    step_ms = d["pass_ns"] / 1e6 / max(d["timed_passes"], 1)
    params = shape.pass_weight_params() + 256 * shape.d_model
    return {
        "shape": {"layers": 24, "d_model": 2048, "heads": 16, "d_ffn": 5632, "params": params},
        "step_ms": step_ms,
        "weight_gb_per_step": 2.0 * params / 1e9,
        "achieved_gbs": 2.0 * params / (step_ms / 1000.0) / 1e9,
        "frac_of_peak": 2.0 * params / (step_ms / 1000.0) / 1e9 / peak,
        "path": "per-phase kernels (d 2048 exceeds the persistent kernel's d <= 1024)",
        "note": "synthetic stand-in for the pages' 1B global model (1.28B); random weights shared across layers "
        "(timing only); one token per step over a cache of %d tokens" % tokens,
    }


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="engine", choices=["engine", "reference"])
    ap.add_argument("--workload", default="d4_b1", choices=sorted(CONFIGS))
    ap.add_argument("--ref-seconds", type=float, default=20.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extras", action="store_true", help="skip the batch-16 job and the BLT-S / BLT-DV / AR comparison")
    ap.add_argument("--no-ar-baseline", action="store_true", help="same as --no-extras (kept for old command lines)")
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
    persistent = args.path == "persistent"

    def barrier():
        torch.cuda.synchronize()
        if dist:
            dist.barrier()

    def engine_for(w, ws_, tensor_cores=True):
        # a batch decodes until its slowest sequence has gen_bytes: room for the faster sequences' extra rounds
        max_ctx = w.prefix_len + (2 * w.gen_bytes if w.batch > 1 else w.gen_bytes) + 4 * max(w.block, 16) + 16
        return Engine(w.shape, ws_, max_batch=w.batch, max_ctx=max_ctx, max_block=max(w.block, 16), max_rows=1024,
                      time_passes=True, persistent=persistent, tensor_cores=tensor_cores)

    ws = WeightSet(wl.shape, seed=wl.seed).materialize()
    nb = wl.batch
    eng = engine_for(wl, ws)
    seq_ids = shard_ids(rank, world, nb)
    prefixes = [[int(b) for b in prefix_bytes(wl.seed, wl.cfg_index, s, wl.prefix_len)] for s in seq_ids]

    with Clocks(local) as clk:
        ms, d, h2d, d2h, one_step = time_job(eng, wl, prefixes, seq_ids, args.steps, args.warmup, barrier, generate, B)
    clocks = clk.summary()
    ms = max_over_ranks(ms, "cuda")
    total_bytes = wl.gen_bytes * nb * world * args.steps
    value = total_bytes / (ms / 1000.0)

    # e2e: the public API from host buffers (prefix bytes from pinned memory; the
    # generated bytes read back every step) -- generate() stages all inputs from the host
    barrier()
    t0 = time.perf_counter()
    e2e_steps = max(1, min(args.steps, 3))
    for _ in range(e2e_steps):
        one_step()
    barrier()
    e2e_s = max_over_ranks((time.perf_counter() - t0) / e2e_steps, "cuda")
    e2e_value = wl.gen_bytes * nb * world / e2e_s

    pk, pk_kind = peaks()
    peak = float(pk["hbm_gbs"])
    roof, dec = pass_figures(d, args.steps, ms, peak, pk_kind)
    roof["traffic"] = measured_traffic(wl.name, bool(d["persistent_calls"]))
    roof["traffic_unit"] = "bytes per pass (dram__bytes_read.sum + dram__bytes_write.sum)"
    roof["kernel"] = "k_mega (persistent decoder pass)" if d["persistent_calls"] else "decoder pass (all kernels of one pass)"
    dec["path"] = args.path
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
        "roofline": roof,
        "decoder": dec,
        "clocks": clocks,
    }
    p_dec = float(wl.shape.pass_weight_params() + 256 * wl.shape.d_model)
    if world == 1 and not (args.no_extras or args.no_ar_baseline) and args.workload == "d4_b1":
        from dataclasses import replace

        # BLT-S k=8, BLT-DV-16 (one step) and greedy AR on the same engine, prefix and length:
        # wall clock beside the decoder-NFE ratio and the pages' proxy bandwidth from counted passes
        modes = {}
        for name, w in (("AR", replace(wl, name="ar_b1", mode="AR", block=1, alpha=0.0)),
                        ("BLT-D-4", wl),
                        ("BLT-S-8", replace(wl, name="s8_p1024", mode="S", block=8, alpha=0.0)),
                        ("BLT-DV-16", replace(wl, name="dv16_p1024", mode="DV", block=16, alpha=0.0))):
            e2 = engine_for(w, ws)
            try:
                msm, dm, _, _, _ = time_job(e2, w, prefixes, seq_ids, 1, 1, barrier, generate, B)
            finally:
                e2.close()
            modes[name] = {
                "value": w.gen_bytes * nb / (msm / 1000.0),
                "unit": "bytes/s",
                "ms_per_step": msm,
                "decoder_passes": dm["passes"],
                "global_calls": dm["latents"],
                "proxy_gb": proxy_gb_counted(dm["passes"], dm["latents"], p_dec),
            }
        ar = modes["AR"]
        for name, mrec in modes.items():
            mrec["speedup_wallclock_vs_ar"] = mrec["value"] / ar["value"]
            mrec["decoder_nfe_ratio_vs_ar"] = ar["decoder_passes"] / max(mrec["decoder_passes"], 1)
            mrec["proxy_reduction_vs_ar"] = 1.0 - mrec["proxy_gb"] / ar["proxy_gb"]
        line["modes"] = {
            "note": "same engine, weights, prefix 1024 and 512 bytes; proxy_gb = 2 [decoder passes x decoder params + "
            "global calls x (19M + 1.28B)] / 1e9 (the pages' formula, 1B encoder/global sizes, calls counted as latents consumed)",
            **modes,
        }
    if world == 1 and not (args.no_extras or args.no_ar_baseline) and args.workload == "d4_b1":
        # decoded bytes/s at batch 16: BLT-S k=8, prefix 4096, 512 bytes per sequence
        w16 = CONFIGS["s8_b16"]
        ids16 = list(range(w16.batch))
        pre16 = [[int(b) for b in prefix_bytes(w16.seed, w16.cfg_index, s, w16.prefix_len)] for s in ids16]
        runs16 = {}
        for tc in (True, False):  # verification passes (128 rows) on the tcgen05 GEMM, then on the GEMV kernels
            e16 = engine_for(w16, ws, tensor_cores=tc)
            try:
                runs16[tc] = time_job(e16, w16, pre16, ids16, 2, 1, barrier, generate, B)
            finally:
                e16.close()
        ms16, d16, h16, o16, _ = runs16[True]
        roof16, dec16 = pass_figures(d16, 2, ms16, peak, pk_kind)
        dec16["path"] = args.path
        dec16["tc_gemms_per_step"] = d16["tc_gemms"] / 2
        ms16g = runs16[False][0]
        line["batch16"] = {
            "config": workload_config(w16),
            "value": w16.gen_bytes * w16.batch * 2 / (ms16 / 1000.0),
            "unit": "bytes/s",
            "steps": 2,
            "warmup": 1,
            "ms_per_step": ms16 / 2,
            "roofline": roof16,
            "decoder": dec16,
            "gemv_value": w16.gen_bytes * w16.batch * 2 / (ms16g / 1000.0),
            "gemv_ms_per_step": ms16g / 2,
            "tcgen05_speedup": ms16g / ms16,
            "note": "drafting passes (16 rows over 16 x ~4100 cached bytes: ~57 attention items per SM) run in the per-phase "
            "kernels, whose attention blocks overlap on each SM (the persistent kernel takes small passes with <= 8 items per SM); "
            "verification passes (128 rows) and prefill chunks project on the tcgen05 GEMM (value) or on the mma.sync GEMV "
            "kernels (gemv_value); roofline over all decoder passes of the job",
        }
    if world == 1 and not args.no_extras and args.workload == "d4_b1":
        # per-pass time across the decoder-step sweep (1 to 1024 rows per pass)
        line["sweep"] = {
            "note": "d_global 4096, BLT-D alpha 0.7, two blocks per sequence; per point one warm-up job and one timed job; "
            "roofline over the timed job's decoder passes (weights + K/V per pass)",
            "points": sweep_timing(barrier, generate, B, Engine, persistent, peak, pk_kind),
        }
    if world == 1 and not (args.no_extras or args.no_ar_baseline) and args.workload == "d4_b1":
        # the N_enc term of the pages' proxy, timed: one global-model step at the 1B size
        gs = global_step_timing(barrier, generate, B, Engine, peak)
        line["global_step"] = gs
        if "modes" in line:
            for name, mrec in line["modes"].items():
                if isinstance(mrec, dict) and "decoder_passes" in mrec:
                    # wall clock of the whole BLT step: the decoder job as measured plus one global step per latent
                    mrec["with_global_ms"] = mrec["ms_per_step"] + mrec["global_calls"] * gs["step_ms"]
            ar_tot = line["modes"]["AR"]["with_global_ms"]
            for name, mrec in line["modes"].items():
                if isinstance(mrec, dict) and "with_global_ms" in mrec:
                    mrec["speedup_with_global_vs_ar"] = ar_tot / mrec["with_global_ms"]
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = oracle_rate(wl, seconds_cap=args.ref_seconds)
    eng.close()
    if dist:
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
