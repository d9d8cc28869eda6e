"""Host-side generation loops over the bltdec C ABI.

Between engine calls the driver plays the parts of Fast-BLT that are not the
local decoder: the entropy patcher, the local encoder and the global model.
Here they are the synthetic stand-ins of :mod:`workload` (a causal hazard
patcher and content-keyed N(0,1) latents).  The driver

* re-patches committed bytes and derives each byte's latent slot (the
  cross-attention rule of section "BLT-D의 어텐션 마스크" on the Fast-BLT
  summary page: the last byte of a patch sees that patch's latent, every
  other byte the latent of the patch before; slot = closed patches up to and
  including the byte, minus one);
* feeds committed-but-uncached bytes back as the next call's pending rows;
* for BLT-S / BLT-DV, re-patches the draft speculatively, sends the draft's
  latent slots and the latents of patches it would close, and commits the
  accepted bytes plus the correction / free byte ("BLT-S와 BLT-DV").

All decoder work runs in the engine's kernels.
"""

from __future__ import annotations

import time
from dataclasses import dataclass, field
from typing import List, Optional, Sequence

import numpy as np
import torch

from workload import sampling_uniforms, ModelShape, Patcher, PatchState, WeightSet, Workload, latent_vectors

from . import binding as B

_NP_DTYPE = {torch.uint8: np.uint8, torch.int32: np.int32, torch.float32: np.float32, torch.int64: np.int64}


def engine_config(shape: ModelShape, max_batch: int, max_ctx: int, max_latents: int, max_rows: int, max_block: int,
                  page_tokens: int = 64, kv_pages: int = 0, attn_chunk: int = 0, flags: int = 0) -> B.blt_dec_config:
    return B.blt_dec_config(
        n_layers=shape.n_layers,
        d_model=shape.d_model,
        n_heads=shape.n_heads,
        d_ffn=shape.d_ffn,
        d_global=shape.d_global,
        vocab=shape.vocab,
        weight_dtype=B.BLT_W_BF16 if shape.weight_dtype == "bf16" else B.BLT_W_F32,
        rope_theta=shape.rope_theta,
        norm_eps=shape.norm_eps,
        max_batch=max_batch,
        max_ctx=max_ctx,
        max_latents=max_latents,
        max_rows=max_rows,
        max_block=max_block,
        page_tokens=page_tokens,
        kv_pages=kv_pages,
        attn_chunk=attn_chunk,
        flags=flags,
    )


class Engine:
    """An engine handle plus device staging buffers for one workload size."""

    def __init__(self, shape: ModelShape, weights: WeightSet, max_batch: int, max_ctx: int, max_block: int,
                 max_rows: int = 1024, max_latents: Optional[int] = None, page_tokens: int = 64, attn_chunk: int = 0,
                 device: str = "cuda", time_passes: bool = False, persistent: bool = False, extra_flags: int = 0,
                 tensor_cores: bool = True):
        self.shape = shape
        self.max_batch, self.max_ctx, self.max_block, self.max_rows = max_batch, max_ctx, max_block, max_rows
        self.max_latents = max_latents or (max_ctx // 2 + 64)
        self.device = torch.device(device)
        self.stream = torch.cuda.Stream(device=self.device)
        # tensor_cores: decode passes of >= 128 rows project on the tcgen05 GEMM (bf16 weights; ignored otherwise)
        flags = (B.BLT_FLAG_TIME_PASSES if time_passes else 0) | (B.BLT_FLAG_PERSISTENT if persistent else 0) | extra_flags
        if tensor_cores:
            flags |= B.BLT_FLAG_TENSOR_CORES
        cfg = engine_config(shape, max_batch, max_ctx, self.max_latents, max_rows, max_block, page_tokens, 0, attn_chunk, flags)
        layers = []
        for l in range(shape.n_layers):
            lw = weights.layer(l)
            layers.append([np.ascontiguousarray(lw[n], dtype=np.float32) for n in B.LAYER_ORDER])
        g = {n: np.ascontiguousarray(weights.get(n), dtype=np.float32) for n in ("embed", "head", "final_norm")}
        self.h = B.blt_dec_init(cfg, g["embed"], g["head"], g["final_norm"], layers, self.stream.cuda_stream)
        dev = self.device
        self.d_lat = torch.zeros((max(max_rows, 4 * max_batch * max_block), shape.d_global), dtype=torch.float32, device=dev)
        self.d_out = torch.zeros((max_batch, max_block), dtype=torch.uint8, device=dev)
        self.d_steps = torch.zeros(max_batch, dtype=torch.int32, device=dev)
        self.d_acc = torch.zeros(max_batch, dtype=torch.int32, device=dev)
        self.d_next = torch.zeros(max_batch, dtype=torch.uint8, device=dev)
        self.d_vslots = torch.zeros((max_batch, max_block), dtype=torch.int32, device=dev)
        self.h2d_bytes = 0
        self.d2h_bytes = 0
        self._h_rows = np.empty(1 << 16, dtype=np.uint8)  # a call's rows, packed (host)
        self._d_rows = torch.empty(1 << 16, dtype=torch.uint8, device=dev)

    # -- staging: every host <-> device copy goes through the engine's blt_dec_upload /
    # blt_dec_download (pinned bounce buffers, the handle's stream)
    def _put(self, dst: torch.Tensor, arr: np.ndarray) -> torch.Tensor:
        """Copy ``arr`` into the first rows of ``dst`` (queued on the engine's stream)."""
        n = arr.shape[0]
        if n == 0:
            return dst[:0]
        arr = np.ascontiguousarray(arr, dtype=_NP_DTYPE[dst.dtype])
        if arr.nbytes > dst.numel() * dst.element_size():
            raise ValueError(f"staging overflow: {arr.nbytes} bytes into {dst.numel() * dst.element_size()}")
        B.blt_dec_upload(self.h, dst.data_ptr(), arr.ctypes.data, arr.nbytes)
        self.h2d_bytes += arr.nbytes
        return dst[:n]

    def _get(self, t: torch.Tensor) -> np.ndarray:
        """A device tensor's values on the host, after the engine's queued work."""
        if not t.is_contiguous():
            raise ValueError("_get needs a contiguous tensor")
        out = np.empty(tuple(t.shape), dtype=_NP_DTYPE[t.dtype])
        B.blt_dec_download(self.h, out.ctypes.data, t.data_ptr(), out.nbytes)
        self.d2h_bytes += out.nbytes
        return out

    def rows(self, byte_lists: Sequence[Sequence[int]], slot_lists: Sequence[Sequence[int]], lat_lists: Sequence[Sequence[np.ndarray]]):
        """Stage a call's rows: bytes, latent slots and new latents packed into one upload."""
        ro = np.cumsum([0] + [len(b) for b in byte_lists]).astype(np.int64)
        lo = np.cumsum([0] + [len(v) for v in lat_lists]).astype(np.int64)
        n = int(ro[-1])
        lats = [v for vl in lat_lists for v in vl]
        dg = self.shape.d_global
        o_s = (n + 15) & ~15
        o_l = (o_s + 4 * n + 15) & ~15
        total = o_l + 4 * dg * len(lats) if lats else o_s + 4 * n
        if self._h_rows.nbytes < total:
            self._h_rows = np.empty(total + total // 4, dtype=np.uint8)
        if self._d_rows.numel() < total:
            torch.cuda.synchronize(self.device)  # the old buffer may still be read by queued work
            self._d_rows = torch.empty(total + total // 4, dtype=torch.uint8, device=self.device)
        buf = self._h_rows
        if n:
            buf[:n] = np.fromiter((b for bl in byte_lists for b in bl), dtype=np.uint8, count=n)
            buf[o_s:o_s + 4 * n].view(np.int32)[:] = np.fromiter((v for sl in slot_lists for v in sl), dtype=np.int32, count=n)
        if lats:
            lv = buf[o_l:total].view(np.float32).reshape(len(lats), dg)
            for i, v in enumerate(lats):
                lv[i] = v
        base = self._d_rows.data_ptr()
        if total:
            B.blt_dec_upload(self.h, base, buf.ctypes.data, total)
        self.h2d_bytes += n * 5 + 4 * dg * len(lats)
        return B.rows_in(base, base + o_s, ro.tolist(), base + o_l if lats else None, lo.tolist())

    def out_view(self, nb: int, k: int) -> torch.Tensor:
        """The engine writes [batch, k] byte outputs densely."""
        return self.d_out.view(-1)[: nb * k].view(nb, k)

    def close(self):
        if self.h:
            B.blt_dec_free(self.h)
            self.h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


@dataclass
class SeqHost:
    """Host view of one sequence: patcher state, pending rows, latents to send."""

    patcher: Patcher
    seed: int
    cfg_index: int
    seq: int
    d_global: int
    pstate: PatchState = field(default_factory=PatchState)
    n_sent: int = 0  # latents the engine holds (committed)
    lat_ready: List[np.ndarray] = field(default_factory=list)  # committed latents not sent yet
    pend_bytes: List[int] = field(default_factory=list)
    pend_slots: List[int] = field(default_factory=list)
    out: List[int] = field(default_factory=list)

    def patch(self, state: PatchState, data: Sequence[int]):
        """Latent slots of ``data`` appended after ``state`` and latents of the patches it closes."""
        per, st = self.patcher.advance(state, data)
        n = state.n_closed
        slots, new_slots, new_fnvs = [], [], []
        for closes, fnv in per:
            if closes:
                new_slots.append(n)
                new_fnvs.append(fnv)
                n += 1
            slots.append(n - 1)
        lats = list(latent_vectors(self.seed, self.cfg_index, self.seq, new_slots, new_fnvs, self.d_global))
        return slots, lats, st

    def commit(self, data: Sequence[int]) -> None:
        slots, lats, st = self.patch(self.pstate, data)
        self.pstate = st
        self.pend_bytes += [int(b) for b in data]
        self.pend_slots += slots
        self.lat_ready += lats

    def take_pending(self):
        b, s, l = self.pend_bytes, self.pend_slots, self.lat_ready
        self.n_sent += len(l)
        self.pend_bytes, self.pend_slots, self.lat_ready = [], [], []
        return b, s, l


@dataclass
class GenResult:
    out: List[List[int]]
    rounds: List[dict]
    stats: dict
    seconds: float
    h2d_bytes: int
    d2h_bytes: int


def generate(eng: Engine, wl: Workload, prefixes: Sequence[Sequence[int]], G: Optional[int] = None, record: bool = False,
             seq_ids: Optional[Sequence[int]] = None) -> GenResult:
    """Prefill every prefix, then decode G bytes per sequence with the workload's mode."""
    G = wl.gen_bytes if G is None else G
    nb = len(prefixes)
    ids = list(seq_ids) if seq_ids is not None else list(range(nb))
    sh = wl.shape
    seqs = [SeqHost(Patcher(wl.patch_kind, wl.seed, wl.cfg_index, i), wl.seed, wl.cfg_index, i, sh.d_global) for i in ids]
    h = eng.h
    st0 = B.blt_dec_stats(h)
    h2d0, d2h0 = eng.h2d_bytes, eng.d2h_bytes
    t0 = time.perf_counter()
    # prefill: every prefix byte but the last, which rides in the first pass
    for s, pre in zip(seqs, prefixes):
        s.commit(list(pre))
    bl, sl, ll = [], [], []
    for s in seqs:
        b, sl_, l = s.take_pending()
        bl.append(b[:-1])
        sl.append(sl_[:-1])
        ll.append(l)
        s.pend_bytes, s.pend_slots = b[-1:], sl_[-1:]
    r, keep = eng.rows(bl, sl, ll)
    B.blt_dec_prefill(h, nb, r)
    rounds: List[dict] = []
    k = wl.block
    while any(len(s.out) < G for s in seqs):
        pend = [s.take_pending() for s in seqs]
        r, keep = eng.rows([p[0] for p in pend], [p[1] for p in pend], [p[2] for p in pend])
        if wl.mode == "D":
            if wl.unmask == "entropy":
                B.blt_dec_diffuse_block_eb(h, nb, r, k, wl.gamma, 0, eng.d_out, eng.d_steps)
            else:
                B.blt_dec_diffuse_block(h, nb, r, k, wl.alpha, 0, eng.d_out, eng.d_steps)
            blk = eng._get(eng.out_view(nb, k))
            steps = eng._get(eng.d_steps[:nb]) if record else None
            for i, s in enumerate(seqs):
                new = [int(v) for v in blk[i]]
                s.commit(new)
                s.out += new
            if record:
                rounds.append(dict(block=blk.copy(), steps=steps.copy()))
        elif wl.mode == "AR":
            B.blt_dec_draft(h, nb, r, B.BLT_DRAFT_AR, 1, 0.0, 0, eng.d_out)
            d = eng._get(eng.out_view(nb, 1))
            for i, s in enumerate(seqs):
                s.commit([int(d[i, 0])])
                s.out.append(int(d[i, 0]))
            if record:
                rounds.append(dict(next=d[:, 0].copy()))
        elif wl.mode in ("S", "DV"):
            mode = B.BLT_DRAFT_AR if wl.mode == "S" else B.BLT_DRAFT_DIFFUSION
            B.blt_dec_draft(h, nb, r, mode, k, wl.alpha, 0, eng.d_out)
            draft = eng._get(eng.out_view(nb, k))
            vslots = np.zeros((nb, k), dtype=np.int32)
            prov: List[List[np.ndarray]] = []
            for i, s in enumerate(seqs):
                slots, lats, _ = s.patch(s.pstate, [int(v) for v in draft[i]])
                vslots[i] = slots
                prov.append(lats)
            lo = np.cumsum([0] + [len(p) for p in prov]).tolist()
            allp = [v for p in prov for v in p]
            dl = None
            if allp:
                dl = eng._put(eng.d_lat, np.stack(allp).astype(np.float32))
            dvs = eng._put(eng.d_vslots.view(-1), vslots.reshape(-1))
            B.blt_dec_verify_accept(h, dvs, dl, lo, eng.d_acc, eng.d_next)
            acc = eng._get(eng.d_acc[:nb])
            nxt = eng._get(eng.d_next[:nb])
            for i, s in enumerate(seqs):
                a = int(acc[i])
                new = [int(v) for v in draft[i, :a]] + [int(nxt[i])]
                # the engine kept the latents of patches closed by the accepted draft bytes
                s_slots, s_lats, st = s.patch(s.pstate, new)
                kept = (vslots[i, a - 1] + 1 - s.pstate.n_closed) if a >= 1 else 0
                s.pstate = st
                s.pend_bytes += new[a:]
                s.pend_slots += s_slots[a:]
                s.n_sent += kept
                s.lat_ready += s_lats[kept:]
                s.out += new
            if record:
                rounds.append(dict(draft=draft.copy(), accepted=acc.copy(), next=nxt.copy()))
        else:
            raise ValueError(wl.mode)
    st = B.blt_dec_sync(h)
    if st != 0:
        raise B.BltError(st, "generate", B.blt_dec_last_error(h))
    dt = time.perf_counter() - t0
    st1 = B.blt_dec_stats(h)
    stats = {k_: st1[k_] - st0[k_] for k_ in st1}
    return GenResult([s.out[:G] for s in seqs], rounds, stats, dt, eng.h2d_bytes - h2d0, eng.d2h_bytes - d2h0)


def generate_sampled(eng: Engine, wl: Workload, prefixes: Sequence[Sequence[int]], G: int, temperature: float, top_p: float,
                     seq_ids: Optional[Sequence[int]] = None, record: bool = False) -> GenResult:
    """Prefill, then decode G bytes per sequence with drawn bytes: BLT-D (confidence
    or EB selection), BLT-S / BLT-DV (rejection-sampling verification).  Round r of
    sequence s uses the workload's uniforms for calls 2 r (block / draft) and
    2 r + 1 (verification), 2 k + 1 each."""
    nb = len(prefixes)
    ids = list(seq_ids) if seq_ids is not None else list(range(nb))
    sh = wl.shape
    seqs = [SeqHost(Patcher(wl.patch_kind, wl.seed, wl.cfg_index, i), wl.seed, wl.cfg_index, i, sh.d_global) for i in ids]
    h = eng.h
    st0 = B.blt_dec_stats(h)
    t0 = time.perf_counter()
    for s, pre in zip(seqs, prefixes):
        s.commit(list(pre))
    bl, sl, ll = [], [], []
    for s in seqs:
        b, sl_, l = s.take_pending()
        bl.append(b[:-1])
        sl.append(sl_[:-1])
        ll.append(l)
        s.pend_bytes, s.pend_slots = b[-1:], sl_[-1:]
    r, keep = eng.rows(bl, sl, ll)
    B.blt_dec_prefill(h, nb, r)
    rounds: List[dict] = []
    k = wl.block
    rnd = 0

    def uniforms(call: int):
        # the engine reads them on its own stream: the copy completes first; callers keep the
        # tensor alive until the call's outputs have been read
        u = torch.from_numpy(np.stack([sampling_uniforms(wl.seed, wl.cfg_index, i, call, 2 * k + 1) for i in ids])).to(eng.device)
        torch.cuda.synchronize(eng.device)
        return u

    while any(len(s.out) < G for s in seqs):
        pend = [s.take_pending() for s in seqs]
        r, keep = eng.rows([p[0] for p in pend], [p[1] for p in pend], [p[2] for p in pend])
        u_d = uniforms(2 * rnd)
        samp = B.sampling(temperature, top_p, u_d)
        if wl.mode == "D":
            rule = B.BLT_UNMASK_EB if wl.unmask == "entropy" else B.BLT_UNMASK_CONFIDENCE
            thr = wl.gamma if wl.unmask == "entropy" else wl.alpha
            B.blt_dec_diffuse_block_sampled(h, nb, r, k, thr, rule, 0, samp, eng.d_out, eng.d_steps)
            blk = eng._get(eng.out_view(nb, k))
            for i, s in enumerate(seqs):
                new = [int(v) for v in blk[i]]
                s.commit(new)
                s.out += new
            if record:
                rounds.append(dict(block=blk.copy()))
        elif wl.mode in ("S", "DV"):
            mode = B.BLT_DRAFT_AR if wl.mode == "S" else B.BLT_DRAFT_DIFFUSION
            B.blt_dec_draft_sampled(h, nb, r, mode, k, wl.alpha, 0, samp, eng.d_out)
            draft = eng._get(eng.out_view(nb, k))
            vslots = np.zeros((nb, k), dtype=np.int32)
            prov: List[List[np.ndarray]] = []
            for i, s in enumerate(seqs):
                slots, lats, _ = s.patch(s.pstate, [int(v) for v in draft[i]])
                vslots[i] = slots
                prov.append(lats)
            lo = np.cumsum([0] + [len(p) for p in prov]).tolist()
            allp = [v for p in prov for v in p]
            dl = eng._put(eng.d_lat, np.stack(allp).astype(np.float32)) if allp else None
            dvs = eng._put(eng.d_vslots.view(-1), vslots.reshape(-1))
            u_v = uniforms(2 * rnd + 1)
            B.blt_dec_verify_sampled(h, dvs, dl, lo, B.sampling(temperature, top_p, u_v), eng.d_acc, eng.d_next)
            acc = eng._get(eng.d_acc[:nb])
            nxt = eng._get(eng.d_next[:nb])
            for i, s in enumerate(seqs):
                a = int(acc[i])
                new = [int(v) for v in draft[i, :a]] + [int(nxt[i])]
                s_slots, s_lats, st = s.patch(s.pstate, new)
                kept = (vslots[i, a - 1] + 1 - s.pstate.n_closed) if a >= 1 else 0
                s.pstate = st
                s.pend_bytes += new[a:]
                s.pend_slots += s_slots[a:]
                s.n_sent += kept
                s.lat_ready += s_lats[kept:]
                s.out += new
            if record:
                rounds.append(dict(draft=draft.copy(), accepted=acc.copy(), next=nxt.copy()))
        else:
            raise ValueError(f"sampled decoding has no mode {wl.mode}")
        rnd += 1
    st = B.blt_dec_sync(h)
    if st != 0:
        raise B.BltError(st, "generate_sampled", B.blt_dec_last_error(h))
    st1 = B.blt_dec_stats(h)
    return GenResult([s.out[:G] for s in seqs], rounds, {k_: st1[k_] - st0[k_] for k_ in st1}, time.perf_counter() - t0, 0, 0)
