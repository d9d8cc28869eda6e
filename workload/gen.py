"""Synthetic decoder weights, prefixes, patch boundaries and latents.

All draws are keyed by integers (seed, stream id, config index, sequence,
position ...) through the counter-based SplitMix64 of :mod:`workload.rng`, so
any element can be regenerated independently and both the oracle and the
engine's host driver see the same numbers.

Recipe (the configs' stated distributions):

* weights ~ N(0, 1/d); byte head ~ N(0, (5/sqrt d)^2); RMSNorm gains 1
  (``gain_std`` > 0 draws gains 1 + N(0, gain_std^2) for stronger tests).
  Values are rounded fp64 -> fp32 (RNE), then fp32 -> bf16 (RNE) for bf16
  shapes; they are returned as float32 arrays holding exactly those values.
* prefix bytes uniform over 0..255.
* patch boundaries: a causal hazard process.  The boundary after byte ``j`` is
  decided from bytes ``<= j`` only: byte 0 always closes the first patch
  (one byte long); otherwise with run length ``r`` (bytes in the open patch,
  counting ``j``) the patch closes when ``u_j < T(r)``, ``u_j`` a 32-bit hash of
  (seed, config, sequence, j, x_j).  ``uniform8``: lengths uniform on 1..8,
  ``T(r) = floor(2^32 / (9 - r))``, forced at 8.  ``entropy12``: hazard 0.24,
  forced at 12 (mean length 4.01, range 1..12).
* latent ``o_j`` (0-based slot j = patch j+1 on the page's numbering) ~ N(0,1)
  of width ``d_global``, keyed by (seed, config, sequence, j, FNV-1a-64 of all
  bytes up to the end of that patch): a different patch history gives a
  different latent, which exposes stale-latent bugs.
"""

from __future__ import annotations

from dataclasses import dataclass
from typing import Dict, List, Sequence, Tuple

import numpy as np

from .configs import ModelShape
from .rng import FNV_OFFSET, derive_key, derive_keys, fnv1a64, normals, normals_many, round_bf16, stream, stream_int, uniform53

STREAM_WEIGHT = 1
STREAM_PREFIX = 2
STREAM_PATCH = 3
STREAM_LATENT = 4
STREAM_GAIN = 5
STREAM_SAMPLE = 6

# Per-layer tensors, PyTorch Linear layout [out, in].
LAYER_TENSORS = (
    "wq_c",  # [d, d]    cross-attn query (never needed: one key per row)
    "wk_c",  # [d, dg]   cross-attn key   (never needed: one key per row)
    "wv_c",  # [d, dg]   cross-attn value
    "wo_c",  # [d, d]    cross-attn output
    "norm_c",  # [d]     cross-attn query-side RMSNorm gain
    "attn_norm",  # [d]
    "wqkv",  # [3d, d]   rows: q (d), k (d), v (d); head h owns rows h*dh..h*dh+dh-1 of each
    "wo",  # [d, d]
    "ffn_norm",  # [d]
    "w1",  # [F, d]    SwiGLU gate
    "w3",  # [F, d]    SwiGLU up
    "w2",  # [d, F]    SwiGLU down
)
GLOBAL_TENSORS = ("embed", "head", "final_norm")  # [257, d], [257, d], [d]


def tensor_shape(shape: ModelShape, name: str) -> Tuple[int, ...]:
    d, dg, f, v = shape.d_model, shape.d_global, shape.d_ffn, shape.vocab
    return {
        "wq_c": (d, d),
        "wk_c": (d, dg),
        "wv_c": (d, dg),
        "wo_c": (d, d),
        "norm_c": (d,),
        "attn_norm": (d,),
        "wqkv": (3 * d, d),
        "wo": (d, d),
        "ffn_norm": (d,),
        "w1": (f, d),
        "w3": (f, d),
        "w2": (d, f),
        "embed": (v, d),
        "head": (v, d),
        "final_norm": (d,),
    }[name]


def _tensor_id(name: str, layer: int) -> int:
    if layer < 0:
        return 1 + GLOBAL_TENSORS.index(name)
    return 100 + 32 * layer + LAYER_TENSORS.index(name)


class WeightSet:
    """Lazily generated synthetic weights of one decoder (float32 arrays)."""

    def __init__(self, shape: ModelShape, seed: int = 0, gain_std: float = 0.0):
        self.shape = shape
        self.seed = seed
        self.gain_std = gain_std
        self._cache: Dict[Tuple[str, int], np.ndarray] = {}

    def get(self, name: str, layer: int = -1) -> np.ndarray:
        k = (name, layer)
        if k not in self._cache:
            self._cache[k] = self._make(name, layer)
        return self._cache[k]

    def layer(self, l: int) -> Dict[str, np.ndarray]:
        return {n: self.get(n, l) for n in LAYER_TENSORS}

    def materialize(self, names=None, threads: int = 0) -> "WeightSet":
        """Generate many tensors at once on a thread pool (numpy releases the GIL)."""
        import os
        from concurrent.futures import ThreadPoolExecutor

        names = LAYER_TENSORS if names is None else names
        keys = [(n, -1) for n in GLOBAL_TENSORS] + [(n, l) for l in range(self.shape.n_layers) for n in names]
        keys = [k for k in keys if k not in self._cache]
        with ThreadPoolExecutor(threads or min(16, os.cpu_count() or 1)) as ex:
            for k, arr in zip(keys, ex.map(lambda k: self._make(*k), keys)):
                self._cache[k] = arr
        return self

    def _make(self, name: str, layer: int) -> np.ndarray:
        sh = self.shape
        dims = tensor_shape(sh, name)
        n = int(np.prod(dims))
        tid = _tensor_id(name, layer)
        if name.endswith("norm") or name == "norm_c":
            if self.gain_std == 0.0:
                return np.ones(dims, dtype=np.float32)
            g = 1.0 + self.gain_std * normals(derive_key(self.seed, STREAM_GAIN, tid), n)
            w = g.astype(np.float32)
        else:
            std = (sh.head_std_mult if name == "head" else 1.0) / np.sqrt(sh.d_model)
            w = (std * normals(derive_key(self.seed, STREAM_WEIGHT, tid), n)).astype(np.float32)
        if sh.weight_dtype == "bf16":
            w = round_bf16(w)
        return w.reshape(dims)


def sampling_uniforms(seed: int, cfg_index: int, seq: int, call: int, n: int) -> np.ndarray:
    """``n`` uniforms in [0, 1) for stochastic decoding call ``call`` of sequence
    ``seq``, as float32 (both sides use exactly these values)."""
    u = uniform53(stream(derive_key(seed, STREAM_SAMPLE, cfg_index, seq, call), 0, n)).astype(np.float32)
    return np.minimum(u, np.float32(1.0 - 2.0**-24))


def prefix_bytes(seed: int, cfg_index: int, seq: int, n: int) -> np.ndarray:
    """``n`` prefix bytes, uniform over 0..255 (uint8)."""
    raw = stream(derive_key(seed, STREAM_PREFIX, cfg_index, seq), 0, n)
    return (raw >> np.uint64(56)).astype(np.uint8)


@dataclass(frozen=True)
class PatchState:
    """Patcher state after ``pos`` bytes."""

    pos: int = 0  # bytes seen
    run: int = 0  # bytes in the open patch
    fnv: int = FNV_OFFSET  # FNV-1a-64 of all bytes seen
    n_closed: int = 0  # closed patches


class Patcher:
    """Synthetic causal patcher standing in for BLT's entropy patcher."""

    def __init__(self, kind: str, seed: int, cfg_index: int, seq: int):
        if kind not in ("uniform8", "entropy12"):
            raise ValueError(kind)
        self.kind = kind
        self.key = derive_key(seed, STREAM_PATCH, cfg_index, seq)

    def _threshold(self, run: int) -> int:
        if self.kind == "uniform8":
            return 1 << 32 if run >= 8 else (1 << 32) // (9 - run)
        return 1 << 32 if run >= 12 else 1030792151  # floor(0.24 * 2^32)

    def _u32(self, j: int, b: int) -> int:
        k = (self.key ^ (int(b) & 0xFF)) & 0xFFFFFFFFFFFFFFFF
        return stream_int(k, j) >> 32

    def advance(self, st: PatchState, data: Sequence[int]) -> Tuple[List[Tuple[bool, int]], PatchState]:
        """Patch ``data`` appended after state ``st``.

        Returns per byte ``(closes_patch, fnv_after_byte)`` and the new state.
        Pure: the same state and bytes always give the same answer.
        """
        pos, run, fnv, n_closed = st.pos, st.run, st.fnv, st.n_closed
        out = []
        for b in data:
            fnv = fnv1a64(fnv, (b,))
            run += 1
            closes = pos == 0 or self._u32(pos, b) < self._threshold(run)
            out.append((closes, fnv))
            if closes:
                n_closed += 1
                run = 0
            pos += 1
        return out, PatchState(pos, run, fnv, n_closed)


def latent_vector(seed: int, cfg_index: int, seq: int, slot: int, fnv: int, d_global: int) -> np.ndarray:
    """Latent for 0-based slot ``slot`` closed with content hash ``fnv`` (float32)."""
    return latent_vectors(seed, cfg_index, seq, [slot], [fnv], d_global)[0]


def latent_vectors(seed: int, cfg_index: int, seq: int, slots: Sequence[int], fnvs: Sequence[int], d_global: int) -> np.ndarray:
    """``latent_vector`` for every (slot, fnv) pair at once: float32 [n, d_global]."""
    if len(slots) == 0:
        return np.zeros((0, d_global), dtype=np.float32)
    keys = derive_keys(seed, STREAM_LATENT, cfg_index, seq, list(slots), list(fnvs))
    return normals_many(keys, d_global).astype(np.float32)
