"""Counter-based random numbers for the synthetic workload.

SplitMix64 (Steele, Lea & Flood, "Fast splittable pseudorandom number
generators", OOPSLA 2014; the 64-bit finaliser constants as published by
S. Vigna) is used in counter mode: element ``i`` of a stream with key ``K`` is
``mix64(K + (i + 1) * GAMMA)``, i.e. the (i+1)-th output of a SplitMix64
generator seeded with ``K``.  Keys are derived by chaining ``mix64`` over a
tuple of integers.  Normals use the Box-Muller transform (Box & Muller, 1958).

Everything is vectorised numpy on uint64 with wrap-around arithmetic.
"""

from __future__ import annotations

import numpy as np

GAMMA = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)
_S30 = np.uint64(30)
_S27 = np.uint64(27)
_S31 = np.uint64(31)
_S11 = np.uint64(11)
_TWO_M53 = 2.0 ** -53


def mix64(z: np.ndarray) -> np.ndarray:
    """SplitMix64 output function on a uint64 array (wraps mod 2**64)."""
    z = np.asarray(z, dtype=np.uint64)
    with np.errstate(over="ignore"):
        z = (z ^ (z >> _S30)) * _M1
        z = (z ^ (z >> _S27)) * _M2
    return z ^ (z >> _S31)


_MASK = 0xFFFFFFFFFFFFFFFF


def mix64_int(z: int) -> int:
    """``mix64`` of one value in Python integers (exact, same result as the array form)."""
    z &= _MASK
    z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & _MASK
    z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & _MASK
    return z ^ (z >> 31)


def stream_int(key: int, i: int) -> int:
    """Element ``i`` of the counter stream ``key`` (one value, Python integers)."""
    return mix64_int(key + (i + 1) * 0x9E3779B97F4A7C15)


def derive_key(*words: int) -> int:
    """Chain ``mix64`` over integer words into one 64-bit stream key."""
    h = 0
    for w in words:
        h = mix64_int(((h ^ (int(w) & _MASK)) + 0x9E3779B97F4A7C15) & _MASK)
    return h


def derive_keys(*columns) -> np.ndarray:
    """``derive_key`` over rows of words: column ``j`` holds word ``j`` of every key
    (ints broadcast).  Elementwise the same operations as ``derive_key``."""
    n = max((len(c) for c in columns if not np.isscalar(c)), default=1)
    if n <= 8:  # a few keys: Python integers are faster than numpy's per-call overhead
        return np.asarray([derive_key(*[c if np.isscalar(c) else c[i] for c in columns]) for i in range(n)], dtype=np.uint64)
    h = np.zeros(n, dtype=np.uint64)
    with np.errstate(over="ignore"):
        for c in columns:
            if np.isscalar(c):
                w = np.uint64(int(c) & 0xFFFFFFFFFFFFFFFF)  # broadcast: the same word for every key
            else:
                w = np.asarray([int(v) & 0xFFFFFFFFFFFFFFFF for v in c], dtype=np.uint64)
            h = mix64((h ^ w) + GAMMA)
    return h


def stream(key: int, start: int, count: int) -> np.ndarray:
    """Elements ``start .. start+count-1`` of the counter stream ``key``."""
    i = np.arange(start + 1, start + count + 1, dtype=np.uint64)
    with np.errstate(over="ignore"):
        return mix64(np.uint64(key) + i * GAMMA)


def uniform53(x: np.ndarray) -> np.ndarray:
    """Top 53 bits of a uint64 as a float64 in [0, 1)."""
    return (x >> _S11).astype(np.float64) * _TWO_M53


def normals(key: int, count: int) -> np.ndarray:
    """``count`` standard normals (float64) from stream ``key``.

    Pair ``p`` uses stream elements ``2p`` and ``2p+1``:
    ``r = sqrt(-2 ln(1 - u_a))``, ``t = 2 pi u_b``; element ``2p`` is
    ``r cos t`` and element ``2p+1`` is ``r sin t``.
    """
    return normals_many(np.asarray([key], dtype=np.uint64), count)[0]


def normals_many(keys: np.ndarray, count: int) -> np.ndarray:
    """``normals`` of every key in ``keys`` at once: float64 [len(keys), count].

    The float64 transform runs in torch on the host cores (multi-threaded);
    every element is computed by the same routine whatever the batch size or
    thread count, so a value never depends on how it was requested."""
    import torch

    keys = np.asarray(keys, dtype=np.uint64).reshape(-1, 1)
    npair = (count + 1) // 2
    i = np.arange(1, 2 * npair + 1, dtype=np.uint64).reshape(1, -1)
    with np.errstate(over="ignore"):
        raw = mix64(keys + i * GAMMA).reshape(keys.shape[0], npair, 2)
    u1 = torch.from_numpy(1.0 - uniform53(raw[:, :, 0]))  # (0, 1]
    u2 = torch.from_numpy(uniform53(raw[:, :, 1]))
    r = torch.sqrt(-2.0 * torch.log(u1))
    t = (2.0 * np.pi) * u2
    out = torch.stack([r * torch.cos(t), r * torch.sin(t)], dim=2)
    return out.reshape(keys.shape[0], -1)[:, :count].numpy()


def round_bf16(x: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bfloat16 (ties to even); float32 out."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32).astype(np.uint64)
    u = (u + np.uint64(0x7FFF) + ((u >> np.uint64(16)) & np.uint64(1))) & np.uint64(0xFFFF0000)
    return u.astype(np.uint32).view(np.float32)


def fnv1a64(h: int, data) -> int:
    """FNV-1a 64-bit hash continued from state ``h`` over the byte values in ``data``."""
    prime = 0x100000001B3
    for b in data:
        h ^= int(b) & 0xFF
        h = (h * prime) & 0xFFFFFFFFFFFFFFFF
    return h


FNV_OFFSET = 0xCBF29CE484222325
