"""Stochastic decoding rules: temperature / top-p sampling and rejection-sampling
verification (oracle; test infrastructure only).

Source: "Fast Byte Latent Transformer (Fast-BLT) 연구 소개" (discuss.pytorch.kr):

* "블록 언마스킹 전략": entropy-bounded unmasking can be combined with top-p
  sampling to make generation diverse (the positions to commit are chosen as in
  the greedy rules; the committed bytes are drawn instead of taken as argmax).
* "BLT-S와 BLT-DV": verification as described accepts draft bytes that equal the
  greedy prediction; for non-zero temperature it extends through rejection
  sampling (only the greedy setting is evaluated on the page).

The pages give no formulas for either, so this module writes out the standard
definitions (readings listed in the design notes):

* ``tempered_top_p``: p = softmax(z / T) over the 256 byte logits; the bytes are
  ranked by p (ties: the lower byte first), the shortest leading run whose
  cumulative probability reaches ``top_p`` is kept, and the kept
  probabilities are renormalised.
* ``draw``: inverse-CDF sampling over byte values 0..255 in increasing order:
  the smallest byte b with ``cumsum(dist)[b] > u``.
* ``rejection_verify``: speculative sampling.  Draft byte x_i was drawn from
  the draft distribution q_i; the verification pass gives the target p_i for
  the same slot (slot i is predicted from the row before it, as in greedy
  verification).  x_i is accepted when ``u_i < min(1, p_i(x_i) / q_i(x_i))``;
  at the first rejection the next byte is drawn from ``max(p_i - q_i, 0)``
  renormalised, and the round stops; when all k are accepted, one more byte is
  drawn from p_k.  The emitted bytes are then distributed exactly as
  sampling from the targets one by one.

Every random number is an input: the uniforms come from the workload's seeded
generator (``workload.sampling_uniforms``), the same ones the engine uses.
Near-tie flags mark decisions that fp32 and fp64 may take differently: a
uniform within ``NEAR_U`` of a CDF boundary or of the acceptance ratio, or a
top-p cut whose cumulative sum is within ``NEAR_P`` of ``top_p``.
"""

from __future__ import annotations

from typing import List, Optional, Sequence, Tuple

import numpy as np

NEAR_U = 2e-3  # uniform vs boundary margin below which a sampling decision is a near-tie
NEAR_P = 2e-3  # cumulative-probability margin of a top-p cut below which it is a near-tie


def tempered_top_p(z: np.ndarray, temperature: float, top_p: float) -> Tuple[np.ndarray, float]:
    """Distribution over the 256 byte values for logits z (fp64), and the margin of
    the top-p cut (how far the cumulative sums next to the cut are from top_p)."""
    z = np.asarray(z, dtype=np.float64)[:256]
    t = z / temperature
    t = t - t.max()
    p = np.exp(t)
    p /= p.sum()
    order = sorted(range(256), key=lambda b: (-p[b], b))
    cum = 0.0
    n = 0
    margin = np.inf
    while n < 256:
        prev = cum
        cum += p[order[n]]
        n += 1
        if cum >= top_p:
            margin = min(abs(cum - top_p), abs(prev - top_p) if n > 1 else np.inf)
            break
    keep = np.zeros(256)
    for b in order[:n]:
        keep[b] = p[b]
    return keep / keep.sum(), float(margin)


def draw(dist: np.ndarray, u: float) -> Tuple[int, float]:
    """Inverse-CDF draw over byte values in increasing order: the smallest b with
    cdf[b] > u.  Also returns the distance from u to the nearest CDF boundary
    among the bytes with non-zero probability."""
    cdf = np.cumsum(np.asarray(dist, dtype=np.float64))
    b = int(np.searchsorted(cdf, u, side="right"))
    b = min(b, 255)
    while dist[b] == 0.0 and b > 0:  # u at or past the total mass (rounding): the last byte with mass
        b -= 1
    nz = np.nonzero(dist)[0]
    bounds = cdf[nz]
    return b, float(np.min(np.abs(bounds - u)))


def rejection_verify(draft: Sequence[int], q: Sequence[np.ndarray], p: Sequence[np.ndarray], u_acc: Sequence[float],
                     u_draw: Sequence[float]) -> Tuple[int, int, List[Tuple[int, str, float]]]:
    """Speculative-sampling verification of k draft bytes.

    q[i]: the draft distribution x_i was drawn from; p[i] (i = 0..k): the target
    distribution of slot i; u_acc[i]: the acceptance uniform of slot i;
    u_draw[i] (i = 0..k): the uniform of the byte drawn at slot i after a
    rejection there (or of the extra byte when i = k).  Returns (accepted,
    next byte, near-tie flags as (slot, kind, margin))."""
    k = len(draft)
    flags: List[Tuple[int, str, float]] = []
    for i in range(k):
        x = int(draft[i])
        qi, pi = np.asarray(q[i], np.float64), np.asarray(p[i], np.float64)
        ratio = 1.0 if qi[x] <= 0.0 else min(1.0, pi[x] / qi[x])
        if ratio < 1.0 and abs(u_acc[i] - ratio) < NEAR_U:
            flags.append((i, "accept", abs(u_acc[i] - ratio)))
        if u_acc[i] < ratio:
            continue
        res = np.maximum(pi - qi, 0.0)
        s = res.sum()
        res = pi if s <= 0.0 else res / s
        b, m = draw(res, u_draw[i])
        if m < NEAR_U:
            flags.append((i, "draw", m))
        return i, b, flags
    b, m = draw(np.asarray(p[k], np.float64), u_draw[k])
    if m < NEAR_U:
        flags.append((k, "draw", m))
    return k, b, flags


def sample_byte(z: np.ndarray, temperature: float, top_p: float, u: float) -> Tuple[int, np.ndarray, Optional[str], float]:
    """One sampled byte from logits z: (byte, the distribution it was drawn from,
    near-tie kind or None, margin)."""
    dist, cut = tempered_top_p(z, temperature, top_p)
    b, m = draw(dist, u)
    if cut < NEAR_P:
        return b, dist, "top_p", cut
    if m < NEAR_U:
        return b, dist, "draw", m
    return b, dist, None, min(m, cut)
