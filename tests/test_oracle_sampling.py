"""Pins of the oracle's stochastic decoding rules (oracle/sampling.py), on the CPU.

Each test checks the oracle against something other than its own formulas: a
library softmax, hand-worked distributions, the zero-temperature limit, and the
defining property of rejection sampling (the emitted byte is distributed as the
target, whatever the draft distribution), measured by Monte Carlo.
"""

import numpy as np
import pytest
from scipy.special import softmax

from oracle.sampling import draw, rejection_verify, sample_byte, tempered_top_p


def _logits_for(probs: dict) -> np.ndarray:
    """Logits whose softmax puts exactly `probs` on the listed bytes (others ~0)."""
    z = np.full(256, -1e4)
    for b, p in probs.items():
        z[b] = np.log(p)
    return z


def test_full_top_p_at_unit_temperature_is_softmax():
    rng = np.random.default_rng(1)
    z = rng.normal(0, 3, 256)
    dist, _ = tempered_top_p(z, 1.0, 1.0)
    assert np.allclose(dist, softmax(z), atol=1e-15, rtol=1e-12)


def test_temperature_scales_logits():
    rng = np.random.default_rng(2)
    z = rng.normal(0, 2, 256)
    dist, _ = tempered_top_p(z, 0.5, 1.0)
    assert np.allclose(dist, softmax(2.0 * z), atol=1e-15, rtol=1e-12)


def test_top_p_worked_example():
    # byte 7: 0.5, byte 3: 0.3, byte 200: 0.15, byte 0: 0.05 (ranked 7, 3, 200, 0)
    z = _logits_for({7: 0.5, 3: 0.3, 200: 0.15, 0: 0.05})
    d, _ = tempered_top_p(z, 1.0, 0.7)
    assert np.isclose(d[7], 0.5 / 0.8) and np.isclose(d[3], 0.3 / 0.8) and d[200] == 0 and d[0] == 0
    d, _ = tempered_top_p(z, 1.0, 0.85)
    assert np.isclose(d[200], 0.15 / 0.95) and d[0] == 0
    d, _ = tempered_top_p(z, 1.0, 0.4)  # the top byte alone reaches 0.4
    assert d[7] == 1.0 and d.sum() == 1.0
    d, margin = tempered_top_p(z, 1.0, 0.8)  # the cut falls on 0.5 + 0.3: a near-tie
    assert margin < 1e-9


def test_zero_temperature_limit_is_argmax():
    rng = np.random.default_rng(3)
    for _ in range(20):
        z = rng.normal(0, 1, 256)
        d, _ = tempered_top_p(z, 1e-4, 0.9)
        for u in (0.0, 0.3, 0.999999):
            assert draw(d, u)[0] == int(np.argmax(z))


def test_inverse_cdf_worked_example():
    d = np.zeros(256)
    d[0], d[1], d[2] = 0.2, 0.5, 0.3
    assert draw(d, 0.1)[0] == 0
    assert draw(d, 0.2)[0] == 1  # the smallest b with cdf[b] > u
    assert draw(d, 0.69)[0] == 1
    assert draw(d, 0.7)[0] == 2
    assert draw(d, 0.999999)[0] == 2
    assert draw(d, 0.7)[1] < 1e-12  # u on a boundary: margin 0


def test_rejection_sampling_emits_the_target_distribution():
    """Whatever q is, the first byte a verification round emits (the draft byte if
    accepted, else the redrawn byte) is distributed as p."""
    rng = np.random.default_rng(4)
    support = [5, 17, 99, 128, 200, 255]
    p = np.zeros(256)
    q = np.zeros(256)
    p[support] = rng.dirichlet(np.ones(6))
    q[support[1:]] = rng.dirichlet(np.ones(5))  # q misses byte 5 entirely
    n = 200_000
    u = rng.random((n, 3))
    counts = np.zeros(256)
    for i in range(n):
        x, _ = draw(q, u[i, 0])
        a, nxt, _ = rejection_verify([x], [q], [p, p], [u[i, 1]], [u[i, 2], 0.5])
        counts[x if a == 1 else nxt] += 1
    emp = counts / n
    sigma = np.sqrt(p * (1 - p) / n)
    assert np.all(np.abs(emp - p) <= 5 * sigma + 1e-12), (emp[support], p[support])


def test_rejection_sampling_accepts_everything_when_draft_equals_target():
    rng = np.random.default_rng(5)
    k = 6
    p = [rng.dirichlet(np.ones(256)) for _ in range(k + 1)]
    draft = [int(np.argmax(pi)) for pi in p[:k]]
    ud = list(rng.random(k + 1))
    a, nxt, _ = rejection_verify(draft, p[:k], p, list(rng.random(k) * 0.999), ud)
    assert a == k and nxt == draw(p[k], ud[k])[0]


def test_rejection_sampling_rejects_bytes_the_target_excludes():
    q = np.zeros(256)
    p = np.zeros(256)
    q[10], q[20] = 0.5, 0.5
    p[20], p[30] = 0.5, 0.5
    # byte 10 has target probability 0: rejected for any u; the redraw is from
    # max(p - q, 0) = {30: 0.5} -> byte 30
    for u in (0.0, 0.5, 0.999):
        a, nxt, _ = rejection_verify([10], [q], [p, p], [u], [0.3, 0.3])
        assert (a, nxt) == (0, 30)
    # byte 20: ratio min(1, 0.5 / 0.5) = 1, always accepted; the extra byte comes from p
    a, nxt, _ = rejection_verify([20], [q], [p, p], [0.999], [0.1, 0.75])
    assert (a, nxt) == (1, 30)


def test_near_tie_flags():
    q = np.zeros(256)
    p = np.zeros(256)
    q[1], q[2] = 0.8, 0.2
    p[1], p[2] = 0.4, 0.6
    # ratio for byte 1 = 0.5: a uniform next to it is flagged
    a, nxt, flags = rejection_verify([1], [q], [p, p], [0.5 + 1e-4], [0.1, 0.1])
    assert any(f[1] == "accept" for f in flags)
    b, dist, kind, margin = sample_byte(_logits_for({3: 0.25, 4: 0.75}), 1.0, 1.0, 0.25 + 1e-5)
    assert kind == "draw" and b == 4
