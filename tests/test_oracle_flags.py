"""Worked cases for every near-tie flag the oracle raises.

The flags decide which divergences between the engine and the oracle the GPU
tests excuse, so each kind is pinned here on constructed logits (the decoder
pass is replaced by a fake that returns them):

* ``argmax``    a committed byte whose top-2 logit gap is below 0.05;
* ``threshold`` a masked position whose confidence is within 0.03 of alpha
  (confidence unmasking, "블록 언마스킹 전략");
* ``fallback``  no position reaches alpha and the two most confident masked
  positions are within 0.03;
* ``eb_bound``  EB sampling: a running entropy sum at the cut is within 0.05
  nats of gamma;
* ``eb_order``  EB sampling: the entropies on either side of the cut are
  within 0.05 nats.

Each kind has a case that must raise it and one that must not.
"""

from dataclasses import replace

import numpy as np
import pytest

from oracle.policies import NEAR_ALPHA, NEAR_EB, NEAR_TIE_GAP, OracleSequence, entropy
from workload import prefix_bytes

FLOOR = -1e3  # logits of the bytes outside a constructed distribution


def conf_row(conf: float, n: int = 2, top: int = 0) -> np.ndarray:
    """Logits whose softmax puts ``conf`` on byte ``top`` and splits the rest evenly
    over n - 1 other bytes (top-2 gap = ln((n - 1) conf / (1 - conf)))."""
    z = np.full(256, FLOOR)
    g = -np.log((1.0 / conf - 1.0) / (n - 1))
    others = [b for b in range(256) if b != top][: n - 1]
    z[top] = 0.0
    z[others] = -g
    return z


def tie_row(gap: float, top: int = 3) -> np.ndarray:
    """A top logit ``gap`` above the runner-up, both far above the rest."""
    z = np.full(256, FLOOR)
    z[top] = 0.0
    z[top + 1] = -gap
    return z


def flat_row(n: int, lift: float = 0.2, top: int = 0) -> np.ndarray:
    """n bytes at equal logits except the top one, ``lift`` higher: entropy just below ln n."""
    z = np.full(256, FLOOR)
    z[top : top + n] = 0.0
    z[top] = lift
    return z


def _seq(tiny, **kw):
    wl, ws, m = tiny
    s = OracleSequence(m, replace(wl, **kw), 0, [int(b) for b in prefix_bytes(0, 0, 0, 64)])
    s.prefill()  # the last prefix byte stays pending: it rides in the first pass
    return s


def _feed(s, passes):
    """Replace the decoder pass by constructed logits; every pass must use its rows."""
    it = iter(passes)

    def fake(rows):
        z = np.stack(next(it))
        assert z.shape == (len(rows), 256)
        s.c.passes += 1
        return z

    s._pass = fake


def _kinds(s):
    return sorted((f.what, f.pos) for f in s.flags)


def test_gap_of_the_constructions():
    assert abs(np.diff(np.sort(conf_row(0.7))[-2:])[0] - np.log(0.7 / 0.3)) < 1e-12
    z = tie_row(0.01)
    assert np.sort(z)[-1] - np.sort(z)[-2] == pytest.approx(0.01)


def test_threshold_and_argmax_flags(tiny):
    s = _seq(tiny, block=4, alpha=0.7)
    N = len(s.bytes)
    pend = tie_row(0.2)  # the pending row's prediction y_l: gap 0.2, no flag
    # pass 1: pos 0 at 0.71 (within 0.03 of alpha, committed), pos 1 at 0.9 (committed),
    # pos 2 at 0.68 (within 0.03, left masked), pos 3 at 0.2 (far below)
    p1 = [pend, conf_row(0.71), conf_row(0.9), conf_row(0.68), conf_row(0.2, n=6)]
    # pass 2: pos 2 at 0.6 (0.1 from alpha: no flag), pos 3 at 0.99 (committed)
    p2 = [conf_row(0.99), conf_row(0.99), conf_row(0.6), conf_row(0.99)]
    # pass 3: pos 2 alone, a near-tie argmax (gap 0.01) committed by the fallback
    p3 = [conf_row(0.99), conf_row(0.99), tie_row(0.01), conf_row(0.99)]
    _feed(s, [p1, p2, p3])
    block, steps, y_last = s.diffuse(4, 0.7)
    assert steps == 3 and y_last == 3
    assert block == [0, 0, 3, 0]
    assert _kinds(s) == [("argmax", N + 2), ("threshold", N + 0), ("threshold", N + 2)]


def test_argmax_flag_on_a_committed_near_tie(tiny):
    s = _seq(tiny, block=2, alpha=0.0)
    N = len(s.bytes)
    # y_l (pending row, predicts position N) gap 0.01; block row 0 (position N) gap 0.025;
    # block row 1 (position N + 1) gap 0.1
    _feed(s, [[tie_row(0.01), tie_row(NEAR_TIE_GAP / 2), tie_row(2 * NEAR_TIE_GAP)]])
    block, steps, y_last = s.diffuse(2, 0.0)
    assert steps == 1 and block == [3, 3] and y_last == 3
    assert _kinds(s) == [("argmax", N), ("argmax", N)]


def test_fallback_flag(tiny):
    # nobody reaches alpha; the two most confident masked positions are 0.01 apart -> flagged
    s = _seq(tiny, block=3, alpha=0.9)
    N = len(s.bytes)
    _feed(s, [[tie_row(1.0), conf_row(0.50, n=3), conf_row(0.51, n=3), conf_row(0.3, n=4)],
              [conf_row(0.99), conf_row(0.99), conf_row(0.99)]])
    block, steps, _ = s.diffuse(3, 0.9)
    assert steps == 2
    assert _kinds(s) == [("fallback", N + 1)]
    # the same with the two confidences 0.06 apart: no fallback flag
    t = _seq(tiny, block=3, alpha=0.9)
    _feed(t, [[tie_row(1.0), conf_row(0.50, n=3), conf_row(0.56, n=3), conf_row(0.3, n=4)],
              [conf_row(0.99), conf_row(0.99), conf_row(0.99)]])
    t.diffuse(3, 0.9)
    assert _kinds(t) == []
    # a single masked position left: the fallback has no competitor, no flag
    u = _seq(tiny, block=2, alpha=0.9)
    _feed(u, [[tie_row(1.0), conf_row(0.95), conf_row(0.5, n=3)], [conf_row(0.95), conf_row(0.5, n=3)]])
    _, steps, _ = u.diffuse(2, 0.9)
    assert steps == 2 and _kinds(u) == []


def _eb_rows():
    # entropies just below ln 2, ln 3, ln 5, ln 8 (distinct by > 0.05)
    rows = [flat_row(8), flat_row(2), flat_row(5), flat_row(3)]
    return rows, entropy(np.stack(rows))


def test_eb_bound_flag(tiny):
    rows, e = _eb_rows()
    order = np.argsort(e)  # 1, 3, 2, 0
    gamma = float(e[order[0]] + e[order[1]] + NEAR_EB / 2)  # the cut's running sum is within 0.05 of gamma
    s = _seq(tiny, block=4, alpha=0.0, unmask="entropy", gamma=gamma)
    N = len(s.bytes)
    _feed(s, [[tie_row(1.0)] + rows, rows, rows])
    block, steps, _ = s.diffuse(4, 0.0, unmask="entropy", gamma=gamma)
    assert ("eb_bound", N + int(order[1])) in _kinds(s)
    assert not any(k == "eb_order" for k, _ in _kinds(s))
    # gamma in the middle of the gap between the second and third running sums: no flag
    gamma2 = float(e[order[0]] + e[order[1]] + e[order[2]] / 2)
    t = _seq(tiny, block=4, alpha=0.0, unmask="entropy", gamma=gamma2)
    _feed(t, [[tie_row(1.0)] + rows, rows, rows])
    t.diffuse(4, 0.0, unmask="entropy", gamma=gamma2)
    assert not any(k in ("eb_bound", "eb_order") for k, _ in _kinds(t))


def test_eb_order_flag(tiny):
    # two positions whose entropies differ by 0.01 nats sit on either side of the cut
    a = flat_row(4, lift=0.20)
    b = flat_row(4, lift=0.23)
    lo = flat_row(2)
    e = entropy(np.stack([lo, a, b]))
    assert 0 < abs(e[1] - e[2]) < NEAR_EB
    gamma = float(e[0] + min(e[1], e[2]) + 0.3)  # takes lo and the lower of a, b; the other is next
    s = _seq(tiny, block=3, alpha=0.0, unmask="entropy", gamma=gamma)
    N = len(s.bytes)
    _feed(s, [[tie_row(1.0), lo, a, b], [lo, a, b]])
    s.diffuse(3, 0.0, unmask="entropy", gamma=gamma)
    nxt = 1 if e[1] > e[2] else 2
    assert ("eb_order", N + nxt) in _kinds(s)
    # entropies 0.5 nats apart: no order flag
    c = flat_row(6)
    e2 = entropy(np.stack([lo, a, c]))
    gamma2 = float(e2[0] + e2[1] + 0.3)
    t = _seq(tiny, block=3, alpha=0.0, unmask="entropy", gamma=gamma2)
    _feed(t, [[tie_row(1.0), lo, a, c], [lo, a, c]])
    t.diffuse(3, 0.0, unmask="entropy", gamma=gamma2)
    assert not any(k == "eb_order" for k, _ in _kinds(t))


def test_verify_flags_only_accepted_near_ties(tiny):
    """Verification flags the argmax of every accepted draft slot that is a near-tie."""
    s = _seq(tiny, block=3, alpha=0.0)
    l = len(s.bytes)
    # draft [3, 3, 9]: y_l = 3 (given), row 0 predicts 3 with gap 0.01 (accepted slot 1 is a
    # near-tie), row 1 predicts 5 (mismatch with draft[2] = 9: a = 2), row 2 is never used
    _feed(s, [[tie_row(0.01, top=3), tie_row(0.5, top=5), tie_row(0.01, top=7)]])
    a, nxt = s.verify([3, 3, 9], 3)
    assert (a, nxt) == (2, 5)
    kinds = _kinds(s)
    assert ("argmax", l + 1) in kinds
    assert ("argmax", l + 2) not in kinds  # gap 0.5
    assert ("argmax", l + 3) not in kinds  # beyond the accepted prefix


def test_flag_margins_are_the_stated_ones():
    assert NEAR_TIE_GAP == 0.05 and NEAR_ALPHA == 0.03 and NEAR_EB == 0.05
