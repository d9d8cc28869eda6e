"""Decoding rules of Fast-BLT on top of the fp64 decoder pass (oracle; test infrastructure only).

Source: "Fast Byte Latent Transformer (Fast-BLT) 연구 소개" (discuss.pytorch.kr):

* "BLT-D 추론": append B [MASK] ids to the clean prefix, run decoder passes
  that each fill 1..B masked positions until none is left, append the block,
  re-patch, repeat.  The clean prefix's K/V and the first latents are cached;
  only the current block (and the newest latent) is recomputed.
* "블록 언마스킹 전략", confidence-based unmasking: confidence is the largest
  predicted probability; every masked position whose confidence reaches the
  threshold alpha is committed; if none does, the single most confident one is.
* "블록 언마스킹 전략", entropy-bounded (EB) sampling: the masked positions are
  ordered by the entropy of their predicted distribution, lowest first, and
  the largest leading set whose summed entropy stays within the bound gamma
  is committed in one pass (the wangzhan123.com page, section on the two
  unmasking rules, says the same: accumulate in that order, stop once the
  running sum passes the bound).
* "BLT-S와 BLT-DV", the shared greedy verification: one causal pass over the
  draft gives greedy next-byte predictions y; draft byte i is accepted while
  it equals y_{i-1}; the first mismatch is replaced by the model's byte and the
  round stops; if every draft byte matches, one more (free) byte is taken.
* "BLT-S": the decoder keeps decoding autoregressively past the patch boundary
  up to a window of k bytes, then the draft is verified.
* "BLT-DV": the diffusion decoder fills a masked block (one step when alpha is
  0), then the same weights under a causal mask verify it.

The wangzhan123.com page (section "六、测量效能之方式") restates the proxy
bandwidth ``GB = b * [N_dec * P_dec + N_enc * (P_enc + P_global)] / 1e9`` with
b = 2 bytes (``proxy_gb``).

Readings (where the pages are silent): ``conf >= alpha`` commits; argmax ties
go to the lowest byte, fallback ties to the lowest position; committed
positions are never re-masked; block rows and BLT-S draft rows see the newest
closed latent; committed-but-uncached rows ride as causal rows in the next
pass; exactly ``G`` bytes are produced, the last block or round cut at ``G``.
EB sampling: entropy in nats over the 256 byte values (the mask id excluded,
as for the confidence); equal entropies are ordered by position; when even
the lowest entropy exceeds gamma, that one position is committed (so every
pass makes progress, as with the confidence fallback); committed bytes are the
greedy argmax.
"""

from __future__ import annotations

from dataclasses import dataclass, field
from typing import List, Optional, Tuple

import numpy as np

from workload import Patcher, PatchState, Workload, latent_vector

from .model import BLOCK, CAUSAL, OracleModel, Row, SeqState, decoder_pass
from .sampling import rejection_verify, sample_byte, tempered_top_p

NEAR_TIE_GAP = 0.05  # top-2 logit gap below which an argmax is a near-tie
NEAR_ALPHA = 0.03  # |conf - alpha| below which a threshold decision is a near-tie
NEAR_EB = 0.05  # nats: entropy or cumulative-entropy margin below which an EB decision is a near-tie


class StepLimit(RuntimeError):
    pass


def head_stats(z: np.ndarray):
    """Per row: confidence (largest softmax probability), argmax byte, top-2 logit gap."""
    zmax = z.max(axis=1)
    pred = np.argmax(z, axis=1)  # first maximum: lowest byte on ties
    conf = 1.0 / np.exp(z - zmax[:, None]).sum(axis=1)
    srt = np.sort(z, axis=1)
    gap = srt[:, -1] - srt[:, -2]
    return conf, pred, gap


def unmask_select(masked: List[int], conf: np.ndarray, alpha: float) -> Tuple[List[int], bool]:
    """Positions committed by one confidence-unmasking step, and whether the fallback fired."""
    chosen = [i for i in masked if conf[i] >= alpha]
    if chosen:
        return chosen, False
    best = masked[0]
    for i in masked[1:]:
        if conf[i] > conf[best]:
            best = i
    return [best], True


def entropy(z: np.ndarray) -> np.ndarray:
    """Per row: Shannon entropy (nats) of softmax(z) over the 256 byte logits."""
    zs = z - z.max(axis=1, keepdims=True)
    p = np.exp(zs)
    p /= p.sum(axis=1, keepdims=True)
    with np.errstate(divide="ignore", invalid="ignore"):
        t = np.where(p > 0, p * np.log(p), 0.0)
    return -t.sum(axis=1)


def eb_select(masked: List[int], ent: np.ndarray, gamma: float) -> Tuple[List[int], List[int], List[float]]:
    """Positions committed by one EB step: the masked positions sorted by entropy
    (position breaks ties), the longest leading run whose running sum of
    entropies is <= gamma, at least the first.  Also returns the order and the
    running sums (for near-tie flags)."""
    order = sorted(masked, key=lambda i: (float(ent[i]), i))
    cums, c = [], 0.0
    for i in order:
        c += float(ent[i])
        cums.append(c)
    n = 0
    while n < len(order) and cums[n] <= gamma:
        n += 1
    return order[: max(n, 1)], order, cums


def accept_length(draft: List[int], y: List[int]) -> Tuple[int, int]:
    """Greedy verification.  ``y[t]`` is the greedy prediction for draft slot t
    (``y[0]`` comes from the last committed byte).  Returns (accepted, next byte)."""
    a = 0
    while a < len(draft) and draft[a] == y[a]:
        a += 1
    return a, y[a]


def proxy_gb(n_dec: float, p_dec: float, n_enc: float, p_enc: float, p_global: float, b: int = 2) -> float:
    """Proxy memory bandwidth in GB: 16-bit parameter loads times forward passes."""
    return b * (n_dec * p_dec + n_enc * (p_enc + p_global)) / 1e9


@dataclass
class Flag:
    pos: int
    what: str  # "argmax" | "threshold" | "fallback"
    value: float


@dataclass
class Counters:
    passes: int = 0  # decoder forward passes (decoder NFE) after the prefill
    rows: int = 0
    prefill_rows: int = 0
    global_calls: int = 0  # encoder/global invocations that supply new latents


class OracleSequence:
    """One sequence decoded by the oracle."""

    def __init__(self, model: OracleModel, wl: Workload, seq: int, prefix: List[int]):
        self.m = model
        self.wl = wl
        self.seq = seq
        self.sh = wl.shape
        self.patcher = Patcher(wl.patch_kind, wl.seed, wl.cfg_index, seq)
        self.pstate = PatchState()
        self.bytes: List[int] = []
        self.lat: List[int] = []  # latent slot of every committed byte
        self.st = SeqState(self.sh, len(prefix) + wl.gen_bytes + 2 * wl.block + 8)
        self.cached = 0  # committed positions whose K/V are final
        self.c = Counters()
        self.flags: List[Flag] = []
        self.commit(prefix)

    # ----------------------------------------------------------- patching
    def _slots(self, closes: List[bool], n_closed_before: int) -> List[int]:
        """Latent rule of "BLT-D의 어텐션 마스크" for appended bytes.

        With patches numbered from 1, a byte of patch p attends o_{p-1}, except
        the last byte of a patch, which attends o_p.  Latent o_j is stored at
        0-based slot j-1.
        """
        out = []
        closed = n_closed_before
        for c in closes:
            p = closed + 1  # the patch this byte belongs to
            j = p if c else p - 1
            out.append(j - 1)
            if c:
                closed += 1
        return out

    @property
    def n_closed(self) -> int:
        return self.pstate.n_closed

    def _new_latents(self, per_byte, n_closed_before: int) -> List[np.ndarray]:
        out = []
        slot = n_closed_before
        for closes, fnv in per_byte:
            if closes:
                out.append(latent_vector(self.wl.seed, self.wl.cfg_index, self.seq, slot, fnv, self.sh.d_global).astype(np.float64))
                slot += 1
        return out

    def commit(self, new: List[int]) -> None:
        """Append committed bytes: re-patch, extend latents and latent slots."""
        if not new:
            return
        per_byte, st = self.patcher.advance(self.pstate, new)
        self.lat += self._slots([c for c, _ in per_byte], self.pstate.n_closed)
        self.st.latents += self._new_latents(per_byte, self.pstate.n_closed)
        self.bytes += [int(b) for b in new]
        self.pstate = st

    # ----------------------------------------------------------- passes
    def _pass(self, rows: List[Row]) -> np.ndarray:
        self.c.passes += 1
        self.c.rows += len(rows)
        return decoder_pass(self.m, self.st, rows)

    def _pending(self) -> List[Row]:
        return [Row(self.bytes[p], p, self.lat[p], CAUSAL) for p in range(self.cached, len(self.bytes))]

    def prefill(self, chunk: int = 512) -> None:
        """Cache K/V of every committed byte but the last (which rides in the next pass)."""
        end = len(self.bytes) - 1
        while self.cached < end:
            hi = min(end, self.cached + chunk)
            rows = [Row(self.bytes[p], p, self.lat[p], CAUSAL) for p in range(self.cached, hi)]
            decoder_pass(self.m, self.st, rows)
            self.c.prefill_rows += len(rows)
            self.cached = hi

    def _flag_argmax(self, pos: int, gap: float) -> None:
        if gap < NEAR_TIE_GAP:
            self.flags.append(Flag(pos, "argmax", float(gap)))

    # ----------------------------------------------------------- BLT-D
    def diffuse(self, B: int, alpha: float, max_steps: Optional[int] = None, unmask: str = "confidence", gamma: float = 0.0,
                samp: Optional[Tuple[float, float, List[float]]] = None):
        """Fill one masked block of B bytes; returns (block, steps, y_last).
        ``unmask`` selects confidence unmasking (threshold ``alpha``) or EB
        sampling (bound ``gamma``).

        ``y_last`` is the greedy prediction of the last pending committed row
        (None when no row was pending), used by BLT-DV verification.

        ``samp`` = (temperature, top_p, uniforms): the committed positions are
        chosen as above, their bytes drawn from the tempered top-p distribution
        of their rows with uniforms[i] for block position i (oracle.sampling);
        the distributions are kept in ``self.q_dists`` (per position) and the
        last pending row's in ``self.p0_dist``.
        """
        if samp is not None:
            self.q_dists = [None] * B
            self.p0_dist = None
        N = len(self.bytes)
        m_slot = self.n_closed - 1  # newest closed latent o_M
        mask_id = self.sh.mask_id
        pend = self._pending()
        block: List[Optional[int]] = [None] * B
        steps = 0
        y_last = None
        while any(b is None for b in block):
            steps += 1
            if max_steps is not None and steps > max_steps:
                raise StepLimit(f"block not filled after {max_steps} passes")
            rows = list(pend) if steps == 1 else []
            rows += [Row(mask_id if block[i] is None else block[i], N + i, m_slot, BLOCK, N + B) for i in range(B)]
            z = self._pass(rows)
            if steps == 1:
                self.cached = N
                if pend:
                    _, p_, g_ = head_stats(z[len(pend) - 1 : len(pend)])
                    y_last = int(p_[0])
                    if samp is None:
                        self._flag_argmax(N, float(g_[0]))
                    else:
                        self.p0_dist, cut = tempered_top_p(z[len(pend) - 1], samp[0], samp[1])
                        if cut < 2e-3:
                            self.flags.append(Flag(N, "top_p", cut))
            conf, pred, gap = head_stats(z[len(rows) - B :])
            masked = [i for i in range(B) if block[i] is None]
            if unmask == "entropy":
                ent = entropy(z[len(rows) - B :])
                chosen, order, cums = eb_select(masked, ent, gamma)
                n = len(chosen)
                # the cut could move: a running sum near gamma, or entropies near the cut close together
                for j in (n - 1, n):
                    if 0 <= j < len(order) and abs(cums[j] - gamma) < NEAR_EB:
                        self.flags.append(Flag(N + order[j], "eb_bound", float(cums[j] - gamma)))
                if n < len(order) and abs(float(ent[order[n]]) - float(ent[order[n - 1]])) < NEAR_EB:
                    self.flags.append(Flag(N + order[n], "eb_order", float(ent[order[n]] - ent[order[n - 1]])))
            else:
                chosen, fallback = unmask_select(masked, conf, alpha)
                for i in masked:
                    if abs(conf[i] - alpha) < NEAR_ALPHA:
                        self.flags.append(Flag(N + i, "threshold", float(conf[i])))
                if fallback and len(masked) > 1:
                    c = np.sort(conf[masked])
                    if c[-1] - c[-2] < NEAR_ALPHA:
                        self.flags.append(Flag(N + chosen[0], "fallback", float(c[-1] - c[-2])))
            for i in chosen:
                if samp is None:
                    self._flag_argmax(N + i, float(gap[i]))
                    block[i] = int(pred[i])
                else:
                    b, dist, kind, margin = sample_byte(z[len(rows) - B + i], samp[0], samp[1], samp[2][i])
                    if kind:
                        self.flags.append(Flag(N + i, kind, margin))
                    block[i] = b
                    self.q_dists[i] = dist
        return [int(b) for b in block], steps, y_last

    # ----------------------------------------------------------- AR
    def ar_step(self) -> int:
        N = len(self.bytes)
        z = self._pass(self._pending())
        self.cached = N
        _, pred, gap = head_stats(z[-1:])
        self._flag_argmax(N, float(gap[0]))
        return int(pred[0])

    # ----------------------------------------------------------- drafts + verification
    def speculative_slots(self, draft: List[int]):
        """Latent slots of draft bytes and the latents of patches they would close."""
        per_byte, _ = self.patcher.advance(self.pstate, draft)
        slots = self._slots([c for c, _ in per_byte], self.n_closed)
        return slots, self._new_latents(per_byte, self.n_closed)

    def verify(self, draft: List[int], y_last: int):
        """One causal pass over the draft, then the accept scan.  Returns (accepted, next byte)."""
        l = len(self.bytes)
        k = len(draft)
        slots, prov = self.speculative_slots(draft)
        n_lat = len(self.st.latents)
        self.st.latents += prov
        z = self._pass([Row(draft[t], l + t, slots[t], CAUSAL) for t in range(k)])
        del self.st.latents[n_lat:]
        _, pred, gap = head_stats(z)
        y = [y_last] + [int(v) for v in pred]
        a, nxt = accept_length(draft, y)
        for t in range(1, a + 1):
            self._flag_argmax(l + t, float(gap[t - 1]))
        self.cached = l + a  # the verify pass wrote the accepted rows' final K/V
        return a, nxt

    def verify_sampled(self, draft: List[int], q: List[np.ndarray], p0: np.ndarray, samp: Tuple[float, float, List[float]]):
        """One causal pass over the draft, then rejection sampling (oracle.sampling):
        targets p_0 = p0 and p_t = dist(verification row t - 1).  Returns (accepted, next byte)."""
        T, top_p, u = samp
        l = len(self.bytes)
        k = len(draft)
        slots, prov = self.speculative_slots(draft)
        n_lat = len(self.st.latents)
        self.st.latents += prov
        z = self._pass([Row(draft[t], l + t, slots[t], CAUSAL) for t in range(k)])
        del self.st.latents[n_lat:]
        ps = [p0]
        for t in range(k):
            d, cut = tempered_top_p(z[t], T, top_p)
            if cut < 2e-3:
                self.flags.append(Flag(l + t + 1, "top_p", cut))
            ps.append(d)
        a, nxt, fl = rejection_verify(draft, q, ps, u[:k], u[k : 2 * k + 1])
        for slot, kind, margin in fl:
            self.flags.append(Flag(l + slot, kind, margin))
        self.cached = l + a
        return a, nxt

    def blt_s_round_sampled(self, k: int, T: float, top_p: float, u_draft: List[float], u_verify: List[float]):
        """Self-speculation with drawn draft bytes, verified by rejection sampling."""
        l = len(self.bytes)
        m_slot = self.n_closed - 1
        N = len(self.bytes)
        z = self._pass(self._pending())
        self.cached = N
        draft, q = [], []
        for t in range(k):
            if t > 0:
                z = self._pass([Row(draft[-1], l + t - 1, m_slot, CAUSAL)])
            b, dist, kind, margin = sample_byte(z[-1], T, top_p, u_draft[t])
            if kind:
                self.flags.append(Flag(l + t, kind, margin))
            draft.append(b)
            q.append(dist)
        a, nxt = self.verify_sampled(draft, q, q[0], (T, top_p, u_verify))
        return draft, a, nxt

    def blt_dv_round_sampled(self, k: int, alpha: float, T: float, top_p: float, u_draft: List[float], u_verify: List[float]):
        """Diffusion draft with drawn bytes, verified by rejection sampling."""
        if len(self.bytes) == self.cached:
            raise ValueError("BLT-DV needs the last committed byte pending")
        draft, steps, _ = self.diffuse(k, alpha, samp=(T, top_p, u_draft))
        a, nxt = self.verify_sampled(draft, self.q_dists, self.p0_dist, (T, top_p, u_verify))
        return draft, a, nxt, steps

    def blt_s_round(self, k: int):
        """Self-speculation: k autoregressive draft bytes, then verification."""
        l = len(self.bytes)
        m_slot = self.n_closed - 1
        y_last = self.ar_step()
        draft = [y_last]
        for t in range(1, k):
            z = self._pass([Row(draft[-1], l + t - 1, m_slot, CAUSAL)])
            _, pred, gap = head_stats(z)
            self._flag_argmax(l + t, float(gap[0]))
            draft.append(int(pred[0]))
        a, nxt = self.verify(draft, y_last)
        return draft, a, nxt

    def blt_dv_round(self, k: int, alpha: float):
        """Diffusion draft of k bytes (one pass when alpha is 0), then verification."""
        if len(self.bytes) == self.cached:
            raise ValueError("BLT-DV needs the last committed byte pending")
        draft, steps, y_last = self.diffuse(k, alpha)
        a, nxt = self.verify(draft, y_last)
        return draft, a, nxt, steps

    # ----------------------------------------------------------- whole generation
    def generate(self, G: int, record: Optional[list] = None) -> List[int]:
        """Produce exactly G bytes with the workload's mode; returns them."""
        wl = self.wl
        out: List[int] = []
        while len(out) < G:
            if wl.mode == "D":
                new, steps, _ = self.diffuse(wl.block, wl.alpha, unmask=wl.unmask, gamma=wl.gamma)
                info = dict(steps=steps)
            elif wl.mode == "AR":
                new = [self.ar_step()]
                info = {}
            elif wl.mode == "S":
                draft, a, nxt = self.blt_s_round(wl.block)
                new = draft[:a] + [nxt]
                info = dict(draft=draft, accepted=a)
            elif wl.mode == "DV":
                draft, a, nxt, steps = self.blt_dv_round(wl.block, wl.alpha)
                new = draft[:a] + [nxt]
                info = dict(draft=draft, accepted=a, steps=steps)
            else:
                raise ValueError(wl.mode)
            new = new[: G - len(out)]
            if record is not None:
                info["bytes"] = list(new)
                info["start"] = len(self.bytes)
                record.append(info)
            self.commit(new)
            self.cached = min(self.cached, len(self.bytes))
            self.c.global_calls += 1
            out += new
        return out
