"""fp64 decoder pass of the Fast-BLT local decoder (oracle; test infrastructure only).

Source: "Fast Byte Latent Transformer (Fast-BLT) 연구 소개" (discuss.pytorch.kr),

* section "계층적 BLT: 인코더, 글로벌 모델, 디코더", the layer equation
  ``B_l = D_{l-1} + W_o softmax(Q K^T / sqrt(d_k)) V``, ``D_l = DecoderTransformerLayer(B_l)``:
  a cross-attention from the byte stream to the latents O, then a transformer
  layer.
* section "BLT-D의 어텐션 마스크": which latent a row may attend to (exactly
  one), and the self-attention mask (clean prefix causal, masked block
  bidirectional and seeing the whole prefix).
* section "BLT-D 학습", block construction: every byte keeps its original
  position index for RoPE.

Readings (the pages do not say): pre-norm RMSNorm (eps 1e-5) before the
cross-attention query, the self-attention and the FFN, and before the byte
head; SwiGLU FFN ``W2 (silu(W1 x) * W3 x)``; rotate-half RoPE with theta 1e4 on
0-based positions; 256-way byte head (the [MASK] row is never predicted);
decoder input = embedding of the byte or [MASK] id.  Everything is float64;
weights are the (bf16- or fp32-) values the workload generator produced.
"""

from __future__ import annotations

from dataclasses import dataclass
from typing import Dict, List

import numpy as np

from workload import GLOBAL_TENSORS, LAYER_TENSORS, ModelShape, WeightSet

CAUSAL = "causal"
BLOCK = "block"


@dataclass(frozen=True)
class Row:
    """One query row of a decoder pass.

    ``byte``  input id (0..255, or the [MASK] id)
    ``pos``   0-based original byte position (RoPE, mask)
    ``lat``   0-based latent slot the row's cross-attention may see
    ``kind``  CAUSAL (clean prefix / draft / verify row) or BLOCK (masked block row)
    ``block_end`` for BLOCK rows: one past the last position of the block
    """

    byte: int
    pos: int
    lat: int
    kind: str
    block_end: int = -1


def may_attend(row: Row, key_pos: int) -> bool:
    """Self-attention mask of section "BLT-D의 어텐션 마스크".

    A clean-prefix (causal) row sees every position up to and including its
    own.  A masked-block row sees the whole clean prefix and every position of
    its block, in both directions.
    """
    if row.kind == CAUSAL:
        return key_pos <= row.pos
    return key_pos < row.block_end


def rmsnorm(x: np.ndarray, g: np.ndarray, eps: float) -> np.ndarray:
    """RMSNorm over the last axis: ``x / sqrt(mean(x^2) + eps) * g``."""
    return x / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps) * g


def silu(x: np.ndarray) -> np.ndarray:
    return x / (1.0 + np.exp(-x))


def rope(x: np.ndarray, pos: np.ndarray, theta: float) -> np.ndarray:
    """Rotate-half rotary embedding.

    ``x``: [..., n_heads, dh]; ``pos``: positions broadcastable to ``x[..., 0, 0]``.
    Pair ``(i, i + dh/2)`` of every head is rotated by angle
    ``pos * theta^(-2i/dh)``.
    """
    dh = x.shape[-1]
    half = dh // 2
    inv = theta ** (-np.arange(half, dtype=np.float64) * 2.0 / dh)
    ang = np.asarray(pos, dtype=np.float64)[..., None, None] * inv  # [..., 1, half]
    c, s = np.cos(ang), np.sin(ang)
    a, b = x[..., :half], x[..., half:]
    return np.concatenate([a * c - b * s, b * c + a * s], axis=-1)


class OracleModel:
    """Decoder weights widened to float64."""

    def __init__(self, shape: ModelShape, weights: WeightSet):
        self.shape = shape
        self.g: Dict[str, np.ndarray] = {n: weights.get(n).astype(np.float64) for n in GLOBAL_TENSORS}
        self.layers: List[Dict[str, np.ndarray]] = [
            {n: weights.get(n, l).astype(np.float64) for n in LAYER_TENSORS} for l in range(shape.n_layers)
        ]

    def n_params(self) -> int:
        tot = sum(a.size for a in self.g.values())
        for L in self.layers:
            tot += sum(a.size for a in L.values())
        return tot


class SeqState:
    """Per-sequence self-attention K/V by position, and latents by slot."""

    def __init__(self, shape: ModelShape, capacity: int):
        H, dh = shape.n_heads, shape.head_dim
        self.K = np.zeros((shape.n_layers, capacity, H, dh))
        self.V = np.zeros((shape.n_layers, capacity, H, dh))
        self.latents: List[np.ndarray] = []  # o_j, float64 [d_global]

    def ensure(self, n: int) -> None:
        if n > self.K.shape[1]:
            cap = max(n, 2 * self.K.shape[1])
            for name in ("K", "V"):
                old = getattr(self, name)
                new = np.zeros((old.shape[0], cap) + old.shape[2:])
                new[:, : old.shape[1]] = old
                setattr(self, name, new)


def cross_attention(m: OracleModel, L: Dict[str, np.ndarray], h: np.ndarray, rows: List[Row], st: SeqState) -> np.ndarray:
    """Cross-attention term of the layer equation, with the latent rule of
    section "BLT-D의 어텐션 마스크": a row's allowed latent set is ``{o_lat}``.

    Written as the literal multi-head softmax over the allowed latents.
    """
    sh = m.shape
    H, dh = sh.n_heads, sh.head_dim
    q = rmsnorm(h, L["norm_c"], sh.norm_eps) @ L["wq_c"].T  # [r, d]
    used = sorted({r.lat for r in rows})
    O = np.stack([st.latents[j] for j in used])  # [u, dg]
    kc = dict(zip(used, (O @ L["wk_c"].T).reshape(len(used), H, dh)))
    vc = dict(zip(used, (O @ L["wv_c"].T).reshape(len(used), H, dh)))
    out = np.zeros_like(h)
    for i, row in enumerate(rows):
        allowed = [row.lat]
        k = np.stack([kc[j] for j in allowed])  # [n_allowed, H, dh]
        v = np.stack([vc[j] for j in allowed])
        s = np.einsum("hd,nhd->hn", q[i].reshape(H, dh), k) / np.sqrt(dh)
        p = np.exp(s - s.max(axis=1, keepdims=True))
        p = p / p.sum(axis=1, keepdims=True)
        out[i] = np.einsum("hn,nhd->hd", p, v).reshape(-1)
    return out @ L["wo_c"].T


def self_attention(m: OracleModel, l: int, q: np.ndarray, rows: List[Row], st: SeqState) -> np.ndarray:
    """Masked softmax attention of every row over the K/V positions it may see.

    The mask is built from ``may_attend`` for every (row, position) pair; masked
    scores are -inf, so they get weight exactly 0.
    """
    sh = m.shape
    H, dh = sh.n_heads, sh.head_dim
    limit = max(max(r.pos for r in rows) + 1, max(r.block_end for r in rows))
    t = np.arange(limit)
    mask = np.stack([may_attend(r, t) for r in rows])  # [r, limit]
    K = st.K[l, :limit]  # [limit, H, dh]
    V = st.V[l, :limit]
    s = np.einsum("ihd,thd->hit", q, K) / np.sqrt(dh)
    s = np.where(mask[None], s, -np.inf)
    p = np.exp(s - s.max(axis=2, keepdims=True))
    p = p / p.sum(axis=2, keepdims=True)
    return np.einsum("hit,thd->ihd", p, V).reshape(len(rows), H * dh)


def decoder_pass(m: OracleModel, st: SeqState, rows: List[Row], want_hidden: bool = False):
    """Run every decoder layer over ``rows`` and return the 256 byte logits.

    Each row's K/V are written into ``st`` at the row's position before the
    layer's attention runs, so rows of this pass see one another as the mask
    allows.  Returns ``logits`` [r, 256] (and the final hidden state if asked).
    """
    sh = m.shape
    H, dh = sh.n_heads, sh.head_dim
    pos = np.array([r.pos for r in rows])
    st.ensure(max(int(pos.max()) + 1, max(r.block_end for r in rows)))
    h = m.g["embed"][np.array([r.byte for r in rows])]  # D_0  [r, d]
    for l, L in enumerate(m.layers):
        h = h + cross_attention(m, L, h, rows, st)  # B_l
        x = rmsnorm(h, L["attn_norm"], sh.norm_eps)
        qkv = x @ L["wqkv"].T
        d = sh.d_model
        q = rope(qkv[:, :d].reshape(-1, H, dh), pos, sh.rope_theta)
        k = rope(qkv[:, d : 2 * d].reshape(-1, H, dh), pos, sh.rope_theta)
        v = qkv[:, 2 * d :].reshape(-1, H, dh)
        st.K[l, pos] = k
        st.V[l, pos] = v
        h = h + self_attention(m, l, q, rows, st) @ L["wo"].T
        x = rmsnorm(h, L["ffn_norm"], sh.norm_eps)
        h = h + (silu(x @ L["w1"].T) * (x @ L["w3"].T)) @ L["w2"].T  # D_l
    z = rmsnorm(h, m.g["final_norm"], sh.norm_eps) @ m.g["head"][:256].T
    if want_hidden:
        return z, h
    return z


def dense_reference_pass(m: OracleModel, byte_ids: np.ndarray, lat: np.ndarray, mask: np.ndarray, latents: np.ndarray) -> np.ndarray:
    """Cache-free pass over a whole sequence with an explicit dense mask.

    ``mask[i, j]`` says whether row i may attend position j; ``lat[i]`` is the
    latent slot of row i; ``latents`` [M, dg].  Used to pin ``decoder_pass``
    (which caches K/V and applies the mask row by row) on tiny shapes.
    """
    sh = m.shape
    H, dh, d = sh.n_heads, sh.head_dim, sh.d_model
    n = len(byte_ids)
    pos = np.arange(n)
    h = m.g["embed"][byte_ids]
    scale = 1.0 / np.sqrt(dh)
    neg = np.where(mask, 0.0, -np.inf)
    for L in m.layers:
        q = rmsnorm(h, L["norm_c"], sh.norm_eps) @ L["wq_c"].T
        kc = (latents @ L["wk_c"].T).reshape(-1, H, dh)
        vc = (latents @ L["wv_c"].T).reshape(-1, H, dh)
        cmask = np.where(np.arange(len(latents))[None, :] == lat[:, None], 0.0, -np.inf)  # [n, M]
        s = np.einsum("nhd,mhd->hnm", q.reshape(n, H, dh), kc) * scale + cmask[None]
        p = np.exp(s - s.max(axis=2, keepdims=True))
        p /= p.sum(axis=2, keepdims=True)
        h = h + np.einsum("hnm,mhd->nhd", p, vc).reshape(n, d) @ L["wo_c"].T
        x = rmsnorm(h, L["attn_norm"], sh.norm_eps)
        qkv = x @ L["wqkv"].T
        q = rope(qkv[:, :d].reshape(n, H, dh), pos, sh.rope_theta)
        k = rope(qkv[:, d : 2 * d].reshape(n, H, dh), pos, sh.rope_theta)
        v = qkv[:, 2 * d :].reshape(n, H, dh)
        s = np.einsum("ihd,jhd->hij", q, k) * scale + neg[None]
        p = np.exp(s - s.max(axis=2, keepdims=True))
        p /= p.sum(axis=2, keepdims=True)
        h = h + np.einsum("hij,jhd->ihd", p, v).reshape(n, d) @ L["wo"].T
        x = rmsnorm(h, L["ffn_norm"], sh.norm_eps)
        h = h + (silu(x @ L["w1"].T) * (x @ L["w3"].T)) @ L["w2"].T
    return rmsnorm(h, m.g["final_norm"], sh.norm_eps) @ m.g["head"][:256].T
