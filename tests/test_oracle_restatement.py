"""Second, independent statement of one decoder pass, in torch fp64, pinning the
oracle's layer composition.

The oracle (``oracle.model.decoder_pass``) is the decoder of "Fast Byte Latent
Transformer (Fast-BLT) 연구 소개", section "계층적 BLT: 인코더, 글로벌 모델,
디코더" (``B_l = D_{l-1} + W_o softmax(QK^T/sqrt(d_k)) V``, then the transformer
layer), with the masks of section "BLT-D의 어텐션 마스크" and original byte
positions for RoPE (section "BLT-D 학습").  The layer internals are readings:
pre-norm RMSNorm before the cross-attention query, the self-attention, the FFN
and the byte head; a SwiGLU FFN ``W2 (silu(W1 x) * W3 x)``; rotate-half RoPE.

This file restates that pass with library operators only
(``torch.nn.functional.linear``, ``rms_norm``, ``silu``,
``scaled_dot_product_attention``), the cross-attention as a literal multi-head
attention over every latent with a one-hot mask, RoPE as a complex rotation of
the pairs (i, i + dh/2), and the self-attention mask built from the page's
rule.  It shares no helper with the oracle.  Planted mistakes in the oracle
(W1/W3 swapped, the pre-FFN norm dropped, the RoPE pairing changed) must make
the two disagree.
"""

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle.model as om_mod
from oracle.model import BLOCK, CAUSAL, OracleModel, Row, SeqState, decoder_pass
from oracle.policies import OracleSequence
from workload import CONFIGS, WeightSet, prefix_bytes

TOL = 1e-12


def _t(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float64))


def _rope_complex(x, pos, theta):
    """x [n, H, dh]: the pair (i, i + dh/2) is the complex number x_i + j x_{i+dh/2},
    rotated by pos * theta^(-2i/dh)."""
    dh = x.shape[-1]
    half = dh // 2
    inv = theta ** (-torch.arange(half, dtype=torch.float64) * 2.0 / dh)
    z = torch.complex(x[..., :half], x[..., half:])
    rot = torch.polar(torch.ones(len(pos), half, dtype=torch.float64), pos[:, None].to(torch.float64) * inv[None, :])
    z = z * rot[:, None, :]
    return torch.cat([z.real, z.imag], dim=-1)


def torch_pass(model: OracleModel, ids, pos, lat, allowed, latents):
    """Cache-free decoder pass over every row at once; ``allowed[i, j]``: row i may see position j."""
    sh = model.shape
    d, H, dh, eps = sh.d_model, sh.n_heads, sh.head_dim, sh.norm_eps
    n = len(ids)
    O = _t(latents)
    M = O.shape[0]
    pos_t = torch.as_tensor(pos)
    h = _t(model.g["embed"])[torch.as_tensor(ids)]
    one_latent = torch.arange(M)[None, :] == torch.as_tensor(lat)[:, None]  # [n, M]
    self_mask = torch.as_tensor(allowed)
    for L in model.layers:
        W = {k: _t(v) for k, v in L.items()}
        # cross-attention: literal multi-head attention over the latents, one allowed per row
        qc = F.linear(F.rms_norm(h, (d,), W["norm_c"], eps), W["wq_c"]).view(n, H, dh).transpose(0, 1)
        kc = F.linear(O, W["wk_c"]).view(M, H, dh).transpose(0, 1)
        vc = F.linear(O, W["wv_c"]).view(M, H, dh).transpose(0, 1)
        ca = F.scaled_dot_product_attention(qc, kc, vc, attn_mask=one_latent)
        h = h + F.linear(ca.transpose(0, 1).reshape(n, d), W["wo_c"])
        # pre-norm self-attention
        x = F.rms_norm(h, (d,), W["attn_norm"], eps)
        q, k, v = F.linear(x, W["wqkv"]).split(d, dim=-1)
        q = _rope_complex(q.reshape(n, H, dh), pos_t, sh.rope_theta)
        k = _rope_complex(k.reshape(n, H, dh), pos_t, sh.rope_theta)
        a = F.scaled_dot_product_attention(q.transpose(0, 1), k.transpose(0, 1), v.reshape(n, H, dh).transpose(0, 1), attn_mask=self_mask)
        h = h + F.linear(a.transpose(0, 1).reshape(n, d), W["wo"])
        # pre-norm SwiGLU FFN
        x = F.rms_norm(h, (d,), W["ffn_norm"], eps)
        h = h + F.linear(F.silu(F.linear(x, W["w1"])) * F.linear(x, W["w3"]), W["w2"])
    z = F.linear(F.rms_norm(h, (d,), _t(model.g["final_norm"]), eps), _t(model.g["head"])[:256])
    return z.numpy()


def _case(wl, model, B=4, seq=0):
    """A whole sequence in one pass: the clean prefix (causal) and a masked block of B."""
    o = OracleSequence(model, wl, seq, [int(b) for b in prefix_bytes(wl.seed, wl.cfg_index, seq, wl.prefix_len)])
    N = len(o.bytes)
    m_slot = o.n_closed - 1
    ids = o.bytes + [wl.shape.mask_id] * B
    lat = o.lat + [m_slot] * B
    pos = list(range(N + B))
    rows = [Row(o.bytes[p], p, o.lat[p], CAUSAL) for p in range(N)] + [Row(wl.shape.mask_id, N + i, m_slot, BLOCK, N + B) for i in range(B)]
    allowed = np.zeros((N + B, N + B), dtype=bool)
    for i in range(N + B):
        for j in range(N + B):
            allowed[i, j] = j <= i if i < N else j < N + B  # prefix causal; block sees the prefix and the whole block
    return rows, np.array(ids), np.array(pos), np.array(lat), allowed, np.stack(o.st.latents), N + B


def _oracle(model, wl, rows, latents, cap):
    st = SeqState(wl.shape, cap)
    st.latents = [v for v in latents]
    return decoder_pass(model, st, rows)


@pytest.fixture(scope="module")
def tiny_gains():
    wl = CONFIGS["tiny_d4"]
    ws = WeightSet(wl.shape, seed=0, gain_std=0.1).materialize()
    return wl, ws, OracleModel(wl.shape, ws)


def test_decoder_pass_equals_torch_restatement(tiny_gains):
    wl, ws, model = tiny_gains
    rows, ids, pos, lat, allowed, latents, cap = _case(wl, model)
    z_or = _oracle(model, wl, rows, latents, cap)
    z_t = torch_pass(model, ids, pos, lat, allowed, latents)
    assert z_or.shape == z_t.shape == (len(rows), 256)
    err = np.abs(z_or - z_t).max()
    assert err < TOL, err
    assert np.abs(z_t).max() > 1.0  # non-trivial logits


def test_restatement_separates_layer_mistakes(tiny_gains, monkeypatch):
    """Mistakes planted in the oracle fail the comparison by far more than its tolerance."""
    wl, ws, model = tiny_gains
    rows, ids, pos, lat, allowed, latents, cap = _case(wl, model)
    z_t = torch_pass(model, ids, pos, lat, allowed, latents)

    # W1 and W3 swapped (silu on the up projection instead of the gate)
    swapped = OracleModel(wl.shape, ws)
    for L in swapped.layers:
        L["w1"], L["w3"] = L["w3"], L["w1"]
    assert np.abs(_oracle(swapped, wl, rows, latents, cap) - z_t).max() > 1e-3

    # the pre-FFN RMSNorm dropped (gain only)
    ffn_gains = [L["ffn_norm"] for L in model.layers]
    real_norm = om_mod.rmsnorm
    monkeypatch.setattr(om_mod, "rmsnorm", lambda x, g, eps: x * g if any(g is f for f in ffn_gains) else real_norm(x, g, eps))
    assert np.abs(_oracle(model, wl, rows, latents, cap) - z_t).max() > 1e-3
    monkeypatch.setattr(om_mod, "rmsnorm", real_norm)

    # RoPE on adjacent pairs (2i, 2i+1) instead of (i, i + dh/2)
    real_rope = om_mod.rope

    def rope_adjacent(x, p, theta):
        y = x.reshape(x.shape[:-1] + (x.shape[-1] // 2, 2)).swapaxes(-1, -2).reshape(x.shape)
        r = real_rope(y, p, theta)
        return r.reshape(x.shape[:-1] + (2, x.shape[-1] // 2)).swapaxes(-1, -2).reshape(x.shape)

    monkeypatch.setattr(om_mod, "rope", rope_adjacent)
    assert np.abs(_oracle(model, wl, rows, latents, cap) - z_t).max() > 1e-3
    monkeypatch.setattr(om_mod, "rope", real_rope)

    # the self-attention output projection transposed
    transposed = OracleModel(wl.shape, ws)
    for L in transposed.layers:
        L["wo"] = L["wo"].T.copy()
    assert np.abs(_oracle(transposed, wl, rows, latents, cap) - z_t).max() > 1e-3


def test_restatement_on_the_nine_layer_shape():
    """The bf16 9-layer d=1024 decoder (the benchmarked model), on a short prefix."""
    from dataclasses import replace

    wl = replace(CONFIGS["d4_b1"], prefix_len=24)
    ws = WeightSet(wl.shape, seed=0, gain_std=0.1).materialize()
    model = OracleModel(wl.shape, ws)
    rows, ids, pos, lat, allowed, latents, cap = _case(wl, model, B=4)
    err = np.abs(_oracle(model, wl, rows, latents, cap) - torch_pass(model, ids, pos, lat, allowed, latents)).max()
    assert err < 1e-10, err
