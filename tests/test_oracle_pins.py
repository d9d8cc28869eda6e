"""Pins of the fp64 oracle against what the pages and the mathematics fix.

Each test is chosen so that a plausible mistake (a dropped term, a wrong mask
index, a transposed operand, a wrong latent slot, an off-by-one in the accept
scan) fails at least one of them.
"""

import itertools
import os
from dataclasses import replace

import numpy as np
import pytest
import torch

from oracle.model import BLOCK, CAUSAL, OracleModel, Row, SeqState, decoder_pass, dense_reference_pass, may_attend, rmsnorm, rope, silu
from oracle.policies import OracleSequence, accept_length, eb_select, entropy, head_stats, proxy_gb, unmask_select
from workload import CONFIGS, WeightSet, prefix_bytes

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _seq(tiny, mode="D", k=4, alpha=0.7, seed_seq=0, n=64):
    wl, ws, m = tiny
    w = replace(wl, mode=mode, block=k, alpha=alpha)
    return OracleSequence(m, w, seed_seq, list(prefix_bytes(0, 0, seed_seq, n)))


# ------------------------------------------------------------------ primitives vs library routines
def test_rmsnorm_matches_torch():
    x = np.random.default_rng(0).standard_normal((5, 128))
    g = np.random.default_rng(1).standard_normal(128)
    ref = torch.nn.functional.rms_norm(torch.from_numpy(x), (128,), torch.from_numpy(g), eps=1e-5).numpy()
    assert np.allclose(rmsnorm(x, g, 1e-5), ref, rtol=1e-13, atol=1e-13)


def test_silu_matches_torch():
    x = np.linspace(-30, 30, 1001)
    assert np.allclose(silu(x), torch.nn.functional.silu(torch.from_numpy(x)).numpy(), rtol=1e-14, atol=1e-300)


def test_rope_invariants():
    rng = np.random.default_rng(2)
    q = rng.standard_normal((1, 4, 64))
    k = rng.standard_normal((1, 4, 64))
    # position 0 is the identity
    assert np.array_equal(rope(q, np.array([0]), 1e4), q)
    # a rotation: norms per head are preserved
    r = rope(q, np.array([123]), 1e4)
    assert np.allclose(np.linalg.norm(r, axis=-1), np.linalg.norm(q, axis=-1), rtol=1e-13)
    # relative: <rope(q, m), rope(k, n)> depends only on m - n
    def dot(m, n):
        return np.einsum("ahd,ahd->ah", rope(q, np.array([m]), 1e4), rope(k, np.array([n]), 1e4))

    assert np.allclose(dot(17, 5), dot(112, 100), rtol=1e-11, atol=1e-11)
    assert not np.allclose(dot(17, 5), dot(17, 6))
    # closed form on a basis vector: e_i -> cos * e_i + sin * e_{i+32}, angle = pos * theta^(-2i/64)
    e = np.zeros((1, 1, 64))
    e[0, 0, 3] = 1.0
    out = rope(e, np.array([7]), 1e4)[0, 0]
    ang = 7 * 1e4 ** (-6 / 64)
    want = np.zeros(64)
    want[3], want[35] = np.cos(ang), np.sin(ang)
    assert np.allclose(out, want, atol=1e-15)


def test_attention_core_matches_torch_sdpa(tiny):
    """The oracle's masked self-attention equals torch's SDPA with the same boolean mask."""
    wl, ws, m = tiny
    sh = wl.shape
    H, dh = sh.n_heads, sh.head_dim
    st = SeqState(sh, 40)
    rng = np.random.default_rng(3)
    st.K[0, :40] = rng.standard_normal((40, H, dh))
    st.V[0, :40] = rng.standard_normal((40, H, dh))
    rows = [Row(0, p, 0, CAUSAL) for p in (30, 31)] + [Row(256, 32 + i, 0, BLOCK, 40) for i in range(8)]
    q = rng.standard_normal((len(rows), H, dh))
    from oracle.model import self_attention

    got = self_attention(m, 0, q, rows, st)
    mask = torch.tensor(np.stack([may_attend(r, np.arange(40)) for r in rows]))
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q).transpose(0, 1), torch.from_numpy(st.K[0, :40]).transpose(0, 1), torch.from_numpy(st.V[0, :40]).transpose(0, 1), attn_mask=mask
    )
    assert np.allclose(got, ref.transpose(0, 1).reshape(len(rows), -1).numpy(), rtol=1e-12, atol=1e-12)


# ------------------------------------------------------------------ masks and latents (the pages' rules)
def _lam_rule_bruteforce(closes):
    """Latent of byte i from the page's wording: o_{p(i)-1}, the last byte of a patch o_{p(i)}."""
    patches, cur = [], []
    for i, c in enumerate(closes):
        cur.append(i)
        if c:
            patches.append(cur)
            cur = []
    if cur:
        patches.append(cur)
    lam = {}
    for p_idx, members in enumerate(patches, start=1):
        closed = p_idx <= sum(closes)
        for i in members:
            last = closed and i == members[-1]
            lam[i] = (p_idx if last else p_idx - 1) - 1  # 0-based slot
    return [lam[i] for i in range(len(closes))]


def test_latent_slots_follow_page_rule(tiny):
    s = _seq(tiny)
    per, _ = s.patcher.advance(type(s.pstate)(), s.bytes)
    assert s.lat == _lam_rule_bruteforce([c for c, _ in per])
    assert s.lat[0] == 0  # the one-byte first patch attends its own latent o_1
    assert len(s.st.latents) == s.n_closed


def test_cached_pass_equals_dense_masked_pass(tiny):
    """Prefill + one block pass == a cache-free pass over [prefix; MASK x B] with the dense mask."""
    wl, ws, m = tiny
    s = _seq(tiny)
    s.prefill()
    N, B = len(s.bytes), 4
    m_slot = s.n_closed - 1
    rows = s._pending() + [Row(256, N + i, m_slot, BLOCK, N + B) for i in range(B)]
    z = decoder_pass(m, s.st, rows)
    ids = np.array(s.bytes + [256] * B)
    lat = np.array(s.lat + [m_slot] * B)
    n = N + B
    dense = np.zeros((n, n), dtype=bool)
    for i in range(n):
        for j in range(n):
            # clean prefix: causal; masked block: all of the prefix and the whole block
            dense[i, j] = (j <= i) if i < N else True
    zd = dense_reference_pass(m, ids, lat, dense, np.stack(s.st.latents))
    assert np.allclose(z, zd[N - 1 :], rtol=1e-10, atol=1e-10)
    # the structured mask itself equals the dense one
    for i in range(n):
        r = Row(0, i, 0, CAUSAL) if i < N else Row(0, i, 0, BLOCK, N + B)
        assert np.array_equal(may_attend(r, np.arange(n)), dense[i])


def test_cross_attention_independent_of_query_and_key_weights(tiny):
    """One allowed latent per row: the softmax weight is exactly 1, so W_q^c, W_k^c cannot matter."""
    wl, ws, m = tiny
    m2 = OracleModel(wl.shape, ws)
    rng = np.random.default_rng(4)
    for L in m2.layers:
        L["wq_c"] = L["wq_c"] + rng.standard_normal(L["wq_c"].shape)
        L["wk_c"] = 3.0 * rng.standard_normal(L["wk_c"].shape)
        L["norm_c"] = L["norm_c"] * 7.0
    outs = []
    for mm in (m, m2):
        s = _seq((wl, ws, mm))
        s.prefill()
        outs.append(decoder_pass(mm, s.st, s._pending() + [Row(256, 64 + i, s.n_closed - 1, BLOCK, 68) for i in range(4)]))
    assert np.array_equal(outs[0], outs[1])


def test_layer_equation_residual_structure(tiny):
    """With self-attention output and FFN down-projection zeroed, each layer adds exactly W_o^c W_v^c o."""
    wl, ws, m = tiny
    m2 = OracleModel(wl.shape, ws)
    for L in m2.layers:
        L["wo"] = np.zeros_like(L["wo"])
        L["w2"] = np.zeros_like(L["w2"])
    s = _seq((wl, ws, m2))
    rows = [Row(s.bytes[p], p, s.lat[p], CAUSAL) for p in range(10)]
    _, h = decoder_pass(m2, s.st, rows, want_hidden=True)
    want = m2.g["embed"][np.array(s.bytes[:10])].copy()
    for L in m2.layers:
        for i in range(10):
            want[i] += L["wo_c"] @ (L["wv_c"] @ s.st.latents[s.lat[i]])
    assert np.allclose(h, want, rtol=1e-12, atol=1e-12)


def test_prefix_rows_blind_to_block(tiny):
    wl, ws, m = tiny
    outs, kvs = [], []
    for fill in (256, 7):
        s = _seq(tiny)
        s.prefill()
        N = len(s.bytes)
        rows = s._pending() + [Row(fill, N + i, s.n_closed - 1, BLOCK, N + 4) for i in range(4)]
        z = decoder_pass(m, s.st, rows)
        outs.append(z[0])
        kvs.append(s.st.K[:, : N].copy())
    assert np.array_equal(outs[0], outs[1])
    assert np.array_equal(kvs[0], kvs[1])


def test_block_of_one_is_a_causal_row(tiny):
    """B = 1: the block row sees positions 0..N, exactly what a causal row at N sees."""
    wl, ws, m = tiny
    zs = []
    for kind in (BLOCK, CAUSAL):
        s = _seq(tiny)
        s.prefill()
        N = len(s.bytes)
        rows = s._pending() + [Row(256, N, s.n_closed - 1, kind, N + 1)]
        zs.append(decoder_pass(m, s.st, rows)[-1])
    assert np.array_equal(zs[0], zs[1])


# ------------------------------------------------------------------ unmasking
def test_head_stats_definitions():
    z = np.array([[0.0, 1.0, 1.0, -2.0] + [-50.0] * 252])
    conf, pred, gap = head_stats(z)
    assert pred[0] == 1  # tie -> lowest byte
    assert gap[0] == 0.0
    p = np.exp(z[0]) / np.exp(z[0]).sum()
    assert np.isclose(conf[0], p.max(), rtol=1e-14)


def test_unmask_select_bruteforce():
    rng = np.random.default_rng(5)
    for _ in range(300):
        B = int(rng.integers(1, 7))
        conf = np.round(rng.random(B), 1)
        masked = sorted(rng.choice(B, size=int(rng.integers(1, B + 1)), replace=False).tolist())
        alpha = float(rng.choice([0.0, 0.3, 0.5, 0.7, 1.1]))
        got, _ = unmask_select(masked, conf, alpha)
        # brute force: the largest subset of masked positions all at or above alpha;
        # if it is empty, the most confident single position (lowest index on ties)
        best = []
        for r in range(len(masked), 0, -1):
            for sub in itertools.combinations(masked, r):
                if all(conf[i] >= alpha for i in sub):
                    best = list(sub)
                    break
            if best:
                break
        if not best:
            top = max(conf[i] for i in masked)
            best = [min(i for i in masked if conf[i] == top)]
        assert got == best


def test_alpha_zero_fills_block_in_one_pass(tiny):
    s = _seq(tiny, alpha=0.0)
    s.prefill()
    for _ in range(3):
        blk, steps, _ = s.diffuse(8, 0.0)
        assert steps == 1 and len(blk) == 8
        s.commit(blk)


def test_alpha_above_one_takes_B_passes(tiny):
    s = _seq(tiny, alpha=1.5)
    s.prefill()
    blk, steps, _ = s.diffuse(6, 1.5)
    assert steps == 6


def test_block_one_step_one_is_ar(tiny):
    """B = 1 with one step per block: one decoder pass per generated byte, and the
    committed byte is the argmax of a row that sees positions 0..N."""
    s = _seq(tiny, mode="D", k=1, alpha=0.0)
    s.prefill()
    out = s.generate(10)
    assert s.c.passes == 10 and len(out) == 10


# ------------------------------------------------------------------ verification (Algorithm 2 of the summary page)
def test_accept_scan_bruteforce():
    rng = np.random.default_rng(6)
    for _ in range(2000):
        k = int(rng.integers(1, 9))
        draft = rng.integers(0, 3, size=k).tolist()
        y = rng.integers(0, 3, size=k + 1).tolist()
        a, nxt = accept_length(draft, y)
        # brute force: largest prefix length whose every byte equals the prediction before it
        want = max(t for t in range(k + 1) if all(draft[i] == y[i] for i in range(t)))
        assert a == want and nxt == y[want]
    assert accept_length([1, 2, 3], [1, 2, 3, 9]) == (3, 9)  # perfect draft: all + free byte
    assert accept_length([5, 2, 3], [1, 2, 3, 9]) == (0, 1)  # wrong first byte: correction


@pytest.mark.parametrize("seq", [0, 1, 2])
def test_blt_s_equals_ar_greedy(tiny, seq):
    """BLT-S preserves greedy decoding exactly (summary page, "BLT-S")."""
    ref = _seq(tiny, mode="AR", k=1, seed_seq=seq)
    ref.prefill()
    want = ref.generate(40)
    for k in (2, 5, 8):
        s = _seq(tiny, mode="S", k=k, seed_seq=seq)
        s.prefill()
        assert s.generate(40) == want


@pytest.mark.parametrize("k,alpha", [(4, 0.0), (8, 0.0), (6, 0.7)])
def test_blt_dv_equals_ar_greedy(tiny, k, alpha):
    """Same weights: every byte BLT-DV commits is the argmax of a causal row."""
    ref = _seq(tiny, mode="AR", k=1, seed_seq=3)
    ref.prefill()
    want = ref.generate(40)
    s = _seq(tiny, mode="DV", k=k, alpha=alpha, seed_seq=3)
    s.prefill()
    assert s.generate(40) == want


def test_blt_s_pass_count(tiny):
    s = _seq(tiny, mode="S", k=5)
    s.prefill()
    rec = []
    s.generate(30, rec)
    assert s.c.passes == 6 * len(rec)  # k draft passes + one verification pass per round
    assert all(1 <= r["accepted"] <= 5 for r in rec)  # the first draft byte is the greedy byte


# ------------------------------------------------------------------ proxy bandwidth
def _gold(name):
    vals = {}
    for line in open(os.path.join(GOLD, name)):
        line = line.split("#")[0].strip()
        if line:
            k, v = line.split("=")
            vals[k.strip()] = float(v)
    return vals


def test_proxy_bandwidth_from_counted_passes():
    g = _gold("proxy_bandwidth.txt")
    # one decoder pass of the 160M decoder at 16 bits loads 0.32 GB
    assert proxy_gb(1, g["p_dec_3b"], 0, 0, 0) == pytest.approx(2 * 160e6 / 1e9)
    # AR BLT per 4-byte patch: 4 decoder calls + 1 encoder/global call (3B sizes)
    per_patch = proxy_gb(g["dec_calls_per_patch_ar"], g["p_dec_3b"], g["global_calls_per_patch_ar"], g["p_enc_3b"], g["p_global_3b"])
    assert per_patch == pytest.approx(4 * 0.32 + 2 * (26e6 + 2.82e9) / 1e9)
    # linear in the counts
    assert proxy_gb(8, 1.0, 2, 1.0, 1.0) == pytest.approx(2 * proxy_gb(4, 1.0, 1, 1.0, 1.0))
    # the 1B model's global term is smaller
    assert proxy_gb(0, 0, 1, g["p_enc_1b"], g["p_global_1b"]) < proxy_gb(0, 0, 1, g["p_enc_3b"], g["p_global_3b"])


def test_entropy_closed_forms_and_library():
    """Entropy (nats) of softmax(z): uniform -> ln 256, two equal maxima far above the
    rest -> ln 2, a single dominant logit -> 0; random logits agree with SciPy."""
    from scipy.stats import entropy as sp_entropy

    z = np.zeros((3, 256))
    z[1, :] = -1e4
    z[1, [7, 200]] = 0.0
    z[2, 5] = 1e4
    e = entropy(z)
    assert abs(e[0] - np.log(256)) < 1e-12
    assert abs(e[1] - np.log(2)) < 1e-12
    assert abs(e[2]) < 1e-12
    r = np.random.default_rng(3).normal(0, 3, (20, 256))
    p = np.exp(r - r.max(axis=1, keepdims=True))
    p /= p.sum(axis=1, keepdims=True)
    assert np.allclose(entropy(r), sp_entropy(p, axis=1), rtol=1e-12, atol=1e-12)


def test_eb_select_worked_cases():
    """EB sampling: sort by entropy, commit the leading run within gamma, at least one."""
    ent = np.array([2.0, 0.5, 1.0, 3.0])
    assert eb_select([0, 1, 2, 3], ent, 1.6)[0] == [1, 2]          # running sums 0.5, 1.5, 3.5, 6.5
    assert eb_select([0, 1, 2, 3], ent, 1.5)[0] == [1, 2]          # the bound is inclusive
    assert eb_select([0, 1, 2, 3], ent, 0.1)[0] == [1]             # nothing within gamma: the lowest one
    assert eb_select([0, 1, 2, 3], ent, 100.0)[0] == [1, 2, 0, 3]  # everything
    assert eb_select([0, 3], ent, 2.5)[0] == [0]                   # only masked positions count
    assert eb_select([2, 0, 1], np.array([1.0, 1.0, 1.0]), 2.0)[0] == [0, 1]  # ties: lower position first


def test_eb_select_is_the_largest_feasible_set():
    """The committed set has the largest size over all subsets of the masked positions
    whose summed entropy is <= gamma (brute force), and when several subsets share
    that size it is the one with the lowest entropies."""
    rng = np.random.default_rng(11)
    for _ in range(200):
        k = int(rng.integers(1, 8))
        ent = rng.uniform(0.0, 3.0, k)
        masked = sorted(rng.choice(k, int(rng.integers(1, k + 1)), replace=False).tolist())
        gamma = float(rng.uniform(0.0, 6.0))
        chosen = eb_select(masked, ent, gamma)[0]
        best = 0
        for n in range(len(masked) + 1):
            for sub in itertools.combinations(masked, n):
                if sum(ent[list(sub)]) <= gamma:
                    best = max(best, n)
        assert len(chosen) == max(best, 1)
        if best >= 1:
            assert sum(ent[chosen]) <= gamma + 1e-12
            rest = [i for i in masked if i not in chosen]
            assert all(ent[i] >= max(ent[chosen]) for i in rest)


def test_eb_extremes(tiny):
    """EB with an unbounded gamma fills the block in one pass, the same block as the
    confidence rule with alpha 0; with gamma 0 (every entropy is > 0) it commits one
    position per pass, so a block of B takes B passes."""
    a = _seq(tiny, alpha=0.0)
    a.prefill()
    blk_c, steps_c, _ = a.diffuse(6, 0.0)
    b = _seq(tiny, alpha=0.0)
    b.prefill()
    blk_e, steps_e, _ = b.diffuse(6, 0.0, unmask="entropy", gamma=1e9)
    assert steps_c == steps_e == 1 and blk_c == blk_e
    c = _seq(tiny, alpha=0.0)
    c.prefill()
    _, steps0, _ = c.diffuse(6, 0.0, unmask="entropy", gamma=0.0)
    assert steps0 == 6
