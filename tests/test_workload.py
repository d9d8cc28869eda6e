"""The seeded workload generator (shared by the oracle and the engine's driver)."""

import os

import numpy as np

from workload import CONFIGS, Patcher, PatchState, WeightSet, latent_vector, prefix_bytes
from workload.rng import normals, round_bf16, stream

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def test_splitmix64_published_vectors():
    want = [int(l, 16) for l in open(os.path.join(GOLD, "splitmix64_seed0.txt")) if l.startswith("0x")]
    got = [int(v) for v in stream(0, 0, len(want))]
    assert got == want


def test_normals_moments_and_determinism():
    z = normals(12345, 200_001)
    assert z.shape == (200_001,)
    assert abs(z.mean()) < 0.01 and abs(z.var() - 1.0) < 0.01
    assert np.array_equal(z[:1000], normals(12345, 1000))
    # fourth moment of a standard normal is 3
    assert abs(np.mean(z**4) - 3.0) < 0.05


def test_round_bf16_ties_to_even():
    # 1 + 2^-8 is halfway between bf16 1.0 and 1 + 2^-7: ties to even (1.0)
    x = np.array([1.0 + 2.0**-8, 1.0 + 3 * 2.0**-8, -1.5, 3.0e-3], dtype=np.float32)
    r = round_bf16(x)
    assert r[0] == 1.0
    assert r[1] == np.float32(1.0 + 2.0**-6)
    assert r[2] == -1.5
    assert (r.view(np.uint32) & 0xFFFF).max() == 0
    assert abs(r[3] - 3.0e-3) <= 3.0e-3 * 2.0**-8


def test_weight_recipe():
    sh = CONFIGS["d4_b1"].shape
    ws = WeightSet(sh)
    w = ws.get("wo", 3)
    assert w.shape == (1024, 1024) and w.dtype == np.float32
    assert (w.view(np.uint32) & 0xFFFF).max() == 0  # bf16 values
    assert abs(w.std() * np.sqrt(1024) - 1.0) < 0.01
    h = ws.get("head")
    assert h.shape == (257, 1024) and abs(h.std() * np.sqrt(1024) - 5.0) < 0.05
    assert np.all(ws.get("ffn_norm", 0) == 1.0)
    assert not np.array_equal(ws.get("w1", 0), ws.get("w3", 0))


def test_patcher_causal_and_lengths():
    for kind, lo, hi, mean in (("uniform8", 1, 8, 4.5), ("entropy12", 1, 12, 4.01)):
        p = Patcher(kind, 0, 1, 0)
        x = prefix_bytes(0, 1, 0, 20000)
        flags, st = p.advance(PatchState(), x)
        closes = [c for c, _ in flags]
        assert closes[0]  # first patch is one byte
        lens, run = [], 0
        for c in closes:
            run += 1
            if c:
                lens.append(run)
                run = 0
        assert min(lens) >= lo and max(lens) == hi
        assert abs(np.mean(lens[1:]) - mean) < 0.15
        # causality: boundaries of a prefix never depend on later bytes
        f2, st2 = p.advance(PatchState(), x[:777])
        assert [c for c, _ in f2] == closes[:777]
        # incremental == one-shot
        f3, _ = p.advance(st2, x[777:1000])
        assert [c for c, _ in f3] == closes[777:1000]


def test_latents_content_keyed():
    a = latent_vector(0, 1, 0, 5, 111, 64)
    b = latent_vector(0, 1, 0, 5, 112, 64)
    assert a.dtype == np.float32 and a.shape == (64,)
    assert not np.array_equal(a, b)
    assert np.array_equal(a, latent_vector(0, 1, 0, 5, 111, 64))


def test_prefix_uniform():
    x = prefix_bytes(0, 1, 0, 1 << 16)
    counts = np.bincount(x, minlength=256)
    assert counts.min() > 150 and counts.max() < 370


def test_scalar_and_batched_generators_agree():
    """The scalar SplitMix64 path (patcher, key derivation) equals the array form,
    and latents generated together equal latents generated one at a time."""
    from workload.gen import latent_vector, latent_vectors
    from workload.rng import GAMMA, derive_keys, mix64, stream, stream_int

    rng = np.random.default_rng(5)
    keys = rng.integers(0, 2**63, 64, dtype=np.uint64) * np.uint64(2) + np.uint64(1)
    for k in keys[:16]:
        for i in (0, 1, 7, 1023, 2**40):
            assert stream_int(int(k), i) == int(stream(int(k), i, 1)[0])
    words = [(3, 4, 1, 9, int(s), int(f)) for s, f in zip(range(20), keys[:20])]
    batched = derive_keys(3, 4, 1, 9, [w[4] for w in words], [w[5] for w in words])
    for w, kb in zip(words, batched):
        h = np.array([0], dtype=np.uint64)
        with np.errstate(over="ignore"):
            for x in w:
                h = mix64((h ^ np.uint64(x & 0xFFFFFFFFFFFFFFFF)) + GAMMA)
        assert int(h[0]) == int(kb)
    # 48 x 2048 values: large enough for the transform to run on several host threads
    a = latent_vectors(0, 1, 3, list(range(48)), [int(k) for k in keys[:48]], 2048)
    b = np.stack([latent_vector(0, 1, 3, i, int(k), 2048) for i, k in enumerate(keys[:48])])
    assert np.array_equal(a.view(np.uint32), b.view(np.uint32))


def test_driver_latent_slots_and_latents_match_oracle():
    """The host harness (driver.SeqHost) derives latent slots and the latents to send with
    its own code; on random commit sequences it agrees with the oracle's rule."""
    from dataclasses import replace

    from block_diffusion_byte_b200.driver import SeqHost
    from oracle.model import OracleModel
    from oracle.policies import OracleSequence
    from workload import CONFIGS, Patcher, WeightSet

    for kind in ("uniform8", "entropy12"):
        wl = replace(CONFIGS["tiny_d4"], patch_kind=kind)
        om = OracleModel(wl.shape, WeightSet(wl.shape).materialize())
        rng = np.random.default_rng(7)
        pre = [int(b) for b in rng.integers(0, 256, 40)]
        o = OracleSequence(om, wl, 0, pre)
        h = SeqHost(Patcher(kind, wl.seed, wl.cfg_index, 0), wl.seed, wl.cfg_index, 0, wl.shape.d_global)
        h.commit(pre)
        for _ in range(30):  # commits of 1..6 bytes, as blocks and accepted drafts arrive
            new = [int(b) for b in rng.integers(0, 256, int(rng.integers(1, 7)))]
            o.commit(new)
            h.commit(new)
        # nothing was taken, so the host holds every byte's slot and every latent
        slots, lats = list(h.pend_slots), list(h.lat_ready)
        assert slots == o.lat
        assert len(lats) == len(o.st.latents) == o.n_closed
        for a, b in zip(lats, o.st.latents):
            assert np.array_equal(np.asarray(a, dtype=np.float64), np.asarray(b, dtype=np.float64))
