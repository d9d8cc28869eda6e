"""Host logic of the driver's staging (no GPU): a call's rows, latent slots and new
latents are packed into one upload, at 16-byte aligned offsets, and the row
descriptor points at them."""

import ctypes as C
import types

import numpy as np
import torch

from block_diffusion_byte_b200 import binding as B
from block_diffusion_byte_b200.driver import Engine
from workload import ModelShape


def _fake_engine(d_global=8):
    eng = types.SimpleNamespace()
    eng.shape = ModelShape(n_layers=1, d_model=32, n_heads=2, d_ffn=64, d_global=d_global, weight_dtype="f32")
    eng.h = 1234
    eng.device = torch.device("cpu")
    eng.h2d_bytes = 0
    eng._h_rows = np.empty(16, dtype=np.uint8)
    eng._d_rows = torch.empty(16, dtype=torch.uint8)
    return eng


def test_rows_packs_one_upload(monkeypatch):
    uploads = []

    def fake_upload(h, dst, src, n):
        uploads.append((h, int(dst), bytes(C.string_at(src, n))))

    monkeypatch.setattr(B, "blt_dec_upload", fake_upload)
    monkeypatch.setattr(torch.cuda, "synchronize", lambda *a, **k: None)
    eng = _fake_engine()
    byte_lists = [[1, 2, 3], [250, 7]]
    slot_lists = [[0, 0, 1], [5, -1]]
    lat = [np.arange(8, dtype=np.float32) + 0.5, -np.arange(8, dtype=np.float32)]
    lat_lists = [[lat[0]], [lat[1]]]
    r, keep = Engine.rows(eng, byte_lists, slot_lists, lat_lists)

    assert len(uploads) == 1
    h, dst, data = uploads[0]
    base = eng._d_rows.data_ptr()
    assert h == 1234 and dst == base
    o_s, o_l = 16, 16 + 32  # 5 bytes -> slots at 16; 5 slots (20 B) -> latents at 48
    assert len(data) == o_l + 2 * 8 * 4
    assert list(data[:5]) == [1, 2, 3, 250, 7]
    assert np.frombuffer(data[o_s:o_s + 20], dtype=np.int32).tolist() == [0, 0, 1, 5, -1]
    got = np.frombuffer(data[o_l:], dtype=np.float32).reshape(2, 8)
    assert np.array_equal(got, np.stack(lat))
    assert r.bytes == base and r.row_latent == base + o_s and r.new_latents == base + o_l
    assert [r.row_offsets[i] for i in range(3)] == [0, 3, 5]
    assert [r.latent_offsets[i] for i in range(3)] == [0, 1, 2]
    assert eng.h2d_bytes == 5 * 5 + 2 * 8 * 4


def test_rows_without_latents(monkeypatch):
    uploads = []
    monkeypatch.setattr(B, "blt_dec_upload", lambda h, dst, src, n: uploads.append(n))
    monkeypatch.setattr(torch.cuda, "synchronize", lambda *a, **k: None)
    eng = _fake_engine()
    r, keep = Engine.rows(eng, [[9]], [[0]], [[]])
    assert uploads == [16 + 4]  # one byte, its slot at 16
    assert not r.new_latents
