"""Model shapes and decoding workloads.

Shapes follow the Fast-BLT decoder as read from the Korean summary page
("배경: BLT 아키텍처", "사전 학습 및 실험 설정"): a local decoder of
``n_layers`` layers, width ``d_model``, ``n_heads`` heads, SwiGLU FFN of width
``d_ffn``, cross-attending to latents of width ``d_global``; vocabulary 256
bytes + one [MASK] id (257).
"""

from __future__ import annotations

from dataclasses import dataclass, replace


@dataclass(frozen=True)
class ModelShape:
    n_layers: int
    d_model: int
    n_heads: int
    d_ffn: int
    d_global: int
    weight_dtype: str  # "f32" or "bf16"
    vocab: int = 257
    rope_theta: float = 10000.0
    norm_eps: float = 1e-5
    head_std_mult: float = 5.0  # byte-head std = mult / sqrt(d)

    @property
    def head_dim(self) -> int:
        return self.d_model // self.n_heads

    @property
    def mask_id(self) -> int:
        return self.vocab - 1

    def pass_weight_params(self) -> int:
        """Decoder parameters streamed by one pass (self-attn + FFN of every layer)."""
        d, f = self.d_model, self.d_ffn
        return self.n_layers * (4 * d * d + 3 * d * f)


@dataclass(frozen=True)
class Workload:
    name: str
    shape: ModelShape
    mode: str  # "D" (BLT-D), "S" (BLT-S), "DV" (BLT-DV), "AR" (plain greedy)
    block: int  # B for BLT-D, k for BLT-S / BLT-DV
    alpha: float
    gen_bytes: int
    batch: int
    prefix_len: int
    patch_kind: str  # "uniform8" or "entropy12"
    seed: int = 0
    cfg_index: int = 0
    unmask: str = "confidence"  # BLT-D block unmasking: "confidence" (threshold alpha) or "entropy" (EB, bound gamma)
    gamma: float = 0.0  # EB sampling: bound on the cumulative entropy (nats) of the positions committed per pass


TINY = ModelShape(n_layers=2, d_model=128, n_heads=4, d_ffn=512, d_global=256, weight_dtype="f32")
DEC9 = ModelShape(n_layers=9, d_model=1024, n_heads=16, d_ffn=4096, d_global=2048, weight_dtype="bf16")
DEC9_G4096 = replace(DEC9, d_global=4096)

CONFIGS = {
    # Tiny BLT-D-4 decoder, fp32: parity-only case the oracle finishes in seconds.
    "tiny_d4": Workload("tiny_d4", TINY, "D", 4, 0.7, 32, 1, 64, "uniform8", 0, 0),
    # BLT-D-4, 9 layers d=1024, prefix 1024, generate 512, batch 1.
    "d4_b1": Workload("d4_b1", DEC9, "D", 4, 0.7, 512, 1, 1024, "entropy12", 0, 1),
    # BLT-DV-16: one-step diffusion draft (alpha 0) + causal verify; prefix 2048, batch 8.
    "dv16_b8": Workload("dv16_b8", DEC9, "DV", 16, 0.0, 1024, 8, 2048, "entropy12", 0, 2),
    # BLT-S k=8 greedy self-speculation; prefix 4096; batch 1 and 16; 512 bytes.
    "s8_b1": Workload("s8_b1", DEC9, "S", 8, 0.0, 512, 1, 4096, "entropy12", 0, 3),
    "s8_b16": Workload("s8_b16", DEC9, "S", 8, 0.0, 512, 16, 4096, "entropy12", 0, 3),
    # BLT-D-4 with entropy-bounded sampling (gamma 4.5 nats: about two positions per pass on
    # this model, whose block rows carry about 2 nats each); otherwise config 2.
    "d4eb_b1": Workload("d4eb_b1", DEC9, "D", 4, 0.0, 512, 1, 1024, "entropy12", 0, 1, unmask="entropy", gamma=4.5),
}

# Decoder-step throughput sweep: batch x block x prefix, d_global 4096.
SWEEP = [
    Workload(f"sweep_b{b}_k{k}_p{p}", DEC9_G4096, "D", k, 0.7, 2 * k, b, p, "entropy12", 0, 4)
    for b in (1, 4, 16, 64)
    for k in (4, 8, 16)
    for p in (512, 2048, 8192)
]


def tiny_variant(w: Workload, **kw) -> Workload:
    """The same decoding rule on the tiny decoder (for full oracle parity)."""
    base = dict(shape=TINY, prefix_len=64, patch_kind="uniform8")
    base.update(kw)
    return replace(w, name=w.name + "_tiny", **base)
