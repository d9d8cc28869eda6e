"""Seeded synthetic workload for the Fast-BLT local-decoder step.

This package is the one piece shared by the fp64 oracle and the CUDA engine's
host driver.  It holds no decoder arithmetic: it only draws numbers.

* ``rng``      -- SplitMix64 (Steele, Lea & Flood, OOPSLA 2014) used as a
                  counter-based generator, Box-Muller normals, bf16 rounding.
* ``configs``  -- the model shapes and decoding workloads (sizes, seeds).
* ``gen``      -- decoder weights, prefix bytes, the synthetic causal patcher
                  that stands in for the entropy model, and the content-keyed
                  latents that stand in for the local encoder + global model.

Which latent a byte attends to (the cross-attention rule of "BLT-D의 어텐션
마스크") is decoder arithmetic and is NOT computed here; each side derives it
from the patch boundaries on its own.
"""

from .configs import ModelShape, Workload, CONFIGS, SWEEP, tiny_variant  # noqa: F401
from .gen import (  # noqa: F401
    LAYER_TENSORS,
    GLOBAL_TENSORS,
    WeightSet,
    PatchState,
    Patcher,
    prefix_bytes,
    sampling_uniforms,
    latent_vector,
    latent_vectors,
)
