"""Seeded synthetic inputs for tests and benchmarks.

The pages measure on model activations (Ouro-1.4B, Huginn-3.5B) and datasets
that are not available here; these generators stand in for them with tensors
of the same shapes and the structure the pages describe: per-loop keys and
values that trace a low-rank trajectory across loops (LLA abstract) plus
small noise, and codecs fitted by SVD of such activations.

This module holds none of the decode arithmetic: it draws random numbers and
fits codec matrices (an offline step of the method, not part of the decode
path), nothing else.  In particular it applies no rotary rotation: the exact
window ring holds keys drawn from the same distribution as the latent keys,
which both the CUDA path and the oracle take as given.

Everything is generated on the CPU with explicit seeds (torch.Generator /
numpy default_rng), so the same seed gives the same bits on every machine.
"""

from .gen import (  # noqa: F401
    CONFIGS, ConfigShape, tiny_hla, hla_codec, hla_hidden, lla_perhead_codec,
    lla_folded_codec, lla_kv, queries, window_ring, random_latents, random_fp8_rows,
)
