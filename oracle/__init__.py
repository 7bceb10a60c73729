"""fp64 CPU oracle of VideoMLA latent-window attention (test infrastructure only).

Only tests/, the smoke check and the benchmark's CPU-baseline leg may import this package.
"""
from .mla_oracle import (  # noqa: F401
    OracleLayer, cache_scalars, dense_mha, dense_scalars_per_token, latent_scalars_per_token,
    ring_slot, rope3d, rope_bands, token_hw, valid_frames,
)
