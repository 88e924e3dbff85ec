"""fp64 CPU oracle of the streaming paged KV-cache hot path.

TEST INFRASTRUCTURE ONLY: imported by tests/, by the smoke check and by the
benchmark's CPU-baseline leg, never by the product library.
"""
from .kvcache_oracle import (  # noqa: F401
    OracleConfig, StreamOracle, bf16_round, to_f32, e4m3_encode, e4m3_decode,
    fp8_quantise_block, fp8_quantise_channels, fp8_quantise_tokens, is_keyframe, BF16_MAX, E4M3_MAX,
)
from .rolling_oracle import RollingOracle, diversity_scores, layer_budgets, top_k  # noqa: F401
