"""Float64 CPU oracle (test infrastructure only; never imported by the product path)."""
from .qi21_oracle import (HEAD_DIM, AXES_DIM, THETA, positions, positions_original, allowed_matrix, rope_angles,
                          rope, rms_norm, attention_head, attn_full, prefix_cache, attn_cached, linear, silu,
                          block_attention, block_ffn, block, embed, velocity, denoise, allowed_pairs)
