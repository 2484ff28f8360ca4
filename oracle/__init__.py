"""Float64 CPU oracle of the PT-DiT block-attention path.

TEST INFRASTRUCTURE ONLY: imported by the tests, by ``__graft_entry__.smoke()``
and by the bench's CPU-baseline / reference leg, never by the product path.
"""
from .ptdit_oracle import *  # noqa: F401,F403
from .ptdit_oracle import (  # noqa: F401
    attention_heads, attention_heads_bwd, averaging, averaging_bwd, block_attn, block_attn_bwd,
    block_attn_rows, gelu_tanh, giim, giim_bwd, layer_norm, masked_self_attention, mlp, pt_block,
    multihead_attention, num_tokens, project, proxy_index, proxy_self_attention, proxy_tokens,
    softmax_rows,
    tcm, tcm_bwd, token_coords, window_allow_matrix, window_region_labels, window_self_attention,
    window_self_attention_bwd, window_members, window_token_map,
)
