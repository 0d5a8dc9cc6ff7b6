"""B200-native shifted sparse attention (S2-Attn, LongLoRA's "shift short
attention"), forward and backward, as hand-written sm_100a CUDA behind a C ABI
(include/s2attn.h, libs2attn.so).  PyTorch provides device memory and streams.
"""
from .api import (ChunkAttention, S2Attention, S2RopeAttention, bwd_workspace_bytes,  # noqa: F401
                  dense_causal_attn, device_status, hga_backward, hga_forward, lse_merge, nf4_dequantize, nf4_levels,
                  nf4_qkv, rope_apply, rope_table, s2_attn, s2attn_backward, s2attn_backward_rope, s2attn_forward,
                  s2attn_forward_rope, seg_backward, seg_forward)
from ._lib import S2AttnError  # noqa: F401
