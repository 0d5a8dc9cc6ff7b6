"""B200-native shifted sparse attention (S2-Attn, LongLoRA's "shift short
attention"), forward and backward, as hand-written sm_100a CUDA behind a C ABI
(include/s2attn.h, libs2attn.so).  PyTorch provides device memory and streams.
"""
from .api import (S2Attention, S2RopeAttention, bwd_workspace_bytes, dense_causal_attn,  # noqa: F401
                  device_status, rope_apply, rope_table, s2_attn, s2attn_backward, s2attn_backward_rope,
                  s2attn_forward, s2attn_forward_rope)
from ._lib import S2AttnError  # noqa: F401
