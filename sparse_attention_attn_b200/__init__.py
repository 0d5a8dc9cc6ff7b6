"""B200-native shifted sparse attention (S2-Attn, LongLoRA's "shift short
attention"), forward and backward, as hand-written sm_100a CUDA behind a C ABI
(include/s2attn.h, libs2attn.so).  PyTorch provides device memory and streams.
"""
from .api import (S2Attention, bwd_workspace_bytes, dense_causal_attn, device_status,  # noqa: F401
                  s2_attn, s2attn_backward, s2attn_forward)
from ._lib import S2AttnError  # noqa: F401
