"""B200-native shifted sparse attention (S²-Attn) forward and backward.

The computation runs in libs2attn.so (hand-written sm_100a CUDA kernels behind
the C ABI in include/s2attn.h); this package is the Python binding.
"""
from .binding import (  # noqa: F401
    DENSE_CAUSAL, ROLLED, STRICT, S2AttnError, S2Attention, backward, check_status, debug_adjacency, forward,
    s2_attention, s2attn_bwd, s2attn_bwd_stages_v, s2attn_bwd_v, s2attn_bwd_workspace_size, s2attn_check_status,
    s2attn_debug_adjacency, s2attn_fwd, s2attn_fwd_v, s2attn_last_error,
)
