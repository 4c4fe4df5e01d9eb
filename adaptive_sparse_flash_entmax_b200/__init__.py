"""B200-native fused alpha-entmax attention (AdaSplash-style), forward and backward.

The computation lives in ``libentattn.so`` (hand-written CUDA for sm_100a,
C ABI in ``include/entattn.h``); ``capi`` binds it with ctypes under the same
names, and ``attention`` wraps it for PyTorch tensors.
"""
from . import capi
from .attention import (EntmaxAttention, entmax_attention, entmax_attn_bwd, entmax_attn_fwd,
                        read_status, workspace)

__all__ = ["capi", "EntmaxAttention", "entmax_attention", "entmax_attn_fwd", "entmax_attn_bwd",
           "read_status", "workspace"]
