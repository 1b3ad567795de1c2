"""B200-native fused scaled-dot-product attention (prefill + split-KV decode,
the backward pass, and the rotary-embedding/KV-cache append step that feeds the decode).

The compute path is libsdpa_b200.so (hand-written sm_100a CUDA behind a C
ABI, ``include/sdpa_b200.h``); this package is a thin ctypes binding over it.
"""
from .ops import (CAUSAL_BOTTOM_RIGHT, CAUSAL_NONE, CAUSAL_TOP_LEFT, LAYOUT_BHSD, LAYOUT_BSHD, attn_decode_splitkv,
                  attn_bwd, attn_decode_splitkv_static, attn_decode_splitkv_varlen, attn_fwd, attn_fwd_varlen,
                  attn_rope_append,
                  bwd_workspace_size, check_device_error, decode_num_splits, decode_workspace,
                  decode_workspace_size)

__all__ = ["attn_fwd", "attn_fwd_varlen", "attn_decode_splitkv", "attn_decode_splitkv_varlen", "attn_decode_splitkv_static",
           "attn_rope_append", "attn_bwd", "bwd_workspace_size", "decode_num_splits", "decode_workspace", "decode_workspace_size", "check_device_error",
           "CAUSAL_NONE", "CAUSAL_TOP_LEFT", "CAUSAL_BOTTOM_RIGHT", "LAYOUT_BHSD", "LAYOUT_BSHD"]
