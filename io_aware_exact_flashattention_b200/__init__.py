"""B200 (sm_100a) exact attention: fused tiled forward with online softmax
(bf16 or E4M3 inputs), its backward, split-KV decode over contiguous or paged
caches and the LSE merge, and the blockwise feed-forward network after
attention, behind the C ABI of libfa.so."""
from .fa import (FAError, attention_backward, bpt_ffn, bpt_layer, decode_attention,
                 decode_attention_paged,
                 decode_default_splits, fa_bwd, fa_combine, fa_decode_paged_splitkv,
                 fa_decode_splitkv, fa_fwd, fa_fwd_fp8, flash_attention, flash_attention_fp8,
                 get_device_status, lib, status_string)

__all__ = ["FAError", "attention_backward", "bpt_ffn", "bpt_layer", "decode_attention",
           "decode_attention_paged",
           "decode_default_splits", "fa_bwd", "fa_combine", "fa_decode_paged_splitkv",
           "fa_decode_splitkv", "fa_fwd", "fa_fwd_fp8", "flash_attention", "flash_attention_fp8",
           "get_device_status", "lib", "status_string"]
