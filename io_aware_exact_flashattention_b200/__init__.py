"""B200 (sm_100a) exact attention: fused tiled forward with online softmax,
split-KV decode and its LSE merge, behind the C ABI of libfa.so."""
from .fa import (FAError, decode_attention, decode_default_splits, fa_combine,
                 fa_decode_splitkv, fa_fwd, flash_attention, get_device_status, lib,
                 status_string)

__all__ = ["FAError", "decode_attention", "decode_default_splits", "fa_combine",
           "fa_decode_splitkv", "fa_fwd", "flash_attention", "get_device_status", "lib",
           "status_string"]
