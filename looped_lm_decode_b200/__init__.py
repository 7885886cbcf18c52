"""LoopVQ hot path on B200: loop-axis VQ encode and decode attention over the coded cache.

The compute runs in libloopvq.so (CUDA, sm_100a) behind the C ABI in
include/loopvq.h; this package is its thin Python binding.
"""
from .loopvq import (Cache, CacheDesc, LoopVQError, prepare, encode, decode_attn, decode_workspace_bytes,  # noqa: F401
                     dequant_debug, default_scale, lib, LIB_PATH, EXPORTS, decode_attn_noalloc,
                     decode_attn_range, Bf16Cache, Bf16CacheDesc, bf16_decode_attn, bf16_decode_workspace_bytes,
                     merge2, Window, WindowDesc, window_advance, window_append, window_workspace_bytes,
                     window_decode_attn, window_append_decode_attn, Tasq, TasqDesc, tasq_encode,
                     tasq_decode_attn, fault_check, set_wait_limit_ns, wait_limit_ns)
