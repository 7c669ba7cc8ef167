"""B200-native (sm_100a) 4-bit FlashAttention forward in the HiFA4 style.

QK^T and PV run as block-scaled FP4 (E2M1 + E4M3 per 16) tcgen05 GEMMs, the
online-softmax state stays in fp32, Smooth-QK rescales Q/K per channel before
quantization, and P-Reordering takes the softmax normalizer from the same
quantized probabilities that feed PV. The computation lives in libhifa4.so
(C ABI, include/hifa4.h); this package is the PyTorch-facing binding.
"""
from ._lib import HiFA4Error, load  # noqa: F401
from .api import (PackedQKV, Rope, alloc_packed, alloc_workspace, append_kv, attention_fwd,  # noqa: F401
                  attention_fwd_debug, attention_fwd_ex, attention_fwd_q, attention_fwd_noalloc, attention_splits, calibrate_smooth,
                  debug_set_wait_limit, get_status, packed_bytes, q_mean, quantize_kv, quantize_q, quantize_qkv,
                  tile_stats, workspace_bytes)

__version__ = "0.1.0"
