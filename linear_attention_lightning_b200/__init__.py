"""MiniMax-M1 Lightning Attention for NVIDIA B200 (sm_100a).

The compute lives in liblightning.so (hand-written CUDA behind a C ABI, see
include/lightning.h). This package adds a thin torch-facing layer that only
marshals tensors into that ABI: torch provides device memory and streams.
"""
from . import abi
from .api import (decode, gqa_decode, gqa_prefill, norm_gate, prefill, prefill_backward, prefill_norm_gate,
                  prefill_snapshots, prefill_variant)

__all__ = ["abi", "prefill", "prefill_snapshots", "prefill_backward", "norm_gate", "prefill_norm_gate", "decode", "gqa_decode", "gqa_prefill",
           "prefill_variant"]
