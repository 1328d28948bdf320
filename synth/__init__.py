"""Seeded synthetic inputs for the masked WIDE layer.

This package is the only code shared by the CUDA path's tests/bench and the
CPU oracle.  It draws random tensors and masks and formats them (bf16 bit
patterns, bit-packed mask words); it holds none of the layer's arithmetic.
"""
from .gen import (  # noqa: F401
    FFNCase, AttnCase, LayerCase,
    bf16_bits_from_f32, f32_from_bf16_bits,
    pack_mask, unpack_mask,
    bernoulli_mask, prototype_masks,
    tiny_ffn, decode_ffn, prefill_ffn, decode_layer, prefill_layer, small_layer,
    ffn_case, CONFIGS,
    RouterCase, router_case,
)
