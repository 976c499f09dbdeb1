"""Seeded synthetic inputs shared by the oracle tests and the benchmark (inputs only)."""
from .heads import (CONFIGS, Head, HeadConfig, Hidden, bf16_bits_to_f32, intra_cluster_cosine,
                    make_config, make_head, make_hidden, make_uniforms, quantize_int4_g32,
                    quantize_int8_g32, to_bf16_bits)

__all__ = ["CONFIGS", "Head", "HeadConfig", "Hidden", "bf16_bits_to_f32", "intra_cluster_cosine",
           "make_config", "make_head", "make_hidden", "make_uniforms", "quantize_int4_g32",
           "quantize_int8_g32", "to_bf16_bits"]
