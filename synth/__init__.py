"""Seeded synthetic inputs for the weight-informed activation-sparse linear layer.

This package holds random draws, shapes and storage-format casts only. It contains
none of the method's arithmetic (no norms, scores, selection or products), so both
the CPU oracle's tests and the CUDA path's tests and benchmark may draw from it.
"""

from .gen import (  # noqa: F401
    WORKLOADS,
    bf16_bits_from_f32,
    f32_from_bf16_bits,
    keep_count,
    make_linear_512x256_f32,
    make_llama7b_ffn,
    make_llama3_8b_layer,
    make_gemma2_2b_spark,
    make_ultrasparse_down,
    make_ds_decode,
    make_weight,
    spark_keep_count,
)
