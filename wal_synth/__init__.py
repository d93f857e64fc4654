"""Seeded synthetic inputs for the direct-packed body-matrix product.

This module only draws random numbers and rounds them to the storage types
(fp16 / bf16).  It holds none of the method's arithmetic: no packing, no
decoding, no products.  Both the FP64 oracle and the CUDA path take their
inputs from here, so neither ever derives an input from the other.

Distributions follow the workload description of the WAL-Ternary-8B model
card ("Representation": T in {-1,0,+1}, exactly 8 signed residual sites per
group of 128, FP16 scales, a binary low-rank correction) with the shapes of
Qwen3-8B / 27B-sized body matrices.
"""
from .gen import (  # noqa: F401
    Components,
    MatrixSpec,
    rng_for,
    gen_components,
    gen_x,
    bf16_bits_from_f32,
    bf16_bits_to_f32,
    body_plan,
    config_plan,
    gen_matrix,
    gen_pq2,
    gen_base3,
    gen_rc1,
    gen_int4,
    gen_int3,
    f24_bytes_from_f32,
    workload_id,
    WORKLOAD_IDS,
    CONFIG_SEED,
    LAYER_8B,
    LAYER_27B,
    ROLE_K_27B,
    stream_seed,
)
