"""Seeded synthetic inputs for the DSA hot path (indexer -> top-k -> sparse MLA).

This package is the one thing the CUDA path and the fp64 oracle share: it draws
the random tensors and encodes them into the storage formats the hot path
consumes (bf16 bit patterns, FP8 e4m3 bytes with per-128 fp32 scales).  It holds
none of the method's arithmetic -- no index scores, no selection, no attention.
"""

from .workloads import (  # noqa: F401
    WORKLOADS,
    Batch,
    DSAInputs,
    Workload,
    bf16_bits_to_f32,
    custom_workload,
    e4m3_encode,
    f32_to_bf16_bits,
    make_inputs,
    quantize_fp8_blocks,
)
