"""Seeded synthetic inputs shared by the oracle tests, the CUDA path tests and the bench."""
from .flux_inputs import (FluxDims, Flux3Dims, Workload, WORKLOADS, TINY_DIMS, FULL_DIMS, F3_TINY_DIMS,
                          F3_FULL_DIMS, F3_BASE_DIMS, F3_TINY_BASE_DIMS, tensor_specs, tensor_specs3,
                          blob_layout, make_weights, make_inputs, make_uncond_text, round_to_bf16_bits,
                          bf16_bits_to_f32)
