"""Seeded synthetic inputs for the OmniKVQuant cache write and decode attention.

This package draws random numbers and lays out token modalities; it holds none
of the method's arithmetic (no rotation of keys, no quantisation, no attention).
Both the CUDA path and the CPU oracle receive the tensors it returns.
"""
from .workloads import (WORKLOADS, WorkloadSpec, codebook, decode_inputs, layer_params,  # noqa: F401
                        modality_layout, prefill_inputs, seq_lengths)
