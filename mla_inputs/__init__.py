"""Seeded synthetic workloads for Multi-Latent Attention (MLA).

This package holds only shapes and seeded random tensors.  It contains none of
the method's arithmetic, so that both the CUDA path and the fp64 oracle can
draw the very same inputs from it without sharing any computation.
"""
from .configs import MlaConfig, WORKLOADS, workload
from .generate import (PrefillInputs, DecodeInputs, make_prefill_inputs,
                       make_decode_inputs, decode_context_lengths,
                       varlen_seq_lengths, make_varlen_inputs)

__all__ = ["MlaConfig", "WORKLOADS", "workload", "PrefillInputs",
           "DecodeInputs", "make_prefill_inputs", "make_decode_inputs",
           "decode_context_lengths", "varlen_seq_lengths", "make_varlen_inputs"]
