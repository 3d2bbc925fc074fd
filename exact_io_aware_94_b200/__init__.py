"""Exact IO-aware attention for B200 (sm_100a): thin Python binding over the C-ABI library.

The binding only marshals arguments; every step of the attention path runs in
the library's CUDA kernels.  There is no CPU fallback: if the compiled library
is missing, every call raises.
"""
from .inputs import AttentionInputs, DecodeInputs, attention_inputs, decode_inputs  # noqa: F401
