"""Kimi Delta Attention (KDA) for NVIDIA B200 (sm_100a).

`chunk_kda` (chunkwise forward) and `recurrent_step` (one decode token per
sequence, state updated in place) call the C-ABI library libkda.so built
from csrc/ (`python -m kimi_delta_attention_20_b200.build`).
"""
from .ops import chunk_kda, chunk_workspace_bytes, recurrent_step  # noqa: F401

__all__ = ["chunk_kda", "recurrent_step", "chunk_workspace_bytes"]
