"""Kimi Delta Attention (KDA) for NVIDIA B200 (sm_100a).

`chunk_kda` (chunkwise forward, with autograd through `chunk_kda_bwd`), `recurrent_step` (one decode token per
sequence, state updated in place) and `decode_token` (the serving token: conv
update + SiLU, the recurrent step and the output gate in one launch) call the
C-ABI library libkda.so built from csrc/
(`python -m kimi_delta_attention_20_b200.build`).
"""
from .ops import chunk_bwd_workspace_bytes, chunk_kda, chunk_kda_bwd, chunk_workspace_bytes, decode_token, recurrent_step  # noqa: F401

__all__ = ["chunk_kda", "chunk_kda_bwd", "recurrent_step", "decode_token", "chunk_workspace_bytes",
           "chunk_bwd_workspace_bytes"]
