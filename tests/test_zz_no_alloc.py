"""kda_chunk_fwd_noalloc: the chunkwise forward for callers that cannot allocate.

Callers that run under a fixed device-memory plan (an inference engine that
reserves its memory at start-up, a plug-in whose host owns every device buffer,
a C host with no allocator at the call site) cannot hand kda_chunk_fwd a
workspace; this entry point uses a small scratch array in the library's own
device memory instead. The test calls it through the C ABI, twice in a row
(the scratch keeps the previous call's contents), and checks each result
against kda_chunk_fwd with the bf16 tolerance the parity tests use.

This file is named so that pytest collects it last.
"""
import ctypes

import pytest
import torch

import kda_inputs as KI
from kda_check import check

pytestmark = pytest.mark.gpu


def _chunk_args(_abi, d, o, S):
    a = _abi.ChunkArgs()
    a.dtype = _abi.KDA_DTYPE_BF16
    B, T, H, Dk = d["q"].shape
    a.B, a.T, a.H, a.Dk, a.Dv = B, T, H, Dk, d["v"].shape[-1]
    for name in ("q", "k", "v", "g", "beta"):
        setattr(a, name, ctypes.c_void_p(d[name].data_ptr()))
    a.o = ctypes.c_void_p(o.data_ptr())
    a.scale = float("nan")
    a.initial_state = ctypes.c_void_p(d["initial_state"].data_ptr())
    a.final_state = ctypes.c_void_p(S.data_ptr())
    a.cu_seqlens = ctypes.c_void_p(d["cu_seqlens"].data_ptr())
    a.cu_seqlens_host = ctypes.c_void_p(d["cu_host"].data_ptr())
    a.N = d["cu_host"].numel() - 1
    a.use_qk_l2norm = 1
    a.has_lower_bound = 1
    a.lower_bound = -5.0
    a.chunk_size = 64
    return a


def test_noalloc_entry_matches_chunk_fwd_on_two_calls():
    import kimi_delta_attention_20_b200 as kda
    from kimi_delta_attention_20_b200 import _abi

    lib = _abi.load()
    inp = KI.draw_chunk(1, 200, 3, 128, 128, dtype=torch.bfloat16, seed=31, seqlens=(130, 70),
                        init_state=True)
    d = {k: v.cuda() for k, v in inp.items()}
    d["cu_host"] = inp["cu_seqlens"].to(torch.int32).contiguous()
    d["cu_seqlens"] = d["cu_seqlens"].to(torch.int32).contiguous()
    o_ref, S_ref = kda.chunk_kda(d["q"], d["k"], d["v"], d["g"], d["beta"],
                                 initial_state=d["initial_state"], output_final_state=True,
                                 use_qk_l2norm_in_kernel=True, lower_bound=-5.0,
                                 cu_seqlens=d["cu_seqlens"])
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for _ in range(2):
        o = torch.full_like(o_ref, float("nan"))
        S = torch.full_like(S_ref, float("nan"))
        args = _chunk_args(_abi, d, o, S)
        status = lib.kda_chunk_fwd_noalloc(ctypes.byref(args), stream)
        assert status == _abi.KDA_OK, lib.kda_status_string(status).decode()
        torch.cuda.synchronize()
        check("no-alloc o", o, o_ref, torch.bfloat16)
        check("no-alloc final state", S, S_ref, torch.bfloat16)
