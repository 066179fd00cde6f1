"""kda_chunk_fwd_noalloc: the chunkwise forward for callers that cannot allocate.

Callers that run under a fixed device-memory plan (an inference engine that
reserves its memory at start-up, a plug-in whose host owns every device buffer,
a C host with no allocator at the call site) cannot hand kda_chunk_fwd a
workspace; this entry point uses a small scratch array in the library's own
device memory instead. The tests call it through the C ABI:
  * twice in a row on the tensor-core shape, each result checked against
    kda_chunk_fwd and against the oracle with the bf16 tolerance of the parity
    tests;
  * on shapes whose kernels need no scratch (fp32 d32, 32-token chunks);
  * with the first device wait made to run out, so the status word in the
    shared array is left at 1: kda_chunk_fwd_noalloc_status reports the
    timeout, and the next call clears the word and is correct again.
The path's rejection of problems needing more than its 4096-byte scratch cannot
be reached: no kernel asks for more than 256 bytes.

This file is named so that pytest collects it last.
"""
import ctypes

import pytest
import torch

import kda_inputs as KI
from kda_cabi import chunk_args, stream_ptr, to_device
from kda_check import check, oracle_chunk

pytestmark = pytest.mark.gpu


def _reference(d, **kw):
    import kimi_delta_attention_20_b200 as kda
    return kda.chunk_kda(d["q"], d["k"], d["v"], d["g"], d["beta"], initial_state=d.get("initial_state"),
                         output_final_state=True, use_qk_l2norm_in_kernel=True,
                         cu_seqlens=d.get("cu_seqlens"), cu_seqlens_cpu=d.get("cu_host"), **kw)


def _check_oracle(inp, o, S, dtype, lower_bound):
    ref = oracle_chunk({k: (v.cpu() if isinstance(v, torch.Tensor) else v) for k, v in inp.items()},
                       lower_bound=lower_bound)
    B, T, H = inp["q"].shape[:3]
    o_flat = o.reshape(B * T, H, -1)
    for n, (a, b, o_ref, S_ref) in enumerate(ref):
        if b > a:
            check(f"no-alloc o seq{n} vs oracle", o_flat[a:b], o_ref, dtype)
        check(f"no-alloc S seq{n} vs oracle", S[n], S_ref, dtype)


def test_noalloc_entry_matches_chunk_fwd_on_two_calls():
    from kimi_delta_attention_20_b200 import _abi

    lib = _abi.load()
    inp = KI.draw_chunk(1, 200, 3, 128, 128, dtype=torch.bfloat16, seed=31, seqlens=(130, 70),
                        init_state=True)
    d = to_device(inp)
    o_ref, S_ref = _reference(d, lower_bound=-5.0)
    for _ in range(2):
        o = torch.full_like(o_ref, float("nan"))
        S = torch.full_like(S_ref, float("nan"))
        args = chunk_args(d, o, S, lower_bound=-5.0)
        status = lib.kda_chunk_fwd_noalloc(ctypes.byref(args), stream_ptr())
        assert status == _abi.KDA_OK, lib.kda_status_string(status).decode()
        assert lib.kda_chunk_fwd_noalloc_status(ctypes.byref(args), stream_ptr()) == _abi.KDA_OK
        check("no-alloc o", o, o_ref, torch.bfloat16)
        check("no-alloc final state", S, S_ref, torch.bfloat16)
        _check_oracle(inp, o, S, torch.bfloat16, -5.0)


@pytest.mark.parametrize("case", ["fp32_d32", "chunk32_bf16_d128"])
def test_noalloc_entry_on_shapes_without_scratch(case):
    from kimi_delta_attention_20_b200 import _abi

    lib = _abi.load()
    if case == "fp32_d32":
        inp = KI.draw_chunk(2, 150, 2, 32, 32, dtype=torch.float32, seed=32, init_state=True)
        dtype, chunk = torch.float32, 64
    else:
        inp = KI.draw_chunk(1, 100, 2, 128, 128, dtype=torch.bfloat16, seed=33, init_state=True)
        dtype, chunk = torch.bfloat16, 32
    d = to_device(inp)
    o_ref, S_ref = _reference(d, chunk_size=chunk)
    o = torch.full_like(o_ref, float("nan"))
    S = torch.full_like(S_ref, float("nan"))
    args = chunk_args(d, o, S, chunk_size=chunk)
    assert lib.kda_chunk_fwd_noalloc(ctypes.byref(args), stream_ptr()) == _abi.KDA_OK
    assert lib.kda_chunk_fwd_noalloc_status(ctypes.byref(args), stream_ptr()) == _abi.KDA_OK
    check("no-alloc o", o, o_ref, dtype)
    check("no-alloc final state", S, S_ref, dtype)
    _check_oracle(inp, o, S, dtype, None)


def test_noalloc_timeout_is_visible_and_cleared_by_the_next_call():
    from kimi_delta_attention_20_b200 import _abi

    lib = _abi.load()
    inp = KI.draw_chunk(1, 150, 2, 128, 128, dtype=torch.bfloat16, seed=34, seqlens=(100, 50),
                        init_state=True)
    d = to_device(inp)
    o = torch.zeros_like(d["v"])
    S = torch.zeros(2, 2, 128, 128, device="cuda")
    stalled = chunk_args(d, o, S, lower_bound=-5.0, debug_flags=_abi.KDA_DEBUG_STALL_FIRST_WAIT)
    assert lib.kda_chunk_fwd_noalloc(ctypes.byref(stalled), stream_ptr()) == _abi.KDA_OK
    assert lib.kda_chunk_fwd_noalloc_status(ctypes.byref(stalled), stream_ptr()) == _abi.KDA_ERR_TIMEOUT
    args = chunk_args(d, o, S, lower_bound=-5.0)
    assert lib.kda_chunk_fwd_noalloc(ctypes.byref(args), stream_ptr()) == _abi.KDA_OK
    assert lib.kda_chunk_fwd_noalloc_status(ctypes.byref(args), stream_ptr()) == _abi.KDA_OK
    _check_oracle(inp, o, S, torch.bfloat16, -5.0)
