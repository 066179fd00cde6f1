"""Device-side failure reporting and host behaviour of the chunk forward.

The tensor-core kernels bound every wait (2 s); a wait that gives up makes its
CTA drain its copies and products, free its tensor memory and leave, and sets
the status word that kda_chunk_fwd_status reads. These tests make the first
wait run out on purpose -- the debug flag leaves the first input copy unissued,
so that wait waits for nothing -- and check that the status reads
KDA_ERR_TIMEOUT, that the context stays usable and that the next call on the
same stream is correct against the oracle. Nothing faults, traps or hangs.
"""
import ctypes

import pytest
import torch

import kda_inputs as KI
from kda_cabi import chunk_args, stream_ptr, to_device
from kda_check import check, oracle_chunk

pytestmark = pytest.mark.gpu


def _lib():
    from kimi_delta_attention_20_b200 import _abi
    return _abi, _abi.load()


def _inputs(seed):
    inp = KI.draw_chunk(1, 330, 4, 128, 128, dtype=torch.bfloat16, seed=seed, seqlens=(200, 130),
                        init_state=True)
    return inp, to_device(inp)


def _compare(inp, o, S):
    ref = oracle_chunk({k: (v.cpu() if isinstance(v, torch.Tensor) else v) for k, v in inp.items()},
                       lower_bound=-5.0)
    for n, (a, b, o_ref, S_ref) in enumerate(ref):
        check(f"o seq{n}", o[0, a:b], o_ref, torch.bfloat16)
        check(f"S seq{n}", S[n], S_ref, torch.bfloat16)


@pytest.mark.parametrize("path", ["two_pass", "single_pass"])
def test_timeout_is_reported_and_the_next_call_is_correct(path):
    import kimi_delta_attention_20_b200 as kda
    _abi, lib = _lib()
    inp, d = _inputs(61)
    if path == "two_pass":
        nbytes = kda.chunk_workspace_bytes(1, 330, 4, 128, 128, N=2, varlen=True)
    else:
        nbytes = 256  # below the record size: the single-pass kernel
    ws = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    o = torch.zeros_like(d["v"])
    S = torch.zeros(2, 4, 128, 128, device="cuda")
    st = stream_ptr()

    stalled = chunk_args(d, o, S, lower_bound=-5.0, workspace=ws,
                         debug_flags=_abi.KDA_DEBUG_STALL_FIRST_WAIT)
    assert lib.kda_chunk_fwd(ctypes.byref(stalled), st) == _abi.KDA_OK
    assert lib.kda_chunk_fwd_status(ctypes.byref(stalled), st) == _abi.KDA_ERR_TIMEOUT
    assert torch.cuda.current_stream().query()  # the status query waited for the stream

    o.fill_(float("nan"))
    S.fill_(float("nan"))
    normal = chunk_args(d, o, S, lower_bound=-5.0, workspace=ws)
    assert lib.kda_chunk_fwd(ctypes.byref(normal), st) == _abi.KDA_OK
    assert lib.kda_chunk_fwd_status(ctypes.byref(normal), st) == _abi.KDA_OK
    _compare(inp, o, S)


def test_status_of_a_shape_without_device_waits_is_ok():
    """fp32 inputs run a kernel without device waits: the status query reads nothing."""
    _abi, lib = _lib()
    inp = KI.draw_chunk(1, 100, 2, 32, 32, dtype=torch.float32, seed=62)
    d = to_device(inp)
    o = torch.empty_like(d["v"])
    S = torch.empty(1, 2, 32, 32, device="cuda")
    a = chunk_args(d, o, S)
    assert lib.kda_chunk_fwd(ctypes.byref(a), stream_ptr()) == _abi.KDA_OK
    assert lib.kda_chunk_fwd_status(ctypes.byref(a), stream_ptr()) == _abi.KDA_OK


@pytest.mark.parametrize("host_copy", ["cpu_tensor", "cu_seqlens_cpu"])
def test_varlen_call_does_not_wait_for_the_gpu(host_copy):
    """With the offsets' host copy at hand (a CPU cu_seqlens, or cu_seqlens_cpu next
    to a CUDA one) chunk_kda returns while the stream is still busy: no blocking
    device-to-host read. The result equals that of a call given only the CUDA
    offsets (same kernels, bit for bit)."""
    import kimi_delta_attention_20_b200 as kda
    inp, d = _inputs(63)
    kw = dict(initial_state=d["initial_state"], output_final_state=True, use_qk_l2norm_in_kernel=True,
              lower_bound=-5.0)
    o_ref, S_ref = kda.chunk_kda(d["q"], d["k"], d["v"], d["g"], d["beta"], cu_seqlens=d["cu_seqlens"], **kw)
    torch.cuda.synchronize()
    cu = dict(cpu_tensor=dict(cu_seqlens=d["cu_host"]),
              cu_seqlens_cpu=dict(cu_seqlens=d["cu_seqlens"], cu_seqlens_cpu=d["cu_host"]))[host_copy]
    torch.cuda._sleep(2_000_000_000)  # about a second of GPU time queued ahead of the call
    o, S = kda.chunk_kda(d["q"], d["k"], d["v"], d["g"], d["beta"], **cu, **kw)
    busy = not torch.cuda.current_stream().query()
    torch.cuda.synchronize()
    assert busy, "the call waited for the GPU"
    assert torch.equal(o, o_ref) and torch.equal(S, S_ref)
