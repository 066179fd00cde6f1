"""Host-side checks of the C ABI that need no GPU: the library loads, exports
every symbol include/kda.h declares, and rejects bad arguments on the host
before anything is launched."""
import ctypes
import os
import re

import pytest

from kimi_delta_attention_20_b200 import _abi

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "kda.h")


def declared_symbols():
    txt = open(HEADER).read()
    return sorted(set(re.findall(r"KDA_API\s+[\w\s\*]+?\b(kda_\w+)\s*\(", txt)))


def test_header_declarations_match_binding():
    assert declared_symbols() == sorted(_abi.EXPORTS)


def test_library_exports_every_declared_symbol():
    lib = _abi.load()
    for name in declared_symbols():
        assert hasattr(lib, name), name
    assert lib.kda_version() >= 100


def test_status_strings():
    lib = _abi.load()
    for s in range(6):
        assert lib.kda_status_string(s)
    assert lib.kda_status_string(0) == b"ok"
    assert lib.kda_status_string(99) == b"unknown status"


FAKE = 0x10000  # 16-byte aligned, never dereferenced: validation fails first


def chunk_args(**over):
    a = _abi.ChunkArgs()
    a.dtype = _abi.KDA_DTYPE_BF16
    a.B, a.T, a.H, a.Dk, a.Dv = 1, 64, 2, 128, 128
    for f in ("q", "k", "v", "g", "o"):
        setattr(a, f, FAKE)
    a.beta = FAKE
    a.N = 1
    a.use_qk_l2norm = 1
    for kk, vv in over.items():
        setattr(a, kk, vv)
    return a


def step_args(**over):
    a = _abi.StepArgs()
    a.dtype = _abi.KDA_DTYPE_BF16
    a.N, a.H, a.Dk, a.Dv = 2, 2, 128, 128
    for f in ("q", "k", "v", "g", "beta", "state", "o"):
        setattr(a, f, FAKE)
    a.use_qk_l2norm = 1
    for kk, vv in over.items():
        setattr(a, kk, vv)
    return a


@pytest.mark.parametrize("over,want", [
    (dict(dtype=7), _abi.KDA_ERR_INVALID_ARGUMENT),
    (dict(B=0), _abi.KDA_ERR_INVALID_ARGUMENT),
    (dict(T=-1), _abi.KDA_ERR_INVALID_ARGUMENT),
    (dict(H=0), _abi.KDA_ERR_INVALID_ARGUMENT),
    (dict(Dk=96), _abi.KDA_ERR_UNSUPPORTED),
    (dict(Dv=256), _abi.KDA_ERR_UNSUPPORTED),
    (dict(chunk_size=32), _abi.KDA_ERR_UNSUPPORTED),
    (dict(q=None), _abi.KDA_ERR_INVALID_ARGUMENT),
    (dict(o=None), _abi.KDA_ERR_INVALID_ARGUMENT),
    (dict(beta=None), _abi.KDA_ERR_INVALID_ARGUMENT),
    (dict(k=FAKE + 8), _abi.KDA_ERR_INVALID_ARGUMENT),
    (dict(beta=FAKE + 1), _abi.KDA_ERR_INVALID_ARGUMENT),
    (dict(initial_state=FAKE + 4), _abi.KDA_ERR_INVALID_ARGUMENT),
    (dict(has_lower_bound=1, lower_bound=0.0), _abi.KDA_ERR_INVALID_ARGUMENT),
    (dict(has_lower_bound=1, lower_bound=float("nan")), _abi.KDA_ERR_INVALID_ARGUMENT),
    (dict(B=2, N=3), _abi.KDA_ERR_INVALID_ARGUMENT),
    (dict(B=2, cu_seqlens=FAKE, N=2), _abi.KDA_ERR_INVALID_ARGUMENT),
    (dict(cu_seqlens=FAKE, N=0), _abi.KDA_ERR_INVALID_ARGUMENT),
])
def test_chunk_fwd_rejects(over, want):
    lib = _abi.load()
    a = chunk_args(**over)
    assert lib.kda_chunk_fwd(ctypes.byref(a), None) == want
    assert lib.kda_chunk_fwd(None, None) == _abi.KDA_ERR_INVALID_ARGUMENT


@pytest.mark.parametrize("cu,want", [
    ([1, 64], _abi.KDA_ERR_INVALID_ARGUMENT),      # does not start at 0
    ([0, 63], _abi.KDA_ERR_INVALID_ARGUMENT),      # does not end at T
    ([0, 40, 30, 64], _abi.KDA_ERR_INVALID_ARGUMENT),  # decreasing
])
def test_chunk_fwd_rejects_bad_cu_seqlens(cu, want):
    lib = _abi.load()
    host = (ctypes.c_int32 * len(cu))(*cu)
    a = chunk_args(cu_seqlens=FAKE, cu_seqlens_host=ctypes.addressof(host), N=len(cu) - 1)
    assert lib.kda_chunk_fwd(ctypes.byref(a), None) == want


def test_host_cu_seqlens_without_device_copy_is_rejected():
    lib = _abi.load()
    host = (ctypes.c_int32 * 2)(0, 64)
    a = chunk_args(cu_seqlens_host=ctypes.addressof(host))
    assert lib.kda_chunk_fwd(ctypes.byref(a), None) == _abi.KDA_ERR_INVALID_ARGUMENT


def test_workspace_query_reads_shapes_only():
    lib = _abi.load()
    a = chunk_args(q=None, k=None, v=None, g=None, o=None, beta=None)
    n = ctypes.c_size_t(123)
    assert lib.kda_chunk_fwd_workspace_size(ctypes.byref(a), ctypes.byref(n)) == _abi.KDA_OK
    assert lib.kda_chunk_fwd_workspace_size(ctypes.byref(a), None) == _abi.KDA_ERR_INVALID_ARGUMENT
    bad = chunk_args(Dk=48)
    assert lib.kda_chunk_fwd_workspace_size(ctypes.byref(bad), ctypes.byref(n)) == _abi.KDA_ERR_UNSUPPORTED


@pytest.mark.parametrize("over,want", [
    (dict(dtype=3), _abi.KDA_ERR_INVALID_ARGUMENT),
    (dict(N=-1), _abi.KDA_ERR_INVALID_ARGUMENT),
    (dict(H=0), _abi.KDA_ERR_INVALID_ARGUMENT),
    (dict(Dk=100), _abi.KDA_ERR_UNSUPPORTED),
    (dict(state=None), _abi.KDA_ERR_INVALID_ARGUMENT),
    (dict(state=FAKE + 4), _abi.KDA_ERR_INVALID_ARGUMENT),
    (dict(q=FAKE + 2), _abi.KDA_ERR_INVALID_ARGUMENT),
    (dict(has_lower_bound=1, lower_bound=1.0), _abi.KDA_ERR_INVALID_ARGUMENT),
])
def test_recurrent_step_rejects(over, want):
    lib = _abi.load()
    a = step_args(**over)
    assert lib.kda_recurrent_step(ctypes.byref(a), None) == want


def test_recurrent_step_empty_batch_is_a_noop():
    lib = _abi.load()
    a = step_args(N=0, q=None, k=None, v=None, g=None, beta=None, state=None, o=None)
    assert lib.kda_recurrent_step(ctypes.byref(a), None) == _abi.KDA_OK


def test_python_binding_refuses_cpu_tensors():
    import torch
    import kimi_delta_attention_20_b200 as kda
    x = torch.zeros(1, 4, 1, 32)
    with pytest.raises(ValueError):
        kda.chunk_kda(x, x, x, x, torch.zeros(1, 4, 1), use_qk_l2norm_in_kernel=True)
    with pytest.raises(ValueError):
        kda.recurrent_step(x[0], x[0], x[0], x[0], torch.zeros(4, 1), torch.zeros(4, 1, 32, 32))
