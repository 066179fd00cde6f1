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
    with open(os.path.join(ROOT, "include", "kda.h")) as f:
        header = int(re.search(r"#define KDA_VERSION (\d+)", f.read()).group(1))
    assert lib.kda_version() == header >= 200


def test_status_queries_on_the_host():
    """The status queries validate like the forward, need a workspace where the
    tensor-core kernels would run, and read nothing for shapes whose kernels have
    no device waits (fp32, or head dims other than 128) -- no GPU needed."""
    lib = _abi.load()
    for fn in (lib.kda_chunk_fwd_status, lib.kda_chunk_fwd_noalloc_status):
        assert fn(None, None) == _abi.KDA_ERR_INVALID_ARGUMENT
        assert fn(ctypes.byref(chunk_args(Dk=48)), None) == _abi.KDA_ERR_UNSUPPORTED
        assert fn(ctypes.byref(chunk_args(dtype=_abi.KDA_DTYPE_F32)), None) == _abi.KDA_OK
        assert fn(ctypes.byref(chunk_args(Dk=64, Dv=64)), None) == _abi.KDA_OK
    assert lib.kda_chunk_fwd_status(ctypes.byref(chunk_args()), None) == _abi.KDA_ERR_WORKSPACE


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
    (dict(chunk_size=48), _abi.KDA_ERR_UNSUPPORTED),
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
    # in-kernel gate: unknown mode, missing A_log, misaligned pointers, bound rules
    (dict(gate_mode=3, A_log=FAKE), _abi.KDA_ERR_INVALID_ARGUMENT),
    (dict(gate_mode=_abi.KDA_GATE_SOFTPLUS), _abi.KDA_ERR_INVALID_ARGUMENT),
    (dict(gate_mode=_abi.KDA_GATE_SOFTPLUS, A_log=FAKE + 2), _abi.KDA_ERR_INVALID_ARGUMENT),
    (dict(gate_mode=_abi.KDA_GATE_SOFTPLUS, A_log=FAKE, dt_bias=FAKE + 1), _abi.KDA_ERR_INVALID_ARGUMENT),
    (dict(gate_mode=_abi.KDA_GATE_SOFTPLUS, A_log=FAKE, has_lower_bound=1, lower_bound=-5.0),
     _abi.KDA_ERR_INVALID_ARGUMENT),
    (dict(gate_mode=_abi.KDA_GATE_SAFE, A_log=FAKE), _abi.KDA_ERR_INVALID_ARGUMENT),
    (dict(gate_mode=_abi.KDA_GATE_SAFE, A_log=FAKE, has_lower_bound=1, lower_bound=1.0),
     _abi.KDA_ERR_INVALID_ARGUMENT),
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
    (dict(state_out=FAKE + 0x40000 + 4), _abi.KDA_ERR_INVALID_ARGUMENT),   # misaligned
    (dict(state_out=FAKE + 1024), _abi.KDA_ERR_INVALID_ARGUMENT),          # overlaps state
    (dict(state=FAKE + 0x3fc00, state_out=FAKE), _abi.KDA_ERR_INVALID_ARGUMENT),  # state starts inside it
])
def test_recurrent_step_rejects(over, want):
    lib = _abi.load()
    a = step_args(**over)
    assert lib.kda_recurrent_step(ctypes.byref(a), None) == want


def test_recurrent_step_empty_batch_is_a_noop():
    lib = _abi.load()
    a = step_args(N=0, q=None, k=None, v=None, g=None, beta=None, state=None, o=None)
    assert lib.kda_recurrent_step(ctypes.byref(a), None) == _abi.KDA_OK


def token_args(**over):
    a = _abi.TokenArgs()
    a.dtype = _abi.KDA_DTYPE_BF16
    a.N, a.H, a.Dk, a.Dv, a.conv_kernel = 2, 2, 128, 128, 4
    for f in ("x", "conv_w", "conv_state", "g", "beta", "state", "o"):
        setattr(a, f, FAKE)
    a.norm_eps = 1e-6
    a.use_qk_l2norm = 1
    for kk, vv in over.items():
        setattr(a, kk, vv)
    return a


@pytest.mark.parametrize("over,want", [
    (dict(dtype=3), _abi.KDA_ERR_INVALID_ARGUMENT),
    (dict(N=-1), _abi.KDA_ERR_INVALID_ARGUMENT),
    (dict(H=0), _abi.KDA_ERR_INVALID_ARGUMENT),
    (dict(Dv=48), _abi.KDA_ERR_UNSUPPORTED),
    (dict(conv_kernel=0), _abi.KDA_ERR_UNSUPPORTED),
    (dict(conv_kernel=9), _abi.KDA_ERR_UNSUPPORTED),
    (dict(norm_eps=-1.0), _abi.KDA_ERR_INVALID_ARGUMENT),
    (dict(norm_eps=float("nan")), _abi.KDA_ERR_INVALID_ARGUMENT),
    (dict(conv_state=None), _abi.KDA_ERR_INVALID_ARGUMENT),
    (dict(x=FAKE + 1), _abi.KDA_ERR_INVALID_ARGUMENT),
    (dict(state=FAKE + 4), _abi.KDA_ERR_INVALID_ARGUMENT),
    (dict(conv_w=FAKE + 2), _abi.KDA_ERR_INVALID_ARGUMENT),
    (dict(g_out=FAKE + 1), _abi.KDA_ERR_INVALID_ARGUMENT),
    (dict(has_lower_bound=1, lower_bound=0.5), _abi.KDA_ERR_INVALID_ARGUMENT),
    (dict(gate_mode=_abi.KDA_GATE_SOFTPLUS), _abi.KDA_ERR_INVALID_ARGUMENT),
    (dict(state_out=FAKE + 0x40000 + 4), _abi.KDA_ERR_INVALID_ARGUMENT),
    (dict(state_out=FAKE + 0x3fff0), _abi.KDA_ERR_INVALID_ARGUMENT),
])
def test_decode_token_rejects(over, want):
    lib = _abi.load()
    a = token_args(**over)
    assert lib.kda_decode_token(ctypes.byref(a), None) == want


def test_decode_token_empty_batch_is_a_noop():
    lib = _abi.load()
    a = token_args(N=0, x=None, conv_w=None, conv_state=None, g=None, beta=None, state=None, o=None)
    assert lib.kda_decode_token(ctypes.byref(a), None) == _abi.KDA_OK


def test_python_binding_refuses_cpu_tensors():
    import torch
    import kimi_delta_attention_20_b200 as kda
    x = torch.zeros(1, 4, 1, 32)
    with pytest.raises(ValueError):
        kda.chunk_kda(x, x, x, x, torch.zeros(1, 4, 1), use_qk_l2norm_in_kernel=True)
    with pytest.raises(ValueError):
        kda.recurrent_step(x[0], x[0], x[0], x[0], torch.zeros(4, 1), torch.zeros(4, 1, 32, 32))


@pytest.mark.parametrize("over", [
    dict(gate_mode=_abi.KDA_GATE_SOFTPLUS, A_log=FAKE, q=None),
    dict(gate_mode=_abi.KDA_GATE_SAFE, A_log=FAKE, has_lower_bound=1, lower_bound=-5.0, o=None),
])
def test_valid_gate_modes_pass_gate_checks(over):
    """A request whose gate fields are valid fails only on the pointer planted as bad."""
    lib = _abi.load()
    a = chunk_args(**over)
    assert lib.kda_chunk_fwd(ctypes.byref(a), None) == _abi.KDA_ERR_INVALID_ARGUMENT
    n = ctypes.c_size_t(0)
    assert lib.kda_chunk_fwd_workspace_size(ctypes.byref(a), ctypes.byref(n)) == _abi.KDA_OK


@pytest.mark.parametrize("over,want", [
    (dict(gate_mode=_abi.KDA_GATE_SOFTPLUS), _abi.KDA_ERR_INVALID_ARGUMENT),
    (dict(gate_mode=_abi.KDA_GATE_SAFE, A_log=FAKE), _abi.KDA_ERR_INVALID_ARGUMENT),
    (dict(gate_mode=-1), _abi.KDA_ERR_INVALID_ARGUMENT),
])
def test_step_rejects_bad_gate(over, want):
    lib = _abi.load()
    a = step_args(**over)
    assert lib.kda_recurrent_step(ctypes.byref(a), None) == want


_LAYOUT_C = r"""
#include <stdio.h>
#include <stddef.h>
#include "kda.h"
#define F(S, m) printf(#S " " #m " %zu\n", offsetof(S, m));
int main(void) {
    printf("kda_chunk_args sizeof %zu\n", sizeof(kda_chunk_args));
    printf("kda_step_args sizeof %zu\n", sizeof(kda_step_args));
    printf("kda_token_args sizeof %zu\n", sizeof(kda_token_args));
    CHUNK_FIELDS
    STEP_FIELDS
    TOKEN_FIELDS
    return 0;
}
"""


def test_ctypes_structs_match_header_layout(tmp_path):
    """Every field of the ctypes mirrors sits at the offset the C compiler gives it."""
    import subprocess
    chunk = "".join(f"F(kda_chunk_args, {n})" for n, _ in _abi.ChunkArgs._fields_)
    step = "".join(f"F(kda_step_args, {n})" for n, _ in _abi.StepArgs._fields_)
    token = "".join(f"F(kda_token_args, {n})" for n, _ in _abi.TokenArgs._fields_)
    src = tmp_path / "layout.c"
    src.write_text(_LAYOUT_C.replace("CHUNK_FIELDS", chunk).replace("STEP_FIELDS", step)
                   .replace("TOKEN_FIELDS", token))
    exe = tmp_path / "layout"
    subprocess.run(["gcc", "-std=c11", "-I", os.path.join(ROOT, "include"), "-o", str(exe), str(src)],
                   check=True)
    got = {}
    for line in subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout.splitlines():
        struct, field, val = line.split()
        got[(struct, field)] = int(val)
    assert got[("kda_chunk_args", "sizeof")] == ctypes.sizeof(_abi.ChunkArgs)
    assert got[("kda_step_args", "sizeof")] == ctypes.sizeof(_abi.StepArgs)
    assert got[("kda_token_args", "sizeof")] == ctypes.sizeof(_abi.TokenArgs)
    for cls, name in ((_abi.ChunkArgs, "kda_chunk_args"), (_abi.StepArgs, "kda_step_args"),
                      (_abi.TokenArgs, "kda_token_args")):
        for field, _ in cls._fields_:
            assert got[(name, field)] == getattr(cls, field).offset, (name, field)
