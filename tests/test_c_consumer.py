"""The library as a plain C program sees it: include/kda.h compiled by gcc, libkda.so
linked directly (no Python, no torch). Only calls that need no GPU are made: the
version, status strings, the workspace queries, and argument checks that fail
before any launch."""
import os
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "kimi_delta_attention_20_b200")

_MAIN_C = r"""
#include <stdint.h>
#include <stdio.h>
#include <string.h>
#include "kda.h"

#define CHECK(c) do { if (!(c)) { printf("failed: %s (line %d)\n", #c, __LINE__); return 1; } } while (0)

int main(void) {
    CHECK(kda_version() == KDA_VERSION);
    for (int s = KDA_OK; s <= KDA_ERR_WORKSPACE; ++s) {
        const char *name = kda_status_string((kda_status)s);
        CHECK(name != NULL && strlen(name) > 0);
    }
    CHECK(kda_last_cuda_error() == 0);

    /* workspace queries read shapes only */
    kda_chunk_args c;
    memset(&c, 0, sizeof c);
    c.dtype = KDA_DTYPE_BF16;
    c.B = 1; c.T = 8192; c.H = 16; c.Dk = 128; c.Dv = 128; c.N = 1;
    c.use_qk_l2norm = 1;
    size_t bytes = 0;
    CHECK(kda_chunk_fwd_workspace_size(&c, &bytes) == KDA_OK);
    CHECK(bytes >= (size_t)128 * 16 * 65536);  /* one record of > 64 KiB per (chunk, head) */
    c.Dk = 48;
    CHECK(kda_chunk_fwd_workspace_size(&c, &bytes) == KDA_ERR_UNSUPPORTED);
    CHECK(kda_chunk_fwd_workspace_size(&c, NULL) == KDA_ERR_INVALID_ARGUMENT);

    /* argument checks fail before any launch */
    CHECK(kda_chunk_fwd(NULL, NULL) == KDA_ERR_INVALID_ARGUMENT);
    CHECK(kda_chunk_fwd_noalloc(NULL, NULL) == KDA_ERR_INVALID_ARGUMENT);
    CHECK(kda_recurrent_step(NULL, NULL) == KDA_ERR_INVALID_ARGUMENT);
    CHECK(kda_decode_token(NULL, NULL) == KDA_ERR_INVALID_ARGUMENT);

    kda_step_args s;
    memset(&s, 0, sizeof s);
    s.dtype = KDA_DTYPE_F32;
    s.N = 2; s.H = 2; s.Dk = 64; s.Dv = 64;
    void *fake = (void *)(uintptr_t)0x10000;  /* aligned, never dereferenced */
    s.q = s.k = s.v = s.g = s.beta = fake;
    s.o = fake;
    s.state = (float *)((uintptr_t)0x10000 + 8);  /* misaligned state */
    CHECK(kda_recurrent_step(&s, NULL) == KDA_ERR_INVALID_ARGUMENT);
    s.state = (float *)fake;
    s.state_out = (float *)((uintptr_t)0x10000 + 4096);  /* overlaps the state */
    CHECK(kda_recurrent_step(&s, NULL) == KDA_ERR_INVALID_ARGUMENT);
    s.N = 0;  /* an empty batch is a no-op */
    CHECK(kda_recurrent_step(&s, NULL) == KDA_OK);
    printf("ok\n");
    return 0;
}
"""


def test_plain_c_program_links_and_calls_the_library(tmp_path):
    lib = os.path.join(PKG, "libkda.so")
    if not os.path.exists(lib):
        pytest.fail("libkda.so is not built (python -m kimi_delta_attention_20_b200.build)")
    src = tmp_path / "main.c"
    src.write_text(_MAIN_C)
    exe = tmp_path / "main"
    subprocess.run(["gcc", "-std=c11", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"), "-o", str(exe),
                    str(src), "-L", PKG, "-l:libkda.so", f"-Wl,-rpath,{PKG}"], check=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0, r.stdout + r.stderr
    assert r.stdout.strip() == "ok"
