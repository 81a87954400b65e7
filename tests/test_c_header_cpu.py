"""The public header from C: include/rwkv_wkv.h compiles as plain C99 with warnings as
errors, and a C program links libwkv.so and gets the documented answers from calls that
need no GPU (version, status strings, host-side argument errors)."""
import os
import shutil
import subprocess

import pytest

from wkv_recurrence_02_b200 import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

C_SOURCE = r"""
#include <stdio.h>
#include <string.h>
#include "rwkv_wkv.h"

int main(void)
{
    size_t bytes = 1;
    int fails = 0;
    if (rwkv_abi_version() != RWKV_ABI_VERSION) fails |= 1;
    if (strcmp(rwkv_status_string(RWKV_ERR_ALIAS), "output overlaps an input") != 0) fails |= 2;
    /* host-side validation: no CUDA call is made */
    if (rwkv_wkv4_forward(-1, 4, 16, 0, 0, 0, 0, 0) != RWKV_ERR_SHAPE) fails |= 4;
    if (rwkv_wkv6_forward(1, 4, 2, 32, 0, 0, 0, 0, 0, 0, 0, 0) != RWKV_ERR_UNSUPPORTED) fails |= 8;
    if (rwkv_wkv6_forward_bf16(0, 4, 2, 64, 0, 0, 0, 0, 0, 0, 0, 0) != RWKV_OK) fails |= 16;
    if (rwkv_wkv6_backward_workspace_bytes(2, 20, 3, 64, &bytes) != RWKV_OK ||
        /* the walks' three fp32 checkpoints per (b, h), then du shares per (b, h) and per
           (b, h, chunk), then the (b, h) flags rounded up to 16 bytes */
        bytes != (size_t)2 * 3 * (3 * 64 * 64) * 4 + 2 * 3 * 64 * 4 + 2 * 3 * 1 * 64 * 4 + 32) fails |= 32;
    if (rwkv_set_wkv6_algo(99) != RWKV_ERR_ARG) fails |= 64;
    printf("fails=%d\n", fails);
    return fails;
}
"""


@pytest.mark.skipif(shutil.which("gcc") is None, reason="no C compiler")
def test_header_is_c99_and_links(tmp_path):
    lib = build.build()
    src = tmp_path / "abi_from_c.c"
    src.write_text(C_SOURCE)
    exe = tmp_path / "abi_from_c"
    libdir = os.path.dirname(lib)
    cmd = ["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic", "-I", os.path.join(ROOT, "include"),
           str(src), "-o", str(exe), "-L", libdir, "-l:" + os.path.basename(lib), "-Wl,-rpath," + libdir]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0 and r.stdout.strip() == "fails=0", (r.returncode, r.stdout, r.stderr)
