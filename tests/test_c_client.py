"""The C ABI from a plain C program: include/rb_api.h compiles as C99 (no
C++ or torch types), and a client linked against librb.so gets the host-side
answers (sizes, status strings, refusals before any launch). No GPU needed."""
import os
import shutil
import subprocess

import pytest

from residual_binary_weight_b200 import build as rb_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

C_SRC = r"""
#include <stdio.h>
#include <string.h>
#include "rb_api.h"

int main(void) {
    rb_layout L = {4096, 4096, 2, 0, RB_SLICED, 0};
    if (rb_planes_words(L) != (size_t)2 * 4096 * 16 * 8) return 1;
    if (rb_scales_count(L) != (size_t)2 * 4096) return 2;
    if (strcmp(rb_status_string(RB_ERR_ALIGNMENT), "RB_ERR_ALIGNMENT") != 0) return 3;
    rb_layout bad = {4096, 4000, 2, 0, RB_ROWS, 0};          /* K not a multiple of 128 */
    if (rb_gemv_workspace_bytes(bad, 1) != 0) return 4;
    if (rb_gemm_workspace_bytes(L, 2048) != 256) return 5;
    /* refused before anything touches a device: null pointers */
    if (rb_gemv(NULL, NULL, RB_F32, L, NULL, 4096, 1, NULL, RB_F16, 4096, NULL, 0, NULL) != RB_ERR_INVALID_ARG)
        return 6;
    if (rb_gemm_from_weight(NULL, RB_F16, 4096, L, NULL, 4096, 16, NULL, RB_F16, 4096, NULL, 0, NULL)
        != RB_ERR_INVALID_ARG)
        return 7;
    if (strlen(rb_last_error()) == 0) return 8;
    printf("ok\n");
    return 0;
}
"""


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_header_compiles_as_c_and_links(tmp_path):
    lib = rb_build.build()
    src = tmp_path / "client.c"
    src.write_text(C_SRC)
    exe = tmp_path / "client"
    subprocess.check_call(["gcc", "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"), str(src),
                           "-o", str(exe), os.path.abspath(lib), f"-Wl,-rpath,{os.path.dirname(os.path.abspath(lib))}"])
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert out.returncode == 0, (out.returncode, out.stdout, out.stderr)
    assert out.stdout.strip() == "ok"
