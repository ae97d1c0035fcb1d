"""The boundary is a C ABI: include/gqe.h compiles as C99 (gcc -Wall -Werror -pedantic), and a
C program linked against libgqe.so calls the entry points that need no GPU (status strings,
stage names, workspace sizes, the shape and null-pointer checks that run before any CUDA
call, null-handle paths of gqe_forward and gqe_decode). CPU only."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
LIBDIR = os.path.join(ROOT, "moe_query_head_b200")

C_SOURCE = r"""
#include <stdio.h>
#include <string.h>
#include "gqe.h"

#define CHECK(c) do { if (!(c)) { printf("FAILED line %d: %s\n", __LINE__, #c); return 1; } } while (0)

int main(void) {
    gqe_handle h = NULL;
    int i;
    CHECK(strcmp(gqe_status_str(GQE_OK), "GQE_OK") == 0);
    for (i = 0; i < GQE_NUM_STAGES; ++i) CHECK(gqe_stage_name(i) != NULL);
    CHECK(gqe_stage_name(GQE_NUM_STAGES) == NULL);
    CHECK(gqe_workspace_bytes(768, 16, 8, 1, 48, GQE_BF16, 16384) > (int64_t)2 * 8 * 16384 * 48 * 2);
    CHECK(gqe_workspace_bytes(768, 15, 8, 1, 48, GQE_BF16, 16384) == -1);
    CHECK(gqe_create(&h, 768, 15, 8, 1, 48, GQE_BF16, 1024) == GQE_ERR_INVALID_ARG);
    CHECK(gqe_create(&h, 768, 16, 8, 1, 40, GQE_BF16, 1024) == GQE_ERR_UNSUPPORTED);
    CHECK(gqe_create(NULL, 768, 16, 8, 1, 48, GQE_BF16, 1024) == GQE_ERR_INVALID_ARG);
    CHECK(h == NULL);
    CHECK(gqe_forward(NULL, NULL, 1, 1, NULL, NULL, NULL, NULL, NULL, NULL, 16, 8, 1, 48,
                      GQE_VARIANT_GQE, 1, NULL, NULL, NULL) == GQE_ERR_INVALID_ARG);
    CHECK(gqe_decode(NULL, NULL, 1, NULL, NULL, 16, NULL, NULL, NULL, NULL, NULL, NULL, NULL,
                     16, 8, 1, 48, GQE_VARIANT_GQE, NULL, NULL, NULL) == GQE_ERR_INVALID_ARG);
    CHECK(gqe_check_device_status(NULL, NULL) == GQE_ERR_INVALID_ARG);
    CHECK(gqe_kernel_launches(NULL) == -1);
    gqe_destroy(NULL);
    printf("ok\n");
    return 0;
}
"""


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_header_is_c99_and_library_links_from_c(tmp_path):
    lib = os.path.join(LIBDIR, "libgqe.so")
    assert os.path.exists(lib), "libgqe.so not built"
    src = tmp_path / "abi.c"
    src.write_text(C_SOURCE)
    exe = tmp_path / "abi"
    cmd = ["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic",
           "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe),
           "-L", LIBDIR, "-lgqe", f"-Wl,-rpath,{LIBDIR}"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stdout + r.stderr
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0 and r.stdout.strip() == "ok", r.stdout + r.stderr
