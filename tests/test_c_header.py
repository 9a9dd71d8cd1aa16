"""The boundary is plain C: include/macaq.h compiles as C99 with warnings as
errors, a C program links against the built libmacaq.so, and the host-only
calls behave as the header states (sizes, status names, refusals of bad
arguments before any device work)."""
import os
import subprocess

import pytest

import w4a4_mxfp4_quantize_b200 as mq

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

PROGRAM = r"""
#include <stdio.h>
#include <string.h>
#include "macaq.h"

static int fails = 0;
#define CHECK(c) do { if (!(c)) { printf("FAIL line %d: %s\n", __LINE__, #c); fails++; } } while (0)

int main(void) {
    CHECK(macaq_abi_version() == MACAQ_ABI_VERSION);
    /* prepared weights: pairs of 128-row tiles per 256-wide K tile */
    CHECK(macaq_weight_code_bytes(1, 1024, 1024) == (size_t)1024 * 512);
    CHECK(macaq_weight_scale_bytes(1, 1024, 1024) == (size_t)1024 * 32);
    CHECK(macaq_weight_code_bytes(2, 48, 256) == (size_t)2 * 256 * 128);   /* rows padded to 256 */
    CHECK(macaq_weight_code_bytes(1, 130, 1024) == 0);                     /* N % 16 != 0 */
    CHECK(macaq_weight_code_bytes(1, 1024, 1000) == 0);                    /* K % 256 != 0 */
    CHECK(macaq_weight_code_bytes(1, 1024, 288) == 0);                     /* K % 32 == 0, K % 256 != 0 */
    CHECK(macaq_weight_code_bytes(1025, 1024, 1024) == 0);                 /* E > 1024 */
    CHECK(macaq_workspace_bytes(128, 1024, 1024, 1) == 0);                 /* fused: no scratch */
    CHECK(macaq_workspace_bytes(4096, 1024, 1024, 1) > 0);
    CHECK(strcmp(macaq_status_string(MACAQ_OK), "MACAQ_OK") == 0);
    CHECK(strcmp(macaq_status_string(MACAQ_ERR_ACT_TYPE), "MACAQ_ERR_ACT_TYPE") == 0);
    /* refusals that need no device */
    CHECK(macaq_dense_mm(NULL, NULL, NULL, NULL, NULL, 16, 1024, 1024, NULL, 0, NULL, NULL) == MACAQ_ERR_NULL);
    CHECK(macaq_dense_mm(NULL, NULL, NULL, NULL, NULL, 16, 1024, 1000, NULL, 0, NULL, NULL) == MACAQ_ERR_SHAPE);
    CHECK(macaq_dense_mm(NULL, NULL, NULL, NULL, NULL, 0, 1024, 1024, NULL, 0, NULL, NULL) == MACAQ_OK);
    CHECK(macaq_prepare_weights(NULL, NULL, 1, 1024, 1024, NULL, NULL, NULL) == MACAQ_ERR_NULL);
    printf("%s\n", fails ? "failed" : "ok");
    return fails != 0;
}
"""


@pytest.fixture(scope="module")
def libdir():
    mq.build()
    return os.path.dirname(mq.build())


def test_header_is_c99_and_links_from_c(tmp_path, libdir):
    src = tmp_path / "use_macaq.c"
    src.write_text(PROGRAM)
    exe = tmp_path / "use_macaq"
    subprocess.check_call(["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic",
                           "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe),
                           "-L", libdir, "-lmacaq", f"-Wl,-rpath,{libdir}"])
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert out.returncode == 0 and out.stdout.strip().endswith("ok"), out.stdout + out.stderr
