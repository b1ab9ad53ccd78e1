"""The boundary is a C ABI: include/stief.h compiles as strict C11 and as C++17, and a plain C
program links against libstief.so and calls it (argument checks and planning only: no CUDA
call is made, so this runs without a GPU)."""
import os
import subprocess

import pytest

from decode_attention_stief_b200 import build as stief_build
import decode_attention_stief_b200 as stief

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
INCLUDE = os.path.join(ROOT, "include")

PROGRAM = r"""
#include "stief.h"
#include <stdio.h>
#include <string.h>

#define CHECK(cond) do { if (!(cond)) { printf("FAILED: %s (line %d)\n", #cond, __LINE__); return 1; } } while (0)

int main(void) {
    static uint16_t dummy[64] __attribute__((aligned(16)));
    int32_t lens[1] = {0};
    CHECK(strcmp(stief_status_string(STIEF_OK), "STIEF_OK") == 0);
    CHECK(strcmp(stief_status_string(STIEF_ERR_WORKSPACE), "STIEF_ERR_WORKSPACE") == 0);
    /* a null output pointer is an argument error: nothing is launched */
    CHECK(stief_decode_attention(dummy, dummy, dummy, dummy, dummy, lens, NULL, dummy, 1u << 20,
                                 1, 32, 8, 128, 64, 64, 1024, 1024, 0, NULL, NULL)
          == STIEF_ERR_INVALID_ARG);
    /* an unsupported head dimension */
    CHECK(stief_compress_append(dummy, dummy, dummy, dummy, dummy, dummy, lens, 1, 8, 1, 64, 64,
                                64, 1024, NULL, NULL) == STIEF_ERR_INVALID_ARG);
    /* a rank that is not a multiple of 16 */
    CHECK(stief_decode_latent(dummy, dummy, dummy, lens, dummy, dummy, 1u << 20, 1, 32, 8, 128,
                              72, 64, 1024, 1024, 0, NULL, NULL) == STIEF_ERR_INVALID_ARG);
    /* planning functions are plain host arithmetic */
    CHECK(stief_decode_max_splits(32768) >= 1);
    CHECK(stief_decode_auto_splits(1, 32, 8, 32768, 148) >= 1);
    CHECK(stief_decode_workspace_bytes(1, 32, 8, 64, 32768) > 0);
    printf("ok\n");
    return 0;
}
"""


@pytest.fixture(scope="module")
def libdir():
    stief_build.build_library()
    return os.path.dirname(stief.library_path())


def test_header_is_strict_c11_and_cxx17(tmp_path):
    src = tmp_path / "h.c"
    src.write_text('#include "stief.h"\nint main(void) { return (int)STIEF_OK; }\n')
    subprocess.run(["gcc", "-std=c11", "-Wall", "-Wextra", "-Werror", "-pedantic", "-I", INCLUDE,
                    "-fsyntax-only", str(src)], check=True)
    subprocess.run(["g++", "-std=c++17", "-Wall", "-Wextra", "-Werror", "-pedantic", "-I",
                    INCLUDE, "-x", "c++", "-fsyntax-only", str(src)], check=True)


def test_plain_c_program_links_and_calls_the_library(tmp_path, libdir):
    src = tmp_path / "abi_check.c"
    exe = tmp_path / "abi_check"
    src.write_text(PROGRAM)
    subprocess.run(["gcc", "-std=c11", "-Wall", "-Wextra", "-Werror", "-I", INCLUDE, str(src),
                    "-L", libdir, "-lstief", f"-Wl,-rpath,{libdir}", "-o", str(exe)], check=True)
    run = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert run.returncode == 0, run.stdout + run.stderr
    assert run.stdout.strip().endswith("ok")
