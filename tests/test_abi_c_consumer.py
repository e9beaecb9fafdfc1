"""The C ABI from plain C, on the CPU: a C11 program that includes include/swa.h (compiled
as C, not C++) links against the library and calls its device-free entry points and an
argument refusal. No GPU is used."""
import os
import subprocess

import pytest

from sliding_window_causal_b200 import _native, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

PROGRAM = r"""
#include <stdio.h>
#include <string.h>
#include "swa.h"

int main(void) {
    int bad = 0;
    int32_t splits = 0, chunk = 0;
    if (swa_decode_valid_slots(5, 16) != 6) bad |= 1;
    if (swa_decode_valid_slots(100, 16) != 16) bad |= 2;
    if (swa_prefill_tile_class(300, 77, 128, 128, 1, 0) < 0) bad |= 4;
    if (swa_decode_split_plan(64, 32, 128, 4096, &splits, &chunk) != SWA_OK
        || splits < 1 || (int64_t)splits * chunk < 4096) bad |= 8;
    if (swa_backward_workspace_bytes(1, 2, 130) != 8 * 2 * 256) bad |= 16;
    if (swa_mha_workspace_bytes(1, 8, 0, SWA_BF16) != -1) bad |= 32;
    /* a refusal: W < 1, decided before any device call */
    if (swa_forward((const void*)0x10000, (const void*)0x10000, (const void*)0x10000,
                    (void*)0x10000, 1, 1, 8, 64, 0, SWA_BF16, NULL) != SWA_ERR_INVALID_ARG) bad |= 64;
    if (strlen(swa_last_error()) == 0) bad |= 128;
    printf("%d\n", bad);
    return bad != 0;
}
"""


@pytest.fixture(scope="module", autouse=True)
def built_library():
    build.build()


def test_header_compiles_as_c_and_links(tmp_path):
    src = tmp_path / "consumer.c"
    src.write_text(PROGRAM)
    exe = tmp_path / "consumer"
    libdir = os.path.dirname(_native.LIB_PATH)
    name = os.path.basename(_native.LIB_PATH)
    cmd = ["gcc", "-std=c11", "-Wall", "-Werror", "-pedantic", "-I", os.path.join(ROOT, "include"),
           str(src), "-o", str(exe), os.path.join(libdir, name), f"-Wl,-rpath,{libdir}"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0 and r.stdout.strip() == "0", (r.stdout, r.stderr)
