"""The boundary is a C ABI: include/fmoe.h compiles as C99, and a plain C program links
against libfmoe.so and calls its host-only entry points (CPU, no device)."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "bit_dequant_expert_softmax_b200")

C_PROGRAM = r"""
#include <stdio.h>
#include "fmoe.h"

int main(void) {
  fmoe_config cfg = {4096, 1024, 512, 4, 4, 1, 0};
  fmoe_config bad = {4096, 1024, 512, 600, 4, 1, 0};
  fmoe_layer_t layer = NULL;
  fmoe_weights w = {NULL, NULL, NULL, NULL};
  printf("%zu %zu\n", fmoe_record_bytes(4096, 1024, 4), fmoe_record_bytes(4096, 1024, 2));
  printf("%d %d\n", fmoe_workspace_bytes(&cfg) > 0, (int)fmoe_workspace_bytes(&bad));
  printf("%d\n", (int)fmoe_layer_create(&cfg, &w, &layer));
  printf("%s\n", fmoe_status_string(FMOE_ERR_NO_WORKSPACE));
  return 0;
}
"""


@pytest.fixture(scope="module")
def built():
    from bit_dequant_expert_softmax_b200 import build
    build.build()
    if shutil.which("gcc") is None:
        pytest.skip("no C compiler")
    return os.path.join(PKG, "libfmoe.so")


def test_header_is_plain_c99(built):
    out = subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror", "-fsyntax-only", "-x", "c",
                          os.path.join(ROOT, "include", "fmoe.h")], capture_output=True, text=True)
    assert out.returncode == 0, out.stderr


def test_c_program_links_and_calls_host_entry_points(built, tmp_path):
    src = tmp_path / "use_fmoe.c"
    src.write_text(C_PROGRAM)
    exe = tmp_path / "use_fmoe"
    cc = subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror", str(src), "-I", os.path.join(ROOT, "include"),
                         "-L", PKG, "-lfmoe", f"-Wl,-rpath,{PKG}", "-o", str(exe)], capture_output=True, text=True)
    assert cc.returncode == 0, cc.stderr
    run = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert run.returncode == 0, run.stderr
    assert run.stdout.split("\n")[:4] == ["7077888 3932160", "1 0", "1", "workspace missing or too small"]
