"""The boundary from plain C (no GPU, no Python binding): include/kda.h
compiles as C99 and as C++ with warnings as errors, and a C program linked
against libkda.so plans a prefill call and names status codes."""
import os
import subprocess

import pytest

from gated_delta_rule_117_b200 import build as kbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "gated_delta_rule_117_b200")

PROGRAM = r"""
#include <stdio.h>
#include "kda.h"
int main(void) {
  kda_plan_t p;
  kda_status_t s = kda_chunk_fwd_plan(1, 16, 4096, 128, 128, KDA_DTYPE_BF16, 0, &p);
  printf("%d %d %d %d %d %zu\n", (int)s, p.path, p.chunk_size, p.segments, p.launches, p.workspace);
  printf("%d\n", (int)kda_chunk_fwd_plan(1, 2, 64, 24, 16, KDA_DTYPE_F32, 0, &p));
  printf("%s\n", kda_status_string(KDA_ERR_ALIAS));
  printf("%d\n", kda_version());
  return 0;
}
"""


@pytest.mark.parametrize("lang,flags", [("c", ["-std=c99"]), ("c++", ["-std=c++17"])])
def test_header_compiles(tmp_path, lang, flags):
    src = tmp_path / ("h." + ("c" if lang == "c" else "cpp"))
    src.write_text('#include "kda.h"\nint kda_header_probe(void) { return KDA_OK; }\n')
    cc = "gcc" if lang == "c" else "g++"
    subprocess.check_call([cc, *flags, "-Wall", "-Wextra", "-Werror", "-c", "-I", os.path.join(ROOT, "include"),
                           "-o", str(tmp_path / "h.o"), str(src)])


def test_c_program_against_the_library(tmp_path):
    kbuild.build()
    src = tmp_path / "plan.c"
    src.write_text(PROGRAM)
    exe = tmp_path / "plan"
    subprocess.check_call(["gcc", "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"), str(src),
                           "-L", PKG, "-lkda", "-Wl,-rpath," + PKG, "-o", str(exe)])
    out = subprocess.run([str(exe)], capture_output=True, text=True, check=True).stdout.split("\n")
    status, path, chunk, segments, launches, workspace = map(int, out[0].split())
    assert status == 0 and path == 2 and chunk == 32 and segments == 9 and launches == 4 and workspace > 0
    assert int(out[1]) == 2                              # KDA_ERR_SHAPE for dk = 24
    assert out[2].startswith("KDA_ERR_ALIAS")
    assert int(out[3]) >= 100
