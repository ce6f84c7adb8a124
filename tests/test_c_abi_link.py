"""The boundary is a plain C ABI: a C99 program that includes include/dora.h
and links libdora_b200.so builds with gcc and runs without Python or torch.
Only calls that need no GPU are made (version, workspace sizes, argument
validation and its error message).
"""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
LIBDIR = os.path.join(ROOT, "dora_weight_decomposed_b200")

C_SRC = r"""
#include <stdio.h>
#include <string.h>
#include "dora.h"

int main(void) {
  dora_desc_t d = {8192, 8192, 384, DORA_BF16, 0.5f};
  size_t n = dora_workspace_size(&d, 0, DORA_OP_NORM);
  size_t b = dora_workspace_size(&d, 4096, DORA_OP_BACKWARD);
  size_t f = dora_workspace_size(&d, 4096, DORA_OP_BACKWARD_FULL);
  if (dora_version() <= 0 || n == 0 || b == 0 || f <= b) return 1;
  dora_desc_t bad = {8192, 8192, 12, DORA_BF16, 0.5f};
  if (dora_workspace_size(&bad, 0, DORA_OP_NORM) != 0) return 2;
  if (dora_merge(&d, NULL, NULL, NULL, NULL, NULL, NULL, 0, NULL) != DORA_EINVAL) return 3;
  if (strstr(dora_last_error(), "W0") == NULL) return 4;
  printf("ok %zu %zu %zu\n", n, b, f);
  return 0;
}
"""


@pytest.mark.skipif(shutil.which("gcc") is None, reason="no C compiler")
def test_c_program_links_and_calls_the_library(tmp_path):
    lib = os.path.join(LIBDIR, "libdora_b200.so")
    if not os.path.exists(lib):
        from dora_weight_decomposed_b200 import build
        build.build()
    src = tmp_path / "use_dora.c"
    src.write_text(C_SRC)
    exe = tmp_path / "use_dora"
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"), str(src), "-o",
                    str(exe), "-L", LIBDIR, "-ldora_b200", "-Wl,-rpath," + LIBDIR], check=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True)
    assert out.returncode == 0, (out.returncode, out.stdout, out.stderr)
    assert out.stdout.startswith("ok ")
